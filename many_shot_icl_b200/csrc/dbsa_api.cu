// C-ABI entry points of the DBSA library: argument validation, host-side
// planning (tile list, gather segments, split plan), workspace carving and
// kernel launches.  All arithmetic of the method runs in the kernels.
#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <string>
#include <vector>

#include "dbsa_internal.h"

using namespace dbsa;

namespace {

thread_local std::string g_err;
// Calls this library made that allocate or free page-locked host memory or
// create or destroy events (each can synchronise the device).
std::atomic<int64_t> g_host_alloc_calls{0};
void count_host_alloc() { g_host_alloc_calls.fetch_add(1, std::memory_order_relaxed); }
thread_local cudaEvent_t g_prof_start = nullptr, g_prof_stop = nullptr;
// Test hook for the next call on this thread (dbsa_test_wait_expiry): its
// tensor-core kernel loads no tile and its waits give up after this many
// nanoseconds (0: no hook).
thread_local uint64_t g_wait_expiry_ns = 0;

uint64_t take_wait_expiry() {
  const uint64_t w = g_wait_expiry_ns;
  g_wait_expiry_ns = 0;
  return w;
}
std::atomic<int64_t> g_launches{0};

void count_launches(int n) { g_launches.fetch_add(n, std::memory_order_relaxed); }

// Records the profiling events (if any) around the main kernel of a call.
struct ProfileScope {
  cudaStream_t st;
  cudaEvent_t stop;
  explicit ProfileScope(cudaStream_t s) : st(s), stop(g_prof_stop) {
    if (g_prof_start) cudaEventRecord(g_prof_start, st);
    g_prof_start = g_prof_stop = nullptr;
  }
  ~ProfileScope() {
    if (stop) cudaEventRecord(stop, st);
  }
};

dbsa_status fail(dbsa_status s, const char *fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof buf, fmt, ap);
  va_end(ap);
  g_err = buf;
  return s;
}

dbsa_status cuda_fail(cudaError_t e, const char *where) {
  return fail(DBSA_ERR_CUDA, "%s: %s", where, cudaGetErrorString(e));
}

constexpr size_t kAlign = 1024;
// Block-major passes with at most this many query rows per (query, KV head)
// (g * n_new) run the tail attention and the merge as one warp-per-row
// kernel; longer passes (prompt passes) keep the tail on the per-query
// mma.sync kernel, which shares each tail key among all the rows.
constexpr int kTailMergeMaxRows = 32;
// Per-query selections (short segments the block-major path cannot share
// cheaply) with at least this many query rows per (query, KV head) run in
// compact mode on the tensor core; fewer rows stay on the per-query mma.sync
// kernel.
constexpr int kCompactMinRows = 64;
// Tensor-core passes whose items average at least this many key tiles rotate
// the packed query rows inside the kernel (the epilogue warpgroup fills the
// Q tile of the item two ahead while the next one runs); with shorter items
// (demonstration-granular decode steps, one key tile each) every item would
// wait for its rotation, so qhat_kernel packs the rows beforehand and the
// kernel loads them by TMA.
constexpr int kRotateQMinTiles = 4;
size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Copies bytes from page-locked host memory (read over the bus by the SMs)
// into device memory: 16-byte words while both sides allow, then bytes.
__global__ void __launch_bounds__(256) copy_from_host_kernel(uint8_t *dst, const uint8_t *src,
                                                             size_t bytes, uint32_t *clear) {
  pdl_enter();
  // the call's status head, cleared here rather than by a separate memset
  if (clear != nullptr && blockIdx.x == 0 && threadIdx.x < kStatusBytes / 4) clear[threadIdx.x] = 0;
  const size_t stride = (size_t)gridDim.x * blockDim.x;
  const size_t i0 = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
  const bool vec = ((reinterpret_cast<uintptr_t>(dst) | reinterpret_cast<uintptr_t>(src)) & 15u) == 0;
  const size_t words = vec ? bytes / 16 : 0;
  for (size_t i = i0; i < words; i += stride)
    reinterpret_cast<uint4 *>(dst)[i] = reinterpret_cast<const uint4 *>(src)[i];
  for (size_t i = words * 16 + i0; i < bytes; i += stride) dst[i] = src[i];
}

// Host-built plans (tile lists, gather tables, block offsets) reach the device
// through page-locked staging memory that a small kernel reads directly.  Two
// things are avoided: from a pageable source cudaMemcpyAsync holds the calling
// thread until the copy can be staged (stalling a caller that queues later
// layers behind this call), and a copy-engine transfer can be queued behind
// the caller's own large uploads on other streams (the next layer's inputs),
// delaying this call by their whole duration.  Each thread keeps a ring of
// staging slots; a slot is refilled only once the event recorded behind its
// previous read has completed, so a read never sees a slot being rewritten.
// A thread's slots are released when it exits, after their last reads (errors
// are ignored there: at process exit the runtime may already be gone).
// Calls that use the ring cannot be captured into a CUDA graph: the host fills
// the slot at call time.
class StagingRing {
 public:
  StagingRing() = default;
  StagingRing(const StagingRing &) = delete;
  StagingRing &operator=(const StagingRing &) = delete;
  ~StagingRing() {
    for (Slot &s : slots_) {
      if (s.ev != nullptr) {
        cudaEventSynchronize(s.ev);
        cudaEventDestroy(s.ev);
        count_host_alloc();
      }
      if (s.p != nullptr) {
        cudaFreeHost(s.p);
        count_host_alloc();
      }
    }
  }
  // A page-locked buffer of >= bytes for the next upload (waits for the
  // slot's previous read); the caller fills it, then calls send().
  cudaError_t stage(size_t bytes, void **host) {
    Slot &s = slots_[next_];
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (s.ev != nullptr) {
      if ((e = cudaEventSynchronize(s.ev)) != cudaSuccess) return e;
      if (s.dev != dev) {
        cudaEventDestroy(s.ev);
        count_host_alloc();
        s.ev = nullptr;
      }
    }
    // All slots share one capacity, which doubles when a plan outgrows it;
    // each slot is brought up to it on its next use, so that after one round
    // of the ring no plan of that size reallocates (freeing a page-locked
    // buffer synchronizes the device).
    if (bytes > cap_all_) cap_all_ = align_up(std::max(bytes, 2 * cap_all_), size_t(1) << 16);
    if (s.cap < cap_all_) {
      if (s.p != nullptr) {
        cudaFreeHost(s.p);  // its last read has completed
        count_host_alloc();
      }
      s.p = nullptr;
      const size_t cap = cap_all_;
      s.cap = 0;
      count_host_alloc();
      if ((e = cudaHostAlloc(&s.p, cap, cudaHostAllocPortable | cudaHostAllocMapped)) !=
          cudaSuccess)
        return e;
      s.cap = cap;
    }
    if (s.ev == nullptr) {
      count_host_alloc();
      if ((e = cudaEventCreateWithFlags(&s.ev, cudaEventDisableTiming)) != cudaSuccess) return e;
      s.dev = dev;
    }
    *host = s.p;
    return cudaSuccess;
  }
  // Copies the first bytes of the buffer stage() returned to dst on stream st
  // and, when clear is given, zeroes the kStatusBytes status head there.
  cudaError_t send(void *dst, size_t bytes, cudaStream_t st, void *clear = nullptr) {
    Slot &s = slots_[next_];
    next_ = (next_ + 1) % kSlots;
    if (bytes > 0 || clear != nullptr) {
      const int grid = (int)std::max<size_t>(1, std::min<size_t>((bytes + 4095) / 4096, 148));
      pdl_launch(copy_from_host_kernel, dim3(grid), dim3(256), 0, st, static_cast<uint8_t *>(dst),
                                                 static_cast<const uint8_t *>(s.p), bytes,
                                                 static_cast<uint32_t *>(clear));
      cudaError_t e = cudaGetLastError();
      if (e != cudaSuccess) return e;
      count_launches(1);
    }
    return cudaEventRecord(s.ev, st);
  }
  cudaError_t upload(void *dst, const void *src, size_t bytes, cudaStream_t st,
                     void *clear = nullptr) {
    if (bytes == 0 && clear == nullptr) return cudaSuccess;
    void *h = nullptr;
    cudaError_t e = stage(std::max<size_t>(bytes, 16), &h);
    if (e != cudaSuccess) return e;
    if (bytes > 0) std::memcpy(h, src, bytes);
    return send(dst, bytes, st, clear);
  }

 private:
  struct Slot {
    void *p = nullptr;
    size_t cap = 0;
    cudaEvent_t ev = nullptr;
    int dev = -1;
  };
  static constexpr int kSlots = 8;
  Slot slots_[kSlots];
  int next_ = 0;
  size_t cap_all_ = 0;
};

StagingRing &staging_ring() {
  static thread_local StagingRing ring;
  return ring;
}
// Uploads a host-built plan through the staging ring; `clear` (a workspace
// head, or null) gets its status bytes zeroed by the same kernel.
cudaError_t upload_async(void *dst, const void *src, size_t bytes, cudaStream_t st,
                         void *clear = nullptr) {
  return staging_ring().upload(dst, src, bytes, st, clear);
}

// Sequential sub-allocation of the caller's workspace.
struct Carve {
  size_t off = kStatusBytes;
  size_t take(size_t bytes) {
    const size_t o = align_up(off, kAlign);
    off = o + bytes;
    return o;
  }
  size_t total() const { return align_up(off, kAlign); }
};

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

dbsa_status check_cfg(const dbsa_config *cfg) {
  if (cfg == nullptr) return fail(DBSA_ERR_INVALID_ARG, "cfg is NULL");
  if (cfg->n_q_heads <= 0 || cfg->n_kv_heads <= 0)
    return fail(DBSA_ERR_INVALID_ARG, "head counts must be positive");
  if (cfg->n_q_heads % cfg->n_kv_heads != 0)
    return fail(DBSA_ERR_UNSUPPORTED, "n_q_heads must be a multiple of n_kv_heads");
  if (cfg->n_q_heads / cfg->n_kv_heads > 64)
    return fail(DBSA_ERR_UNSUPPORTED, "more than 64 query heads per KV head");
  if (cfg->head_dim != 64 && cfg->head_dim != 128)
    return fail(DBSA_ERR_UNSUPPORTED, "head_dim must be 64 or 128 (got %d)", cfg->head_dim);
  if (cfg->dtype != DBSA_BF16 && cfg->dtype != DBSA_F32)
    return fail(DBSA_ERR_UNSUPPORTED, "dtype must be DBSA_BF16 or DBSA_F32");
  if (!(cfg->rope_theta > 1.0) || !std::isfinite(cfg->rope_theta))
    return fail(DBSA_ERR_INVALID_ARG, "rope_theta must be a finite value > 1");
  if (cfg->window_j < 0) return fail(DBSA_ERR_INVALID_ARG, "window_j must be >= 0");
  if (cfg->pattern < 0 || cfg->pattern > 3) return fail(DBSA_ERR_INVALID_ARG, "unknown pattern");
  if (cfg->reserved != 0) return fail(DBSA_ERR_INVALID_ARG, "reserved must be 0");
  if (!std::isfinite(cfg->softmax_scale)) return fail(DBSA_ERR_INVALID_ARG, "bad softmax_scale");
  return DBSA_OK;
}

dbsa_status check_offs(const int32_t *offs, int32_t nb) {
  if (offs == nullptr) return fail(DBSA_ERR_INVALID_ARG, "offs is NULL");
  if (nb < 1) return fail(DBSA_ERR_INVALID_ARG, "need at least one block (nb = %d)", nb);
  if (offs[0] != 0) return fail(DBSA_ERR_INVALID_ARG, "offs[0] must be 0");
  for (int32_t b = 0; b < nb; ++b)
    if (offs[b + 1] <= offs[b])
      return fail(DBSA_ERR_INVALID_ARG, "block %d is empty or offsets decrease", b);
  if (offs[nb] > (1 << 30)) return fail(DBSA_ERR_INVALID_ARG, "context too long");
  return DBSA_OK;
}

float scale_log2(const dbsa_config *cfg) {
  const double s = cfg->softmax_scale > 0.f ? (double)cfg->softmax_scale
                                            : 1.0 / std::sqrt((double)cfg->head_dim);
  return (float)(s * 1.4426950408889634);  // * log2(e)
}

int num_sms() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
    return 148;
  return n;
}

// -------------------------------------------------------------- Stage-1 plan
// Key ranges (positions [rs, re)) a block may attend to before the causal
// clip, in processing order: the sink first, then the contiguous window that
// ends with the block itself.  [DBSA notes] §Stage 1, item 2 and §Ablations.
int key_ranges(int pattern, int j, const int32_t *offs, int b, int32_t rs[2], int32_t re[2]) {
  const bool sink = pattern == DBSA_PATTERN_SINK_PREV_SELF || pattern == DBSA_PATTERN_SINK_SELF;
  int w0;
  if (pattern == DBSA_PATTERN_SINK_PREV_SELF) w0 = std::max(0, b - j);
  else if (pattern == DBSA_PATTERN_FULL) w0 = 0;
  else w0 = b;
  if (!sink || w0 <= 1) {
    rs[0] = offs[sink ? 0 : w0];
    re[0] = offs[b + 1];
    return 1;
  }
  rs[0] = offs[0];
  re[0] = offs[1];
  rs[1] = offs[w0];
  re[1] = offs[b + 1];
  return 2;
}

int64_t tiles_of(const dbsa_tile_item &it) {
  int64_t n = 0;
  for (int r = 0; r < it.n_ranges; ++r) n += (it.len[r] + kTileKeys - 1) / kTileKeys;
  return n;
}

// Items of one block: one per (query head, 128-row tile).  Rows of the tile
// at positions q_pos0.., stored at rows q_row0.. of q / out.  Key rows of
// range r start at k_row_of[r] in the rotated-K buffer, v_row_of[r] in V.
void block_items(const dbsa_config *cfg, const int32_t *offs, int b, int32_t q_row_shift,
                 const int32_t k_row_of[2], const int32_t v_row_of[2], int nr, const int32_t rs[2],
                 const int32_t re[2], std::vector<dbsa_tile_item> &items) {
  const int Hq = cfg->n_q_heads, Hkv = cfg->n_kv_heads, g = Hq / Hkv;
  const int L = offs[b + 1] - offs[b];
  const int n_qt = (L + kTileRows - 1) / kTileRows;
  for (int c = 0; c < Hkv; ++c)
    for (int m = 0; m < n_qt; ++m)
      for (int hl = 0; hl < g; ++hl) {
        dbsa_tile_item it;
        std::memset(&it, 0, sizeof it);
        it.head = c * g + hl;
        it.q_pos0 = offs[b] + m * kTileRows;
        it.q_row0 = it.q_pos0 - q_row_shift;
        it.n_rows = std::min(kTileRows, offs[b + 1] - it.q_pos0);
        it.block = b;
        const int32_t qend = it.q_pos0 + it.n_rows;
        int n = 0;
        for (int r = 0; r < nr; ++r) {
          const int32_t e = std::min(re[r], qend);
          if (e <= rs[r]) continue;
          it.k_row0[n] = k_row_of[r];
          it.v_row0[n] = v_row_of[r];
          it.pos0[n] = rs[r];
          it.len[n] = e - rs[r];
          ++n;
        }
        it.n_ranges = n;
        items.push_back(it);
      }
}

// The encode tile list: blocks in decreasing order of work (the light blocks
// at the start of the context go last), then KV head, query tile, query head
// so that neighbouring CTAs share K/V tiles in L2.
void encode_items(const dbsa_config *cfg, const int32_t *offs, int32_t nb,
                  std::vector<dbsa_tile_item> &items) {
  std::vector<std::pair<int64_t, int>> order;
  for (int b = 0; b < nb; ++b) {
    int32_t rs[2], re[2];
    const int nr = key_ranges(cfg->pattern, cfg->window_j, offs, b, rs, re);
    int64_t keys = 0;
    for (int r = 0; r < nr; ++r) keys += re[r] - rs[r];
    order.push_back({-keys * (offs[b + 1] - offs[b]), b});
  }
  std::stable_sort(order.begin(), order.end(),
                   [](const auto &x, const auto &y) { return x.first < y.first; });
  for (const auto &ob : order) {
    const int b = ob.second;
    int32_t rs[2], re[2];
    const int nr = key_ranges(cfg->pattern, cfg->window_j, offs, b, rs, re);
    block_items(cfg, offs, b, 0, rs, rs, nr, rs, re, items);
  }
}

// Append plan: the new block nb (positions T0..T0+L-1) attends to ranges of
// the extended offset table; the rotated keys of those ranges are packed
// contiguously ("compact rows").
struct AppendPlan {
  std::vector<int32_t> offs;  // extended, nb + 2 entries
  int nr;
  int32_t rs[2], re[2], cs[2];
  int32_t k_rows;             // compact rows
  int32_t new_row;            // compact row of position T0
};
AppendPlan append_plan(const dbsa_config *cfg, const int32_t *offs, int32_t nb, int32_t L) {
  AppendPlan p;
  p.offs.assign(offs, offs + nb + 1);
  p.offs.push_back(offs[nb] + L);
  p.nr = key_ranges(cfg->pattern, cfg->window_j, p.offs.data(), nb, p.rs, p.re);
  p.cs[0] = 0;
  p.cs[1] = p.re[0] - p.rs[0];
  p.k_rows = 0;
  for (int r = 0; r < p.nr; ++r) p.k_rows += p.re[r] - p.rs[r];
  const int rl = p.nr - 1;  // the last range holds the new block
  p.new_row = p.cs[rl] + (offs[nb] - p.rs[rl]);
  return p;
}

// -------------------------------------------------------------- Stage-2 plan
struct GatherPlan {
  std::vector<S2Query> queries;
  std::vector<S2Segment> segs;
  std::vector<S2Item> items;
  int32_t max_pos;  // largest key / query position + 1
  // items the per-query kernel runs: the tail items (one per query) in the
  // block-major mode, every split item in the per-query mode
  std::vector<int32_t> run_items;
  // per-query mode (short selected segments, e.g. single demonstrations):
  // each query's key sequence is split into a few items that the per-query
  // kernel gathers segment by segment; no packed rows, no tensor-core tiles
  bool per_query = false;
  // compact mode (a per-query selection of short segments with many query
  // rows, e.g. a demonstration-granular prompt pass): every query's gathered
  // keys, rotated at their fresh positions, and its values are written to a
  // compact buffer (query q's rows start at compact_base[q]); the tensor-core
  // kernel then attends per (KV head, query, 128-row tile) over them
  bool compact = false;
  std::vector<int32_t> compact_base;
  int64_t compact_rows = 0;
  // the query rows of all (query, block) items packed block by block, and the
  // tile list of the tensor-core kernel over them
  int32_t tc_rows = 0;
  int32_t nb = 0;
  int64_t cache_rows = 0;  // offs[nb]
  // packed_items[k]: the item owning packed rows [k R, (k + 1) R), R = g n_new
  std::vector<int32_t> packed_items;
  // per item: (first packed row or -1 for a tail item, the position its query
  // rows are rotated at for token 0, its query, 0), read by the packing kernel
  std::vector<int4> item_meta;
  std::vector<dbsa_tile_item> tc_tiles;
};

int32_t offs_count(const GatherPlan &gp) { return gp.nb + 1; }

// Whether the pass's tensor-core kernel rotates its packed query rows itself.
bool rotates_q(const GatherPlan &gp) {
  int64_t tiles = 0;
  for (const dbsa_tile_item &t : gp.tc_tiles) tiles += (t.len[0] + kTileKeys - 1) / kTileKeys;
  return tiles >= (int64_t)kRotateQMinTiles * (int64_t)gp.tc_tiles.size();
}

// Orders a tile list for the persistent kernel, whose CTA j (of G = min(n,
// sms)) takes entries j, j + G, j + 2G, ...: largest items (by key tiles)
// first, dealt to the CTAs in rows of G that alternate in direction (a
// snake), so that a CTA that drew a large item in one row draws a small one
// in the next.  The last, partial row runs in ascending CTA order (CTAs
// 0 .. of it take an extra item), so the rows are oriented from there back.
constexpr int kBalanceItemsPerSm = 8;
void balance_tiles(std::vector<dbsa_tile_item> &tiles, int sms) {
  const int64_t n = (int64_t)tiles.size();
  const int64_t G = std::min<int64_t>(n, std::max(1, sms));
  if (G <= 1) return;
  auto key_tiles = [&](int64_t i) { return (tiles[i].len[0] + kTileKeys - 1) / kTileKeys; };
  std::vector<int64_t> order(n);
  for (int64_t i = 0; i < n; ++i) order[i] = i;
  std::stable_sort(order.begin(), order.end(),
                   [&](int64_t a, int64_t b) { return key_tiles(a) > key_tiles(b); });
  const int64_t last_row = (n - 1) / G;
  std::vector<dbsa_tile_item> sorted(n);
  for (int64_t k = 0; k < n; ++k) {
    const int64_t r = k / G, j = k % G;
    sorted[r * G + (((last_row - r) & 1) == 0 ? j : G - 1 - j)] = tiles[order[k]];
  }
  tiles.swap(sorted);
}

// Packed rows of the items: packed_items[k] owns rows [k R, (k + 1) R), and
// its query rows are rotated at (the query's token position - the item's
// p_begin); the other items (tails) have no packed rows.
void set_item_meta(GatherPlan &gp, int R, int32_t n_new, int32_t tail_len) {
  gp.item_meta.assign(gp.items.size(), make_int4(-1, 0, 0, 0));
  for (size_t k = 0; k < gp.packed_items.size(); ++k) {
    const int32_t i = gp.packed_items[k];
    const S2Item &it = gp.items[i];
    const int32_t pos0 = gp.queries[it.query].n_gathered + tail_len - n_new - it.p_begin;
    gp.item_meta[i] = make_int4((int32_t)(k * R), pos0, it.query, 0);
  }
}

dbsa_status gather_plan(const dbsa_config *cfg, const int32_t *offs, int32_t nb, int32_t nq,
                        const int32_t *sel_ptr, const int32_t *sel, int32_t n_new,
                        int32_t tail_len, GatherPlan &gp) {
  gp.nb = nb;
  gp.cache_rows = offs[nb];
  if (nq < 1) return fail(DBSA_ERR_INVALID_ARG, "nq must be >= 1");
  if (sel_ptr == nullptr || sel == nullptr) return fail(DBSA_ERR_INVALID_ARG, "selection is NULL");
  if (sel_ptr[0] != 0) return fail(DBSA_ERR_INVALID_ARG, "sel_ptr[0] must be 0");
  if (n_new < 1 || tail_len < n_new)
    return fail(DBSA_ERR_INVALID_ARG, "need 1 <= n_new <= tail_len (n_new=%d tail_len=%d)", n_new,
                tail_len);
  const int g = cfg->n_q_heads / cfg->n_kv_heads;
  const int R = g * n_new;
  std::vector<char> seen(nb, 0);
  gp.max_pos = 0;
  int64_t total_keys = 0;
  // capacity hints only (the loop below validates the selection); a valid
  // selection has at most nb blocks per query
  const size_t n_sel = (size_t)std::max<int64_t>(
      0, std::min<int64_t>(sel_ptr[nq], (int64_t)nq * nb));
  gp.queries.reserve(nq);
  gp.segs.reserve(n_sel);
  gp.items.reserve(n_sel + nq);
  for (int q = 0; q < nq; ++q) {
    const int32_t a = sel_ptr[q], e = sel_ptr[q + 1];
    if (e <= a) return fail(DBSA_ERR_INVALID_ARG, "query %d selects no block", q);
    // distinct blocks only, so at most nb: checked before sel is read
    if ((int64_t)e - a > nb)
      return fail(DBSA_ERR_INVALID_ARG, "query %d selects %lld blocks of %d", q,
                  (long long)e - a, nb);
    if (sel[a] != 0) return fail(DBSA_ERR_INVALID_ARG, "query %d: first block must be the sink (0)", q);
    S2Query qi;
    std::memset(&qi, 0, sizeof qi);
    qi.seg_begin = (int32_t)gp.segs.size();
    qi.n_seg = e - a;
    int64_t p = 0;
    for (int32_t i = a; i < e; ++i) {
      const int32_t b = sel[i];
      if (b < 0 || b >= nb) return fail(DBSA_ERR_INVALID_ARG, "query %d: block %d out of range", q, b);
      if (seen[b]) return fail(DBSA_ERR_INVALID_ARG, "query %d: block %d selected twice", q, b);
      seen[b] = 1;
      S2Segment s;
      s.cache_row0 = offs[b];
      s.pos0 = (int32_t)p;
      s.len = offs[b + 1] - offs[b];
      s.query = q;
      gp.segs.push_back(s);
      p += s.len;
    }
    for (int32_t i = a; i < e; ++i) seen[sel[i]] = 0;
    if (p + tail_len > (1 << 30)) return fail(DBSA_ERR_INVALID_ARG, "gathered context too long");
    qi.n_gathered = (int32_t)p;
    total_keys += p + tail_len;
    gp.max_pos = std::max<int32_t>(gp.max_pos, (int32_t)(p + tail_len));
    gp.queries.push_back(qi);
  }
  // Selections of short segments (a demonstration-granular gather: blocks of
  // one demonstration each) go per query when the block-major path's extra
  // traffic would outweigh the K/V it saves: it keeps one partial per (query,
  // segment) row and one packed query row per (query, segment, token, head),
  // each written and read once, and rotates every key of the cache, while
  // the per-query path streams every query's own gathered keys.  Passes with
  // few query tokens (decode steps) still share the keys across queries.
  int64_t gathered = 0;
  for (const auto &qi : gp.queries) gathered += qi.n_gathered;
  bool per_query = gathered < (int64_t)kTileKeys * (int64_t)gp.segs.size();
  if (per_query) {
    const double elt = cfg->dtype == DBSA_F32 ? 4.0 : 2.0;
    const double D = cfg->head_dim, Hkv = cfg->n_kv_heads;
    const double per_query_bytes = (double)(gathered + (int64_t)nq * tail_len) * Hkv * D * elt * 2;
    const double per_pair = (double)cfg->n_q_heads * n_new * ((2.0 * D + 8.0) * 2 + 2.0 * D * 2);
    const double block_bytes =
        (double)offs[nb] * Hkv * D * (2.0 * elt + 4.0) + (double)gp.segs.size() * per_pair;
    per_query = !(block_bytes < per_query_bytes);
  }
  if (per_query && R >= kCompactMinRows) {
    // Compact mode: one block item per query over its whole gathered sequence
    // (fresh positions 0 .. T'_q - 1, already applied to the compact keys, so
    // the query rows are rotated at their own positions) and one tail item.
    gp.compact = true;
    gp.compact_base.resize(nq);
    gp.packed_items.resize(nq);
    gp.run_items.reserve(nq);
    for (int q = 0; q < nq; ++q) {
      S2Query &qi = gp.queries[q];
      gp.compact_base[q] = (int32_t)gp.compact_rows;
      gp.compact_rows += qi.n_gathered;
      qi.item_begin = (int32_t)gp.items.size();
      S2Item it;
      it.query = q;
      it.p_begin = 0;
      it.p_end = qi.n_gathered;
      it.p_lo = 0;
      gp.packed_items[q] = (int32_t)gp.items.size();
      gp.items.push_back(it);
      S2Item tail;
      tail.query = q;
      tail.p_begin = qi.n_gathered & ~(kRopeLo - 1);
      tail.p_end = qi.n_gathered + tail_len;
      tail.p_lo = qi.n_gathered;
      gp.run_items.push_back((int32_t)gp.items.size());
      gp.items.push_back(tail);
      qi.n_items = 2;
    }
    if (gp.compact_rows > (1 << 30))
      return fail(DBSA_ERR_INVALID_ARG, "gathered contexts of the batch too long");
    set_item_meta(gp, R, n_new, tail_len);
    gp.tc_rows = nq * R;
    gp.tc_tiles.reserve((size_t)cfg->n_kv_heads * nq * ((R + kTileRows - 1) / kTileRows));
    for (int c = 0; c < cfg->n_kv_heads; ++c)
      for (int q = 0; q < nq; ++q)
        for (int m = 0; m < R; m += kTileRows) {
          dbsa_tile_item t;
          std::memset(&t, 0, sizeof t);
          t.head = c;
          t.q_row0 = q * R + m;
          t.q_pos0 = 1 << 30;  // after every gathered key: no causal limit
          t.n_rows = std::min(kTileRows, R - m);
          t.n_ranges = 1;
          t.block = q;
          t.k_row0[0] = gp.compact_base[q];
          t.v_row0[0] = gp.compact_base[q];
          t.pos0[0] = 0;
          t.len[0] = gp.queries[q].n_gathered;
          gp.tc_tiles.push_back(t);
        }
    return DBSA_OK;
  }
  if (per_query) {
    gp.per_query = true;
    // Split size: >= 33 keys per query row of a CTA (bounds the partial
    // traffic to ~3 % of the K/V bytes) and enough CTAs for ~4 waves.  Rows
    // per CTA follow the per-query kernel's shape table.
    constexpr int kSplitKeys = 64;
    const int rows_cta = (R <= 16) ? 16 : (R <= 32) ? 32 : (R <= 64) ? 64 : (R <= 128) ? 128 : 160;
    const int zdim = (R + rows_cta - 1) / rows_cta;
    const int64_t min_chunk = std::max<int64_t>(256, (int64_t)33 * std::min(R, rows_cta));
    const int64_t want_ctas = (int64_t)4 * num_sms();
    const int64_t par_chunk =
        (total_keys * cfg->n_kv_heads * zdim + want_ctas - 1) / std::max<int64_t>(1, want_ctas);
    int64_t chunk = std::max(min_chunk, par_chunk);
    chunk = (chunk + kSplitKeys - 1) / kSplitKeys * kSplitKeys;
    for (int q = 0; q < nq; ++q) {
      S2Query &qi = gp.queries[q];
      const int64_t K = (int64_t)qi.n_gathered + tail_len;
      const int64_t n_split = std::max<int64_t>(1, (K + chunk - 1) / chunk);
      int64_t per = (K + n_split - 1) / n_split;
      per = (per + kSplitKeys - 1) / kSplitKeys * kSplitKeys;
      qi.item_begin = (int32_t)gp.items.size();
      for (int64_t s0 = 0; s0 < K; s0 += per) {
        S2Item it;
        it.query = q;
        it.p_begin = (int32_t)s0;
        it.p_end = (int32_t)std::min<int64_t>(K, s0 + per);
        it.p_lo = it.p_begin;
        gp.run_items.push_back((int32_t)gp.items.size());
        gp.items.push_back(it);
      }
      qi.n_items = (int32_t)gp.items.size() - qi.item_begin;
    }
    return DBSA_OK;
  }
  {
    // Block-major on the tensor core.  Items per query = one
    // per selected block + one for its own tail tokens (per-query kernel);
    // the rows of the block items are packed block by block (queries in
    // order, token-major rows within an item) and cut into 128-row tiles
    // that all read the same block of rotated keys, so a block selected by
    // many queries is read and rotated once per pass.
    // items selecting each block, in query order: a counting sort by block
    std::vector<int32_t> block_begin(nb + 1, 0);
    for (int32_t i = 0; i < sel_ptr[nq]; ++i) ++block_begin[sel[i] + 1];
    for (int b = 0; b < nb; ++b) block_begin[b + 1] += block_begin[b];
    std::vector<int32_t> fill(block_begin.begin(), block_begin.end() - 1);
    gp.packed_items.resize(sel_ptr[nq]);
    gp.run_items.reserve(nq);
    for (int q = 0; q < nq; ++q) {
      S2Query &qi = gp.queries[q];
      qi.item_begin = (int32_t)gp.items.size();
      for (int sgi = 0; sgi < qi.n_seg; ++sgi) {
        const S2Segment &sg = gp.segs[qi.seg_begin + sgi];
        S2Item it;
        it.query = q;
        it.p_begin = sg.pos0;  // the block's fresh start P
        it.p_end = sg.pos0 + sg.len;
        it.p_lo = sg.pos0;
        gp.packed_items[fill[sel[sel_ptr[q] + sgi]]++] = (int32_t)gp.items.size();
        gp.items.push_back(it);
      }
      S2Item tail;
      tail.query = q;
      tail.p_begin = qi.n_gathered & ~(kRopeLo - 1);
      tail.p_end = qi.n_gathered + tail_len;
      tail.p_lo = qi.n_gathered;
      gp.run_items.push_back((int32_t)gp.items.size());
      gp.items.push_back(tail);
      qi.n_items = (int32_t)gp.items.size() - qi.item_begin;
    }
    // rows packed block by block: packed_items[k] owns rows [k R, (k + 1) R)
    set_item_meta(gp, R, n_new, tail_len);
    gp.tc_rows = (int32_t)(gp.packed_items.size() * R);
    std::vector<int32_t> block_row0(nb, 0), block_rows(nb, 0);
    size_t n_tiles = 0;
    for (int b = 0; b < nb; ++b) {
      block_row0[b] = block_begin[b] * R;
      block_rows[b] = (block_begin[b + 1] - block_begin[b]) * R;
      n_tiles += (block_rows[b] + kTileRows - 1) / kTileRows;
    }
    gp.tc_tiles.reserve(n_tiles * cfg->n_kv_heads);
    for (int c = 0; c < cfg->n_kv_heads; ++c)
      for (int b = 0; b < nb; ++b)
        for (int m = 0; m < block_rows[b]; m += kTileRows) {
          dbsa_tile_item t;
          std::memset(&t, 0, sizeof t);
          t.head = c;
          t.q_row0 = block_row0[b] + m;
          t.q_pos0 = 1 << 30;  // after every gathered key: no causal limit
          t.n_rows = std::min(kTileRows, block_rows[b] - m);
          t.n_ranges = 1;
          t.block = b;
          t.k_row0[0] = offs[b];
          t.v_row0[0] = offs[b];
          t.pos0[0] = 0;
          t.len[0] = offs[b + 1] - offs[b];
          gp.tc_tiles.push_back(t);
        }
    // A pass with a few items per SM (a decode step: one 128-row tile per (KV
    // head, block)) is ordered for the persistent kernel's balance; longer
    // lists keep the order in which the row tiles of one block run together
    // (their K/V tiles are then read from L2).
    if ((int64_t)gp.tc_tiles.size() < (int64_t)kBalanceItemsPerSm * num_sms())
      balance_tiles(gp.tc_tiles, num_sms());
  }
  return DBSA_OK;
}

// -------------------------------------------------------------- workspace layouts
struct S1Layout {
  size_t rope, items, k_rot, v_bf16, total;
  int32_t n_hi;
};
S1Layout s1_layout(const dbsa_config *cfg, int64_t max_pos, int64_t n_items, int64_t k_rows) {
  S1Layout l;
  Carve cv;
  l.n_hi = (int32_t)(std::max<int64_t>(max_pos - 1, 0) / kRopeLo + 1);
  l.rope = cv.take(rope_table_bytes(l.n_hi, cfg->head_dim));
  l.items = cv.take((size_t)n_items * sizeof(dbsa_tile_item));
  l.k_rot = cv.take((size_t)cfg->n_kv_heads * k_rows * cfg->head_dim * 2);
  l.v_bf16 = cfg->dtype == DBSA_F32 ? cv.take((size_t)cfg->n_kv_heads * k_rows * cfg->head_dim * 2)
                                    : 0;
  l.total = cv.total();
  return l;
}

struct S2Layout {
  size_t rope, queries, packed_items, item_meta, tc_tiles, offs, compact_base, core_end, segs,
      items, run_items, blob_end, q_rot_pos, k_hat, v_hat, q_hat, part_acc, part_ml, total;
  int32_t n_hi;
};
// prepared: the block-relative keys (and bf16 V of fp32 caches) come from a
// dbsa_block_keys() buffer instead of the workspace.
S2Layout s2_layout(const dbsa_config *cfg, const GatherPlan &gp, int32_t n_new,
                   bool prepared = false) {
  S2Layout l;
  Carve cv;
  l.n_hi = (int32_t)(std::max<int64_t>(gp.max_pos - 1, 0) / kRopeLo + 1);
  l.rope = cv.take(rope_table_bytes(l.n_hi, cfg->head_dim));
  // the plan tables, uploaded as one blob: first those every mode reads,
  // then those only the per-query kernel, the compact gather and the gather
  // map read (a decode step's block-major pass needs none of them)
  l.queries = cv.take(gp.queries.size() * sizeof(S2Query));
  l.packed_items = cv.take(gp.packed_items.size() * sizeof(int32_t));
  l.item_meta = cv.take(gp.item_meta.size() * sizeof(int4));
  l.tc_tiles = cv.take(gp.tc_tiles.size() * sizeof(dbsa_tile_item));
  l.offs = cv.take((size_t)(offs_count(gp)) * sizeof(int32_t));
  l.compact_base = cv.take(gp.compact_base.size() * sizeof(int32_t));
  l.core_end = cv.take(0);
  l.segs = cv.take(gp.segs.size() * sizeof(S2Segment));
  l.items = cv.take(gp.items.size() * sizeof(S2Item));
  l.run_items = cv.take(gp.run_items.size() * sizeof(int32_t));
  l.blob_end = cv.take(0);
  // rows packed by qhat_kernel (passes of short items only)
  const bool packs_q = !gp.per_query && !rotates_q(gp);
  l.q_rot_pos = cv.take(packs_q ? gp.items.size() * sizeof(int32_t) : 0);
  const int64_t T = gp.cache_rows;
  if (gp.compact) {
    // every query's gathered keys (rotated) and values, bf16 [Hkv][rows][D]
    l.k_hat = cv.take((size_t)cfg->n_kv_heads * gp.compact_rows * cfg->head_dim * 2);
    l.v_hat = cv.take((size_t)cfg->n_kv_heads * gp.compact_rows * cfg->head_dim * 2);
  } else {
    const bool own_keys = !prepared && !gp.per_query;
    l.k_hat = cv.take(own_keys ? (size_t)cfg->n_kv_heads * T * cfg->head_dim * 2 : 0);
    l.v_hat = cv.take(own_keys && cfg->dtype == DBSA_F32
                          ? (size_t)cfg->n_kv_heads * T * cfg->head_dim * 2
                          : 0);
  }
  l.q_hat = cv.take(packs_q ? (size_t)cfg->n_kv_heads * gp.tc_rows * cfg->head_dim * 2 : 0);
  const size_t rows = gp.items.size() * (size_t)cfg->n_q_heads * n_new;
  l.part_acc = cv.take(rows * cfg->head_dim * sizeof(uint16_t));
  l.part_ml = cv.take(rows * sizeof(float2));
  l.total = cv.total();
  return l;
}

// dbsa_block_keys() buffer: status word, RoPE tables for positions inside a
// block, the offset table, K-hat [Hkv][T][D] bf16 and (fp32 caches) bf16 V.
struct BKLayout {
  size_t rope, offs, k_hat, v_hat, total;
  int32_t n_hi;
};
// The block-keys tables also cover every position a gather from the same
// cache reaches with up to this many tail tokens (a query's gathered length is
// at most T), so a prepared gather reads them instead of building its own.
constexpr int64_t kBlockKeysTailPositions = 8192;

BKLayout bk_layout(const dbsa_config *cfg, const int32_t *offs, int32_t nb) {
  BKLayout l;
  Carve cv;
  const int64_t T = offs[nb];
  l.n_hi = (int32_t)((T + kBlockKeysTailPositions - 1) / kRopeLo + 1);
  l.rope = cv.take(rope_table_bytes(l.n_hi, cfg->head_dim));
  l.offs = cv.take((size_t)(nb + 1) * sizeof(int32_t));
  l.k_hat = cv.take((size_t)cfg->n_kv_heads * T * cfg->head_dim * 2);
  l.v_hat = cv.take(cfg->dtype == DBSA_F32 ? (size_t)cfg->n_kv_heads * T * cfg->head_dim * 2 : 0);
  l.total = cv.total();
  return l;
}

dbsa_status check_ws(void *ws, size_t ws_bytes, size_t need) {
  if (ws == nullptr) return fail(DBSA_ERR_WORKSPACE, "workspace is NULL");
  if ((reinterpret_cast<uintptr_t>(ws) & 255u) != 0)
    return fail(DBSA_ERR_WORKSPACE, "workspace must be 256-byte aligned");
  if (ws_bytes < need)
    return fail(DBSA_ERR_WORKSPACE, "workspace too small: %zu < %zu bytes", ws_bytes, need);
  return DBSA_OK;
}

template <typename T>
T *at(void *ws, size_t off) {
  return reinterpret_cast<T *>(static_cast<uint8_t *>(ws) + off);
}

// Builds the RoPE tables at `off` in the workspace (enqueued) and returns them.
cudaError_t build_tables(void *ws, size_t off, int32_t n_hi, const dbsa_config *cfg,
                         cudaStream_t st, RopeTables *out) {
  float *base = at<float>(ws, off);
  *out = rope_tables_at(base, n_hi, cfg->head_dim);
  return launch_rope_tables(base, n_hi, cfg->head_dim, cfg->rope_theta, st);
}

int64_t encode_item_bound(const dbsa_config *cfg, int64_t T, int32_t nb) {
  return (int64_t)cfg->n_q_heads * ((T + kTileRows - 1) / kTileRows + nb);
}

}  // namespace

void dbsa::set_last_error(const char *msg) { g_err = msg; }

// ============================================================== public ABI
extern "C" {

const char *dbsa_version(void) { return "dbsa-b200 0.1 (sm_100a)"; }

const char *dbsa_last_error(void) { return g_err.c_str(); }

int64_t dbsa_kernel_launches(void) { return g_launches.load(std::memory_order_relaxed); }

void dbsa_test_wait_expiry(uint64_t limit_ns) { g_wait_expiry_ns = limit_ns; }

void dbsa_set_profile_events(void *start, void *stop) {
  g_prof_start = static_cast<cudaEvent_t>(start);
  g_prof_stop = static_cast<cudaEvent_t>(stop);
}

int32_t dbsa_group_blocks(const int32_t *demo_len, int32_t n_demos, int32_t k, int32_t *offs_out) {
  if (demo_len == nullptr || offs_out == nullptr || n_demos <= 0 || k <= 0) {
    fail(DBSA_ERR_INVALID_ARG, "group_blocks: bad arguments");
    return -1;
  }
  const int32_t nb = (n_demos + k - 1) / k;
  int64_t acc = 0;
  offs_out[0] = 0;
  for (int32_t i = 0; i < n_demos; ++i) {
    if (demo_len[i] < 1) {
      fail(DBSA_ERR_INVALID_ARG, "group_blocks: demonstration %d has no tokens", i);
      return -1;
    }
    acc += demo_len[i];
    if (acc > (1 << 30)) {
      fail(DBSA_ERR_INVALID_ARG, "group_blocks: context too long");
      return -1;
    }
    if ((i + 1) % k == 0 || i + 1 == n_demos) offs_out[(i + k) / k] = (int32_t)acc;
  }
  return nb;
}

int64_t dbsa_stage1_plan(const dbsa_config *cfg, const int32_t *offs_host, int32_t nb,
                         dbsa_tile_item *items, int64_t max_items) {
  if (check_cfg(cfg) != DBSA_OK || check_offs(offs_host, nb) != DBSA_OK) return -1;
  std::vector<dbsa_tile_item> v;
  encode_items(cfg, offs_host, nb, v);
  if (items != nullptr)
    std::memcpy(items, v.data(), sizeof(dbsa_tile_item) * (size_t)std::min<int64_t>(max_items, v.size()));
  return (int64_t)v.size();
}

int64_t dbsa_stage1_tile_count(const dbsa_config *cfg, const int32_t *offs_host, int32_t nb) {
  if (check_cfg(cfg) != DBSA_OK || check_offs(offs_host, nb) != DBSA_OK) return -1;
  std::vector<dbsa_tile_item> v;
  encode_items(cfg, offs_host, nb, v);
  int64_t n = 0;
  for (const auto &it : v) n += tiles_of(it);
  return n;
}

size_t dbsa_encode_workspace_size(const dbsa_config *cfg, int64_t n_tokens, int32_t nb) {
  if (check_cfg(cfg) != DBSA_OK || n_tokens <= 0 || nb <= 0) return 0;
  return s1_layout(cfg, n_tokens, encode_item_bound(cfg, n_tokens, nb), n_tokens).total;
}

dbsa_status dbsa_encode_blocks(const dbsa_config *cfg, const void *q, const void *k,
                               const void *v, const int32_t *offs_host, int32_t nb,
                               void *k_cache, void *v_cache, int64_t cap, void *out,
                               void *workspace, size_t ws_bytes, void *stream) {
  const uint64_t wait_expiry = take_wait_expiry();
  dbsa_status s = check_cfg(cfg);
  if (s != DBSA_OK) return s;
  if ((s = check_offs(offs_host, nb)) != DBSA_OK) return s;
  if (!q || !k || !v || !k_cache || !v_cache || !out)
    return fail(DBSA_ERR_INVALID_ARG, "a tensor pointer is NULL");
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(k_cache) ||
      !aligned16(v_cache) || !aligned16(out))
    return fail(DBSA_ERR_INVALID_ARG, "tensor pointers must be 16-byte aligned");
  const int64_t T = offs_host[nb];
  if (cap < T) return fail(DBSA_ERR_CAPACITY, "cache capacity %lld < %lld tokens", (long long)cap,
                           (long long)T);
  std::vector<dbsa_tile_item> items;
  encode_items(cfg, offs_host, nb, items);
  const S1Layout L = s1_layout(cfg, T, encode_item_bound(cfg, T, nb), T);
  if ((s = check_ws(workspace, ws_bytes, L.total)) != DBSA_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const bool f32 = cfg->dtype == DBSA_F32;
  cudaError_t e;
  RopeTables rope;
  if ((e = build_tables(workspace, L.rope, L.n_hi, cfg, st, &rope)) != cudaSuccess)
    return cuda_fail(e, "rope tables");
  count_launches(1);
  // the upload kernel also clears the status word
  if ((e = upload_async(at<void>(workspace, L.items), items.data(),
                        items.size() * sizeof(dbsa_tile_item), st, workspace)) != cudaSuccess)
    return cuda_fail(e, "tile list upload");
  IngestArgs ia{};
  ia.k = k;
  ia.v = v;
  ia.n_tok = (int32_t)T;
  ia.pos0 = 0;
  ia.Hkv = cfg->n_kv_heads;
  ia.k_rot = at<void>(workspace, L.k_rot);
  ia.k_rows = T;
  ia.k_row_base = 0;
  ia.v_bf16 = f32 ? at<void>(workspace, L.v_bf16) : nullptr;
  ia.k_cache = k_cache;
  ia.v_cache = v_cache;
  ia.cap = cap;
  ia.rope = rope;
  if ((e = launch_ingest(ia, cfg->head_dim, f32, st)) != cudaSuccess) return cuda_fail(e, "ingest");
  count_launches(1);
  Stage1Args sa{};
  sa.q_src = q;
  sa.q_f32 = f32;
  sa.q_heads = cfg->n_q_heads;
  sa.rope = rope;
  sa.k_rot = ia.k_rot;
  sa.k_rows = T;
  sa.v = f32 ? ia.v_bf16 : v_cache;
  sa.v_rows = T;
  sa.v_head_stride = f32 ? T : cap;
  sa.out = out;
  sa.Hq = cfg->n_q_heads;
  sa.Hkv = cfg->n_kv_heads;
  sa.items = at<dbsa_tile_item>(workspace, L.items);
  sa.n_items = (int32_t)items.size();
  sa.scale_log2 = scale_log2(cfg);
  sa.status = at<int>(workspace, 0);
  sa.wait_limit_ns = wait_expiry;
  sa.withhold_tiles = wait_expiry != 0;
  {
    ProfileScope prof(st);
    e = launch_stage1(sa, cfg->head_dim, f32, num_sms(), st);
  }
  if (e != cudaSuccess) return cuda_fail(e, "stage-1 attention");
  count_launches(1);
  return DBSA_OK;
}

size_t dbsa_append_workspace_size(const dbsa_config *cfg, const int32_t *offs_host, int32_t nb,
                                  int32_t L) {
  if (check_cfg(cfg) != DBSA_OK || check_offs(offs_host, nb) != DBSA_OK || L < 1) return 0;
  const AppendPlan ap = append_plan(cfg, offs_host, nb, L);
  const int64_t n_items = (int64_t)cfg->n_q_heads * ((L + kTileRows - 1) / kTileRows);
  return s1_layout(cfg, (int64_t)offs_host[nb] + L, n_items, ap.k_rows).total;
}

dbsa_status dbsa_append_block(const dbsa_config *cfg, const void *q, const void *k, const void *v,
                              int32_t L, const int32_t *offs_host, int32_t nb, void *k_cache,
                              void *v_cache, int64_t cap, void *out, void *workspace,
                              size_t ws_bytes, void *stream) {
  const uint64_t wait_expiry = take_wait_expiry();
  dbsa_status s = check_cfg(cfg);
  if (s != DBSA_OK) return s;
  if ((s = check_offs(offs_host, nb)) != DBSA_OK) return s;
  if (L < 1) return fail(DBSA_ERR_INVALID_ARG, "the new block needs at least one token");
  if (!q || !k || !v || !k_cache || !v_cache || !out)
    return fail(DBSA_ERR_INVALID_ARG, "a tensor pointer is NULL");
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(k_cache) ||
      !aligned16(v_cache) || !aligned16(out))
    return fail(DBSA_ERR_INVALID_ARG, "tensor pointers must be 16-byte aligned");
  const int64_t T0 = offs_host[nb];
  if (T0 + L > (1 << 30)) return fail(DBSA_ERR_INVALID_ARG, "context too long");
  if (cap < T0 + L)
    return fail(DBSA_ERR_CAPACITY, "cache capacity %lld < %lld tokens", (long long)cap,
                (long long)(T0 + L));
  const AppendPlan ap = append_plan(cfg, offs_host, nb, L);
  const bool f32 = cfg->dtype == DBSA_F32;
  std::vector<dbsa_tile_item> items;
  {
    int32_t krow[2] = {ap.cs[0], ap.cs[1]};
    int32_t vrow[2];
    for (int r = 0; r < 2; ++r) vrow[r] = f32 ? ap.cs[r] : ap.rs[r];
    block_items(cfg, ap.offs.data(), nb, (int32_t)T0, krow, vrow, ap.nr, ap.rs, ap.re, items);
  }
  const int64_t n_items_bound = (int64_t)cfg->n_q_heads * ((L + kTileRows - 1) / kTileRows);
  const S1Layout Ly = s1_layout(cfg, T0 + L, n_items_bound, ap.k_rows);
  if ((s = check_ws(workspace, ws_bytes, Ly.total)) != DBSA_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e;
  RopeTables rope;
  if ((e = build_tables(workspace, Ly.rope, Ly.n_hi, cfg, st, &rope)) != cudaSuccess)
    return cuda_fail(e, "rope tables");
  count_launches(1);
  // the upload kernel also clears the status word
  if ((e = upload_async(at<void>(workspace, Ly.items), items.data(),
                        items.size() * sizeof(dbsa_tile_item), st, workspace)) != cudaSuccess)
    return cuda_fail(e, "tile list upload");
  void *k_rot = at<void>(workspace, Ly.k_rot);
  void *v_bf16 = f32 ? at<void>(workspace, Ly.v_bf16) : nullptr;
  // window rows already in the cache
  for (int r = 0; r < ap.nr; ++r) {
    const int32_t e_in_cache = std::min<int32_t>(ap.re[r], (int32_t)T0);
    if (e_in_cache <= ap.rs[r]) continue;
    WindowArgs wa{};
    wa.k_cache = k_cache;
    wa.v_cache = v_cache;
    wa.cap = cap;
    wa.Hkv = cfg->n_kv_heads;
    wa.row0 = ap.rs[r];
    wa.n = e_in_cache - ap.rs[r];
    wa.k_rot = k_rot;
    wa.k_rows = ap.k_rows;
    wa.dst_row0 = ap.cs[r];
    wa.v_bf16 = v_bf16;
    wa.rope = rope;
    if ((e = launch_window(wa, cfg->head_dim, f32, st)) != cudaSuccess)
      return cuda_fail(e, "window rotation");
    count_launches(1);
  }
  IngestArgs ia{};
  ia.k = k;
  ia.v = v;
  ia.n_tok = L;
  ia.pos0 = (int32_t)T0;
  ia.Hkv = cfg->n_kv_heads;
  ia.k_rot = k_rot;
  ia.k_rows = ap.k_rows;
  ia.k_row_base = ap.new_row;
  ia.v_bf16 = v_bf16;
  ia.k_cache = k_cache;
  ia.v_cache = v_cache;
  ia.cap = cap;
  ia.rope = rope;
  if ((e = launch_ingest(ia, cfg->head_dim, f32, st)) != cudaSuccess) return cuda_fail(e, "ingest");
  count_launches(1);
  Stage1Args sa{};
  sa.q_src = q;
  sa.q_f32 = f32;
  sa.q_heads = cfg->n_q_heads;
  sa.rope = rope;
  sa.k_rot = k_rot;
  sa.k_rows = ap.k_rows;
  sa.v = f32 ? v_bf16 : v_cache;
  sa.v_rows = f32 ? ap.k_rows : T0 + L;
  sa.v_head_stride = f32 ? ap.k_rows : cap;
  sa.out = out;
  sa.Hq = cfg->n_q_heads;
  sa.Hkv = cfg->n_kv_heads;
  sa.items = at<dbsa_tile_item>(workspace, Ly.items);
  sa.n_items = (int32_t)items.size();
  sa.scale_log2 = scale_log2(cfg);
  sa.status = at<int>(workspace, 0);
  sa.wait_limit_ns = wait_expiry;
  sa.withhold_tiles = wait_expiry != 0;
  {
    ProfileScope prof(st);
    e = launch_stage1(sa, cfg->head_dim, f32, num_sms(), st);
  }
  if (e != cudaSuccess) return cuda_fail(e, "stage-1 attention");
  count_launches(1);
  return DBSA_OK;
}

size_t dbsa_gather_workspace_size(const dbsa_config *cfg, const int32_t *offs_host, int32_t nb,
                                  int32_t nq, const int32_t *sel_ptr_host,
                                  const int32_t *sel_blocks_host, int32_t n_new,
                                  int32_t tail_len) {
  if (check_cfg(cfg) != DBSA_OK || check_offs(offs_host, nb) != DBSA_OK) return 0;
  GatherPlan gp;
  if (gather_plan(cfg, offs_host, nb, nq, sel_ptr_host, sel_blocks_host, n_new, tail_len, gp) !=
      DBSA_OK)
    return 0;
  return s2_layout(cfg, gp, n_new).total;
}

}  // extern "C"

namespace {

// Stage 2 behind both entry points; block_keys = null rotates the cache keys
// at block-relative positions into the workspace, else takes them from a
// dbsa_block_keys() buffer.
// The last gather plan built on this thread, with the inputs it came from.
// The layers of one prompt pass or decode step share the cache layout, the
// selection and the pass shape, so every layer after the first reuses it.
struct PlanCache {
  std::vector<int32_t> key;
  GatherPlan gp;
  bool valid = false;
};

// The plan inputs as one array (configuration fields, sizes, offsets and the
// selection); false if sel_ptr is not a well-formed CSR pointer array, in which
// case the caller plans afresh (and reports the error).
bool plan_key(const dbsa_config *cfg, const int32_t *offs, int32_t nb, int32_t nq,
              const int32_t *sel_ptr, const int32_t *sel, int32_t n_new, int32_t tail_len,
              std::vector<int32_t> &key) {
  if (nq < 1 || sel_ptr == nullptr || sel == nullptr || sel_ptr[0] != 0) return false;
  for (int32_t q = 0; q < nq; ++q)
    if (sel_ptr[q + 1] <= sel_ptr[q]) return false;
  if ((int64_t)sel_ptr[nq] > (int64_t)nq * nb) return false;
  const int32_t head[] = {cfg->n_q_heads, cfg->n_kv_heads, cfg->head_dim, (int32_t)cfg->dtype,
                          cfg->window_j, cfg->pattern, num_sms(), nb, nq, n_new, tail_len};
  key.clear();
  key.reserve(sizeof head / sizeof head[0] + (size_t)nb + 1 + (size_t)nq + 1 + sel_ptr[nq]);
  key.insert(key.end(), head, head + sizeof head / sizeof head[0]);
  key.insert(key.end(), offs, offs + nb + 1);
  key.insert(key.end(), sel_ptr, sel_ptr + nq + 1);
  key.insert(key.end(), sel, sel + sel_ptr[nq]);
  return true;
}

// The query rows of a partial-mode tensor-core pass.  Passes of long items
// hand the kernel the unrotated q_new (it rotates the packed rows itself);
// passes of short items run qhat_kernel first (recording, when a gather map
// is requested, the position each item's token 0 was rotated at) and the
// kernel loads the packed rows by TMA.
cudaError_t set_query_rows(Stage1Args &sa, const dbsa_config *cfg, const GatherPlan &gp,
                           const S2Layout &L, const void *q_new, int32_t n_new, int32_t tail_len,
                           int32_t n_items, const RopeTables &rope, void *workspace,
                           const int32_t *dbg_map, cudaStream_t st) {
  const bool f32 = cfg->dtype == DBSA_F32;
  sa.part.item_meta = at<int4>(workspace, L.item_meta);
  if (rotates_q(gp)) {
    sa.q_src = q_new;
    sa.q_f32 = f32;
    sa.q_heads = cfg->n_q_heads;
    sa.rope = rope;
    return cudaSuccess;
  }
  QHatArgs qa{};
  qa.q_new = q_new;
  qa.n_new = n_new;
  qa.tail_len = tail_len;
  qa.Hq = cfg->n_q_heads;
  qa.Hkv = cfg->n_kv_heads;
  qa.n_items = n_items;
  qa.item_meta = sa.part.item_meta;
  qa.rows = gp.tc_rows;
  qa.q_hat = at<void>(workspace, L.q_hat);
  qa.q_rot_pos = dbg_map != nullptr ? at<int32_t>(workspace, L.q_rot_pos) : nullptr;
  qa.rope = rope;
  cudaError_t e = launch_qhat(qa, cfg->head_dim, f32, st);
  if (e != cudaSuccess) return e;
  count_launches(1);
  sa.q_rot = qa.q_hat;
  sa.q_rows = gp.tc_rows;
  sa.part.q_rot_pos = qa.q_rot_pos;
  return cudaSuccess;
}

dbsa_status gather_impl(const dbsa_config *cfg, const void *k_cache, const void *v_cache,
                        int64_t cap, const int32_t *offs_host, int32_t nb, int32_t nq,
                        const int32_t *sel_ptr_host, const int32_t *sel_blocks_host,
                        const void *q_new, int32_t n_new, const void *k_tail, const void *v_tail,
                        int32_t tail_len, int32_t tail_cap, void *out, int32_t *dbg_map,
                        int64_t dbg_cap, const void *block_keys, size_t bk_bytes, void *workspace,
                        size_t ws_bytes, void *stream, const FixedScratch *fixed = nullptr) {
  const uint64_t wait_expiry = take_wait_expiry();
  dbsa_status s = check_cfg(cfg);
  if (s != DBSA_OK) return s;
  if ((s = check_offs(offs_host, nb)) != DBSA_OK) return s;
  if (!k_cache || !v_cache || !q_new || !k_tail || !v_tail || !out)
    return fail(DBSA_ERR_INVALID_ARG, "a tensor pointer is NULL");
  if (!aligned16(k_cache) || !aligned16(v_cache) || !aligned16(q_new) || !aligned16(k_tail) ||
      !aligned16(v_tail) || !aligned16(out))
    return fail(DBSA_ERR_INVALID_ARG, "tensor pointers must be 16-byte aligned");
  if (tail_len > tail_cap)
    return fail(DBSA_ERR_INVALID_ARG, "tail_len %d > tail_cap %d", tail_len, tail_cap);
  if (offs_host[nb] > cap)
    return fail(DBSA_ERR_CAPACITY, "offsets reach %d rows but cap is %lld", offs_host[nb],
                (long long)cap);
  static thread_local PlanCache cache;
  static thread_local std::vector<int32_t> key;
  const bool keyed = plan_key(cfg, offs_host, nb, nq, sel_ptr_host, sel_blocks_host, n_new,
                              tail_len, key);
  if (!(keyed && cache.valid && key == cache.key)) {
    cache.valid = false;
    cache.gp = GatherPlan();
    if ((s = gather_plan(cfg, offs_host, nb, nq, sel_ptr_host, sel_blocks_host, n_new, tail_len,
                         cache.gp)) != DBSA_OK)
      return s;
    if (keyed) {
      cache.key.swap(key);
      cache.valid = true;
    }
  }
  const GatherPlan &gp = cache.gp;
  if (dbg_map != nullptr) {
    if ((reinterpret_cast<uintptr_t>(dbg_map) & 7u) != 0)
      return fail(DBSA_ERR_INVALID_ARG, "dbg_map must be 8-byte aligned");
    for (const auto &qi : gp.queries)
      if (qi.n_gathered > dbg_cap)
        return fail(DBSA_ERR_INVALID_ARG, "dbg_cap %lld < gathered tokens %d", (long long)dbg_cap,
                    qi.n_gathered);
  }
  const bool prepared = block_keys != nullptr;
  const S2Layout L = s2_layout(cfg, gp, n_new, prepared);
  if (fixed != nullptr) {
    // the no-allocation entry point: its fixed scratch, resolved only now
    // that the call has been validated and planned
    if (L.total > fixed->bytes)
      return fail(DBSA_ERR_WORKSPACE,
                  "dbsa_gather_rope_attend_noalloc: this batch needs %zu bytes of scratch but the "
                  "entry point holds %zu; use dbsa_gather_rope_attend with a workspace or split "
                  "the batch",
                  L.total, fixed->bytes);
    cudaError_t re = fixed->resolve(&workspace);
    if (re != cudaSuccess) return cuda_fail(re, "dbsa_gather_rope_attend_noalloc: scratch address");
    ws_bytes = fixed->bytes;
  }
  if ((s = check_ws(workspace, ws_bytes, L.total)) != DBSA_OK) return s;
  BKLayout B{};
  if (prepared) {
    B = bk_layout(cfg, offs_host, nb);
    if ((reinterpret_cast<uintptr_t>(block_keys) & 255u) != 0)
      return fail(DBSA_ERR_WORKSPACE, "block_keys must be 256-byte aligned");
    if (bk_bytes < B.total)
      return fail(DBSA_ERR_WORKSPACE, "block_keys too small: %zu < %zu bytes", bk_bytes, B.total);
  }
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e;
  // the status word: cleared here for the plain-copy upload of a fixed
  // scratch, else by the staging upload's kernel below
  if (fixed != nullptr && (e = cudaMemsetAsync(workspace, 0, kStatusBytes, st)) != cudaSuccess)
    return cuda_fail(e, "status clear");
  RopeTables rope;
  if (prepared && B.n_hi >= L.n_hi) {
    // the block-keys tables cover this call's positions (same rows, same values)
    rope = rope_tables_at(at<float>(const_cast<void *>(block_keys), B.rope), B.n_hi,
                          cfg->head_dim);
  } else {
    if ((e = build_tables(workspace, L.rope, L.n_hi, cfg, st, &rope)) != cudaSuccess)
      return cuda_fail(e, "rope tables");
    count_launches(1);
  }
  // one upload of the three small plan arrays (they are contiguous in the carve)
  {
    // the tables, laid out as in the workspace, written straight into staging
    // (the no-allocation entry point: into a host vector, then one
    // cudaMemcpyAsync from that pageable memory, which returns once the
    // driver has taken the bytes)
    // a block-major pass whose tails run in the tail-and-merge kernel, with
    // no gather map requested, reads none of the segment, item and run-item
    // tables: they stay on the host
    const bool block_major = !gp.per_query && !gp.compact;
    const bool tail_merge = (cfg->n_q_heads / cfg->n_kv_heads) * n_new <= kTailMergeMaxRows;
    const bool core_only = block_major && tail_merge && dbg_map == nullptr;
    const size_t blob_bytes = (core_only ? L.core_end : L.blob_end) - L.queries;
    static thread_local std::vector<uint8_t> plain;
    uint8_t *blob = nullptr;
    if (fixed != nullptr) {
      if (plain.size() < blob_bytes) plain.resize(blob_bytes);
      blob = plain.data();
    } else if ((e = staging_ring().stage(blob_bytes, reinterpret_cast<void **>(&blob))) !=
               cudaSuccess) {
      return cuda_fail(e, "gather plan staging");
    }
    std::memcpy(blob, gp.queries.data(), gp.queries.size() * sizeof(S2Query));
    if (!core_only) {
      std::memcpy(blob + (L.segs - L.queries), gp.segs.data(),
                  gp.segs.size() * sizeof(S2Segment));
      std::memcpy(blob + (L.items - L.queries), gp.items.data(),
                  gp.items.size() * sizeof(S2Item));
      std::memcpy(blob + (L.run_items - L.queries), gp.run_items.data(),
                  gp.run_items.size() * sizeof(int32_t));
    }
    std::memcpy(blob + (L.packed_items - L.queries), gp.packed_items.data(),
                gp.packed_items.size() * sizeof(int32_t));
    std::memcpy(blob + (L.item_meta - L.queries), gp.item_meta.data(),
                gp.item_meta.size() * sizeof(int4));
    std::memcpy(blob + (L.tc_tiles - L.queries), gp.tc_tiles.data(),
                gp.tc_tiles.size() * sizeof(dbsa_tile_item));
    std::memcpy(blob + (L.offs - L.queries), offs_host, (size_t)(nb + 1) * sizeof(int32_t));
    std::memcpy(blob + (L.compact_base - L.queries), gp.compact_base.data(),
                gp.compact_base.size() * sizeof(int32_t));
    if (fixed != nullptr)
      e = cudaMemcpyAsync(at<void>(workspace, L.queries), blob, blob_bytes,
                          cudaMemcpyHostToDevice, st);
    else
      e = staging_ring().send(at<void>(workspace, L.queries), blob_bytes, st, workspace);
    if (e != cudaSuccess) return cuda_fail(e, "gather plan upload");
  }
  Stage2Args a{};
  a.k_cache = k_cache;
  a.v_cache = v_cache;
  a.cap = cap;
  a.q_new = q_new;
  a.k_tail = k_tail;
  a.v_tail = v_tail;
  a.tail_len = tail_len;
  a.tail_cap = tail_cap;
  a.n_new = n_new;
  a.Hq = cfg->n_q_heads;
  a.Hkv = cfg->n_kv_heads;
  a.queries = at<S2Query>(workspace, L.queries);
  a.segs = at<S2Segment>(workspace, L.segs);
  a.items = at<S2Item>(workspace, L.items);
  a.n_items = (int32_t)gp.items.size();
  a.n_queries = nq;
  a.run_items = at<int32_t>(workspace, L.run_items);
  a.n_run = (int32_t)gp.run_items.size();
  a.part_acc = at<uint16_t>(workspace, L.part_acc);
  a.part_ml = at<float2>(workspace, L.part_ml);
  a.out = out;
  a.dbg_map = dbg_map;
  a.dbg_cap = dbg_cap;
  a.scale_log2 = scale_log2(cfg);
  a.rope = rope;
  const bool f32 = cfg->dtype == DBSA_F32;
  if (gp.compact) {
    // every query's gathered keys (rotated at their fresh positions) and
    // values into the compact buffers (the gather map comes from this
    // kernel), the packed query rows at their own positions, the tensor-core
    // kernel over (kv head, query, 128-row tile) in partial mode, then the
    // tail keys on the per-query kernel and the merge below
    CompactArgs ca{};
    ca.k_cache = k_cache;
    ca.v_cache = v_cache;
    ca.cap = cap;
    ca.Hkv = cfg->n_kv_heads;
    ca.segs = a.segs;
    ca.n_segs = (int32_t)gp.segs.size();
    ca.base = at<int32_t>(workspace, L.compact_base);
    ca.rows = gp.compact_rows;
    ca.k_hat = at<void>(workspace, L.k_hat);
    ca.v_hat = at<void>(workspace, L.v_hat);
    ca.dbg = dbg_map;
    ca.dbg_cap = dbg_cap;
    ca.rope = rope;
    if ((e = launch_compact(ca, cfg->head_dim, f32, st)) != cudaSuccess)
      return cuda_fail(e, "compact gather");
    count_launches(1);
    a.dbg_map = nullptr;  // written by the compact gather above
    Stage1Args sa{};
    if ((e = set_query_rows(sa, cfg, gp, L, q_new, n_new, tail_len, a.n_items, rope, workspace,
                            nullptr, st)) != cudaSuccess)
      return cuda_fail(e, "query rotation");
    sa.k_rot = ca.k_hat;
    sa.k_rows = gp.compact_rows;
    sa.v = ca.v_hat;
    sa.v_rows = gp.compact_rows;
    sa.v_head_stride = gp.compact_rows;
    sa.out = nullptr;
    sa.Hq = cfg->n_kv_heads;  // packed rows are per kv head
    sa.Hkv = cfg->n_kv_heads;
    sa.items = at<dbsa_tile_item>(workspace, L.tc_tiles);
    sa.n_items = (int32_t)gp.tc_tiles.size();
    sa.scale_log2 = a.scale_log2;
    sa.status = at<int>(workspace, 0);
    sa.part.acc = a.part_acc;
    sa.part.ml = a.part_ml;
    sa.part.packed_items = at<int32_t>(workspace, L.packed_items);
    sa.part.group = cfg->n_q_heads / cfg->n_kv_heads;
    sa.part.Hq = cfg->n_q_heads;
    sa.part.n_new = n_new;
    sa.part.dbg = nullptr;
    sa.wait_limit_ns = wait_expiry;
    sa.withhold_tiles = wait_expiry != 0;
    {
      ProfileScope prof(st);
      e = launch_stage1(sa, cfg->head_dim, false, num_sms(), st);
    }
    if (e != cudaSuccess) return cuda_fail(e, "stage-2 tensor-core attention");
    count_launches(1);
    if ((e = launch_stage2_main(a, cfg->head_dim, f32, st)) != cudaSuccess)  // tail items
      return cuda_fail(e, "stage-2 tail attention");
    count_launches(1);
  } else if (gp.per_query) {
    // the per-query kernel over every split item (it writes the gather map
    // from its own segment walk)
    {
      ProfileScope prof(st);
      e = launch_stage2_main(a, cfg->head_dim, f32, st);
    }
    if (e != cudaSuccess) return cuda_fail(e, "stage-2 per-query attention");
    count_launches(1);
  } else {
    // keys at block-relative positions, packed query rows, then the
    // tensor-core kernel over (kv head, block, 128-row tile) in partial mode
    RelRopeArgs ra{};
    ra.k_cache = k_cache;
    ra.v_cache = v_cache;
    ra.cap = cap;
    ra.Hkv = cfg->n_kv_heads;
    ra.T = (int32_t)gp.cache_rows;
    ra.nb = nb;
    ra.offs = at<int32_t>(workspace, L.offs);
    void *bk = const_cast<void *>(block_keys);
    ra.k_hat = prepared ? at<void>(bk, B.k_hat) : at<void>(workspace, L.k_hat);
    ra.v_bf16 = !f32 ? nullptr : prepared ? at<void>(bk, B.v_hat) : at<void>(workspace, L.v_hat);
    ra.rope = rope;
    if (!prepared) {
      if ((e = launch_rel_rope(ra, cfg->head_dim, f32, st)) != cudaSuccess)
        return cuda_fail(e, "block-relative rotation");
      count_launches(1);
    }
    a.dbg_map = nullptr;  // written by the tensor-core kernel's epilogue (sa.part.dbg)
    Stage1Args sa{};
    if ((e = set_query_rows(sa, cfg, gp, L, q_new, n_new, tail_len, a.n_items, rope, workspace,
                            dbg_map, st)) != cudaSuccess)
      return cuda_fail(e, "query rotation");
    sa.k_rot = ra.k_hat;
    sa.k_rows = gp.cache_rows;
    sa.v = f32 ? ra.v_bf16 : v_cache;
    sa.v_rows = gp.cache_rows;
    sa.v_head_stride = f32 ? gp.cache_rows : cap;
    sa.out = nullptr;
    sa.Hq = cfg->n_kv_heads;  // packed rows are per kv head
    sa.Hkv = cfg->n_kv_heads;
    sa.items = at<dbsa_tile_item>(workspace, L.tc_tiles);
    sa.n_items = (int32_t)gp.tc_tiles.size();
    sa.scale_log2 = a.scale_log2;
    sa.status = at<int>(workspace, 0);
    sa.part.acc = a.part_acc;
    sa.part.ml = a.part_ml;
    sa.part.packed_items = at<int32_t>(workspace, L.packed_items);
    sa.part.group = cfg->n_q_heads / cfg->n_kv_heads;
    sa.part.Hq = cfg->n_q_heads;
    sa.part.n_new = n_new;
    sa.part.dbg = dbg_map;   // written by the kernel's epilogue when given
    sa.part.dbg_cap = dbg_cap;
    sa.part.items = a.items;
    sa.part.queries = a.queries;
    sa.part.tail_len = tail_len;
    sa.wait_limit_ns = wait_expiry;
    sa.withhold_tiles = wait_expiry != 0;
    {
      ProfileScope prof(st);
      e = launch_stage1(sa, cfg->head_dim, false, num_sms(), st);
    }
    if (e != cudaSuccess) return cuda_fail(e, "stage-2 tensor-core attention");
    count_launches(1);
    const int rows = (cfg->n_q_heads / cfg->n_kv_heads) * n_new;
    if (rows <= kTailMergeMaxRows) {
      // few rows per (query, KV head), e.g. a decode step: each query's own
      // tail tokens and the merge of its block partials in one kernel
      if ((e = launch_stage2_tail_merge(a, cfg->head_dim, f32, st)) != cudaSuccess)
        return cuda_fail(e, "stage-2 tail attention and merge");
      count_launches(1);
      return DBSA_OK;
    }
    // many rows (a prompt pass): the tail keys on the per-query tensor-core
    // (mma.sync) kernel, then the merge below
    if ((e = launch_stage2_main(a, cfg->head_dim, f32, st)) != cudaSuccess)  // tail items
      return cuda_fail(e, "stage-2 tail attention");
    count_launches(1);
  }
  if ((e = launch_stage2_merge(a, cfg->head_dim, f32, st)) != cudaSuccess)
    return cuda_fail(e, "stage-2 merge");
  count_launches(1);
  return DBSA_OK;
}

}  // namespace

dbsa_status dbsa::gather_fixed_scratch(
    const dbsa_config *cfg, const void *k_cache, const void *v_cache, int64_t cap,
    const int32_t *offs_host, int32_t nb, int32_t nq, const int32_t *sel_ptr_host,
    const int32_t *sel_blocks_host, const void *q_new, int32_t n_new, const void *k_tail,
    const void *v_tail, int32_t tail_len, int32_t tail_cap, void *out, int32_t *dbg_map,
    int64_t dbg_cap, const FixedScratch &fixed, void *stream) {
  return gather_impl(cfg, k_cache, v_cache, cap, offs_host, nb, nq, sel_ptr_host,
                     sel_blocks_host, q_new, n_new, k_tail, v_tail, tail_len, tail_cap, out,
                     dbg_map, dbg_cap, nullptr, 0, nullptr, 0, stream, &fixed);
}

extern "C" {

dbsa_status dbsa_gather_rope_attend(const dbsa_config *cfg, const void *k_cache,
                                    const void *v_cache, int64_t cap, const int32_t *offs_host,
                                    int32_t nb, int32_t nq, const int32_t *sel_ptr_host,
                                    const int32_t *sel_blocks_host, const void *q_new,
                                    int32_t n_new, const void *k_tail, const void *v_tail,
                                    int32_t tail_len, int32_t tail_cap, void *out,
                                    int32_t *dbg_map, int64_t dbg_cap, void *workspace,
                                    size_t ws_bytes, void *stream) {
  return gather_impl(cfg, k_cache, v_cache, cap, offs_host, nb, nq, sel_ptr_host,
                     sel_blocks_host, q_new, n_new, k_tail, v_tail, tail_len, tail_cap, out,
                     dbg_map, dbg_cap, nullptr, 0, workspace, ws_bytes, stream);
}

size_t dbsa_block_keys_size(const dbsa_config *cfg, const int32_t *offs_host, int32_t nb) {
  if (check_cfg(cfg) != DBSA_OK || check_offs(offs_host, nb) != DBSA_OK) return 0;
  return bk_layout(cfg, offs_host, nb).total;
}

dbsa_status dbsa_block_keys(const dbsa_config *cfg, const void *k_cache, const void *v_cache,
                            int64_t cap, const int32_t *offs_host, int32_t nb, void *block_keys,
                            size_t bk_bytes, void *stream) {
  dbsa_status s = check_cfg(cfg);
  if (s != DBSA_OK) return s;
  if ((s = check_offs(offs_host, nb)) != DBSA_OK) return s;
  if (!k_cache || !v_cache) return fail(DBSA_ERR_INVALID_ARG, "a tensor pointer is NULL");
  if (!aligned16(k_cache) || !aligned16(v_cache))
    return fail(DBSA_ERR_INVALID_ARG, "tensor pointers must be 16-byte aligned");
  if (offs_host[nb] > cap)
    return fail(DBSA_ERR_CAPACITY, "offsets reach %d rows but cap is %lld", offs_host[nb],
                (long long)cap);
  const BKLayout B = bk_layout(cfg, offs_host, nb);
  if ((s = check_ws(block_keys, bk_bytes, B.total)) != DBSA_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e;
  RopeTables rope;
  if ((e = build_tables(block_keys, B.rope, B.n_hi, cfg, st, &rope)) != cudaSuccess)
    return cuda_fail(e, "rope tables");
  count_launches(1);
  if ((e = upload_async(at<void>(block_keys, B.offs), offs_host,
                        (size_t)(nb + 1) * sizeof(int32_t), st)) != cudaSuccess)
    return cuda_fail(e, "offset upload");
  RelRopeArgs ra{};
  ra.k_cache = k_cache;
  ra.v_cache = v_cache;
  ra.cap = cap;
  ra.Hkv = cfg->n_kv_heads;
  ra.T = offs_host[nb];
  ra.nb = nb;
  ra.offs = at<int32_t>(block_keys, B.offs);
  ra.k_hat = at<void>(block_keys, B.k_hat);
  ra.v_bf16 = cfg->dtype == DBSA_F32 ? at<void>(block_keys, B.v_hat) : nullptr;
  ra.rope = rope;
  if ((e = launch_rel_rope(ra, cfg->head_dim, cfg->dtype == DBSA_F32, st)) != cudaSuccess)
    return cuda_fail(e, "block-relative rotation");
  count_launches(1);
  return DBSA_OK;
}

dbsa_status dbsa_gather_rope_attend_prepared(
    const dbsa_config *cfg, const void *k_cache, const void *v_cache, int64_t cap,
    const int32_t *offs_host, int32_t nb, int32_t nq, const int32_t *sel_ptr_host,
    const int32_t *sel_blocks_host, const void *q_new, int32_t n_new, const void *k_tail,
    const void *v_tail, int32_t tail_len, int32_t tail_cap, void *out, int32_t *dbg_map,
    int64_t dbg_cap, const void *block_keys, size_t bk_bytes, void *workspace, size_t ws_bytes,
    void *stream) {
  if (block_keys == nullptr) return fail(DBSA_ERR_INVALID_ARG, "block_keys is NULL");
  return gather_impl(cfg, k_cache, v_cache, cap, offs_host, nb, nq, sel_ptr_host,
                     sel_blocks_host, q_new, n_new, k_tail, v_tail, tail_len, tail_cap, out,
                     dbg_map, dbg_cap, block_keys, bk_bytes, workspace, ws_bytes, stream);
}

int64_t dbsa_host_allocation_calls(void) {
  return g_host_alloc_calls.load(std::memory_order_relaxed);
}

dbsa_status dbsa_read_status(const void *workspace, void *stream) {
  if (workspace == nullptr) return fail(DBSA_ERR_INVALID_ARG, "workspace is NULL");
  int word = 0;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaMemcpyAsync(&word, workspace, sizeof word, cudaMemcpyDeviceToHost, st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return cuda_fail(e, "status read");
  if (word == DBSA_ERR_TIMEOUT) {
    fail(DBSA_ERR_TIMEOUT, "a device-side wait expired");
    return DBSA_ERR_TIMEOUT;
  }
  return word == 0 ? DBSA_OK : (dbsa_status)word;
}

}  // extern "C"
