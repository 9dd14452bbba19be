// Stage-1 block-sparse streaming attention on the 5th-generation tensor core.
//
// [DBSA notes] §Stage 1, item 2: every token of block b_i attends to the sink
// block b_1, the previous j blocks and (causally) its own block.  The host
// planner turns this pattern into a tile list: one item per (query head,
// 128-row query tile inside one block), each with at most two contiguous key
// ranges (the sink, then the window up to the diagonal).  Masked tiles are
// never enumerated (the page's implementation skipped masked blocks with
// Flex Attention for a speed-up proportional to the sparsity; here the list
// holds only the tiles that contain an allowed pair).
//
// One persistent CTA per SM walks items round-robin.  Warp roles:
//   warp 0      TMA producer: two independent cursors, one for the K tiles
//               (3-stage ring, preceded by each item's Q tile when the Q
//               rows come pre-rotated), one for the V tiles (2-stage ring)
//   warp 1      TMEM owner; one thread issues O_h += P_h V_h for the two key
//               halves of each tile (tcgen05, A from TMEM)
//   warp 10     one thread issues S = Q K^T (tcgen05, both operands in SMEM)
//   warps 2..9  softmax, two warpgroups splitting every tile by keys:
//               warpgroup w takes keys 64w..64w+63 of each tile, one thread
//               per query row (TMEM lane), with its own fp32 running max and
//               sum (lazy rescale threshold) and its own O accumulator O_w
//               (the PV of its half of the keys).  Both halves of a tile are
//               exponentiated at once, so a tile's P is ready in half the
//               time one warpgroup would take; each thread makes one pass
//               over its 64 scores held in registers (mask, max, rescale,
//               exp2).  At an item's end they publish the merge factors of
//               the two states and go on.
//   warps 11..14 Q tiles and epilogue: rotate each item's query rows into
//               its Q tile (double-buffered, two items ahead; launches with
//               ROTQ), then, at the item's end, combine O_0 and O_1, free O
//               for the next item's first PV, and write the rows out (bf16:
//               staged in the item's Q tile, then one bulk copy per row).
// S = Q K^T lives in TMEM in two 128-column buffers (tile parity); each
// warpgroup writes its 64 keys' P as bf16 pairs over the first 32 columns of
// its own half of the S buffer, and O_0, O_1 take D columns each: 512 columns
// in all.  With ROTQ the query rows are read unrotated and rotated in the
// kernel (one thread per row, fp32, rounded once to bf16); without it they
// arrive rotated (bf16, packed by a preceding kernel) and are loaded by TMA.
// K arrives already rotated (bf16) from the preparation pass and V is read
// straight from the pre-RoPE cache.  Every wait is bounded and reports
// DBSA_ERR_TIMEOUT.
//
// Measured on B200: the tensor core runs a 128x128x16
// MMA in 64 cycles but keeps only about one MMA queued, so the issuing
// threads must not stall between MMAs; softmax warps that saturate the FMA
// pipe starve an issuer on the same SM sub-partition, hence the packed
// (f32x2) and 3-input arithmetic in the softmax and two issuer threads.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cudaTypedefs.h>

#include <cmath>
#include <mutex>

#include "dbsa_internal.h"
#include "sm100.cuh"
#include "vec8.cuh"

namespace dbsa {
namespace {

using namespace sm100;

constexpr uint64_t kWaitLimitNs = 4000000000ull;   // default: 4 s, far above any legitimate wait
constexpr uint64_t kDrainLimitNs = 200000000ull;   // 0.2 s for the exit drain
constexpr uint32_t kFull = 0xFFFFFFFFu;

// Ring depths (tiles in flight).  A K slot frees when its QK^T has run and is
// needed again kStagesK tiles later; a V slot frees only after its PV, about
// two tiles after the QK, and is needed kStagesV tiles later.  Q is double
// buffered: the epilogue warpgroup writes an item's Q tile once it has
// finished the item two before it in the same slot (ROTQ), or the producer
// loads it once that item's last QK^T has run or its staged rows have been
// copied out.
constexpr int kStagesK = 3;
constexpr int kStagesV = 2;
// The epilogue stages an item's bf16 rows in its Q tile only when the item
// has at least this many key tiles: the Q slot then frees once the rows are
// copied out, which for shorter items would hold up the next-but-one item's
// Q tile.  Shorter items store their rows directly.
constexpr int kStageMinTiles = 3;
constexpr int kStagesQ = 2;

enum Bar {
  B_Q_FULL = 0,                // [Q stage]: the Q tile is in place
  B_Q_EMPTY = B_Q_FULL + kStagesQ,   // [Q stage]: an unstaged item's last QK^T (TMA Q tiles)
  B_K_FULL = B_Q_EMPTY + kStagesQ, B_K_EMPTY = B_K_FULL + kStagesK,
  B_V_FULL = B_K_EMPTY + kStagesK, B_V_EMPTY = B_V_FULL + kStagesV,
  B_S_FULL = B_V_EMPTY + kStagesV,  // [buffer]
  B_P_FULL = B_S_FULL + 2,     // [buffer][half]: P of keys 64h.. written by warpgroup h
  B_PV_DONE = B_P_FULL + 4,    // [buffer]: both PV halves of the buffer's tile done
  B_O_FREE = B_PV_DONE + 2, B_DRAIN = B_O_FREE + 1,
  B_ML_A = B_DRAIN + 1,       // end of item: warpgroup 1 has published (m, l)
  B_ML_B = B_ML_A + 1,        // end of item: warpgroup 0 has published the merge factors
  B_ML_FREE = B_ML_B + 1,     // the epilogue warpgroup has read the merge factors
  B_DRAIN_QK = B_ML_FREE + 1,
  B_Q_COPIED = B_DRAIN_QK + 1,  // [Q stage]: every row staged there has been copied out
  B_COUNT = B_Q_COPIED + kStagesQ
};

constexpr int kSoftmaxThreads = 256;              // warps 2..9: two warpgroups
constexpr int kQKWarp = 10;                       // QK^T issuer (after the softmax warps)
constexpr int kEpiWarp0 = 11;                     // warps 11..14: epilogue warpgroup
constexpr int kThreads = 32 * (kEpiWarp0 + 4);

struct Item {
  int head, q_row0, q_pos0, n_rows, n_ranges;
  int k_row0[2], v_row0[2], pos0[2], len[2];
  int nt0, ntiles;
};

__device__ __forceinline__ Item load_item(const dbsa_tile_item *items, int idx) {
  const dbsa_tile_item *s = items + idx;
  Item it;
  it.head = __ldg(&s->head);
  it.q_row0 = __ldg(&s->q_row0);
  it.q_pos0 = __ldg(&s->q_pos0);
  it.n_rows = __ldg(&s->n_rows);
  it.n_ranges = __ldg(&s->n_ranges);
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    it.k_row0[r] = __ldg(&s->k_row0[r]);
    it.v_row0[r] = __ldg(&s->v_row0[r]);
    it.pos0[r] = __ldg(&s->pos0[r]);
    it.len[r] = it.n_ranges > r ? __ldg(&s->len[r]) : 0;
  }
  it.nt0 = (it.len[0] + kTileKeys - 1) / kTileKeys;
  it.ntiles = it.nt0 + (it.len[1] + kTileKeys - 1) / kTileKeys;
  return it;
}

__device__ __forceinline__ void tile_of(const Item &it, int t, int &r, int &kt) {
  if (t < it.nt0) {
    r = 0;
    kt = t * kTileKeys;
  } else {
    r = 1;
    kt = (t - it.nt0) * kTileKeys;
  }
}

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// The softmax warps share each SM sub-partition with the MMA-issuing thread,
// and every FMA-pipe instruction they issue can delay an MMA issue; the
// per-score arithmetic therefore uses sm_100's packed and 3-input forms.
__device__ __forceinline__ float max3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}
using f32x2 = unsigned long long;
__device__ __forceinline__ f32x2 f2_pack(float a, float b) {
  f32x2 r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
  return r;
}
__device__ __forceinline__ void f2_unpack(f32x2 r, float &a, float &b) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(a), "=f"(b) : "l"(r));
}
__device__ __forceinline__ f32x2 f2_fma(f32x2 a, f32x2 b, f32x2 c) {
  f32x2 d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ f32x2 f2_add(f32x2 a, f32x2 b) {
  f32x2 d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}

// 2^x for a pair of scores on the FMA pipe.  The exponential unit delivers 16
// results per clock per SM, which for a 128x128 tile is as long as its two
// MMAs; evaluating a share of P here keeps it off the critical path.  With
// n = round(x) and f = x - n in [-1/2, 1/2], 2^x = 2^n * 2^f: n is added to the
// exponent field and 2^f is a cubic fitted to it on that interval (weighted
// least squares at Chebyshev nodes, reweighted toward equal ripple), with a
// relative error below 7.5e-5, far under the half-ulp (2^-9) of the bf16 P it
// feeds.  The rounding adds and subtracts 1.5 * 2^23, which leaves round(x) in
// the low bits of the sum.  x is clamped at -125 so the exponent field stays
// normal: a masked (-inf) score gives 2^-125 rather than 0.
constexpr float kExp2C0 = 0.99992806f, kExp2C1 = 0.69326097f, kExp2C2 = 0.24261113f,
                kExp2C3 = 0.05517166f;
// Pairs (of the 16 in a 32-score chunk) whose P is evaluated by exp2_poly2.
constexpr uint32_t kPolyPairMask = 0x8080u;
__device__ __forceinline__ f32x2 exp2_poly2(f32x2 x) {
  float x0, x1;
  f2_unpack(x, x0, x1);
  const f32x2 xc = f2_pack(fmaxf(x0, -125.f), fmaxf(x1, -125.f));
  const f32x2 j = f2_add(xc, f2_pack(12582912.f, 12582912.f));
  const f32x2 n = f2_add(j, f2_pack(-12582912.f, -12582912.f));
  const f32x2 f = f2_fma(n, f2_pack(-1.f, -1.f), xc);
  f32x2 q = f2_fma(f2_pack(kExp2C3, kExp2C3), f, f2_pack(kExp2C2, kExp2C2));
  q = f2_fma(q, f, f2_pack(kExp2C1, kExp2C1));
  q = f2_fma(q, f, f2_pack(kExp2C0, kExp2C0));
  float j0, j1, q0, q1;
  f2_unpack(j, j0, j1);
  f2_unpack(q, q0, q1);
  return f2_pack(__uint_as_float(__float_as_uint(q0) + (__float_as_uint(j0) << 23)),
                 __uint_as_float(__float_as_uint(q1) + (__float_as_uint(j1) << 23)));
}

// Bounded wait used on the way out: ignores the abort flag.
__device__ __forceinline__ void drain_wait(uint64_t *bar, uint32_t parity) {
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (globaltimer_ns() - t0 > kDrainLimitNs) return;
  }
}

struct Params {
  const dbsa_tile_item *items;
  int n_items;
  int group;  // Hq / Hkv
  int Hq;
  void *out;
  float scale_log2;
  int *status;
  uint64_t wait_limit_ns;  // limit of every bounded wait
  int withhold_tiles;      // test hook: the producer loads nothing (every wait runs out)
  Stage1Partial part;  // partial-output mode (part.acc != null)
  // Unrotated query rows.  Stage 1: row q_row0 + r of an item is q_src row
  // (q_row0 + r) x q_heads + head, rotated at q_pos0 + r.  Partial mode:
  // packed row w of an item's query (token w / g, local head w % g) comes
  // from q_src [query][n_new][q_heads], rotated at item_meta.y + token.
  const void *q_src;
  int q_f32;               // q_src is fp32 (else bf16)
  int q_heads;
  RopeTables rope;
};

// One row of a Q tile in the layout a 128-byte-swizzled TMA tile load writes
// and the QK^T descriptor reads: columns 64a..64a+63 in atom column a (HALF
// bytes apart), row r at byte 128 r inside it, and the row's 16-byte chunk c
// at chunk position c ^ (r mod 8).  Chunk j of the row holds columns
// 8j..8j+7, rounded to bf16 here.
__device__ __forceinline__ void put_q_chunk(uint8_t *tile, int row, int j, const float (&f)[8]) {
  constexpr uint32_t HALF = 128 * 64 * 2;
  uint32_t w[4];
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    __nv_bfloat162 h = __floats2bfloat162_rn(f[2 * e], f[2 * e + 1]);
    w[e] = *reinterpret_cast<uint32_t *>(&h);
  }
  *reinterpret_cast<uint4 *>(tile + (j >> 3) * HALF + row * 128 + (((j & 7) ^ (row & 7)) << 4)) =
      make_uint4(w[0], w[1], w[2], w[3]);
}

// This thread's row of an item's Q tile: the unrotated query vector, rotated
// at its position (rotate-half RoPE with the angle tables, the rounding of
// every other rotation in the library) and stored as bf16; rows past the
// item's n_rows are zero.  Returns the position the row was rotated at.
template <int D, typename T>
__device__ __forceinline__ int rotate_q_row(const Params &p, const Item &it, int row,
                                            uint8_t *tile) {
  constexpr int H = D / 2;
  const bool valid = row < it.n_rows;
  int pos = 0;
  int64_t off = 0;
  if (valid) {
    if (p.part.acc != nullptr) {
      const int grow = it.q_row0 + row;                 // row of the kv head's packed rows
      const int R = p.part.group * p.part.n_new;
      const int item = __ldg(p.part.packed_items + grow / R);
      const int w = grow % R;
      const int4 meta = __ldg(p.part.item_meta + item);
      const int tok = w / p.part.group;
      pos = meta.y + tok;
      off = (((int64_t)meta.z * p.part.n_new + tok) * p.q_heads + it.head * p.part.group +
             w % p.part.group) * D;
    } else {
      pos = it.q_pos0 + row;
      off = ((int64_t)(it.q_row0 + row) * p.q_heads + it.head) * D;
    }
  }
  const T *src = static_cast<const T *>(p.q_src) + off;
#pragma unroll 4
  for (int i0 = 0; i0 < H; i0 += 8) {
    float lo[8], hi[8];
    if (valid) {
      float c[8], sn[8];
      load8(src + i0, lo);
      load8(src + H + i0, hi);
      rope_cs8(p.rope, pos, i0, H, c, sn);
      rotate8(lo, hi, c, sn);
    } else {
#pragma unroll
      for (int e = 0; e < 8; ++e) lo[e] = hi[e] = 0.f;
    }
    put_q_chunk(tile, row, i0 / 8, lo);
    put_q_chunk(tile, row, (H + i0) / 8, hi);
  }
  return pos;
}

// STAGE: the launch stages the bf16 rows of its items of at least
// kStageMinTiles key tiles in their Q tiles (Stage 1 and prompt passes); a
// launch without it (decode steps, fp32 outputs) has none of that code.
// ROTQ: the epilogue warpgroup rotates the query rows into the Q tiles (the
// tensor map tmQ is unused); without it the producer loads pre-rotated Q
// tiles through tmQ.
template <int D, bool OUT_F32, bool STAGE, bool ROTQ>
__global__ void __launch_bounds__(kThreads, 1)
    stage1_attn_kernel(const __grid_constant__ CUtensorMap tmQ,
                       const __grid_constant__ CUtensorMap tmK,
                       const __grid_constant__ CUtensorMap tmV, const Params p) {
  constexpr uint32_t HALF = 128 * 64 * 2;        // one 128-row x 64-column swizzled atom column
  constexpr uint32_t TILE = 128 * D * 2;         // Q / K / V tile
  constexpr int NH = D / 64;                     // 64-column halves per row
  constexpr uint32_t IDESC_QK = idesc_bf16_f32(128, 128, false);
  constexpr uint32_t IDESC_PV = idesc_bf16_f32(128, D, true);
  constexpr uint32_t TMEM_COLS = 512;
  constexpr uint32_t COL_S = 0;                  // two S buffers, 128 columns each
  constexpr uint32_t COL_O = 256;                // O of key half h at COL_O + h * D

  // Tiles (1024-byte aligned for the 128-byte swizzle): the Q, K and V rings;
  // then the epilogue exchange and the barriers.  The request leaves room for
  // any alignment pad of the dynamic shared-memory base.
  extern __shared__ uint8_t smem_raw[];
  uint8_t *base = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t *sQ = base;
  uint8_t *sK = sQ + kStagesQ * TILE;
  uint8_t *sV = sK + kStagesK * TILE;
  float2 *sML = reinterpret_cast<float2 *>(sV + kStagesV * TILE);  // epilogue exchange, [128]
  uint64_t *bar = reinterpret_cast<uint64_t *>(sML + 128);
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bar + B_COUNT);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  // whether the epilogue stages an item's rows in its Q tile (bf16 rows of
  // items with at least kStageMinTiles key tiles), which decides who frees
  // the item's Q slot
  auto stages_rows = [&](int ntiles) { return STAGE && ntiles >= kStageMinTiles; };

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStagesQ; ++s) {
      mbar_init(&bar[B_Q_FULL + s], ROTQ ? 128 : 1);   // the epilogue's rows / one TMA load
      mbar_init(&bar[B_Q_EMPTY + s], 1);     // an unstaged item's last QK^T
      mbar_init(&bar[B_Q_COPIED + s], 128);  // a staged item's row copies
    }
    for (int s = 0; s < kStagesK; ++s) {
      mbar_init(&bar[B_K_FULL + s], 1);
      mbar_init(&bar[B_K_EMPTY + s], 1);
    }
    for (int s = 0; s < kStagesV; ++s) {
      mbar_init(&bar[B_V_FULL + s], 1);
      mbar_init(&bar[B_V_EMPTY + s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bar[B_S_FULL + s], 1);
      mbar_init(&bar[B_P_FULL + 2 * s], 128);
      mbar_init(&bar[B_P_FULL + 2 * s + 1], 128);
      mbar_init(&bar[B_PV_DONE + s], 1);
    }
    mbar_init(&bar[B_O_FREE], 128);
    mbar_init(&bar[B_DRAIN], 1);
    mbar_init(&bar[B_DRAIN_QK], 1);
    mbar_init(&bar[B_ML_A], 128);
    mbar_init(&bar[B_ML_B], 128);
    mbar_init(&bar[B_ML_FREE], 128);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, TMEM_COLS);
    tmem_relinquish();
    tc_fence_before();
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // the set-up above touches shared memory and TMEM only
  pdl_enter();

  if (warp == 0 && lane == 0) {
    // ------------------------------------------------------------ producer
    // Two independent cursors over the CTA's tile sequence: K tiles (without
    // ROTQ, each item's Q tile first) and V tiles.  A K slot frees when its
    // QK^T has run, a V slot only when its PV has run, which happens about two
    // tiles later; separate cursors keep the K loads from queueing behind V
    // slots.  A Q slot frees at its item's last QK^T, or, when the epilogue
    // staged the item's rows there, once it has copied them out.  Neither
    // cursor blocks: the thread polls whichever slot it needs next.
    if (!ROTQ) tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
    // Test hook: no tile is loaded, so every wait of the consumers is for a
    // barrier that nothing completes and can only run out at the wait limit.
    // This thread waits for the abort they raise (bounded by twice the limit,
    // then it raises it itself) and issues nothing.
    const bool withhold = p.withhold_tiles != 0;
    if (withhold) {
      const uint64_t t0 = globaltimer_ns();
      while (!*abort_flag) {
        if (globaltimer_ns() - t0 > 2 * p.wait_limit_ns) {
          *abort_flag = 1;
          atomicExch(p.status, DBSA_ERR_TIMEOUT);
          break;
        }
        __nanosleep(256);
      }
    }
    int kidx = withhold ? p.n_items : blockIdx.x, vidx = kidx, kt = 0, vt = 0;
    Item kit, vit;
    if (kidx < p.n_items) kit = vit = load_item(p.items, kidx);
    bool need_q = !ROTQ && kidx < p.n_items;
    uint32_t qn = 0, kn = 0, vn = 0;          // Q, K, V tiles issued
    int armed_q[kStagesQ], armed_k[kStagesK], armed_v[kStagesV];
    // Per Q slot (TMA Q tiles): how its last item frees it (-1 unused, 0 at
    // its last QK^T, 1 after the epilogue's copies of the rows it staged
    // there) and the uses of each kind so far; each kind has its own barrier.
    // The slots are used in turn, so the state is kept in registers as (slot
    // used next, the other slot) and swapped after each Q load.
    static_assert(kStagesQ == 2, "the Q slot state rotates between two slots");
    int qa_prev = -1, qb_prev = -1;
    uint32_t qa_staged = 0, qa_direct = 0, qb_staged = 0, qb_direct = 0;
#pragma unroll
    for (int s = 0; s < kStagesQ; ++s) armed_q[s] = -1;
#pragma unroll
    for (int s = 0; s < kStagesK; ++s) armed_k[s] = -1;
#pragma unroll
    for (int s = 0; s < kStagesV; ++s) armed_v[s] = -1;
    uint64_t t_prog = globaltimer_ns();
    uint32_t idle = 0;
    while (kidx < p.n_items || vidx < p.n_items) {
      bool prog = false;
      if (kidx < p.n_items) {
        const int kvh = kit.head / p.group;
        if (need_q) {
          const uint32_t qs = qn % kStagesQ, nq = qn / kStagesQ;
          const bool free_slot =
              qa_prev < 0 ||
              (qa_prev == 1 ? mbar_try_wait(&bar[B_Q_COPIED + qs], (qa_staged - 1) & 1)
                            : mbar_try_wait(&bar[B_Q_EMPTY + qs], (qa_direct - 1) & 1));
          if (free_slot) {
            mbar_arrive_expect_tx(&bar[B_Q_FULL + qs], TILE);
#pragma unroll
            for (int h = 0; h < NH; ++h)
              tma_load_3d(sQ + qs * TILE + h * HALF, &tmQ, &bar[B_Q_FULL + qs], h * 64, kit.q_row0,
                          kit.head);
            armed_q[qs] = nq & 1;
            qa_prev = stages_rows(kit.ntiles) ? 1 : 0;
            qa_staged += qa_prev;
            qa_direct += 1 - qa_prev;
            // the next Q load goes to the other slot
            const int tp = qa_prev;
            const uint32_t ts = qa_staged, td = qa_direct;
            qa_prev = qb_prev;
            qa_staged = qb_staged;
            qa_direct = qb_direct;
            qb_prev = tp;
            qb_staged = ts;
            qb_direct = td;
            ++qn;
            need_q = false;
            prog = true;
          }
        } else {
          const uint32_t st = kn % kStagesK, n = kn / kStagesK;
          if (n == 0 || mbar_try_wait(&bar[B_K_EMPTY + st], (n - 1) & 1)) {
            int r, k0;
            tile_of(kit, kt, r, k0);
            mbar_arrive_expect_tx(&bar[B_K_FULL + st], TILE);
#pragma unroll
            for (int h = 0; h < NH; ++h)
              tma_load_3d(sK + st * TILE + h * HALF, &tmK, &bar[B_K_FULL + st], h * 64,
                          (r ? kit.k_row0[1] : kit.k_row0[0]) + k0, kvh);
            armed_k[st] = n & 1;
            ++kn;
            prog = true;
            if (++kt == kit.ntiles) {
              kt = 0;
              kidx += gridDim.x;
              if (kidx < p.n_items) {
                kit = load_item(p.items, kidx);
                need_q = !ROTQ;
              }
            }
          }
        }
      }
      if (vidx < p.n_items) {
        const uint32_t st = vn % kStagesV, n = vn / kStagesV;
        if (n == 0 || mbar_try_wait(&bar[B_V_EMPTY + st], (n - 1) & 1)) {
          int r, k0;
          tile_of(vit, vt, r, k0);
          const int kvh = vit.head / p.group;
          mbar_arrive_expect_tx(&bar[B_V_FULL + st], TILE);
#pragma unroll
          for (int h = 0; h < NH; ++h)
            tma_load_3d(sV + st * TILE + h * HALF, &tmV, &bar[B_V_FULL + st], h * 64,
                        (r ? vit.v_row0[1] : vit.v_row0[0]) + k0, kvh);
          armed_v[st] = n & 1;
          ++vn;
          prog = true;
          if (++vt == vit.ntiles) {
            vt = 0;
            vidx += gridDim.x;
            if (vidx < p.n_items) vit = load_item(p.items, vidx);
          }
        }
      }
      if (prog) {
        idle = 0;
        t_prog = globaltimer_ns();
      } else if ((++idle & 63u) == 0u) {
        if (*abort_flag) break;
        if (globaltimer_ns() - t_prog > p.wait_limit_ns) {
          *abort_flag = 1;
          atomicExch(p.status, DBSA_ERR_TIMEOUT);
          break;
        }
      }
    }
    // Every load this thread issued must land before the CTA exits.
    for (int s = 0; s < kStagesQ; ++s)
      if (armed_q[s] >= 0) drain_wait(&bar[B_Q_FULL + s], (uint32_t)armed_q[s]);
    for (int s = 0; s < kStagesK; ++s)
      if (armed_k[s] >= 0) drain_wait(&bar[B_K_FULL + s], (uint32_t)armed_k[s]);
    for (int s = 0; s < kStagesV; ++s)
      if (armed_v[s] >= 0) drain_wait(&bar[B_V_FULL + s], (uint32_t)armed_v[s]);
  } else if ((warp == 1 || warp == kQKWarp) && lane == 0) {
    // ------------------------------------------------------------ MMA issuers
    // Two threads on different SM sub-partitions feed the tensor core: warp
    // kQKWarp issues S = Q K^T, warp 1 issues O += P V.  The tensor core keeps
    // only about one MMA queued, so every instruction an issuer runs between
    // two MMAs is idle time for it: descriptors are precomputed (a descriptor
    // for a byte offset is the base descriptor plus offset / 16), ring stages
    // advance incrementally, and a wait whose phase is complete costs one
    // try_wait.  QK(t) writes the S buffer in which P(t - 2) lived, so it
    // waits for PV(t - 2) to complete (the softmax read S(t - 2) before it
    // signalled P(t - 2)).
    const bool is_qk = warp == kQKWarp;
    const uint64_t dQ = sdesc_sw128(smem_u32(sQ), 16, 1024);
    const uint64_t dK = sdesc_sw128(smem_u32(sK), 16, 1024);
    const uint64_t dV = sdesc_sw128(smem_u32(sV), HALF, 1024);
    constexpr uint64_t kTileDesc = TILE >> 4;
    uint32_t st = 0, ph = 0;        // ring stage / phase of this issuer's operand (K or V)
    uint32_t s_it = 0, item_no = 0;
    bool ok = true;
    auto wait = [&](int b, uint32_t parity) -> bool {
      return mbar_try_wait(&bar[b], parity) ||
             mbar_wait(&bar[b], parity, abort_flag, p.status, p.wait_limit_ns, DBSA_ERR_TIMEOUT);
    };
    for (int idx = blockIdx.x; ok && idx < p.n_items; idx += gridDim.x, ++item_no) {
      const int ntiles = load_item(p.items, idx).ntiles;
      const uint32_t qs = item_no % kStagesQ;
      if (is_qk && !(ok = wait(B_Q_FULL + qs, (item_no / kStagesQ) & 1))) break;
      const uint64_t dq = dQ + qs * kTileDesc;
      for (int t = 0; t < ntiles; ++t, ++s_it) {
        const uint32_t b = s_it & 1;
        if (is_qk) {
          if (!(ok = wait(B_K_FULL + st, ph))) break;
          if (s_it >= 2 && !(ok = wait(B_PV_DONE + b, ((s_it - 2) >> 1) & 1))) break;
          tc_fence_after();
          const uint64_t dk = dK + st * kTileDesc;
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t off16 = ((kk >> 2) * HALF + (kk & 3) * 32) >> 4;
            mma_bf16_ss(tmem + COL_S + b * 128, dq + off16, dk + off16, IDESC_QK,
                        kk > 0 ? 1u : 0u);
          }
          mma_commit(&bar[B_S_FULL + b]);
          mma_commit(&bar[B_K_EMPTY + st]);
          if (!ROTQ && t == ntiles - 1 && !stages_rows(ntiles)) mma_commit(&bar[B_Q_EMPTY + qs]);
        } else {
          // O_h (+)= P_h V_h for the key halves h = 0, 1 of the tile, each as
          // soon as its warpgroup has written P_h; both accumulators must have
          // been read by the previous item's epilogue before the first PV.
          // The item's first tile starts O_0 and O_1.
          if (!(ok = wait(B_V_FULL + st, ph))) break;
          if (t == 0 && item_no > 0 && !(ok = wait(B_O_FREE, (item_no - 1) & 1))) break;
          const uint64_t dv = dV + st * kTileDesc;
          const uint32_t ta = tmem + COL_S + b * 128;
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            if (!(ok = wait(B_P_FULL + 2 * b + h, (s_it >> 1) & 1))) break;
            tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              // P_h: keys 64h..64h+63 packed two per column in the first 32
              // columns of half h of the S buffer; 8 columns per 16 keys
              mma_bf16_ts(tmem + COL_O + h * D, ta + h * 64 + kk * 8, dv + (4 * h + kk) * 128,
                          IDESC_PV, (kk > 0 || t > 0) ? 1u : 0u);
          }
          if (!ok) break;
          mma_commit(&bar[B_PV_DONE + b]);
          mma_commit(&bar[B_V_EMPTY + st]);
        }
        if (++st == (is_qk ? kStagesK : kStagesV)) {
          st = 0;
          ph ^= 1;
        }
      }
    }
    // All issued MMAs must finish before TMEM is released.
    const int drain = is_qk ? B_DRAIN_QK : B_DRAIN;
    mma_commit(&bar[drain]);
    drain_wait(&bar[drain], 0);
  } else if (warp >= 2 && warp < 2 + kSoftmaxThreads / 32) {
    // ------------------------------------------------------------ softmax
    // Two warpgroups split every tile by keys: warpgroup w takes keys
    // 64w..64w+63 (its half of the S buffer), with its own running max / sum
    // and its own O accumulator O_w; the two states are combined once, in
    // the epilogue.  The two warps that share a row quarter sit on the same SM
    // sub-partition and exponentiate their halves at once.
    const int wg = (warp - 2) >> 2;
    const int quad = warp & 3;
    const int row = quad * 32 + lane;
    const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
    const uint32_t col_o = COL_O + wg * D;
    const float sl2 = p.scale_log2;
    uint32_t s_it = 0, item_no = 0;
    bool ok = true;
    for (int idx = blockIdx.x; ok && idx < p.n_items; idx += gridDim.x, ++item_no) {
      const Item it = load_item(p.items, idx);
      const int qpos = it.q_pos0 + row;
      float m_ref = -INFINITY, l = 0.f;
      uint32_t prev = 0;          // CTA-wide index of the previous tile
      for (int t = 0; t < it.ntiles; ++t, ++s_it) {
        int r, kt;
        tile_of(it, t, r, kt);
        const uint32_t col_s = COL_S + (s_it & 1) * 128 + wg * 64;   // this half of S
        ok = __all_sync(kFull, mbar_wait(&bar[B_S_FULL + (s_it & 1)], (s_it >> 1) & 1, abort_flag,
                                         p.status, p.wait_limit_ns, DBSA_ERR_TIMEOUT));
        if (!ok) break;
        tc_fence_after();
        const int klim = (r ? it.len[1] : it.len[0]) - kt;   // valid keys of this tile
        const int kpos0 = (r ? it.pos0[1] : it.pos0[0]) + kt;
        const bool need_mask = klim < 128 || kpos0 + 127 > it.q_pos0;
        // last allowed key of this row, counted from this half's first key
        const int klast = min(klim - 1, qpos - kpos0) - wg * 64;
        // -- one pass over this half's 64 scores, held in registers: masked
        // scores become -inf, the row maximum, the lazy rescale, then
        // P = 2^(s * scale - m) as bf16 pairs over the half's columns 0..31
        // (every score is in registers before the first P column is written).
        uint32_t va[32], vb[32];
        tmem_ld32(tmem + lane_off + col_s, va);
        tmem_ld32(tmem + lane_off + col_s + 32, vb);
        tmem_wait_ld(va);
        tmem_wait_ld(vb);
        if (need_mask) {
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            if (e > klast) va[e] = __float_as_uint(-INFINITY);
            if (32 + e > klast) vb[e] = __float_as_uint(-INFINITY);
          }
        }
        float mt[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
        for (int e = 0; e < 32; e += 2) {
          mt[(e >> 1) & 1] = max3(mt[(e >> 1) & 1], __uint_as_float(va[e]), __uint_as_float(va[e + 1]));
          mt[2 + ((e >> 1) & 1)] =
              max3(mt[2 + ((e >> 1) & 1)], __uint_as_float(vb[e]), __uint_as_float(vb[e + 1]));
        }
        const float mt_x = max3(mt[0], mt[1], fmaxf(mt[2], mt[3])) * sl2;
        if (t == 0) {
          m_ref = mt_x;
        } else {
          const bool need = mt_x > m_ref + 8.0f;
          if (__any_sync(kFull, need)) {
            // O_w must hold the item's earlier tiles before it is rescaled
            ok = __all_sync(kFull, mbar_wait(&bar[B_PV_DONE + (prev & 1)], (prev >> 1) & 1,
                                             abort_flag, p.status, p.wait_limit_ns,
                                             DBSA_ERR_TIMEOUT));
            if (!ok) break;
            tc_fence_after();
            const float m_new = fmaxf(m_ref, mt_x);
            const float alpha = (m_new == -INFINITY) ? 1.f : ex2(m_ref - m_new);
            l *= alpha;
            m_ref = m_new;
#pragma unroll 1
            for (int c = 0; c < D / 32; ++c) {
              uint32_t o[32];
              tmem_ld32(tmem + lane_off + col_o + c * 32, o);
              tmem_wait_ld(o);
#pragma unroll
              for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
              tmem_st32(tmem + lane_off + col_o + c * 32, o);
            }
            tmem_wait_st();
          }
        }
        prev = s_it;
        const float mu = (m_ref == -INFINITY) ? 0.f : m_ref;
        const f32x2 sc2 = f2_pack(sl2, sl2), nmu2 = f2_pack(-mu, -mu);
        f32x2 sum2[2] = {0ull, 0ull};
        // chunk c of 32 scores -> 16 packed P columns.  A chunk whose keys
        // are all masked for every row of the warp (the ragged end of a key
        // range, the far side of the causal diagonal) gets P = 0 without
        // exponentials: the exponential unit bounds this pass.
        auto exp_chunk = [&](const uint32_t (&v)[32], int c, bool masked) {
          uint32_t pw[16];
          if (masked) {
#pragma unroll
            for (int e = 0; e < 16; ++e) pw[e] = 0u;
            tmem_st16(tmem + lane_off + col_s + c * 16, pw);
            return;
          }
#pragma unroll
          for (int e = 0; e < 32; e += 2) {
            const f32x2 x2 =
                f2_fma(f2_pack(__uint_as_float(v[e]), __uint_as_float(v[e + 1])), sc2, nmu2);
            float p0, p1;
            if ((kPolyPairMask >> (e >> 1)) & 1u) {
              f2_unpack(exp2_poly2(x2), p0, p1);
            } else {
              float x0, x1;
              f2_unpack(x2, x0, x1);
              p0 = ex2(x0);
              p1 = ex2(x1);
            }
            sum2[(e >> 1) & 1] = f2_add(sum2[(e >> 1) & 1], f2_pack(p0, p1));
            __nv_bfloat162 hh = __floats2bfloat162_rn(p0, p1);
            pw[e >> 1] = *reinterpret_cast<uint32_t *>(&hh);
          }
          tmem_st16(tmem + lane_off + col_s + c * 16, pw);
        };
        exp_chunk(va, 0, need_mask && __all_sync(kFull, klast < 0));
        exp_chunk(vb, 1, need_mask && __all_sync(kFull, klast < 32));
        tmem_wait_st();
        float sa, sb2, sc, sd;
        f2_unpack(sum2[0], sa, sb2);
        f2_unpack(sum2[1], sc, sd);
        l += (sa + sb2) + (sc + sd);
        // The S(t + 2) that next writes this buffer waits for both PV halves
        // of this tile.
        tc_fence_before();
        mbar_arrive(&bar[B_P_FULL + 2 * (s_it & 1) + wg]);
      }
      if (!ok) break;
      // ---- end of item: merge factors for O = (O_0 e^{m_0 - M} + O_1 e^{m_1 - M}) /
      // (l_0 e^{m_0 - M} + l_1 e^{m_1 - M}).  Warpgroup 1 publishes its (m, l);
      // warpgroup 0 merges the two states and publishes f_w = e^{m_w - M} / L
      // for the epilogue warpgroup (in partial mode (M, L) also go to the
      // split-partial arrays).  Both warpgroups then go on to the next item.
      const bool partial = p.part.acc != nullptr;
      if (wg == 1) {
        if (item_no > 0)
          ok = __all_sync(kFull, mbar_wait(&bar[B_ML_FREE], (item_no - 1) & 1, abort_flag,
                                           p.status, p.wait_limit_ns, DBSA_ERR_TIMEOUT));
        if (!ok) break;
        sML[row] = make_float2(m_ref, l);
        mbar_arrive(&bar[B_ML_A]);
      } else {
        ok = __all_sync(kFull, mbar_wait(&bar[B_ML_A], item_no & 1, abort_flag, p.status,
                                         p.wait_limit_ns, DBSA_ERR_TIMEOUT));
        if (!ok) break;
        const float2 ml1 = sML[row];
        const float M = fmaxf(m_ref, ml1.x);
        const float w0 = (m_ref == -INFINITY) ? 0.f : ex2(m_ref - M);
        const float w1 = (ml1.x == -INFINITY) ? 0.f : ex2(ml1.x - M);
        const float L = l * w0 + ml1.y * w1;
        const float inv = L > 0.f ? 1.f / L : 0.f;
        sML[row] = make_float2(w0 * inv, w1 * inv);
        mbar_arrive(&bar[B_ML_B]);
        if (partial && row < it.n_rows) {
          const int grow = it.q_row0 + row;
          const int R = p.part.group * p.part.n_new;
          const int item = __ldg(p.part.packed_items + grow / R);
          const int w = grow % R;
          const int h = it.head * p.part.group + w % p.part.group;
          p.part.ml[((int64_t)item * p.part.Hq + h) * p.part.n_new + w / p.part.group] =
              make_float2(M, L);
        }
      }
    }
  } else if (warp >= kEpiWarp0 && warp < kEpiWarp0 + 4) {
    // ------------------------------------------------------------ Q tiles and epilogue
    // One thread per row (TMEM lane).  The Q tiles of the CTA's first two
    // items are written first.  Per item: the merge factors, then, once the
    // item's last PV is done (in-order tensor core: so are all of its PVs,
    // and the QK^T that read its Q tile), O_0 and O_1 are read and combined,
    // O is released for the next item's first PV, and the rows are written
    // out; the item's Q slot, which may have staged them, then takes the Q
    // tile of the item two ahead.
    const int quad = warp & 3;
    const int row = quad * 32 + lane;
    const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
    const bool partial = p.part.acc != nullptr;
    // The Q tile of item idx into slot qs; returns the position this
    // thread's row was rotated at.
    auto put_q = [&](int idx, uint32_t qs) -> int {
      const Item it = load_item(p.items, idx);
      uint8_t *tile = sQ + qs * TILE;
      const int pos = p.q_f32 ? rotate_q_row<D, float>(p, it, row, tile)
                              : rotate_q_row<D, bf16>(p, it, row, tile);
      fence_proxy_async_smem();   // visible to the tensor core's reads
      mbar_arrive(&bar[B_Q_FULL + qs]);
      return pos;
    };
    static_assert(kStagesQ == 2, "Q slots alternate between two items");
    int qpos0 = 0, qpos1 = 0;        // positions the rows in Q slots 0 and 1 were rotated at
    uint32_t n_staged0 = 0, n_staged1 = 0;   // staged items per Q slot so far
    if (ROTQ && blockIdx.x < p.n_items) qpos0 = put_q(blockIdx.x, 0);
    if (ROTQ && blockIdx.x + gridDim.x < p.n_items) qpos1 = put_q(blockIdx.x + gridDim.x, 1);
    uint32_t s_it = 0, item_no = 0;
    bool ok = true;
    for (int idx = blockIdx.x; ok && idx < p.n_items; idx += gridDim.x, ++item_no) {
      const Item it = load_item(p.items, idx);
      s_it += it.ntiles;
      const uint32_t last = s_it - 1;
      ok = __all_sync(kFull, mbar_wait(&bar[B_ML_B], item_no & 1, abort_flag, p.status,
                                       p.wait_limit_ns, DBSA_ERR_TIMEOUT));
      if (!ok) break;
      const float2 fw = sML[row];
      mbar_arrive(&bar[B_ML_FREE]);
      ok = __all_sync(kFull, mbar_wait(&bar[B_PV_DONE + (last & 1)], (last >> 1) & 1, abort_flag,
                                       p.status, p.wait_limit_ns, DBSA_ERR_TIMEOUT));
      if (!ok) break;
      tc_fence_after();
      int64_t prow = 0;
      if (partial && row < it.n_rows) {
        const int grow = it.q_row0 + row;                 // row of the packed query buffer
        const int R = p.part.group * p.part.n_new;
        const int item = __ldg(p.part.packed_items + grow / R);
        const int w = grow % R;
        const int h = it.head * p.part.group + w % p.part.group;
        prow = ((int64_t)item * p.part.Hq + h) * p.part.n_new + w / p.part.group;
      }
      const int64_t orow = ((int64_t)(it.q_row0 + row) * p.Hq + it.head) * D;
      uint16_t *pacc = partial ? p.part.acc + prow * D : nullptr;
      const uint32_t qs = item_no % kStagesQ;
      if (!stages_rows(it.ntiles)) {
        // fp32 output, or a short item: read, combine and store O 32 columns
        // at a time
#pragma unroll 1
        for (int col = 0; col < D; col += 32) {
          uint32_t o0[32], o1[32];
          tmem_ld32(tmem + lane_off + COL_O + col, o0);
          tmem_ld32(tmem + lane_off + COL_O + D + col, o1);
          tmem_wait_ld(o0);
          tmem_wait_ld(o1);
          if (row < it.n_rows) {
#pragma unroll
            for (int e = 0; e < 32; ++e)
              o0[e] = __float_as_uint(__uint_as_float(o0[e]) * fw.x + __uint_as_float(o1[e]) * fw.y);
            if (OUT_F32 && !partial) {
              float *dst = static_cast<float *>(p.out) + orow + col;
#pragma unroll
              for (int e = 0; e < 32; e += 4)
                *reinterpret_cast<uint4 *>(dst + e) = make_uint4(o0[e], o0[e + 1], o0[e + 2], o0[e + 3]);
            } else {
              uint16_t *dst = partial ? pacc + col : static_cast<uint16_t *>(p.out) + orow + col;
#pragma unroll
              for (int e = 0; e < 32; e += 8) {
                uint32_t w[4];
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                  __nv_bfloat162 hh = __floats2bfloat162_rn(__uint_as_float(o0[e + 2 * q]),
                                                            __uint_as_float(o0[e + 2 * q + 1]));
                  w[q] = *reinterpret_cast<uint32_t *>(&hh);
                }
                *reinterpret_cast<uint4 *>(dst + e) = make_uint4(w[0], w[1], w[2], w[3]);
              }
            }
          }
        }
        tc_fence_before();
        mbar_arrive(&bar[B_O_FREE]);
      } else {
        // bf16 rows of a long item: O is read, combined, packed and staged in
        // the item's Q tile (its last QK^T completed before its last PV),
        // then released for the next item's first PV, and the rows go out by
        // the bulk-copy engine as one contiguous piece each.  Per-thread
        // 16-byte global stores of 128 rows put 32 rows in flight per warp
        // instruction on the load/store pipe, which the softmax and issuing
        // warps share.
        // Row r of the staging tile holds its NC 16-byte chunks rotated by
        // r mod NC (chunk j in slot (j + r) mod NC), so that the 32 rows of a
        // warp's store fall in distinct bank groups; the copy then takes the
        // row in two contiguous pieces.
        constexpr int NC = D / 8;
        uint8_t *srow = sQ + qs * TILE + row * (D * 2);
        const int rot = row % NC;
#pragma unroll
        for (int col = 0; col < D; col += 16) {
          uint32_t o0[16], o1[16];
          tmem_ld16(tmem + lane_off + COL_O + col, o0);
          tmem_ld16(tmem + lane_off + COL_O + D + col, o1);
          tmem_wait_ld16(o0);
          tmem_wait_ld16(o1);
          uint32_t pk[8];
#pragma unroll
          for (int e = 0; e < 16; e += 2) {
            __nv_bfloat162 hh = __floats2bfloat162_rn(
                __uint_as_float(o0[e]) * fw.x + __uint_as_float(o1[e]) * fw.y,
                __uint_as_float(o0[e + 1]) * fw.x + __uint_as_float(o1[e + 1]) * fw.y);
            pk[e / 2] = *reinterpret_cast<uint32_t *>(&hh);
          }
          const int j = col / 8;   // chunks j, j + 1 of the row
          *reinterpret_cast<uint4 *>(srow + ((j + rot) % NC) * 16) =
              make_uint4(pk[0], pk[1], pk[2], pk[3]);
          *reinterpret_cast<uint4 *>(srow + ((j + 1 + rot) % NC) * 16) =
              make_uint4(pk[4], pk[5], pk[6], pk[7]);
        }
        tc_fence_before();
        mbar_arrive(&bar[B_O_FREE]);
        fence_proxy_async_smem();
        if (row < it.n_rows) {
          uint8_t *dst = reinterpret_cast<uint8_t *>(
              partial ? pacc : static_cast<uint16_t *>(p.out) + orow);
          const uint32_t s0 = smem_u32(srow);
          bulk_store(dst, s0 + rot * 16, (NC - rot) * 16);   // chunks 0 .. NC - rot - 1
          if (rot > 0) bulk_store(dst + (NC - rot) * 16, s0, rot * 16);
          bulk_commit();
        }
        bulk_wait_read();
        // once every row's copy has read the tile, the slot may take the Q
        // tile of the item two ahead (written below, or by the producer)
        mbar_arrive(&bar[B_Q_COPIED + qs]);
        if (ROTQ) {
          const uint32_t n_st = qs ? n_staged1++ : n_staged0++;
          ok = __all_sync(kFull, mbar_wait(&bar[B_Q_COPIED + qs], n_st & 1, abort_flag, p.status,
                                           p.wait_limit_ns, DBSA_ERR_TIMEOUT));
        }
      }
      if (partial && p.part.dbg != nullptr && it.head == 0 && row < it.n_rows) {
        // Gather map: the thread of an item's first packed row records, for
        // every key of the tile's range, the cache row its K and V tiles came
        // from and the fresh position that the two rotations combine to (the
        // query's token-0 position - the position this kernel rotated the
        // item's token-0 rows at + the key's block-relative position).
        const int grow = it.q_row0 + row;
        const int R = p.part.group * p.part.n_new;
        if (grow % R == 0) {
          const int item = __ldg(p.part.packed_items + grow / R);
          const S2Item si = p.part.items[item];
          const int qabs0 = p.part.queries[si.query].n_gathered + p.part.tail_len - p.part.n_new;
          const int shift = qabs0 - (ROTQ ? (qs ? qpos1 : qpos0) : p.part.q_rot_pos[item]);
          const int64_t room = p.part.dbg_cap - si.p_begin;
          const int n = si.p_begin < 0 ? 0 : (int)min((int64_t)it.len[0], room);
          int32_t *m = p.part.dbg + ((int64_t)si.query * p.part.dbg_cap + si.p_begin) * 2;
          const bool same_rows = it.k_row0[0] == it.v_row0[0];
          for (int r = 0; r < n; ++r)
            *reinterpret_cast<int2 *>(m + 2 * r) =
                make_int2(same_rows ? it.k_row0[0] + r : -2, shift + it.pos0[0] + r);
        }
      }
      const int nidx = idx + 2 * gridDim.x;
      if (ROTQ && ok && nidx < p.n_items) {
        const int pos = put_q(nidx, qs);
        if (qs) qpos1 = pos; else qpos0 = pos;
      }
    }
    bulk_wait_all();   // this thread's row copies have landed
  }
  __syncwarp();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

// ---------------------------------------------------------------- host side
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &f, 12000, cudaEnableDefault,
                                         &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
  });
  return fn;
}

// [heads][rows][D] bf16 view (head stride in rows), 128-row x 64-column boxes.
bool make_map(CUtensorMap *m, const void *ptr, int D, int64_t rows, int64_t heads,
              int64_t head_stride_rows) {
  auto enc = tensor_map_encoder();
  if (!enc) return false;
  cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)rows, (cuuint64_t)heads};
  cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)head_stride_rows * D * 2};
  cuuint32_t box[3] = {64, 128, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(ptr), dims, strides,
                   box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

template <int D>
constexpr size_t smem_bytes() {
  // tiles + epilogue exchange + barriers, + 1 KB for the manual 1024-byte
  // alignment of the swizzled tiles.  The request is padded above half an
  // SM's shared memory so that no two CTAs share an SM: each one allocates
  // all 512 TMEM columns.
  constexpr size_t need = 1024 + (size_t)128 * D * 2 * (kStagesQ + kStagesK + kStagesV) + 128 * sizeof(float2) +
                          B_COUNT * 8 + 16;
  constexpr size_t one_per_sm = 232448 / 2 + 1024;
  return need > one_per_sm ? need : one_per_sm;
}

template <int D, bool F32, bool STAGE, bool ROTQ>
cudaError_t launch_t(const CUtensorMap &mq, const CUtensorMap &mk, const CUtensorMap &mv,
                     const Params &p, int grid, cudaStream_t st) {
  constexpr size_t smem = smem_bytes<D>();
  static_assert(smem <= 232448, "shared memory budget");
  static_assert(smem > 232448 / 2, "one CTA per SM (the kernel owns all 512 TMEM columns)");
  cudaError_t e = cudaFuncSetAttribute(stage1_attn_kernel<D, F32, STAGE, ROTQ>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  pdl_launch(stage1_attn_kernel<D, F32, STAGE, ROTQ>, dim3(grid), dim3(kThreads), smem, st, mq, mk,
             mv, p);
  return cudaGetLastError();
}

// The launch shapes in use: Stage 1 always rotates its queries in the kernel
// (fp32 or bf16 outputs); partial-mode passes (bf16 partials) either way.
template <int D>
cudaError_t launch_shape(const CUtensorMap &mq, const CUtensorMap &mk, const CUtensorMap &mv,
                         const Params &p, int grid, bool f32, bool stage, bool rotq,
                         cudaStream_t st) {
  if (f32)
    return rotq ? launch_t<D, true, false, true>(mq, mk, mv, p, grid, st) : cudaErrorInvalidValue;
  if (stage)
    return rotq ? launch_t<D, false, true, true>(mq, mk, mv, p, grid, st)
                : launch_t<D, false, true, false>(mq, mk, mv, p, grid, st);
  return rotq ? launch_t<D, false, false, true>(mq, mk, mv, p, grid, st)
              : launch_t<D, false, false, false>(mq, mk, mv, p, grid, st);
}

}  // namespace

cudaError_t launch_stage1(const Stage1Args &a, int head_dim, bool out_f32, int num_sms,
                          cudaStream_t st) {
  if (a.n_items <= 0) return cudaSuccess;
  // queries rotated here (q_src) or pre-rotated rows loaded by TMA (q_rot)
  const bool rotq = a.q_src != nullptr;
  if (rotq ? (a.part.acc != nullptr && a.part.item_meta == nullptr) : a.q_rot == nullptr)
    return cudaErrorInvalidValue;
  CUtensorMap mq, mk, mv;
  if (!make_map(&mk, a.k_rot, head_dim, a.k_rows, a.Hkv, a.k_rows) ||
      !make_map(&mv, a.v, head_dim, a.v_rows, a.Hkv, a.v_head_stride))
    return cudaErrorInvalidValue;
  if (rotq)
    mq = mk;   // a placeholder: the kernel reads no Q tile through it
  else if (!make_map(&mq, a.q_rot, head_dim, a.q_rows, a.Hq, a.q_rows))
    return cudaErrorInvalidValue;
  Params p;
  p.items = a.items;
  p.n_items = a.n_items;
  p.group = a.Hq / a.Hkv;
  p.Hq = a.Hq;
  p.out = a.out;
  p.scale_log2 = a.scale_log2;
  p.status = a.status;
  p.wait_limit_ns = a.wait_limit_ns != 0 ? a.wait_limit_ns : kWaitLimitNs;
  p.withhold_tiles = a.withhold_tiles;
  p.part = a.part;
  p.q_src = a.q_src;
  p.q_f32 = a.q_f32;
  p.q_heads = a.q_heads;
  p.rope = a.rope;
  const int grid = a.n_items < num_sms ? a.n_items : num_sms;
  // Rows are staged (bf16 outputs) except in passes with few query rows per
  // (query, KV head) (decode steps): those stream their K/V from HBM and keep
  // the TMA unit busy with loads, so their rows are stored directly rather
  // than queued on it as bulk copies.
  const bool stage =
      !out_f32 && (a.part.acc == nullptr || a.part.group * a.part.n_new >= 32);
  if (head_dim == 128) return launch_shape<128>(mq, mk, mv, p, grid, out_f32, stage, rotq, st);
  return launch_shape<64>(mq, mk, mv, p, grid, out_f32, stage, rotq, st);
}

}  // namespace dbsa
