// Internal declarations of the DBSA library: device-visible plan structs and
// the launchers each kernel file provides.  Not part of the public ABI.
#pragma once

#include <cstddef>
#include <cstdint>

#include <cuda_runtime.h>

#include "../../include/dbsa.h"

namespace dbsa {

// Programmatic dependent launch.  Every kernel of the library is launched
// with programmatic stream serialisation and starts with pdl_enter(): it
// waits there until the previous kernel in the stream has completed and its
// memory is visible (griddepcontrol.wait), then lets the next kernel be
// scheduled (griddepcontrol.launch_dependents; the next grid is scheduled
// once every CTA of this one has started, and waits in its own pdl_enter).
// Nothing before pdl_enter() touches global memory, so the overlap is the
// launch latency and the next kernel's block scheduling, not data.
__device__ __forceinline__ void pdl_enter() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
template <typename... KArgs, typename... Args>
cudaError_t pdl_launch(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t st, Args &&...args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<Args &&>(args)...);
}

constexpr int kTileRows = 128;   // Stage-1 query rows per tile (tcgen05 M)
constexpr int kTileKeys = 128;   // Stage-1 keys per score tile (tcgen05 N)
constexpr int kRopeLo = 16;      // positions per RoPE "hi" table step
constexpr int kRopeShift = 4;    // log2(kRopeLo)

// Head of every workspace: the device status word (cleared by each call).
constexpr size_t kStatusBytes = 256;

// RoPE angle factors, built on the device in fp64 and stored as fp32 in
// planar form: hc/hs[a][i] = cos/sin(16a * w_i), lc/ls[r][i] = cos/sin(r * w_i)
// (r < 16), w_i = theta^(-2i/D), each [rows][D/2].  Position p uses the
// complex product hi[p >> 4] * lo[p & 15].
struct RopeTables {
  const float *hc, *hs;
  const float *lc, *ls;
  int32_t n_hi;
};

// Stage 2: per-query metadata, gathered segments and split items.
struct S2Segment {
  int32_t cache_row0;  // first cache row of the block
  int32_t pos0;        // fresh position of its first token
  int32_t len;         // tokens
  int32_t query;       // the query that selected it
};
struct S2Query {
  int32_t seg_begin;   // index into the segment array
  int32_t n_seg;
  int32_t n_gathered;  // T'_q
  int32_t item_begin;  // first split item of this query
  int32_t n_items;
  int32_t pad[3];
};
struct S2Item {
  int32_t query;
  int32_t p_begin;     // key positions [p_begin, p_end) of the query's key sequence;
  int32_t p_end;       // p_begin is a multiple of 16 (the kernel's RoPE step)
  int32_t p_lo;        // keys below p_lo (>= p_begin) belong to other items: masked
};
// ---- launchers (each returns cudaGetLastError() after enqueueing) ----

// Fills the four tables (laid out back to back from `base`: hc, hs, lc, ls).
cudaError_t launch_rope_tables(float *base, int32_t n_hi, int32_t head_dim, double theta,
                               cudaStream_t st);
// Table pointers inside a block of rope_table_bytes() starting at `base`.
RopeTables rope_tables_at(const float *base, int32_t n_hi, int32_t head_dim);
size_t rope_table_bytes(int32_t n_hi, int32_t head_dim);

// Rotate K of n_tok token-major input rows (positions pos0..), copy the raw
// K/V into the cache rows pos0.., and (f32 inputs) write bf16 V.  (The
// queries are rotated by the tensor-core kernel as it reads them.)
struct IngestArgs {
  const void *k, *v;               // [n_tok][Hkv][D] input dtype
  int32_t n_tok, pos0;
  int32_t Hkv;
  void *k_rot;                     // bf16 [Hkv][k_rows][D], row k_row_base + t
  int64_t k_rows;
  int32_t k_row_base;
  void *v_bf16;                    // bf16 [Hkv][k_rows][D] (f32 inputs only) or null
  void *k_cache, *v_cache;         // input dtype [Hkv][cap][D], row pos0 + t
  int64_t cap;
  RopeTables rope;
};
cudaError_t launch_ingest(const IngestArgs &a, int head_dim, bool f32, cudaStream_t st);

// Rotate cache rows [row0, row0+n) (positions = rows) into k_rot rows
// dst_row0.. and (f32) convert the V rows to bf16 scratch rows.
struct WindowArgs {
  const void *k_cache, *v_cache;
  int64_t cap;
  int32_t Hkv;
  int32_t row0, n;
  void *k_rot;
  int64_t k_rows;
  int32_t dst_row0;
  void *v_bf16;
  RopeTables rope;
};
cudaError_t launch_window(const WindowArgs &a, int head_dim, bool f32, cudaStream_t st);

// Split partials (Stage 2): per (item, head, token) row, (M, L) in fp32 (M
// the row's score maximum in log2 units, L the sum of 2^(s - M) over the
// item's keys) and the item's normalised output O_item = sum p v / L as bf16
// (a convex combination of V rows, so it keeps V's range).  The merge forms
// O = sum_i 2^(M_i - M) L_i O_i / sum_i 2^(M_i - M) L_i.
//
// Partial-output mode of the tensor-core attention kernel (Stage 2, block-
// major): every split item owns group * n_new consecutive rows of the packed
// query buffer (token-major: u * group + local head), so row r belongs to item
// packed_items[r / (group * n_new)]; the kernel writes the partial of each row
// at index ((item * Hq + head) * n_new + u).
struct Stage1Partial {
  uint16_t *acc;               // bf16 normalised outputs; null: plain mode
  float2 *ml;
  const int32_t *packed_items; // item of each group * n_new packed rows
  int32_t group, Hq, n_new;
  // Gather map (null: not requested), [nq][dbg_cap][2].  For every item whose
  // first packed row falls in a tile of KV head 0, the epilogue writes, for
  // each key r of the tile's range, entry [query][p_begin + r] = (the cache
  // row its K and V tiles were loaded from, the fresh position the pair of
  // rotations gives it: the query's token-0 position minus the position the
  // kernel rotated the item's token-0 query rows at plus the key's
  // block-relative position).
  int32_t *dbg;
  int64_t dbg_cap;
  const S2Item *items;
  const S2Query *queries;
  // per item (first packed row or -1, the position its query rows are
  // rotated at for token 0, its query, 0): read where the kernel rotates the
  // packed query rows (q_src set)
  const int4 *item_meta;
  // passes whose packed rows qhat_kernel rotated (q_rot set): per item, the
  // position it rotated token 0 at
  const int32_t *q_rot_pos;
  int32_t tail_len;
};

// Stage 2, block-major tensor-core passes: keys of every cache row rotated
// at their position inside their own block (row s of block b at s - offs[b]);
// fp32 caches also get a bf16 copy of V.
struct RelRopeArgs {
  const void *k_cache, *v_cache;   // [Hkv][cap][D], input dtype
  int64_t cap;
  int32_t Hkv, T, nb;
  const int32_t *offs;             // device copy, [nb + 1]
  void *k_hat;                     // bf16 [Hkv][T][D]
  void *v_bf16;                    // bf16 [Hkv][T][D] (fp32 caches only) or null
  RopeTables rope;
};
cudaError_t launch_rel_rope(const RelRopeArgs &a, int head_dim, bool f32, cudaStream_t st);

// Packed query rows of the block-major pass: rows item_meta[i].x .. + g*n_new
// of kv head c are query token u / local head hl (row u * g + hl) of split
// item i (a (query, block) pair), rotated at (its position - the block's
// fresh start), i.e. at item_meta[i].y + u.
struct QHatArgs {
  const void *q_new;               // [nq][n_new][Hq][D]
  int32_t n_new, tail_len, Hq, Hkv;
  int32_t n_items;                 // items (tail items have item_meta.x = -1)
  // per item: (first packed row, position of token 0's rotation, query, 0)
  const int4 *item_meta;
  int32_t rows;                    // packed rows per kv head
  void *q_hat;                     // bf16 [Hkv][rows][D]
  int32_t *q_rot_pos;              // per item: rotation position of token 0, or null
  RopeTables rope;
};
cudaError_t launch_qhat(const QHatArgs &a, int head_dim, bool f32, cudaStream_t st);

// Compact mode of Stage 2: every query's gathered keys, rotated at their fresh
// positions, and its values, bf16 [Hkv][rows][D]; query q's gathered token p
// goes to row base[q] + p.  With dbg non-null, dbg[q][p] = (cache row, p).
struct CompactArgs {
  const void *k_cache, *v_cache;   // [Hkv][cap][D], input dtype
  int64_t cap;
  int32_t Hkv;
  const S2Segment *segs;           // every query's segments
  int32_t n_segs;
  const int32_t *base;             // [nq]: compact row of each query's first gathered token
  int64_t rows;                    // sum of the queries' gathered tokens
  void *k_hat, *v_hat;             // bf16 [Hkv][rows][D]
  int32_t *dbg;
  int64_t dbg_cap;
  RopeTables rope;
};
cudaError_t launch_compact(const CompactArgs &a, int head_dim, bool f32, cudaStream_t st);

// Stage-1 tcgen05 attention over a tile list.
struct Stage1Args {
  // The queries, in one of two forms.  q_src (non-null): unrotated, bf16 or
  // fp32 (q_f32), rotated by the kernel itself as it fills each Q tile.
  // Stage 1: [rows][q_heads][D], row q_row0 + r of an item at position
  // q_pos0 + r.  Partial mode: [queries][n_new][q_heads][D], packed rows
  // found through part.packed_items and part.item_meta.  Otherwise q_rot:
  // already rotated bf16 [Hq][q_rows][D] rows, loaded by TMA.
  const void *q_src;
  int32_t q_f32, q_heads;
  RopeTables rope;
  const void *q_rot;
  int64_t q_rows;
  const void *k_rot;      // bf16 [Hkv][k_rows][D]
  int64_t k_rows;
  const void *v;          // bf16 [Hkv][v_rows] rows, head stride v_head_stride rows
  int64_t v_rows, v_head_stride;
  void *out;              // [out_rows][Hq][D], bf16 or f32
  int32_t Hq, Hkv;
  const dbsa_tile_item *items;
  int32_t n_items;
  float scale_log2;       // softmax scale * log2(e)
  int *status;
  uint64_t wait_limit_ns; // limit of every bounded wait (0: the 4 s default)
  int32_t withhold_tiles; // test hook: load no tile, so every wait runs out
  Stage1Partial part;     // part.acc == null for Stage 1 itself
};
cudaError_t launch_stage1(const Stage1Args &a, int head_dim, bool out_f32, int num_sms,
                          cudaStream_t st);

// Stage-2 split-KV gather + re-RoPE + attention, then the split merge.
struct Stage2Args {
  const void *k_cache, *v_cache;   // [Hkv][cap][D]
  int64_t cap;
  const void *q_new;               // [nq][n_new][Hq][D]
  const void *k_tail, *v_tail;     // [nq][tail_cap][Hkv][D]
  int32_t tail_len, tail_cap, n_new;
  int32_t Hq, Hkv;
  const S2Query *queries;
  const S2Segment *segs;
  const S2Item *items;
  int32_t n_items, n_queries;
  const int32_t *run_items;        // the tail items, which the per-query kernel runs
  int32_t n_run;
  uint16_t *part_acc;              // bf16 [n_items][Hq][n_new][D], normalised (see above)
  float2 *part_ml;                 // [n_items][Hq][n_new] (m in log2 units, l)
  void *out;                       // [nq][n_new][Hq][D]
  // [nq][dbg_cap][2] or null: the per-query kernel writes (cache row, the
  // position its rotation used) for every gathered key it loads (KV head 0,
  // first row group)
  int32_t *dbg_map;
  int64_t dbg_cap;
  float scale_log2;
  RopeTables rope;
};
// Sets the message dbsa_last_error() returns on this thread.
void set_last_error(const char *msg);

// Scratch owned by the library rather than the caller: `bytes` of device
// memory whose address (on the current device) resolve() returns.
struct FixedScratch {
  size_t bytes;
  cudaError_t (*resolve)(void **ptr);
};
// Stage 2 out of a FixedScratch (dbsa_gather_rope_attend_noalloc): the call is
// validated and planned before the scratch is resolved, a batch that does
// not fit is rejected with DBSA_ERR_WORKSPACE, and the plan goes to the
// device with one cudaMemcpyAsync from pageable host memory (no page-locked
// staging, no events).  Otherwise as dbsa_gather_rope_attend.
dbsa_status gather_fixed_scratch(const dbsa_config *cfg, const void *k_cache, const void *v_cache,
                                 int64_t cap, const int32_t *offs_host, int32_t nb, int32_t nq,
                                 const int32_t *sel_ptr_host, const int32_t *sel_blocks_host,
                                 const void *q_new, int32_t n_new, const void *k_tail,
                                 const void *v_tail, int32_t tail_len, int32_t tail_cap,
                                 void *out, int32_t *dbg_map, int64_t dbg_cap,
                                 const FixedScratch &fixed, void *stream);

cudaError_t launch_stage2_main(const Stage2Args &a, int head_dim, bool f32, cudaStream_t st);
// Block-major mode: every query's tail tokens and the merge of all its
// partials, writing the output (replaces the per-query kernel's tail items
// and the merge).
cudaError_t launch_stage2_tail_merge(const Stage2Args &a, int head_dim, bool f32,
                                     cudaStream_t st);
cudaError_t launch_stage2_merge(const Stage2Args &a, int head_dim, bool f32, cudaStream_t st);

}  // namespace dbsa
