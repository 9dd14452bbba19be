/*
 * dbsa.h -- C ABI of the DBSA attention engine for NVIDIA B200 (sm_100a).
 *
 * Dynamic Block-Sparse Attention for many-shot in-context learning, as stated
 * on the paper-notes page "Efficient Many-Shot In-Context Learning with
 * Dynamic Block-Sparse Attention" (ACL 2025), cited below as [DBSA notes]:
 *
 *   Stage 1 (§Stage 1, block-sparse streaming attention encoding): the
 *   demonstrations are grouped into blocks b_1..b_nb; every token of block
 *   b_i attends to the sink block b_1, the previous j blocks and, causally,
 *   its own block, with RoPE at sequential positions; the K/V cache is kept
 *   BEFORE the rotary transform, and a new block can be encoded alone.
 *
 *   Stage 2 (§Stage 2, dynamic demonstration selection and generation): per
 *   query, the retrieved blocks (sink always first) are concatenated, RoPE is
 *   re-applied to their cached keys at fresh sequential positions, and the
 *   query tokens attend with full attention over that cache.
 *
 * Conventions shared by every call
 * --------------------------------
 *  - One call = one transformer layer.  The caller passes that layer's
 *    pointers; layers are independent.
 *  - Blocks are numbered from 0 in this ABI: block 0 is the page's b_1, the
 *    sink.  Block b holds tokens [offs[b], offs[b+1]) of the context.
 *  - Positions are token positions (0..T-1 in Stage 1; 0..T'-1 over the
 *    gathered tokens in Stage 2; query tokens continue at T' + u).
 *  - RoPE is the rotate-half form: for i < d/2 the pair (x_i, x_{i+d/2}) is
 *    rotated by pos * theta^(-2i/d).  Query head h reads KV head
 *    h / (n_q_heads / n_kv_heads).  Scores are scaled by softmax_scale
 *    (1/sqrt(head_dim) when softmax_scale <= 0).
 *  - Element type: cfg->dtype for every activation, cache and output buffer
 *    (DBSA_BF16: bfloat16; DBSA_F32: float).  Tensor-core operands are bf16
 *    in both cases, accumulation and softmax are fp32.
 *  - Ownership: the caller owns every buffer.  Device pointers (marked
 *    "device") must be 16-byte aligned.  Host pointers ("host") are read
 *    during the call only.  The library never allocates or frees device
 *    memory: it works in the caller's `workspace`, whose size the matching
 *    *_workspace_size() call returns.
 *  - Asynchrony: work is enqueued on `stream` (a cudaStream_t; NULL = the
 *    legacy default stream).  A call returns after validation, host
 *    planning and enqueueing.  Host arrays may be freed on return.
 *  - Errors: every call returns a dbsa_status.  On any status other than
 *    DBSA_OK no kernel was enqueued and no output was touched, except
 *    DBSA_ERR_CUDA (a launch failed; outputs undefined).  dbsa_last_error()
 *    returns a per-thread message for the last failure.  A kernel whose
 *    bounded wait expired writes DBSA_ERR_TIMEOUT into the status word at
 *    the head of the workspace; dbsa_read_status() reads it.
 */
#ifndef DBSA_H
#define DBSA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum dbsa_status {
    DBSA_OK = 0,
    DBSA_ERR_INVALID_ARG = 1,  /* bad pointer, size, offset table or selection */
    DBSA_ERR_UNSUPPORTED = 2,  /* head_dim / head ratio / dtype not supported */
    DBSA_ERR_CAPACITY = 3,     /* cache capacity too small */
    DBSA_ERR_WORKSPACE = 4,    /* workspace missing, misaligned or too small */
    DBSA_ERR_CUDA = 5,         /* a CUDA call failed */
    DBSA_ERR_TIMEOUT = 6       /* a device-side bounded wait expired */
} dbsa_status;

typedef enum dbsa_dtype { DBSA_BF16 = 0, DBSA_F32 = 1 } dbsa_dtype;

/* Stage-1 attention patterns: the DBSA pattern (§Stage 1, item 2) and the
 * alternatives of [DBSA notes] §Ablations › sparse attention patterns. */
typedef enum dbsa_pattern {
    DBSA_PATTERN_SINK_PREV_SELF = 0, /* sink + previous j blocks + causal self */
    DBSA_PATTERN_FULL = 1,           /* full causal attention */
    DBSA_PATTERN_SINK_SELF = 2,      /* sink + causal self */
    DBSA_PATTERN_SELF = 3            /* causal self only */
} dbsa_pattern;

typedef struct dbsa_config {
    int32_t n_q_heads;     /* Hq */
    int32_t n_kv_heads;    /* Hkv; Hq % Hkv == 0 and Hq / Hkv <= 64 */
    int32_t head_dim;      /* D: 64 or 128 */
    int32_t dtype;         /* dbsa_dtype */
    double rope_theta;     /* RoPE base, e.g. 1e4 (Llama-2) or 5e5 (Llama-3.1) */
    int32_t window_j;      /* j, previous blocks each block attends to (>= 0) */
    int32_t pattern;       /* dbsa_pattern (Stage 1 only) */
    float softmax_scale;   /* <= 0 selects 1/sqrt(head_dim) */
    int32_t reserved;      /* must be 0 */
} dbsa_config;

/* ---------------------------------------------------------------------------
 * Block table ([DBSA notes] §Stage 1, item 1; §Configuration parameters:
 * 50 demonstrations per block).
 * Groups n_demos demonstrations of lengths demo_len[0..n_demos) (host, each
 * >= 1 token) into blocks of k, in the given order, and writes the token
 * offsets offs_out[0..nb] (host, room for ceil(n_demos/k)+1 entries),
 * offs_out[0] = 0.  The last block holds the remainder when k does not
 * divide n_demos.  Returns nb, or -1 on bad arguments (see dbsa_last_error).
 * ------------------------------------------------------------------------ */
int32_t dbsa_group_blocks(const int32_t *demo_len, int32_t n_demos, int32_t k,
                          int32_t *offs_out);

/* ---------------------------------------------------------------------------
 * Stage 1: block-sparse streaming prefill of a whole demonstration set
 * ([DBSA notes] §Stage 1, items 2-3).
 *
 *   q        device, [T][Hq][D]   pre-RoPE queries of the T context tokens
 *   k, v     device, [T][Hkv][D]  pre-RoPE keys and values
 *   offs_host host, [nb+1]        block offsets, offs[0] = 0, strictly
 *                                 increasing, offs[nb] = T
 *   k_cache, v_cache device, [Hkv][cap][D]  receive the pre-RoPE K and V of
 *                                 every token (rows [0, T) of each head),
 *                                 bit-identical to k and v; cap >= T
 *   out      device, [T][Hq][D]   attention output of every token
 *   workspace device, ws_bytes >= dbsa_encode_workspace_size(cfg, T, nb)
 *
 * Row t of block b attends to the keys s <= t with s in block 0, in blocks
 * b-j .. b-1 or in block b (cfg->pattern selects an ablation instead).
 * q/k/v may not alias k_cache/v_cache/out.
 * Errors: INVALID_ARG (null pointer, bad offsets, T = 0), UNSUPPORTED
 * (head_dim, Hq/Hkv, dtype), CAPACITY (cap < T), WORKSPACE, CUDA.
 * ------------------------------------------------------------------------ */
size_t dbsa_encode_workspace_size(const dbsa_config *cfg, int64_t n_tokens,
                                  int32_t nb);
dbsa_status dbsa_encode_blocks(const dbsa_config *cfg, const void *q,
                               const void *k, const void *v,
                               const int32_t *offs_host, int32_t nb,
                               void *k_cache, void *v_cache, int64_t cap,
                               void *out, void *workspace, size_t ws_bytes,
                               void *stream);

/* ---------------------------------------------------------------------------
 * Stage 1, incremental: encode ONE new block b_{nb+1} after nb encoded
 * blocks ([DBSA notes] §Stage 1, item 4: a new demonstration block costs one
 * more block's encoding, independent of the pool size).
 *
 *   q        device, [L][Hq][D]  pre-RoPE queries of the new block's L tokens
 *   k, v     device, [L][Hkv][D] pre-RoPE keys / values of the new block
 *   offs_host host, [nb+1]       offsets of the EXISTING blocks (offs[nb] =
 *                                T0, the tokens already in the cache)
 *   k_cache, v_cache device, [Hkv][cap][D]: rows [0, T0) hold the encoded
 *                                blocks; rows [T0, T0+L) receive the new
 *                                block's pre-RoPE K/V; cap >= T0 + L
 *   out      device, [L][Hq][D]  output of the new block's tokens
 *
 * The new tokens sit at positions T0 .. T0+L-1 and attend exactly as the
 * last block of dbsa_encode_blocks over nb+1 blocks would.
 * Errors: as dbsa_encode_blocks; L must be >= 1.
 * ------------------------------------------------------------------------ */
size_t dbsa_append_workspace_size(const dbsa_config *cfg,
                                  const int32_t *offs_host, int32_t nb,
                                  int32_t L);
dbsa_status dbsa_append_block(const dbsa_config *cfg, const void *q,
                              const void *k, const void *v, int32_t L,
                              const int32_t *offs_host, int32_t nb,
                              void *k_cache, void *v_cache, int64_t cap,
                              void *out, void *workspace, size_t ws_bytes,
                              void *stream);

/* ---------------------------------------------------------------------------
 * Stage 2: per-query gather + RoPE re-rotation + GQA attention
 * ([DBSA notes] §Stage 2, items 2-4).
 *
 *   k_cache, v_cache device, [Hkv][cap][D]  pre-RoPE cache from Stage 1
 *   offs_host  host, [nb+1]     block offsets of the cache
 *   nq                          number of queries in the batch
 *   sel_ptr_host host, [nq+1]   CSR row pointer into sel_blocks_host
 *   sel_blocks_host host        per query: selected block ids; the first
 *                               MUST be 0 (the sink), ids unique, < nb.
 *                               Their order is the order of concatenation.
 *   q_new    device, [nq][n_new][Hq][D]  pre-RoPE queries of the n_new
 *                               newest tokens of each query (n_new = the
 *                               prompt length for the prompt pass, 1 per
 *                               decode step)
 *   k_tail, v_tail device, [nq][tail_cap][Hkv][D]  pre-RoPE K/V of each
 *                               query's own tokens so far; the last n_new
 *                               of the tail_len tokens are q_new's tokens
 *                               (the caller writes them before the call)
 *   out      device, [nq][n_new][Hq][D]
 *   dbg_map  device or NULL, [nq][dbg_cap][2] int32, 8-byte aligned: when
 *                               given, entry [q][p] receives, for every
 *                               gathered token p of query q, the pair (cache
 *                               row, position) written by the attention
 *                               kernel that consumes that key: the cache row
 *                               its K and V were loaded from (-2 if the two
 *                               differ) and the fresh position its rotation
 *                               used.  On the block-by-block tensor-core path
 *                               that position is the query's token-0
 *                               position minus the position the query rows
 *                               were rotated at, plus the key's offset
 *                               inside its block; on the per-query path it is
 *                               the position of the rotation table entries
 *                               applied.  Correct results have position p.
 *                               Entries p >= T'_q are untouched.
 *
 * Query q's gathered cache is the concatenation of its selected blocks'
 * tokens; gathered token p gets position p (0 .. T'_q-1).  Query token u
 * (tail token tu = tail_len - n_new + u) sits at position T'_q + tu and
 * attends to every gathered token and to tail tokens 0..tu.
 * Errors: INVALID_ARG (selection without leading sink, duplicate or
 * out-of-range block, tail_len < n_new, tail_len > tail_cap, dbg_cap too
 * small), UNSUPPORTED, CAPACITY (offs[nb] > cap), WORKSPACE, CUDA.
 * ------------------------------------------------------------------------ */
size_t dbsa_gather_workspace_size(const dbsa_config *cfg,
                                  const int32_t *offs_host, int32_t nb,
                                  int32_t nq, const int32_t *sel_ptr_host,
                                  const int32_t *sel_blocks_host,
                                  int32_t n_new, int32_t tail_len);
dbsa_status dbsa_gather_rope_attend(
    const dbsa_config *cfg, const void *k_cache, const void *v_cache,
    int64_t cap, const int32_t *offs_host, int32_t nb, int32_t nq,
    const int32_t *sel_ptr_host, const int32_t *sel_blocks_host,
    const void *q_new, int32_t n_new, const void *k_tail, const void *v_tail,
    int32_t tail_len, int32_t tail_cap, void *out, int32_t *dbg_map,
    int64_t dbg_cap, void *workspace, size_t ws_bytes, void *stream);

/* ---------------------------------------------------------------------------
 * Stage 2 with prepared block keys ([DBSA notes] §Stage 2, item 3: RoPE is
 * re-applied to the cached keys at the gathered positions).
 *
 * Gathered token p of query q sits at P + r, where P is the fresh start of
 * its block in that query and r its offset inside the block; since
 * R(a)^T R(b) = R(b - a), the score of (query row, key) factors into the key
 * rotated at r and the query row rotated at (its position - P).  The rotated
 * keys R(r) k depend on the cache only, so one dbsa_block_keys() call serves
 * every query batch and decode step until the cache changes (an encode or an
 * append), and dbsa_gather_rope_attend_prepared() skips that rotation.
 *
 *   block_keys device, bk_bytes >= dbsa_block_keys_size(cfg, offs, nb),
 *              256-byte aligned, owned by the caller: the keys of every cache
 *              row s of block b rotated at s - offs[b] (bf16, [Hkv][T][D]),
 *              a bf16 copy of V for DBSA_F32 caches, and RoPE angle tables
 *              for positions below T + 8192 (a prepared gather whose
 *              positions fit, i.e. tail_len <= 8192, uses them instead of
 *              building its own).
 *
 * dbsa_gather_rope_attend_prepared takes the arguments of
 * dbsa_gather_rope_attend plus block_keys, which must come from
 * dbsa_block_keys() on the same cfg, cache contents, cap and offsets (not
 * checked).  Results are bit-identical to dbsa_gather_rope_attend.  Its
 * workspace may be the size dbsa_gather_workspace_size() returns (an upper
 * bound: the rotated keys are not placed in it).
 * Errors: as dbsa_gather_rope_attend; WORKSPACE also for a missing,
 * misaligned or too small block_keys buffer.
 * ------------------------------------------------------------------------ */
size_t dbsa_block_keys_size(const dbsa_config *cfg, const int32_t *offs_host,
                            int32_t nb);
dbsa_status dbsa_block_keys(const dbsa_config *cfg, const void *k_cache,
                            const void *v_cache, int64_t cap,
                            const int32_t *offs_host, int32_t nb,
                            void *block_keys, size_t bk_bytes, void *stream);
dbsa_status dbsa_gather_rope_attend_prepared(
    const dbsa_config *cfg, const void *k_cache, const void *v_cache,
    int64_t cap, const int32_t *offs_host, int32_t nb, int32_t nq,
    const int32_t *sel_ptr_host, const int32_t *sel_blocks_host,
    const void *q_new, int32_t n_new, const void *k_tail, const void *v_tail,
    int32_t tail_len, int32_t tail_cap, void *out, int32_t *dbg_map,
    int64_t dbg_cap, const void *block_keys, size_t bk_bytes, void *workspace,
    size_t ws_bytes, void *stream);

/* ---------------------------------------------------------------------------
 * Stage 2 without a workspace.  The paper has no counterpart: this is a
 * calling convention of this library, not a step of the method.
 *
 * For callers that cannot allocate device memory when they call in, such as
 * code that runs inside another framework's fixed memory budget or a host
 * thread that must not call cudaMalloc (it may synchronise the device).
 * Same arguments, results and errors as dbsa_gather_rope_attend, minus the
 * workspace; the outputs are bit-identical to that call's.  The scratch is
 * one array of 16 MiB in the library's device memory, held by every GPU that
 * loads the library until the process exits.
 *  - A batch whose dbsa_gather_workspace_size() exceeds 16 MiB is rejected
 *    with DBSA_ERR_WORKSPACE and a message naming both sizes; nothing runs.
 *  - The first call on a device looks up the array's device address (with
 *    that device current) and keeps it; make that first call before any
 *    stream capture.
 *  - Every call on a device shares the one array and leaves its contents
 *    behind; the call clears the status word it needs at zero.  Calls whose
 *    work overlaps on the GPU (other streams, other host threads) race on the
 *    array: serialise them.
 *  - Its device status word is read with dbsa_noalloc_read_status(), not
 *    dbsa_read_status() (there is no caller workspace).
 * It allocates nothing: no cudaMalloc, cudaFree, page-locked host memory,
 * event or other allocating library call.  Its plan tables reach the device
 * with one cudaMemcpyAsync from pageable host memory, which returns once the
 * driver has taken the bytes (it may wait for the stream's earlier copies).
 * ------------------------------------------------------------------------ */
dbsa_status dbsa_gather_rope_attend_noalloc(
    const dbsa_config *cfg, const void *k_cache, const void *v_cache,
    int64_t cap, const int32_t *offs_host, int32_t nb, int32_t nq,
    const int32_t *sel_ptr_host, const int32_t *sel_blocks_host,
    const void *q_new, int32_t n_new, const void *k_tail, const void *v_tail,
    int32_t tail_len, int32_t tail_cap, void *out, int32_t *dbg_map,
    int64_t dbg_cap, void *stream);

/* ---------------------------------------------------------------------------
 * Status and introspection.
 * ------------------------------------------------------------------------ */

/* Message of the last failed call on this thread ("" if none). Never NULL. */
const char *dbsa_last_error(void);

/* Synchronises `stream`, reads the device status word at the head of
 * `workspace` (device) and returns it (DBSA_OK or DBSA_ERR_TIMEOUT), or
 * DBSA_ERR_CUDA if the copy failed.  The word is cleared by each call that
 * uses the workspace. */
dbsa_status dbsa_read_status(const void *workspace, void *stream);

/* The same for the scratch of dbsa_gather_rope_attend_noalloc on the current
 * device: synchronises `stream` and returns the status word its last call
 * left (DBSA_OK or DBSA_ERR_TIMEOUT), or DBSA_ERR_CUDA. */
dbsa_status dbsa_noalloc_read_status(void *stream);

/* Test hook of the failure detection, for the NEXT call on this thread only
 * (0 = no hook).  Every device wait of the tensor-core kernel is bounded (4 s
 * by default); when one runs out, the kernel writes DBSA_ERR_TIMEOUT to the
 * status word, finishes its copies and tensor-core work in flight, releases
 * its tensor memory and returns, leaving the context usable.  With the hook,
 * that call's kernel loads no tile, so each of its waits is for a barrier
 * that nothing completes, and they give up after `limit_ns` nanoseconds: the
 * call's status reads DBSA_ERR_TIMEOUT and its outputs are incomplete.
 * Cleared by the call.  For tests only. */
void dbsa_test_wait_expiry(uint64_t limit_ns);

/* Calls this library has made (all threads) that allocate or free
 * page-locked host memory or create or destroy CUDA events: the plan staging
 * of the workspace-taking calls, on a thread's first calls and when a plan
 * outgrows the staging capacity (which then doubles, and each of the eight
 * staging slots is brought up to it on its next use).
 * dbsa_gather_rope_attend_noalloc makes none. */
int64_t dbsa_host_allocation_calls(void);

/* One Stage-1 tile-list entry: a 128-row query tile of one head, and at most
 * two key ranges (the sink block, then the window up to the diagonal). */
typedef struct dbsa_tile_item {
    int32_t head;       /* query head */
    int32_t q_row0;     /* first query row (row of q / out) */
    int32_t q_pos0;     /* position of that row */
    int32_t n_rows;     /* valid rows, 1..128 */
    int32_t n_ranges;   /* 1 or 2 */
    int32_t block;      /* block of the query rows */
    int32_t k_row0[2];  /* first key row of each range in the rotated-K buffer */
    int32_t v_row0[2];  /* first value row of each range */
    int32_t pos0[2];    /* position of the first key of each range */
    int32_t len[2];     /* keys in each range */
} dbsa_tile_item;

/* Host-only planner behind dbsa_encode_blocks: the tile list (query tiles
 * of 128 rows never straddle a block; key ranges follow the pattern) for
 * blocks [0, nb).  Writes at most max_items entries to items (host, may be
 * NULL to count) and returns the total count, or -1 on bad arguments.  The
 * ordering is the one the kernel uses. */
int64_t dbsa_stage1_plan(const dbsa_config *cfg, const int32_t *offs_host,
                         int32_t nb, dbsa_tile_item *items, int64_t max_items);

/* Number of 128x128 score tiles the Stage-1 kernel evaluates for a plan,
 * i.e. tiles with at least one allowed (query, key) pair, summed over all
 * heads.  Returns -1 on bad arguments. */
int64_t dbsa_stage1_tile_count(const dbsa_config *cfg, const int32_t *offs_host,
                               int32_t nb);

/* Library version string. */
const char *dbsa_version(void);

/* Number of CUDA kernels this process has launched through the library
 * (all threads).  For accounting in benchmarks. */
int64_t dbsa_kernel_launches(void);

/* Profiling hook for the NEXT call on this thread only: `start` and `stop`
 * (cudaEvent_t, either may be NULL) are recorded on the call's stream
 * immediately before and after its main attention kernel (Stage-1 tensor-core
 * kernel, or the Stage-2 split kernel without the merge), so that the
 * kernel's duration can be read with cudaEventElapsedTime.  Cleared by the
 * call. */
void dbsa_set_profile_events(void *start, void *stop);

#ifdef __cplusplus
}
#endif

#endif /* DBSA_H */
