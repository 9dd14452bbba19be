// Stage 2: fused gather + RoPE re-rotation + GQA attention, split over the
// key sequence ("split-KV"), then a log-sum-exp merge of the splits.
//
// [DBSA notes] §Stage 2, items 2-4: the selected blocks (sink first) are
// concatenated, their cached pre-RoPE keys are rotated again at fresh
// sequential positions, and the query tokens attend to the whole gathered
// cache.  Query q's key sequence is [gathered tokens 0..T'_q) ++ [its own tail
// tokens], positions 0..T'_q + tail_len - 1, so one causal rule (key position
// <= row position) covers both parts.
//
// Grid: (split item, KV head, row group).  Every CTA reads each key of its
// split once and scores it against all g * n_new query rows that share the KV
// head (GQA), so the cache is streamed from HBM once per (query, KV head).
// Keys are fetched with 16-byte cp.async through a per-thread segment walk
// (the gather), rotated in shared memory (fp32 math, two-level fp64-built
// table), and multiplied on the tensor cores with mma.sync (bf16 in, fp32
// accumulate); softmax runs online in registers.  Decode passes (<= 16 rows)
// split each key tile across the four warps and merge them through shared
// memory; longer passes give each warp 16 rows.
#include <cuda_bf16.h>

#include <cfloat>
#include <climits>

#include "dbsa_internal.h"
#include "vec8.cuh"

namespace dbsa {
namespace {

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void cp_async16(void *dst, const void *src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(dst)), "l"(src)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;" ::: "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t &r0, uint32_t &r1, uint32_t &r2,
                                        uint32_t &r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t &r0, uint32_t &r1,
                                          uint32_t &r2, uint32_t &r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
// D = A * B + D, m16n8k16, bf16 inputs, fp32 accumulators.
__device__ __forceinline__ void mma16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                         uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, "
      "{%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t *>(&h);
}

// Byte offset of (row, 16-byte chunk) in a swizzled [rows][D] bf16 tile.
template <int D>
__device__ __forceinline__ uint32_t soff(int row, int chunk) {
  return (uint32_t)(row * (D * 2) + ((chunk ^ (row & 7)) << 4));
}

template <int D, typename CT>
__device__ __forceinline__ void zero_chunk_row(uint8_t *tile, int row, int ch0, int nch) {
  for (int ch = ch0; ch < ch0 + nch; ++ch)
    *reinterpret_cast<uint4 *>(tile + soff<D>(row, ch)) = make_uint4(0, 0, 0, 0);
}

template <int D, typename CT>
__device__ __forceinline__ void fetch_row(uint8_t *tile, int row, int ch0, int nch,
                                          const CT *src) {
  if constexpr (sizeof(CT) == 2) {
    for (int ch = ch0; ch < ch0 + nch; ++ch) cp_async16(tile + soff<D>(row, ch), src + ch * 8);
  } else {
    for (int ch = ch0; ch < ch0 + nch; ++ch) {
      float f[8];
      load8(src + ch * 8, f);
      store8_bf16(reinterpret_cast<bf16 *>(tile + soff<D>(row, ch)), f);
    }
  }
}

// KW = keys of each 64-key tile handled by one warp: 64 (each warp owns 16
// query rows) or 16 (<= 16 rows; the four warps split the tile's keys).
template <int D, typename CT, int KW>
__global__ void __launch_bounds__(128) stage2_attn_kernel(const Stage2Args a) {
  constexpr int H = D / 2;
  constexpr int CH = D / 8;                 // 16-byte chunks per row
  constexpr int ROWB = D * 2;
  constexpr int TILEB = kS2Keys * ROWB;
  constexpr int MROWS = (KW == 64) ? 64 : 16;
  constexpr int NB = KW / 8;                // n8 key blocks per warp
  constexpr int ND = D / 8;                 // n8 dim blocks
  extern __shared__ __align__(128) uint8_t sm[];
  uint8_t *sQ = sm;
  uint8_t *sK = sQ + MROWS * ROWB;
  uint8_t *sV = sK + 2 * TILEB;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int c = blockIdx.y;
  const S2Item item = a.items[blockIdx.x];
  const S2Query qi = a.queries[item.query];
  const int q = item.query;
  const int g = a.Hq / a.Hkv;
  const int R = g * a.n_new;
  const int Tq = qi.n_gathered;
  const int pos_first = Tq + a.tail_len - a.n_new;  // position of query token 0
  const int row_base = (KW == 64) ? blockIdx.z * 64 : 0;
  const CT *kc = static_cast<const CT *>(a.k_cache);
  const CT *vc = static_cast<const CT *>(a.v_cache);
  const CT *kt = static_cast<const CT *>(a.k_tail);
  const CT *vt = static_cast<const CT *>(a.v_tail);

  // ---- query rows: rotate at their positions, store bf16 (swizzled)
  for (int u = threadIdx.x; u < MROWS * (H / 8); u += blockDim.x) {
    const int rr = u / (H / 8), cp = u % (H / 8);
    const int r = row_base + rr;
    float lo[8], hi[8];
    if (r < R) {
      const int tok = r / g, h = c * g + r % g;
      const CT *src = static_cast<const CT *>(a.q_new) +
                      (((int64_t)q * a.n_new + tok) * a.Hq + h) * D;
      load8(src + cp * 8, lo);
      load8(src + H + cp * 8, hi);
      float cs[8], sn[8];
      rope_cs8(a.rope, pos_first + tok, cp * 8, H, cs, sn);
      rotate8(lo, hi, cs, sn);
    } else {
#pragma unroll
      for (int e = 0; e < 8; ++e) lo[e] = hi[e] = 0.f;
    }
    store8_bf16(reinterpret_cast<bf16 *>(sQ + soff<D>(rr, cp)), lo);
    store8_bf16(reinterpret_cast<bf16 *>(sQ + soff<D>(rr, cp + H / 8)), hi);
  }

  // ---- gather: thread t fetches row (t >> 1) of every tile, chunk half (t & 1)
  const int frow = threadIdx.x >> 1;
  const int fch0 = (threadIdx.x & 1) * (CH / 2);
  int seg = 0;  // per-thread segment cursor (positions only grow)
  const int n_tiles = (item.p_end - item.p_begin + kS2Keys - 1) / kS2Keys;
  auto issue_tile = [&](int j) {
    const int p = item.p_begin + j * kS2Keys + frow;
    uint8_t *dk = sK + (j & 1) * TILEB;
    uint8_t *dv = sV + (j & 1) * TILEB;
    if (p >= item.p_end) {
      zero_chunk_row<D, CT>(dk, frow, fch0, CH / 2);
      zero_chunk_row<D, CT>(dv, frow, fch0, CH / 2);
      return;
    }
    const CT *ks, *vs;
    if (p < Tq) {
      while (seg + 1 < qi.n_seg && __ldg(&a.segs[qi.seg_begin + seg + 1].pos0) <= p) ++seg;
      const S2Segment sg = a.segs[qi.seg_begin + seg];
      const int64_t crow = (int64_t)sg.cache_row0 + (p - sg.pos0);
      ks = kc + ((int64_t)c * a.cap + crow) * D;
      vs = vc + ((int64_t)c * a.cap + crow) * D;
      if (a.dbg_map != nullptr && c == 0 && blockIdx.z == 0 && fch0 == 0) {
        int32_t *m = a.dbg_map + ((int64_t)q * a.dbg_cap + p) * 2;
        m[0] = (int32_t)crow;
        m[1] = p;
      }
    } else {
      const int64_t w = p - Tq;
      ks = kt + (((int64_t)q * a.tail_cap + w) * a.Hkv + c) * D;
      vs = vt + (((int64_t)q * a.tail_cap + w) * a.Hkv + c) * D;
    }
    fetch_row<D, CT>(dk, frow, fch0, CH / 2, ks);
    fetch_row<D, CT>(dv, frow, fch0, CH / 2, vs);
  };

  if (n_tiles > 0) issue_tile(0);
  cp_async_commit();
  __syncthreads();

  // ---- Q fragments (A operand), kept in registers for the whole split
  const int wrow = (KW == 64) ? warp * 16 : 0;  // first query row of this warp (in sQ)
  uint32_t qf[D / 16][4];
  {
    const int r = wrow + (lane & 7) + ((lane >> 3) & 1) * 8;
#pragma unroll
    for (int ks = 0; ks < D / 16; ++ks)
      ldsm_x4(smem_u32(sQ) + soff<D>(r, 2 * ks + (lane >> 4)), qf[ks][0], qf[ks][1], qf[ks][2],
              qf[ks][3]);
  }
  // positions of this thread's two rows (g and g + 8 of the warp's 16)
  const int gq = lane >> 2, tq = lane & 3;
  int qpos[2];
#pragma unroll
  for (int h2 = 0; h2 < 2; ++h2) {
    const int r = row_base + wrow + gq + 8 * h2;
    qpos[h2] = (r < R) ? pos_first + r / g : INT_MAX;
  }
  const int kw0 = (KW == 64) ? 0 : warp * 16;  // this warp's keys inside a tile

  float o[ND][4];
#pragma unroll
  for (int nd = 0; nd < ND; ++nd) o[nd][0] = o[nd][1] = o[nd][2] = o[nd][3] = 0.f;
  float m_run[2] = {-INFINITY, -INFINITY}, l_run[2] = {0.f, 0.f};
  const float sl2 = a.scale_log2;

  for (int j = 0; j < n_tiles; ++j) {
    if (j + 1 < n_tiles) issue_tile(j + 1);
    cp_async_commit();
    cp_async_wait<1>();
    __syncthreads();
    const int p0 = item.p_begin + j * kS2Keys;
    uint8_t *tk = sK + (j & 1) * TILEB;
    uint8_t *tv = sV + (j & 1) * TILEB;
    // ---- re-rotate the raw keys at their fresh positions p0 + row
    {
      const int row = threadIdx.x >> 1;
      const int i_base = (threadIdx.x & 1) * (H / 2);
#pragma unroll
      for (int cc = 0; cc < H / 16; ++cc) {
        const int i0 = i_base + cc * 8;
        bf16 *plo = reinterpret_cast<bf16 *>(tk + soff<D>(row, i0 / 8));
        bf16 *phi = reinterpret_cast<bf16 *>(tk + soff<D>(row, (H + i0) / 8));
        float lo[8], hi[8], cs[8], sn[8];
        load8(plo, lo);
        load8(phi, hi);
        rope_cs8(a.rope, (int64_t)p0 + row, i0, H, cs, sn);
        rotate8(lo, hi, cs, sn);
        store8_bf16(plo, lo);
        store8_bf16(phi, hi);
      }
    }
    __syncthreads();

    // ---- S = Q K^T for this warp's 16 rows x KW keys
    float s[NB][4];
#pragma unroll
    for (int nb = 0; nb < NB; ++nb) s[nb][0] = s[nb][1] = s[nb][2] = s[nb][3] = 0.f;
#pragma unroll
    for (int ks = 0; ks < D / 16; ++ks) {
#pragma unroll
      for (int nb = 0; nb < NB; nb += 2) {
        const int mi = lane >> 3;
        const int krow = kw0 + (nb + (mi >> 1)) * 8 + (lane & 7);
        uint32_t b0, b1, b2, b3;
        ldsm_x4(smem_u32(tk) + soff<D>(krow, 2 * ks + (mi & 1)), b0, b1, b2, b3);
        mma16816(s[nb], qf[ks], b0, b1);
        mma16816(s[nb + 1], qf[ks], b2, b3);
      }
    }
    // ---- mask (split end, causal inside the query's own tail), online softmax
    const bool need_mask = (p0 + kS2Keys > item.p_end) || (p0 + kS2Keys - 1 > pos_first);
    float tmax[2] = {-INFINITY, -INFINITY};
#pragma unroll
    for (int nb = 0; nb < NB; ++nb)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        float x = s[nb][e] * sl2;
        if (need_mask) {
          const int kp = p0 + kw0 + nb * 8 + 2 * tq + (e & 1);
          if (kp >= item.p_end || kp > qpos[e >> 1]) x = -INFINITY;
        }
        s[nb][e] = x;
        tmax[e >> 1] = fmaxf(tmax[e >> 1], x);
      }
    float alpha[2], mu[2];
#pragma unroll
    for (int h2 = 0; h2 < 2; ++h2) {
      tmax[h2] = fmaxf(tmax[h2], __shfl_xor_sync(0xFFFFFFFFu, tmax[h2], 1));
      tmax[h2] = fmaxf(tmax[h2], __shfl_xor_sync(0xFFFFFFFFu, tmax[h2], 2));
      const float mn = fmaxf(m_run[h2], tmax[h2]);
      alpha[h2] = (mn == -INFINITY) ? 1.f : ex2(m_run[h2] - mn);
      m_run[h2] = mn;
      mu[h2] = (mn == -INFINITY) ? 0.f : mn;
      l_run[h2] *= alpha[h2];
    }
#pragma unroll
    for (int nd = 0; nd < ND; ++nd) {
      o[nd][0] *= alpha[0];
      o[nd][1] *= alpha[0];
      o[nd][2] *= alpha[1];
      o[nd][3] *= alpha[1];
    }
#pragma unroll
    for (int nb = 0; nb < NB; ++nb)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float pv = ex2(s[nb][e] - mu[e >> 1]);
        s[nb][e] = pv;
        l_run[e >> 1] += pv;
      }
    // ---- O += P V
#pragma unroll
    for (int kk = 0; kk < KW / 16; ++kk) {
      uint32_t pa[4];
      pa[0] = pack_bf16(s[2 * kk][0], s[2 * kk][1]);
      pa[1] = pack_bf16(s[2 * kk][2], s[2 * kk][3]);
      pa[2] = pack_bf16(s[2 * kk + 1][0], s[2 * kk + 1][1]);
      pa[3] = pack_bf16(s[2 * kk + 1][2], s[2 * kk + 1][3]);
      const int mi = lane >> 3;
      const int vrow = kw0 + kk * 16 + (mi & 1) * 8 + (lane & 7);
#pragma unroll
      for (int nd = 0; nd < ND; nd += 2) {
        uint32_t b0, b1, b2, b3;
        ldsm_x4_t(smem_u32(tv) + soff<D>(vrow, nd + (mi >> 1)), b0, b1, b2, b3);
        mma16816(o[nd], pa, b0, b1);
        mma16816(o[nd + 1], pa, b2, b3);
      }
    }
    __syncthreads();  // tile j's buffers may be refilled by iteration j + 1
  }
  cp_async_wait<0>();

  // ---- row sums over the quad
#pragma unroll
  for (int h2 = 0; h2 < 2; ++h2) {
    l_run[h2] += __shfl_xor_sync(0xFFFFFFFFu, l_run[h2], 1);
    l_run[h2] += __shfl_xor_sync(0xFFFFFFFFu, l_run[h2], 2);
  }

  auto part_index = [&](int r) -> int64_t {  // r = query row (GQA row) index
    const int tok = r / g, h = c * g + r % g;
    return ((int64_t)blockIdx.x * a.Hq + h) * a.n_new + tok;
  };

  if constexpr (KW == 64) {
#pragma unroll
    for (int h2 = 0; h2 < 2; ++h2) {
      const int r = row_base + wrow + gq + 8 * h2;
      if (r >= R) continue;
      const int64_t pi = part_index(r);
      float *acc = a.part_acc + pi * D;
#pragma unroll
      for (int nd = 0; nd < ND; ++nd)
        *reinterpret_cast<float2 *>(acc + nd * 8 + 2 * tq) =
            make_float2(o[nd][2 * h2], o[nd][2 * h2 + 1]);
      if (tq == 0) a.part_ml[pi] = make_float2(m_run[h2], l_run[h2]);
    }
  } else {
    // merge the four warps' partial states for the 16 rows through shared memory
    __syncthreads();
    float *so = reinterpret_cast<float *>(sK);          // [4][16][D]
    float2 *sml = reinterpret_cast<float2 *>(so + 4 * 16 * D);  // [4][16]
#pragma unroll
    for (int h2 = 0; h2 < 2; ++h2) {
      const int r = gq + 8 * h2;
#pragma unroll
      for (int nd = 0; nd < ND; ++nd)
        *reinterpret_cast<float2 *>(so + (warp * 16 + r) * D + nd * 8 + 2 * tq) =
            make_float2(o[nd][2 * h2], o[nd][2 * h2 + 1]);
      if (tq == 0) sml[warp * 16 + r] = make_float2(m_run[h2], l_run[h2]);
    }
    __syncthreads();
    // 128 threads: row = t / 8, dims [(t % 8) * D/8, +D/8)
    const int r = threadIdx.x >> 3;
    const int d0 = (threadIdx.x & 7) * (D / 8);
    if (r < R) {
      float M = -INFINITY;
#pragma unroll
      for (int w = 0; w < 4; ++w) M = fmaxf(M, sml[w * 16 + r].x);
      float wgt[4], L = 0.f;
#pragma unroll
      for (int w = 0; w < 4; ++w) {
        const float2 ml = sml[w * 16 + r];
        wgt[w] = (ml.x == -INFINITY) ? 0.f : ex2(ml.x - M);
        L += ml.y * wgt[w];
      }
      const int64_t pi = part_index(r);
      float *acc = a.part_acc + pi * D;
      for (int d = d0; d < d0 + D / 8; ++d) {
        float x = 0.f;
#pragma unroll
        for (int w = 0; w < 4; ++w) x += wgt[w] * so[(w * 16 + r) * D + d];
        acc[d] = x;
      }
      if ((threadIdx.x & 7) == 0) a.part_ml[pi] = make_float2(M, L);
    }
  }
}

// One warp per output row (query q, token u, head h): combine the row's split
// partials with their log-sum-exp weights.
template <int D, typename OT>
__global__ void __launch_bounds__(128) stage2_merge_kernel(const Stage2Args a) {
  const int64_t row = (int64_t)blockIdx.x * 4 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  const int64_t n_rows = (int64_t)a.n_queries * a.n_new * a.Hq;
  if (row >= n_rows) return;
  const int h = (int)(row % a.Hq);
  const int tok = (int)((row / a.Hq) % a.n_new);
  const int q = (int)(row / ((int64_t)a.Hq * a.n_new));
  const S2Query qi = a.queries[q];
  float M = -INFINITY;
  for (int i = 0; i < qi.n_items; ++i) {
    const int64_t pi = ((int64_t)(qi.item_begin + i) * a.Hq + h) * a.n_new + tok;
    M = fmaxf(M, a.part_ml[pi].x);
  }
  constexpr int PER = D / 32;
  float acc[PER];
#pragma unroll
  for (int e = 0; e < PER; ++e) acc[e] = 0.f;
  float L = 0.f;
  for (int i = 0; i < qi.n_items; ++i) {
    const int64_t pi = ((int64_t)(qi.item_begin + i) * a.Hq + h) * a.n_new + tok;
    const float2 ml = a.part_ml[pi];
    const float w = (ml.x == -INFINITY) ? 0.f : ex2(ml.x - M);
    L += w * ml.y;
    const float *src = a.part_acc + pi * D + lane * PER;
#pragma unroll
    for (int e = 0; e < PER; ++e) acc[e] += w * src[e];
  }
  const float inv = 1.f / L;
  OT *dst = static_cast<OT *>(a.out) + (((int64_t)q * a.n_new + tok) * a.Hq + h) * D + lane * PER;
#pragma unroll
  for (int e = 0; e < PER; ++e) {
    if constexpr (sizeof(OT) == 2)
      dst[e] = __float2bfloat16_rn(acc[e] * inv);
    else
      dst[e] = acc[e] * inv;
  }
}

template <int D, typename CT, int KW>
cudaError_t launch_main(const Stage2Args &a, cudaStream_t st) {
  constexpr int MROWS = (KW == 64) ? 64 : 16;
  constexpr size_t smem = (size_t)MROWS * D * 2 + 4 * (size_t)kS2Keys * D * 2;
  static_assert(KW == 64 || smem >= 4 * 16 * D * 4 + 4 * 16 * 8, "merge scratch fits");
  cudaError_t e = cudaFuncSetAttribute(stage2_attn_kernel<D, CT, KW>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const int g = a.Hq / a.Hkv;
  const int R = g * a.n_new;
  const int zdim = (KW == 64) ? (R + 63) / 64 : 1;
  dim3 grid(a.n_items, a.Hkv, zdim);
  stage2_attn_kernel<D, CT, KW><<<grid, 128, smem, st>>>(a);
  return cudaGetLastError();
}

template <int D, typename CT>
cudaError_t launch_d(const Stage2Args &a, cudaStream_t st) {
  const int R = (a.Hq / a.Hkv) * a.n_new;
  return (R <= 16) ? launch_main<D, CT, 16>(a, st) : launch_main<D, CT, 64>(a, st);
}

template <int D, typename CT>
cudaError_t launch_merge(const Stage2Args &a, cudaStream_t st) {
  const int64_t rows = (int64_t)a.n_queries * a.n_new * a.Hq;
  stage2_merge_kernel<D, CT><<<(unsigned)((rows + 3) / 4), 128, 0, st>>>(a);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_stage2_main(const Stage2Args &a, int head_dim, bool f32, cudaStream_t st) {
  if (a.n_items <= 0) return cudaSuccess;
  if (head_dim == 128) return f32 ? launch_d<128, float>(a, st) : launch_d<128, bf16>(a, st);
  return f32 ? launch_d<64, float>(a, st) : launch_d<64, bf16>(a, st);
}

cudaError_t launch_stage2_merge(const Stage2Args &a, int head_dim, bool f32, cudaStream_t st) {
  if (a.n_items <= 0) return cudaSuccess;
  if (head_dim == 128) return f32 ? launch_merge<128, float>(a, st) : launch_merge<128, bf16>(a, st);
  return f32 ? launch_merge<64, float>(a, st) : launch_merge<64, bf16>(a, st);
}

}  // namespace dbsa
