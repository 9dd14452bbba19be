// Stage 2, per-query parts: the per-query split kernel and the log-sum-exp
// merge of split partials, and the block-major mode's tail-and-merge kernel.
//
// [DBSA notes] §Stage 2, items 2-4: the selected blocks (sink first) are
// concatenated, their cached pre-RoPE keys are rotated again at fresh
// sequential positions, and the query tokens attend to the whole gathered
// cache and, causally, to the query's own tokens.  Query q's key sequence is
// [gathered tokens 0..T'_q) ++ [its own tail tokens], positions
// 0..T'_q + tail_len - 1.  Normally the gathered blocks are handled block by
// block by the tensor-core kernel (one partial per (query, block)) and
// stage2_tail_merge_kernel runs each query's tail keys [T'_q, T'_q + tail_len)
// and merges all partials of a row into the output.  For selections of short
// segments (a demonstration-granular gather) stage2_attn_kernel runs whole
// split items [p_begin, p_end) of a query's key sequence, fetching the
// gathered keys segment by segment, and stage2_merge_kernel combines them.
//
// Grid: (item, KV head, row group).  A CTA reads each key of its item once
// and scores it against all g * n_new query rows that share the KV head
// (GQA).  Keys are fetched with 16-byte cp.async, rotated in shared
// memory (fp32 math, two-level fp64-built table) at their positions, and
// multiplied with mma.sync (bf16 in, fp32 accumulate); softmax runs online in
// registers and one causal rule (key position <= row position) covers the
// tail.  Passes of <= 16 rows split each key tile across the warps and merge
// them through shared memory; longer passes give each warp 16 rows.
#include <cuda_bf16.h>

#include <cfloat>
#include <climits>
#include <type_traits>

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

// Warps form KG key groups of RT warps.  A key group streams the sub-tiles
// j = kg, kg + KG, ... (KT keys each) of its split through its own NST-stage
// cp.async ring; the group's RT warps own the CTA's 16-row query tiles and
// all read the same keys, so every key is fetched from HBM and rotated once
// per (query, KV head, row group).  Each warp keeps an online-softmax state
// for its 16 rows; the key groups' states are merged through shared memory at
// the end and written as one split partial.
//
template <int D, typename CT, int RT, int KG, int KT, int NST>
__global__ void __launch_bounds__(32 * RT * KG, 1) stage2_attn_kernel(const Stage2Args a) {
  pdl_enter();
  constexpr int H = D / 2;
  constexpr int CH = D / 8;                 // 16-byte chunks per row
  constexpr int ROWB = D * 2;
  constexpr int NT = 32 * RT;               // threads of one key group
  constexpr int NTOT = NT * KG;
  constexpr int MROWS = 16 * RT;            // query rows of the CTA
  constexpr int NB = KT / 8;                // n8 key blocks per sub-tile
  constexpr int ND = D / 8;                 // n8 dim blocks
  static_assert(NB % 2 == 0 && KT % RT == 0, "tile shape");
  constexpr uint32_t STAGEB = KT * ROWB;
  extern __shared__ __align__(128) uint8_t sm[];
  uint8_t *sQ = sm;
  float *sLc = reinterpret_cast<float *>(sQ + MROWS * ROWB);  // RoPE lo table, [16][H] x 2
  float *sLs = sLc + kRopeLo * H;
  uint8_t *sRing = reinterpret_cast<uint8_t *>(sLs + kRopeLo * H);  // [KG][NST][K, V][KT][D]

  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const int kg = warp / RT, wr = warp % RT;
  const int c = blockIdx.y;
  const int g = a.Hq / a.Hkv;
  const int RQ = g * a.n_new;                      // rows of one query
  // keys [p_lo, p_end) of the query's sequence (p_begin is a multiple of the
  // RoPE step; keys in [p_begin, p_lo) belong to other items and are masked)
  const int it_idx = a.run_items[blockIdx.x];
  const S2Item item = a.items[it_idx];
  const int q = item.query;
  const S2Query qi = a.queries[q];
  const int Tq = qi.n_gathered;
  const int k_begin = item.p_begin, k_end = item.p_end, k_lo = item.p_lo;
  const int R = RQ;
  const int pos_first = Tq + a.tail_len - a.n_new;  // position of query token 0 (per query)
  const int row_base = blockIdx.z * MROWS;
  const CT *kc = static_cast<const CT *>(a.k_cache);
  const CT *vc = static_cast<const CT *>(a.v_cache);
  const CT *kt = static_cast<const CT *>(a.k_tail);
  const CT *vt = static_cast<const CT *>(a.v_tail);

  auto group_sync = [&]() {
    if constexpr (RT == 1) {
      __syncwarp();
    } else {
      asm volatile("bar.sync %0, %1;" ::"r"(1 + kg), "r"(NT) : "memory");
    }
  };

  for (int u = tid; u < kRopeLo * H; u += NTOT) {
    sLc[u] = __ldg(a.rope.lc + u);
    sLs[u] = __ldg(a.rope.ls + u);
  }
  // ---- query rows: rotate at their positions, store bf16 (swizzled)
  for (int u = tid; u < MROWS * (H / 8); u += NTOT) {
    const int rr = u / (H / 8), cp = u % (H / 8);
    const int r = row_base + rr;
    float lo[8], hi[8];
    if (r < R) {
      const int tok = r / g, h = c * g + r % g, pos = pos_first + tok;
      const CT *src = static_cast<const CT *>(a.q_new) +
                      (((int64_t)q * a.n_new + tok) * a.Hq + h) * D;
      load8(src + cp * 8, lo);
      load8(src + H + cp * 8, hi);
      float cs[8], sn[8];
      rope_cs8(a.rope, pos, cp * 8, H, cs, sn);
      rotate8(lo, hi, cs, sn);
    } else {
#pragma unroll
      for (int e = 0; e < 8; ++e) lo[e] = hi[e] = 0.f;
    }
    store8_bf16(reinterpret_cast<bf16 *>(sQ + soff<D>(rr, cp)), lo);
    store8_bf16(reinterpret_cast<bf16 *>(sQ + soff<D>(rr, cp + H / 8)), hi);
  }

  // ---- gather: warp wr of a key group loads (and later rotates) rows
  // [wr * RPW, (wr + 1) * RPW) of each sub-tile.  Lane l (l < RPW) resolves
  // the cache or tail row of row l for K, lane 16 + l the same row for V;
  // then every copy instruction moves one whole K row (lanes 0-15) and one
  // whole V row (lanes 16-31).
  constexpr int RPW = KT / RT;
  static_assert(RPW <= 16 && CH <= 16, "one row per half-warp");
  const int n_sub = (k_end - k_begin + KT - 1) / KT;
  int seg = 0;  // segment cursor: this lane's positions only grow
  const int n_local = kg < n_sub ? (n_sub - kg + KG - 1) / KG : 0;
  const int half_id = lane >> 4, hl = lane & 15;  // half-warp: 0 = K, 1 = V
  auto stage_ptr = [&](int jl, int kv) -> uint8_t * {
    return sRing + ((size_t)(kg * NST + jl % NST) * 2 + kv) * STAGEB;
  };
  // Position at which the rotation step turns row r0 + k of the sub-tile that
  // starts at key position t0 (r0 = a warp's first row): the "hi" factor of
  // the 16-position group holding t0 + r0 times the "lo" factor (r0 & 15) + k.
  auto rot_pos = [](int t0, int r0, int k) {
    return (((t0 + r0) >> kRopeShift) << kRopeShift) + (r0 & (kRopeLo - 1)) + k;
  };
  const bool write_map = a.dbg_map != nullptr && c == 0 && blockIdx.z == 0;
  auto issue = [&](int jl) {
    const int t0 = k_begin + (kg + jl * KG) * KT;   // first key position of the sub-tile
    const int p0 = t0 + wr * RPW;
    // this lane's row pointer (lanes hl < RPW); null past the split end
    const CT *my = nullptr;
    if (hl < RPW) {
      const int p = p0 + hl;
      if (p < k_end && p >= k_lo) {
        if (p < Tq) {   // gathered token p: walk to the segment that holds it
          while (seg + 1 < qi.n_seg && __ldg(&a.segs[qi.seg_begin + seg + 1].pos0) <= p) ++seg;
          const int64_t crow = (int64_t)__ldg(&a.segs[qi.seg_begin + seg].cache_row0) +
                               (p - __ldg(&a.segs[qi.seg_begin + seg].pos0));
          my = (half_id ? vc : kc) + ((int64_t)c * a.cap + crow) * D;
          if (write_map && half_id == 0)   // the row this lane loads, and its rotation position
            *reinterpret_cast<int2 *>(a.dbg_map + ((int64_t)q * a.dbg_cap + p) * 2) =
                make_int2((int)crow, rot_pos(t0, wr * RPW, hl));
        } else {        // the query's own tail token p - T'_q
          const int64_t w = p - Tq;
          my = (half_id ? vt : kt) + (((int64_t)q * a.tail_cap + w) * a.Hkv + c) * D;
        }
      }
    }
    uint8_t *dst = stage_ptr(jl, half_id);
#pragma unroll 4
    for (int r = 0; r < RPW; ++r) {
      const CT *src = reinterpret_cast<const CT *>(
          __shfl_sync(0xFFFFFFFFu, reinterpret_cast<unsigned long long>(my), (half_id << 4) + r));
      if (hl < CH) {
        uint8_t *d = dst + soff<D>(wr * RPW + r, hl);
        if (src == nullptr) {
          *reinterpret_cast<uint4 *>(d) = make_uint4(0, 0, 0, 0);
        } else if constexpr (sizeof(CT) == 2) {
          cp_async16(d, src + hl * 8);
        } else {
          float f[8];
          load8(src + hl * 8, f);
          store8_bf16(reinterpret_cast<bf16 *>(d), f);
        }
      }
    }
  };

#pragma unroll
  for (int s0 = 0; s0 < NST - 1; ++s0) {
    if (s0 < n_local) issue(s0);
    cp_async_commit();
  }
  __syncthreads();  // sQ complete

  // ---- Q fragments (A operand) of this warp's 16 rows: kept in registers,
  // or (large CTAs, where registers are scarce) re-read from shared memory
  constexpr bool kQRegs = RT < 8;
  const int qfrow = wr * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
  uint32_t qf[kQRegs ? D / 16 : 1][4];
  if constexpr (kQRegs) {
#pragma unroll
    for (int ks = 0; ks < D / 16; ++ks)
      ldsm_x4(smem_u32(sQ) + soff<D>(qfrow, 2 * ks + (lane >> 4)), qf[ks][0], qf[ks][1], qf[ks][2],
              qf[ks][3]);
  }
  const int gq = lane >> 2, tq = lane & 3;
  int qpos[2];
#pragma unroll
  for (int h2 = 0; h2 < 2; ++h2) {
    const int r = row_base + wr * 16 + gq + 8 * h2;
    qpos[h2] = r < R ? pos_first + r / g : INT_MAX;
  }

  float o[ND][4];
#pragma unroll
  for (int nd = 0; nd < ND; ++nd) o[nd][0] = o[nd][1] = o[nd][2] = o[nd][3] = 0.f;
  float m_run[2] = {-INFINITY, -INFINITY}, l_run[2] = {0.f, 0.f};
  const float sl2 = a.scale_log2;

  for (int jl = 0; jl < n_local; ++jl) {
    cp_async_wait<NST - 2>();
    group_sync();
    if (jl + NST - 1 < n_local) issue(jl + NST - 1);
    cp_async_commit();
    const int p0 = k_begin + (kg + jl * KG) * KT;
    uint8_t *tk = stage_ptr(jl, 0);
    uint8_t *tv = stage_ptr(jl, 1);
    // ---- re-rotate this warp's rows of the sub-tile at their fresh positions
    // p0 + row.  Lane = frequency pair(s); the rows of one warp share one
    // 16-position group, hence one "hi" factor, and the "lo" factors come
    // from shared memory.
    {
      static_assert(RPW <= kRopeLo && kRopeLo % RPW == 0, "a warp's rows share one hi factor");
      const int r0 = wr * RPW;
      const int64_t hoff = (int64_t)((p0 + r0) >> kRopeShift) * H;
      if constexpr (H == 64) {
        // p0 is a multiple of 16 and r0 a multiple of 8, so row r0 + k sits at
        // position offset (r0 & 15) + k of its 16-group and at swizzle phase
        // k & 7: every address below is a per-lane base plus a constant.
        static_assert(RPW % 8 == 0, "rows per warp keep the swizzle phase");
        const int i = 2 * lane;
        const f32x2 hcos = *reinterpret_cast<const f32x2 *>(a.rope.hc + hoff + i);
        const f32x2 hsin = *reinterpret_cast<const f32x2 *>(a.rope.hs + hoff + i);
        const f32x2 nhsin = f2_neg(hsin);
        const float *lcb = sLc + (r0 & (kRopeLo - 1)) * H + i;
        const float *lsb = sLs + (r0 & (kRopeLo - 1)) * H + i;
        uint8_t *rowb = tk + r0 * ROWB + (i & 7) * 2;
#pragma unroll
        for (int k = 0; k < RPW; ++k) {
          const f32x2 lcos = *reinterpret_cast<const f32x2 *>(lcb + k * H);
          const f32x2 lsin = *reinterpret_cast<const f32x2 *>(lsb + k * H);
          const f32x2 cs = f2_fma(hcos, lcos, f2_mul(nhsin, lsin));
          const f32x2 sn = f2_fma(hcos, lsin, f2_mul(hsin, lcos));
          uint32_t *plo = reinterpret_cast<uint32_t *>(rowb + k * ROWB + (((i >> 3) ^ (k & 7)) << 4));
          uint32_t *phi = plo + (H / 8) * 4;  // second half: chunk + H/8, same swizzle
          const f32x2 xl = f2_from_bf16x2(*plo), xh = f2_from_bf16x2(*phi);
          *plo = f2_to_bf16x2(f2_fma(xl, cs, f2_mul(f2_neg(xh), sn)));
          *phi = f2_to_bf16x2(f2_fma(xh, cs, f2_mul(xl, sn)));
        }
      } else {
        static_assert(H == 32, "head_dim 64 or 128");
        const int i = lane;
        const float hcos = a.rope.hc[hoff + i], hsin = a.rope.hs[hoff + i];
#pragma unroll 4
        for (int r = r0; r < r0 + RPW; ++r) {
          const int lr = (r0 & (kRopeLo - 1)) + (r - r0);   // as rot_pos(p0, r0, r - r0)
          const float lcos = sLc[lr * H + i], lsin = sLs[lr * H + i];
          const float cs = __fmaf_rn(hcos, lcos, __fmul_rn(-hsin, lsin));
          const float sn = __fmaf_rn(hcos, lsin, __fmul_rn(hsin, lcos));
          bf16 *plo = reinterpret_cast<bf16 *>(tk + soff<D>(r, i >> 3)) + (i & 7);
          bf16 *phi = reinterpret_cast<bf16 *>(tk + soff<D>(r, (H + i) >> 3)) + (i & 7);
          const float xl = __bfloat162float(*plo), xh = __bfloat162float(*phi);
          *plo = __float2bfloat16_rn(__fmaf_rn(xl, cs, __fmul_rn(-xh, sn)));
          *phi = __float2bfloat16_rn(__fmaf_rn(xh, cs, __fmul_rn(xl, sn)));
        }
      }
    }
    group_sync();

    // ---- S = Q K^T for this warp's 16 rows x KT keys
    float s[NB][4];
#pragma unroll
    for (int nb = 0; nb < NB; ++nb) s[nb][0] = s[nb][1] = s[nb][2] = s[nb][3] = 0.f;
#pragma unroll
    for (int ks = 0; ks < D / 16; ++ks) {
      uint32_t qa[4];
      if constexpr (kQRegs) {
        qa[0] = qf[ks][0]; qa[1] = qf[ks][1]; qa[2] = qf[ks][2]; qa[3] = qf[ks][3];
      } else {
        ldsm_x4(smem_u32(sQ) + soff<D>(qfrow, 2 * ks + (lane >> 4)), qa[0], qa[1], qa[2], qa[3]);
      }
#pragma unroll
      for (int nb = 0; nb < NB; nb += 2) {
        const int mi = lane >> 3;
        const int krow = (nb + (mi >> 1)) * 8 + (lane & 7);
        uint32_t b0, b1, b2, b3;
        ldsm_x4(smem_u32(tk) + soff<D>(krow, 2 * ks + (mi & 1)), b0, b1, b2, b3);
        mma16816(s[nb], qa, b0, b1);
        mma16816(s[nb + 1], qa, b2, b3);
      }
    }
    // ---- mask (split end; causal inside the query's own tail), online softmax
    const bool need_mask = (p0 + KT > k_end) || (p0 < k_lo) || (p0 + KT - 1 > pos_first);
    float tmax[2] = {-INFINITY, -INFINITY};
#pragma unroll
    for (int nb = 0; nb < NB; ++nb)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        float x = s[nb][e] * sl2;
        if (need_mask) {
          const int kp = p0 + nb * 8 + 2 * tq + (e & 1);
          if (kp >= k_end || kp < k_lo || kp > qpos[e >> 1]) x = -INFINITY;
        }
        s[nb][e] = x;
        tmax[e >> 1] = fmaxf(tmax[e >> 1], x);
      }
    // Lazy rescale: the running max only moves (and O, l are rescaled) when
    // a row's new scores exceed it by more than 2^8; until then the stale max
    // keeps every exponent <= 2^8, which fp32 and bf16 P hold without loss.
    float mu[2];
#pragma unroll
    for (int h2 = 0; h2 < 2; ++h2) {
      tmax[h2] = fmaxf(tmax[h2], __shfl_xor_sync(0xFFFFFFFFu, tmax[h2], 1));
      tmax[h2] = fmaxf(tmax[h2], __shfl_xor_sync(0xFFFFFFFFu, tmax[h2], 2));
      if (tmax[h2] > m_run[h2] + 8.0f) {
        const float mn = tmax[h2];
        const float alpha = (m_run[h2] == -INFINITY) ? 0.f : ex2(m_run[h2] - mn);
        m_run[h2] = mn;
        l_run[h2] *= alpha;
#pragma unroll
        for (int nd = 0; nd < ND; ++nd) {
          o[nd][2 * h2] *= alpha;
          o[nd][2 * h2 + 1] *= alpha;
        }
      }
      mu[h2] = (m_run[h2] == -INFINITY) ? 0.f : m_run[h2];
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
    for (int kk = 0; kk < KT / 16; ++kk) {
      uint32_t pa[4];
      pa[0] = pack_bf16(s[2 * kk][0], s[2 * kk][1]);
      pa[1] = pack_bf16(s[2 * kk][2], s[2 * kk][3]);
      pa[2] = pack_bf16(s[2 * kk + 1][0], s[2 * kk + 1][1]);
      pa[3] = pack_bf16(s[2 * kk + 1][2], s[2 * kk + 1][3]);
      const int mi = lane >> 3;
      const int vrow = kk * 16 + (mi & 1) * 8 + (lane & 7);
#pragma unroll
      for (int nd = 0; nd < ND; nd += 2) {
        uint32_t b0, b1, b2, b3;
        ldsm_x4_t(smem_u32(tv) + soff<D>(vrow, nd + (mi >> 1)), b0, b1, b2, b3);
        mma16816(o[nd], pa, b0, b1);
        mma16816(o[nd + 1], pa, b2, b3);
      }
    }
  }
  cp_async_wait<0>();

  // ---- row sums over the quad
#pragma unroll
  for (int h2 = 0; h2 < 2; ++h2) {
    l_run[h2] += __shfl_xor_sync(0xFFFFFFFFu, l_run[h2], 1);
    l_run[h2] += __shfl_xor_sync(0xFFFFFFFFu, l_run[h2], 2);
  }
  auto part_index = [&](int r) -> int64_t {  // r = row index of the CTA (token-major)
    return ((int64_t)it_idx * a.Hq + c * g + r % g) * a.n_new + r / g;
  };

  // partials: (M, L) and the normalised output acc / L as bf16
  if constexpr (KG == 1) {
#pragma unroll
    for (int h2 = 0; h2 < 2; ++h2) {
      const int r = row_base + wr * 16 + gq + 8 * h2;
      if (r >= R) continue;
      const int64_t pi = part_index(r);
      const float inv = l_run[h2] > 0.f ? 1.f / l_run[h2] : 0.f;
      uint16_t *acc = a.part_acc + pi * D;
#pragma unroll
      for (int nd = 0; nd < ND; ++nd)
        *reinterpret_cast<uint32_t *>(acc + nd * 8 + 2 * tq) =
            pack_bf16(o[nd][2 * h2] * inv, o[nd][2 * h2 + 1] * inv);
      if (tq == 0) a.part_ml[pi] = make_float2(m_run[h2], l_run[h2]);
    }
  } else {
    // merge the key groups' states for the CTA's rows through shared memory
    __syncthreads();
    float *so = reinterpret_cast<float *>(sRing);                  // [KG][MROWS][D]
    float2 *sml = reinterpret_cast<float2 *>(so + KG * MROWS * D);  // [KG][MROWS]
#pragma unroll
    for (int h2 = 0; h2 < 2; ++h2) {
      const int rr = wr * 16 + gq + 8 * h2;
#pragma unroll
      for (int nd = 0; nd < ND; ++nd)
        *reinterpret_cast<float2 *>(so + ((size_t)kg * MROWS + rr) * D + nd * 8 + 2 * tq) =
            make_float2(o[nd][2 * h2], o[nd][2 * h2 + 1]);
      if (tq == 0) sml[kg * MROWS + rr] = make_float2(m_run[h2], l_run[h2]);
    }
    __syncthreads();
    for (int idx = tid; idx < MROWS * (D / 4); idx += NTOT) {
      const int rr = idx / (D / 4), d0 = (idx % (D / 4)) * 4;
      const int r = row_base + rr;
      if (r >= R) continue;
      float M = -INFINITY;
#pragma unroll
      for (int k = 0; k < KG; ++k) M = fmaxf(M, sml[k * MROWS + rr].x);
      float L = 0.f;
      float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
      for (int k = 0; k < KG; ++k) {
        const float2 ml = sml[k * MROWS + rr];
        const float w = (ml.x == -INFINITY) ? 0.f : ex2(ml.x - M);
        L += w * ml.y;
        const float4 x = *reinterpret_cast<const float4 *>(so + ((size_t)k * MROWS + rr) * D + d0);
        acc.x += w * x.x;
        acc.y += w * x.y;
        acc.z += w * x.z;
        acc.w += w * x.w;
      }
      const int64_t pi = part_index(r);
      const float inv = L > 0.f ? 1.f / L : 0.f;
      *reinterpret_cast<uint2 *>(a.part_acc + pi * D + d0) =
          make_uint2(pack_bf16(acc.x * inv, acc.y * inv), pack_bf16(acc.z * inv, acc.w * inv));
      if (d0 == 0) a.part_ml[pi] = make_float2(M, L);
    }
  }
}

// One warp per output row (query q, token u, head h): combine the row's split
// partials, O = sum_i 2^(M_i - M) L_i O_i / sum_i 2^(M_i - M) L_i.  The lanes
// read the items' (M_i, L_i) in parallel (lane i % 32 holds item i's weight);
// the items' rows are then added in item order, four loads in flight.  Rows
// run token-fastest, the order of an item's partial rows, so the warps of a
// CTA read adjacent rows of each item.
template <int D, typename OT>
__global__ void __launch_bounds__(128) stage2_merge_kernel(const Stage2Args a) {
  pdl_enter();
  const int64_t row = (int64_t)blockIdx.x * 4 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  const int64_t n_rows = (int64_t)a.n_queries * a.n_new * a.Hq;
  if (row >= n_rows) return;
  const int tok = (int)(row % a.n_new);
  const int h = (int)((row / a.n_new) % a.Hq);
  const int q = (int)(row / ((int64_t)a.Hq * a.n_new));
  const S2Query qi = a.queries[q];
  const int n = qi.n_items;
  auto part = [&](int i) { return ((int64_t)(qi.item_begin + i) * a.Hq + h) * a.n_new + tok; };
  float M = -INFINITY;
  for (int i = lane; i < n; i += 32) M = fmaxf(M, a.part_ml[part(i)].x);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
  constexpr int PER = D / 32;
  float acc[PER];
#pragma unroll
  for (int e = 0; e < PER; ++e) acc[e] = 0.f;
  float L = 0.f;
  auto load_row = [&](int i, uint16_t (&v)[PER]) {
    const uint16_t *src = a.part_acc + part(i) * D + lane * PER;
    if constexpr (PER == 4) {
      *reinterpret_cast<uint2 *>(v) = *reinterpret_cast<const uint2 *>(src);
    } else {
      *reinterpret_cast<uint32_t *>(v) = *reinterpret_cast<const uint32_t *>(src);
    }
  };
  for (int i0 = 0; i0 < n; i0 += 32) {
    float w = 0.f;
    if (i0 + lane < n) {
      const float2 ml = a.part_ml[part(i0 + lane)];
      w = (ml.x == -INFINITY) ? 0.f : ex2(ml.x - M) * ml.y;
    }
    L += w;
    const int cnt = min(32, n - i0);
    for (int j = 0; j < cnt; j += 4) {
      uint16_t v[4][PER];
#pragma unroll
      for (int k = 0; k < 4; ++k)
        if (j + k < cnt) load_row(i0 + j + k, v[k]);
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const float wk = __shfl_sync(0xffffffffu, w, (j + k) & 31);
        if (j + k < cnt) {
#pragma unroll
          for (int e = 0; e < PER; ++e) acc[e] += wk * __uint_as_float((uint32_t)v[k][e] << 16);
        }
      }
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) L += __shfl_xor_sync(0xffffffffu, L, o);
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

// Block-major mode, after the tensor-core pass: each query's own tail tokens
// and the merge of every partial of a row, in one kernel.  CTA = (query q,
// KV head c, group of up to 8 rows of the query's g * n_new rows); two warps
// per output row (query token u, head h), each taking half of the row's
// sources: alternate groups of 4 tail keys, and one half of its partials.
// Lane l holds the elements i = l + 32 j (j < D / 32), so the rotate-half
// pairs (i, i + D/2) sit in the same lane.  The CTA rotates the tail keys its
// rows can see, 32 at a time, into shared memory at their positions T'_q + u'
// (fp32, no rounding), with their values; a warp scores its rotated query row
// against its keys u' <= the row's tail index (the causal rule), in log2
// units, with an online softmax.  It then merges its half of the row's block
// partials (M_i, L_i, O_i), written by the tensor-core pass, into that state
// (m, l, acc):  with M = max(m, max_i M_i),
//   o = 2^(m - M) acc + sum_i 2^(M_i - M) L_i O_i,   n = 2^(m - M) l + sum_i 2^(M_i - M) L_i,
// and the two warps' (M, n, o) are combined into O = o / n.
template <int D, typename CT>
__global__ void __launch_bounds__(512, 2) stage2_tail_merge_kernel(const Stage2Args a) {
  pdl_enter();
  constexpr int H = D / 2;
  constexpr int E = D / 32;           // elements per lane
  constexpr int CH = 32;              // tail keys per shared-memory chunk
  __shared__ float sK[CH][D], sV[CH][D];
  __shared__ float sO[16][D];         // a warp's tail accumulator, regrouped for the merge
  __shared__ float sC[8][D + 2];      // the second warp of each row: (M, n, o)
  const int q = blockIdx.x, c = blockIdx.y;
  const int g = a.Hq / a.Hkv;
  const int R = g * a.n_new;
  const int RW = min(8, R);                     // rows per CTA
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int rw = warp % RW, hf = warp / RW;     // row slot, half of the row's sources
  const int r = blockIdx.z * 8 + rw;            // this warp's row (token-major: u * g + hl)
  const bool live = r < R;
  const S2Query qi = a.queries[q];
  const int Tq = qi.n_gathered;
  const int tok = live ? r / g : 0;
  const int h = c * g + (live ? r % g : 0);
  const int tu = a.tail_len - a.n_new + tok;    // this row's tail index
  const float sl2 = a.scale_log2;
  // the query row, rotated at T'_q + tu
  float qr[E];
  {
    const CT *src = static_cast<const CT *>(a.q_new) + (((int64_t)q * a.n_new + tok) * a.Hq + h) * D;
#pragma unroll
    for (int j = 0; j < E; ++j) qr[j] = to_f32(src[lane + 32 * j]);
    const int64_t pq = (int64_t)Tq + tu;
#pragma unroll
    for (int j = 0; j < E / 2; ++j) {
      float cs, sn;
      rope_cs1(a.rope, pq, lane + 32 * j, H, cs, sn);
      const float lo = qr[j], hi = qr[j + E / 2];
      qr[j] = __fmaf_rn(lo, cs, __fmul_rn(-hi, sn));
      qr[j + E / 2] = __fmaf_rn(hi, cs, __fmul_rn(lo, sn));
    }
  }
  float m = -INFINITY, l = 0.f, acc[E];
#pragma unroll
  for (int j = 0; j < E; ++j) acc[j] = 0.f;
  // the CTA's rows see the tail keys up to its last row's tail index
  const int r_last = min(R, blockIdx.z * 8 + RW) - 1;
  const int k_end = a.tail_len - a.n_new + r_last / g + 1;
  for (int k0 = 0; k0 < k_end; k0 += CH) {
    const int nk = min(CH, k_end - k0);
    __syncthreads();   // the previous chunk has been read by every warp
#pragma unroll 4
    for (int u = threadIdx.x; u < nk * H; u += blockDim.x) {
      const int j = u / H, i = u % H;
      const int64_t row = ((int64_t)q * a.tail_cap + k0 + j) * a.Hkv + c;
      const CT *ks = static_cast<const CT *>(a.k_tail) + row * D;
      const CT *vs = static_cast<const CT *>(a.v_tail) + row * D;
      float cs, sn;
      rope_cs1(a.rope, (int64_t)Tq + k0 + j, i, H, cs, sn);
      const float lo = to_f32(ks[i]), hi = to_f32(ks[i + H]);
      sK[j][i] = __fmaf_rn(lo, cs, __fmul_rn(-hi, sn));
      sK[j][i + H] = __fmaf_rn(hi, cs, __fmul_rn(lo, sn));
      sV[j][i] = to_f32(vs[i]);
      sV[j][i + H] = to_f32(vs[i + H]);
    }
    __syncthreads();
    // keys k0 .. k0 + n - 1 of this chunk are visible to the row (u' <= tu);
    // this warp takes the groups of 4 starting at 4 hf, 4 hf + 8, ...
    const int n = live ? max(0, min(nk, tu - k0 + 1)) : 0;
    for (int j0 = 4 * hf; j0 < n; j0 += 8) {
      float sc[4];
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        float d = 0.f;
        if (j0 + t < n) {
#pragma unroll
          for (int j = 0; j < E; ++j) d = __fmaf_rn(qr[j], sK[j0 + t][lane + 32 * j], d);
        }
        sc[t] = d;
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1)
#pragma unroll
        for (int t = 0; t < 4; ++t) sc[t] += __shfl_xor_sync(0xffffffffu, sc[t], o);
      float mx = m;
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        sc[t] = (j0 + t < n) ? sc[t] * sl2 : -INFINITY;
        mx = fmaxf(mx, sc[t]);
      }
      const float alpha = (m == -INFINITY) ? 0.f : ex2(m - mx);
      l *= alpha;
#pragma unroll
      for (int j = 0; j < E; ++j) acc[j] *= alpha;
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        const float pt = ex2(sc[t] - mx);
        l += pt;
        if (j0 + t < n) {
#pragma unroll
          for (int j = 0; j < E; ++j) acc[j] = __fmaf_rn(pt, sV[j0 + t][lane + 32 * j], acc[j]);
        }
      }
      m = mx;
    }
  }
  // this warp's half of the row's block partials (every item of the query but
  // the last, its tail item).  For the merge each lane takes E consecutive
  // elements (8- or 4-byte loads of every partial row), so the tail
  // accumulator is regrouped through shared memory first.
#pragma unroll
  for (int j = 0; j < E; ++j) sO[warp][lane + 32 * j] = acc[j];
  __syncwarp();
  float acc_c[E];
#pragma unroll
  for (int j = 0; j < E; ++j) acc_c[j] = sO[warp][E * lane + j];
  const int nb = qi.n_items - 1;
  const int nb0 = (nb + 1) / 2;
  const int i_lo = hf == 0 ? 0 : nb0, i_hi = live ? (hf == 0 ? nb0 : nb) : i_lo;
  auto part = [&](int i) { return ((int64_t)(qi.item_begin + i) * a.Hq + h) * a.n_new + tok; };
  float M = m;
  for (int i = i_lo + lane; i < i_hi; i += 32) M = fmaxf(M, a.part_ml[part(i)].x);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
  const float wt = (m == -INFINITY) ? 0.f : ex2(m - M);   // this warp may have no tail key
  float L = 0.f, out[E];
#pragma unroll
  for (int j = 0; j < E; ++j) out[j] = wt * acc_c[j];
  using Vec = typename std::conditional<E == 4, uint2, uint32_t>::type;   // E bf16 values
  constexpr int U = 6;                         // partial rows in flight (64 registers)
  for (int i0 = i_lo; i0 < i_hi; i0 += 32) {
    float w = 0.f;
    if (i0 + lane < i_hi) {
      const float2 ml = a.part_ml[part(i0 + lane)];
      w = (ml.x == -INFINITY) ? 0.f : ex2(ml.x - M) * ml.y;
    }
    L += w;
    const int cnt = min(32, i_hi - i0);
    for (int k0 = 0; k0 < cnt; k0 += U) {
      Vec v[U];
#pragma unroll
      for (int k = 0; k < U; ++k)
        if (k0 + k < cnt)
          v[k] = *reinterpret_cast<const Vec *>(a.part_acc + part(i0 + k0 + k) * D + E * lane);
#pragma unroll
      for (int k = 0; k < U; ++k) {
        const float wk = __shfl_sync(0xffffffffu, w, (k0 + k) & 31);
        if (k0 + k < cnt) {
          const uint32_t *wv = reinterpret_cast<const uint32_t *>(&v[k]);
#pragma unroll
          for (int j = 0; j < E / 2; ++j) {
            out[2 * j] = __fmaf_rn(wk, __uint_as_float(wv[j] << 16), out[2 * j]);
            out[2 * j + 1] = __fmaf_rn(wk, __uint_as_float(wv[j] & 0xFFFF0000u), out[2 * j + 1]);
          }
        }
      }
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) L += __shfl_xor_sync(0xffffffffu, L, o);
  const float nrm = L + wt * l;                // this warp's normaliser at scale M
  // the second warp of the row hands (M, n, o) to the first, which combines
  if (hf == 1) {
    if (lane == 0) {
      sC[rw][0] = M;
      sC[rw][1] = nrm;
    }
#pragma unroll
    for (int j = 0; j < E; ++j) sC[rw][2 + E * lane + j] = out[j];
  }
  __syncthreads();
  if (hf == 1 || !live) return;
  const float M1 = sC[rw][0], n1 = sC[rw][1];
  const float Mx = fmaxf(M, M1);
  const float f0 = (M == -INFINITY) ? 0.f : ex2(M - Mx);
  const float f1 = (M1 == -INFINITY) ? 0.f : ex2(M1 - Mx);
  const float inv = 1.f / (f0 * nrm + f1 * n1);
  CT *dst = static_cast<CT *>(a.out) + (((int64_t)q * a.n_new + tok) * a.Hq + h) * D + E * lane;
#pragma unroll
  for (int j = 0; j < E; ++j) from_f32((f0 * out[j] + f1 * sC[rw][2 + E * lane + j]) * inv, dst[j]);
}

template <int D, typename CT, int RT, int KG, int KT>
cudaError_t launch_main(const Stage2Args &a, cudaStream_t st) {
  constexpr int NST = 3;
  constexpr int MROWS = 16 * RT;
  constexpr size_t ring = (size_t)KG * NST * 2 * KT * D * 2;
  constexpr size_t merge = KG > 1 ? (size_t)KG * MROWS * (D * 4 + 8) : 0;
  constexpr size_t lo_tables = (size_t)2 * kRopeLo * (D / 2) * sizeof(float);
  constexpr size_t smem = (size_t)MROWS * D * 2 + lo_tables + (ring > merge ? ring : merge);
  static_assert(smem <= 232448, "shared memory budget");
  cudaError_t e = cudaFuncSetAttribute(stage2_attn_kernel<D, CT, RT, KG, KT, NST>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const int R = (a.Hq / a.Hkv) * a.n_new;
  if (a.n_run <= 0) return cudaSuccess;
  dim3 grid(a.n_run, a.Hkv, (R + MROWS - 1) / MROWS);
  pdl_launch(stage2_attn_kernel<D, CT, RT, KG, KT, NST>, dim3(grid), dim3(32 * RT * KG), smem, st, a);
  return cudaGetLastError();
}

// Rows per CTA by pass shape: <= 16 rows (decode): 4 key groups of 1 warp;
// <= 32: 4 x 2; <= 64: 2 x 4; <= 128: 1 x 8; larger: 1 x 10 warps (160 rows)
// per row group.
template <int D, typename CT>
cudaError_t launch_d(const Stage2Args &a, cudaStream_t st) {
  const int R = (a.Hq / a.Hkv) * a.n_new;
  // tail items span at most tail_len + 15 keys: 4 key groups of 16 keys cover
  // a decode step's tail (<= 48 tokens) in one round at 2 CTAs per SM
  if (R <= 16) return launch_main<D, CT, 1, 4, 16>(a, st);
  if (R <= 32) return launch_main<D, CT, 2, 4, 32>(a, st);
  if (R <= 64) return launch_main<D, CT, 4, 2, 64>(a, st);
  if (R <= 128) return launch_main<D, CT, 8, 1, 64>(a, st);
  return launch_main<D, CT, 10, 1, 80>(a, st);
}

template <int D, typename CT>
cudaError_t launch_tail_merge(const Stage2Args &a, cudaStream_t st) {
  const int R = (a.Hq / a.Hkv) * a.n_new;
  dim3 grid(a.n_queries, a.Hkv, (R + 7) / 8);
  pdl_launch(stage2_tail_merge_kernel<D, CT>, dim3(grid), dim3(64 * min(8, R)), 0, st, a);   // two warps per row
  return cudaGetLastError();
}

template <int D, typename CT>
cudaError_t launch_merge(const Stage2Args &a, cudaStream_t st) {
  const int64_t rows = (int64_t)a.n_queries * a.n_new * a.Hq;
  pdl_launch(stage2_merge_kernel<D, CT>, dim3((unsigned)((rows + 3) / 4)), dim3(128), 0, st, a);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_stage2_main(const Stage2Args &a, int head_dim, bool f32, cudaStream_t st) {
  if (a.n_items <= 0) return cudaSuccess;
  if (head_dim == 128) return f32 ? launch_d<128, float>(a, st) : launch_d<128, bf16>(a, st);
  return f32 ? launch_d<64, float>(a, st) : launch_d<64, bf16>(a, st);
}

cudaError_t launch_stage2_tail_merge(const Stage2Args &a, int head_dim, bool f32,
                                     cudaStream_t st) {
  if (a.n_queries <= 0) return cudaSuccess;
  if (head_dim == 128)
    return f32 ? launch_tail_merge<128, float>(a, st) : launch_tail_merge<128, bf16>(a, st);
  return f32 ? launch_tail_merge<64, float>(a, st) : launch_tail_merge<64, bf16>(a, st);
}

cudaError_t launch_stage2_merge(const Stage2Args &a, int head_dim, bool f32, cudaStream_t st) {
  if (a.n_items <= 0) return cudaSuccess;
  if (head_dim == 128) return f32 ? launch_merge<128, float>(a, st) : launch_merge<128, bf16>(a, st);
  return f32 ? launch_merge<64, float>(a, st) : launch_merge<64, bf16>(a, st);
}

}  // namespace dbsa
