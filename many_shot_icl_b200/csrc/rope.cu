// RoPE angle tables and the Stage-1 preparation kernels.
//
// [DBSA notes] §Stage 1, item 3: queries and keys are rotated at sequential
// positions, while the cache keeps K/V BEFORE the rotary transform.  The
// preparation pass therefore (a) copies the raw K/V into the head-major cache,
// (b) writes a rotated bf16 copy of K into the workspace for the tensor-core
// kernel (which rotates the queries itself as it reads them), and for fp32
// inputs (c) a bf16 copy of V.  It is pure streaming work (HBM-bound); the
// angle factors come from two small tables built once per call in fp64.
#include <cuda_bf16.h>

#include "dbsa_internal.h"
#include "vec8.cuh"

namespace dbsa {
namespace {

__global__ void rope_tables_kernel(float *base, int32_t n_hi, int32_t half, double theta) {
  pdl_enter();
  const int64_t n = (int64_t)(n_hi + kRopeLo) * half;
  float *hc = base, *hs = hc + (int64_t)n_hi * half;
  float *lc = hs + (int64_t)n_hi * half, *ls = lc + (int64_t)kRopeLo * half;
  for (int64_t u = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; u < n;
       u += (int64_t)gridDim.x * blockDim.x) {
    const int32_t i = (int32_t)(u % half);
    const int64_t row = u / half;
    const double w = pow(theta, -2.0 * (double)i / (double)(2 * half));
    double sn, cs;
    if (row < n_hi) {
      sincos((double)(row * kRopeLo) * w, &sn, &cs);
      hc[row * half + i] = (float)cs;
      hs[row * half + i] = (float)sn;
    } else {
      const int64_t r = row - n_hi;
      sincos((double)r * w, &sn, &cs);
      lc[r * half + i] = (float)cs;
      ls[r * half + i] = (float)sn;
    }
  }
}

// One work unit = (token t, head slot hh, chunk cp): elements [8cp, 8cp+8) of
// the first half and the matching 8 of the second half; slots 0..Hkv-1 are
// the key heads, the rest the value heads.
template <int D, typename T>
__global__ void __launch_bounds__(256) ingest_kernel(IngestArgs a) {
  pdl_enter();
  constexpr int H = D / 2;
  constexpr int CP = H / 8;
  const int slots = 2 * a.Hkv;
  const int64_t n_units = (int64_t)a.n_tok * slots * CP;
  const T *k = static_cast<const T *>(a.k);
  const T *v = static_cast<const T *>(a.v);
  for (int64_t u = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; u < n_units;
       u += (int64_t)gridDim.x * blockDim.x) {
    const int cp = (int)(u % CP);
    const int hh = (int)((u / CP) % slots);
    const int64_t t = u / ((int64_t)CP * slots);
    const int64_t pos = a.pos0 + t;
    const int i0 = cp * 8;
    float lo[8], hi[8];
    if (hh < a.Hkv) {  // key head: cache the raw key, rotate into k_rot
      const int c_ = hh;
      const T *src = k + (t * a.Hkv + c_) * D;
      T *cache = static_cast<T *>(a.k_cache) + ((int64_t)c_ * a.cap + pos) * D;
      copy8(src + i0, cache + i0);
      copy8(src + H + i0, cache + H + i0);
      load8(src + i0, lo);
      load8(src + H + i0, hi);
      float c[8], s[8];
      rope_cs8(a.rope, pos, i0, H, c, s);
      rotate8(lo, hi, c, s);
      bf16 *dst = static_cast<bf16 *>(a.k_rot) + ((int64_t)c_ * a.k_rows + a.k_row_base + t) * D;
      store8_bf16(dst + i0, lo);
      store8_bf16(dst + H + i0, hi);
    } else {  // value head: cache the raw value (and a bf16 copy for fp32 inputs)
      const int c_ = hh - a.Hkv;
      const T *src = v + (t * a.Hkv + c_) * D;
      T *cache = static_cast<T *>(a.v_cache) + ((int64_t)c_ * a.cap + pos) * D;
      copy8(src + i0, cache + i0);
      copy8(src + H + i0, cache + H + i0);
      if (a.v_bf16 != nullptr) {
        load8(src + i0, lo);
        load8(src + H + i0, hi);
        bf16 *dst =
            static_cast<bf16 *>(a.v_bf16) + ((int64_t)c_ * a.k_rows + a.k_row_base + t) * D;
        store8_bf16(dst + i0, lo);
        store8_bf16(dst + H + i0, hi);
      }
    }
  }
}

// Cache rows [row0, row0+n) of every KV head, at positions equal to the row.
template <int D, typename T>
__global__ void __launch_bounds__(256) window_kernel(WindowArgs a) {
  pdl_enter();
  constexpr int H = D / 2;
  constexpr int CP = H / 8;
  const int64_t n_units = (int64_t)a.n * a.Hkv * CP;
  for (int64_t u = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; u < n_units;
       u += (int64_t)gridDim.x * blockDim.x) {
    const int cp = (int)(u % CP);
    const int c_ = (int)((u / CP) % a.Hkv);
    const int64_t r = u / ((int64_t)CP * a.Hkv);
    const int64_t pos = a.row0 + r;
    const int i0 = cp * 8;
    float lo[8], hi[8], c[8], s[8];
    const T *src = static_cast<const T *>(a.k_cache) + ((int64_t)c_ * a.cap + pos) * D;
    load8(src + i0, lo);
    load8(src + H + i0, hi);
    rope_cs8(a.rope, pos, i0, H, c, s);
    rotate8(lo, hi, c, s);
    bf16 *dst = static_cast<bf16 *>(a.k_rot) + ((int64_t)c_ * a.k_rows + a.dst_row0 + r) * D;
    store8_bf16(dst + i0, lo);
    store8_bf16(dst + H + i0, hi);
    if (a.v_bf16 != nullptr) {
      const T *vs = static_cast<const T *>(a.v_cache) + ((int64_t)c_ * a.cap + pos) * D;
      load8(vs + i0, lo);
      load8(vs + H + i0, hi);
      bf16 *vd = static_cast<bf16 *>(a.v_bf16) + ((int64_t)c_ * a.k_rows + a.dst_row0 + r) * D;
      store8_bf16(vd + i0, lo);
      store8_bf16(vd + H + i0, hi);
    }
  }
}

// Key rows at block-relative positions (row s of block b at s - offs[b]).
template <int D, typename T>
__global__ void __launch_bounds__(256) rel_rope_kernel(RelRopeArgs a) {
  pdl_enter();
  constexpr int H = D / 2;
  constexpr int CP = H / 8;
  const int64_t n_units = (int64_t)a.T * a.Hkv * CP;
  for (int64_t u = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; u < n_units;
       u += (int64_t)gridDim.x * blockDim.x) {
    const int cp = (int)(u % CP);
    const int c_ = (int)((u / CP) % a.Hkv);
    const int32_t s = (int32_t)(u / ((int64_t)CP * a.Hkv));
    int lo = 0, hi = a.nb;  // block of row s: offs[lo] <= s < offs[lo + 1]
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (__ldg(a.offs + mid) <= s) lo = mid; else hi = mid;
    }
    const int64_t pos = s - __ldg(a.offs + lo);
    const int i0 = cp * 8;
    float xl[8], xh[8], c[8], sn[8];
    const T *src = static_cast<const T *>(a.k_cache) + ((int64_t)c_ * a.cap + s) * D;
    load8(src + i0, xl);
    load8(src + H + i0, xh);
    rope_cs8(a.rope, pos, i0, H, c, sn);
    rotate8(xl, xh, c, sn);
    bf16 *dst = static_cast<bf16 *>(a.k_hat) + ((int64_t)c_ * a.T + s) * D;
    store8_bf16(dst + i0, xl);
    store8_bf16(dst + H + i0, xh);
    if (a.v_bf16 != nullptr) {
      const T *vs = static_cast<const T *>(a.v_cache) + ((int64_t)c_ * a.cap + s) * D;
      load8(vs + i0, xl);
      load8(vs + H + i0, xh);
      bf16 *vd = static_cast<bf16 *>(a.v_bf16) + ((int64_t)c_ * a.T + s) * D;
      store8_bf16(vd + i0, xl);
      store8_bf16(vd + H + i0, xh);
    }
  }
}

template <int D, typename T>
__global__ void __launch_bounds__(256) qhat_kernel(QHatArgs a) {
  pdl_enter();
  // One thread per (block item, query token, kv head, 8-pair chunk): the g
  // query heads of the kv head share the token's position, so the rotation
  // factors are built once and applied to all g rows (row token * g + local
  // head of the item, in the plane of the kv head).
  constexpr int H = D / 2;
  constexpr int CP = H / 8;
  const int g = a.Hq / a.Hkv;
  const int64_t n_units = (int64_t)a.n_items * a.n_new * a.Hkv * CP;
  for (int64_t u = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; u < n_units;
       u += (int64_t)gridDim.x * blockDim.x) {
    const int cp = (int)(u % CP);
    const int c_ = (int)((u / CP) % a.Hkv);
    const int tok = (int)((u / ((int64_t)CP * a.Hkv)) % a.n_new);
    const int item = (int)(u / ((int64_t)CP * a.Hkv * a.n_new));
    const int4 meta = __ldg(a.item_meta + item);
    const int row0 = meta.x;
    if (row0 < 0) continue;                      // a tail item: no packed rows
    const int q = meta.z;
    const int64_t pos = (int64_t)meta.y + tok;   // (its position - the block's fresh start)
    // the position used for token 0 of the item, for the gather map
    if (a.q_rot_pos != nullptr && tok == 0 && c_ == 0 && cp == 0) a.q_rot_pos[item] = (int32_t)pos;
    const int i0 = cp * 8;
    float c[8], sn[8];
    rope_cs8(a.rope, pos, i0, H, c, sn);
    const T *src =
        static_cast<const T *>(a.q_new) + (((int64_t)q * a.n_new + tok) * a.Hq + c_ * g) * D;
    bf16 *dst = static_cast<bf16 *>(a.q_hat) + ((int64_t)c_ * a.rows + row0 + tok * g) * D;
    for (int hl = 0; hl < g; ++hl) {
      float xl[8], xh[8];
      load8(src + (int64_t)hl * D + i0, xl);
      load8(src + (int64_t)hl * D + H + i0, xh);
      rotate8(xl, xh, c, sn);
      store8_bf16(dst + (int64_t)hl * D + i0, xl);
      store8_bf16(dst + (int64_t)hl * D + H + i0, xh);
    }
  }
}

// Compact mode of Stage 2: compact row r of KV head c holds gathered token p
// of query q (r = base[q] + p): its key rotated at its fresh position p, and
// its value, both bf16.  One warp per (segment, KV head) walks the segment's
// contiguous cache rows, four rows in flight; lane l owns the frequencies
// 2l and 2l + 1 (lanes 2l >= D/2 have none), so each rotate-half pair
// (i, i + D/2) stays in one lane.  With a gather map requested, KV head 0's
// warp records (cache row, p) for every row it reads.
template <int D, typename T>
__global__ void __launch_bounds__(256) compact_kernel(CompactArgs a) {
  pdl_enter();
  constexpr int H = D / 2;
  const int lane = threadIdx.x & 31;
  const bool has_pair = 2 * lane < H;
  const int64_t n_tasks = (int64_t)a.n_segs * a.Hkv;
  const int64_t warp0 = (blockIdx.x * (int64_t)blockDim.x + threadIdx.x) >> 5;
  const int64_t n_warps = ((int64_t)gridDim.x * blockDim.x) >> 5;
  for (int64_t task = warp0; task < n_tasks; task += n_warps) {
    const int c_ = (int)(task % a.Hkv);
    const S2Segment sg = a.segs[task / a.Hkv];
    const int64_t rbase = (int64_t)__ldg(a.base + sg.query) + sg.pos0;
    const T *ksrc = static_cast<const T *>(a.k_cache) + ((int64_t)c_ * a.cap + sg.cache_row0) * D;
    const T *vsrc = static_cast<const T *>(a.v_cache) + ((int64_t)c_ * a.cap + sg.cache_row0) * D;
    bf16 *kdst = static_cast<bf16 *>(a.k_hat) + ((int64_t)c_ * a.rows + rbase) * D;
    bf16 *vdst = static_cast<bf16 *>(a.v_hat) + ((int64_t)c_ * a.rows + rbase) * D;
    const int i = 2 * lane;   // this lane's frequencies i, i + 1
    for (int r0 = 0; r0 < sg.len; r0 += 4) {
      // the four rows' loads first (the stores below could alias them as far
      // as the compiler knows), then rotation and stores
      float kl[4][2], kh[4][2], vl[4][2], vh[4][2];
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const int r = r0 + k;
        if (has_pair && r < sg.len) {
          load2(ksrc + (int64_t)r * D + i, kl[k]);
          load2(ksrc + (int64_t)r * D + H + i, kh[k]);
          load2(vsrc + (int64_t)r * D + i, vl[k]);
          load2(vsrc + (int64_t)r * D + H + i, vh[k]);
        }
      }
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const int r = r0 + k;
        if (r >= sg.len) break;
        const int64_t pos = (int64_t)sg.pos0 + r;
        if (has_pair) {
          float cs[2], sn[2];
#pragma unroll
          for (int e = 0; e < 2; ++e) rope_cs1(a.rope, pos, i + e, H, cs[e], sn[e]);
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const float x = kl[k][e], y = kh[k][e];
            kl[k][e] = __fmaf_rn(x, cs[e], __fmul_rn(-y, sn[e]));
            kh[k][e] = __fmaf_rn(y, cs[e], __fmul_rn(x, sn[e]));
          }
          store2_bf16(kdst + (int64_t)r * D + i, kl[k]);
          store2_bf16(kdst + (int64_t)r * D + H + i, kh[k]);
          store2_bf16(vdst + (int64_t)r * D + i, vl[k]);
          store2_bf16(vdst + (int64_t)r * D + H + i, vh[k]);
        }
        if (a.dbg != nullptr && c_ == 0 && lane == 0)   // the row read and its rotation position
          *reinterpret_cast<int2 *>(a.dbg + ((int64_t)sg.query * a.dbg_cap + pos) * 2) =
              make_int2(sg.cache_row0 + r, (int)pos);
      }
    }
  }
}

int grid_for(int64_t n_units, int block) {
  int64_t g = (n_units + block - 1) / block;
  if (g > 148 * 16) g = 148 * 16;
  if (g < 1) g = 1;
  return (int)g;
}

}  // namespace

cudaError_t launch_rel_rope(const RelRopeArgs &a, int head_dim, bool f32, cudaStream_t st) {
  if (a.T <= 0) return cudaSuccess;
  const int g = grid_for((int64_t)a.T * a.Hkv * (head_dim / 16), 256);
  if (head_dim == 128) {
    if (f32) pdl_launch(rel_rope_kernel<128, float>, dim3(g), dim3(256), 0, st, a);
    else pdl_launch(rel_rope_kernel<128, bf16>, dim3(g), dim3(256), 0, st, a);
  } else {
    if (f32) pdl_launch(rel_rope_kernel<64, float>, dim3(g), dim3(256), 0, st, a);
    else pdl_launch(rel_rope_kernel<64, bf16>, dim3(g), dim3(256), 0, st, a);
  }
  return cudaGetLastError();
}

cudaError_t launch_qhat(const QHatArgs &a, int head_dim, bool f32, cudaStream_t st) {
  if (a.rows <= 0) return cudaSuccess;
  const int g = grid_for((int64_t)a.n_items * a.n_new * a.Hkv * (head_dim / 16), 256);
  if (head_dim == 128) {
    if (f32) pdl_launch(qhat_kernel<128, float>, dim3(g), dim3(256), 0, st, a);
    else pdl_launch(qhat_kernel<128, bf16>, dim3(g), dim3(256), 0, st, a);
  } else {
    if (f32) pdl_launch(qhat_kernel<64, float>, dim3(g), dim3(256), 0, st, a);
    else pdl_launch(qhat_kernel<64, bf16>, dim3(g), dim3(256), 0, st, a);
  }
  return cudaGetLastError();
}

cudaError_t launch_compact(const CompactArgs &a, int head_dim, bool f32, cudaStream_t st) {
  if (a.rows <= 0 || a.n_segs <= 0) return cudaSuccess;
  const int g = grid_for((int64_t)a.n_segs * a.Hkv * 32, 256);
  if (head_dim == 128) {
    if (f32) pdl_launch(compact_kernel<128, float>, dim3(g), dim3(256), 0, st, a);
    else pdl_launch(compact_kernel<128, bf16>, dim3(g), dim3(256), 0, st, a);
  } else {
    if (f32) pdl_launch(compact_kernel<64, float>, dim3(g), dim3(256), 0, st, a);
    else pdl_launch(compact_kernel<64, bf16>, dim3(g), dim3(256), 0, st, a);
  }
  return cudaGetLastError();
}

size_t rope_table_bytes(int32_t n_hi, int32_t head_dim) {
  return (size_t)2 * (n_hi + kRopeLo) * (head_dim / 2) * sizeof(float);
}

RopeTables rope_tables_at(const float *base, int32_t n_hi, int32_t head_dim) {
  const int64_t half = head_dim / 2;
  RopeTables t;
  t.hc = base;
  t.hs = t.hc + n_hi * half;
  t.lc = t.hs + n_hi * half;
  t.ls = t.lc + kRopeLo * half;
  t.n_hi = n_hi;
  return t;
}

cudaError_t launch_rope_tables(float *base, int32_t n_hi, int32_t head_dim, double theta,
                               cudaStream_t st) {
  const int half = head_dim / 2;
  const int64_t n = (int64_t)(n_hi + kRopeLo) * half;
  pdl_launch(rope_tables_kernel, dim3(grid_for(n, 256)), dim3(256), 0, st, base, n_hi, half, theta);
  return cudaGetLastError();
}

cudaError_t launch_ingest(const IngestArgs &a, int head_dim, bool f32, cudaStream_t st) {
  const int64_t n = (int64_t)a.n_tok * 2 * a.Hkv * (head_dim / 16);
  const int g = grid_for(n, 256);
  if (head_dim == 128) {
    if (f32) pdl_launch(ingest_kernel<128, float>, dim3(g), dim3(256), 0, st, a);
    else pdl_launch(ingest_kernel<128, bf16>, dim3(g), dim3(256), 0, st, a);
  } else {
    if (f32) pdl_launch(ingest_kernel<64, float>, dim3(g), dim3(256), 0, st, a);
    else pdl_launch(ingest_kernel<64, bf16>, dim3(g), dim3(256), 0, st, a);
  }
  return cudaGetLastError();
}

cudaError_t launch_window(const WindowArgs &a, int head_dim, bool f32, cudaStream_t st) {
  if (a.n <= 0) return cudaSuccess;
  const int64_t n = (int64_t)a.n * a.Hkv * (head_dim / 16);
  const int g = grid_for(n, 256);
  if (head_dim == 128) {
    if (f32) pdl_launch(window_kernel<128, float>, dim3(g), dim3(256), 0, st, a);
    else pdl_launch(window_kernel<128, bf16>, dim3(g), dim3(256), 0, st, a);
  } else {
    if (f32) pdl_launch(window_kernel<64, float>, dim3(g), dim3(256), 0, st, a);
    else pdl_launch(window_kernel<64, bf16>, dim3(g), dim3(256), 0, st, a);
  }
  return cudaGetLastError();
}

}  // namespace dbsa
