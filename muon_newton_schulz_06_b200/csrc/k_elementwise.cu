// Elementwise passes of the Muon step (HBM-bound):
//
//  * momentum_norm: M <- fl32(fl32(mu*M) + G), U <- fl32(G + fl32(mu*M)) (Nesterov) or
//    M, written to the workspace in wide orientation (transposed for tall matrices),
//    with a deterministic per-matrix sum of U^2 that ends in the scale
//    1/(||U||_F + eps).  Autoresearch train.py review, MuonAdamW paragraph: Muon
//    applies Nesterov momentum to the gradient with a buffer of the parameter's shape;
//    the Frobenius normalisation is the benchmark spec's.
//  * apply: W <- fl32(W - lrs*O) (then, with weight decay, - fl32(lr*wd)*W_old where the
//    decay applies) rounded to the parameter dtype, O read back from the workspace
//    (transposed for tall matrices); or export O into a caller buffer.
//
// One work unit is a 64 x 64 tile of the caller matrix; 256 threads each own 2 rows x 8
// consecutive columns, so rows move as 16-byte vectors (streaming cache hints: every
// byte is touched once per pass), and every load of a unit is issued before its stores.  Tall matrices go through a shared-memory tile to write /
// read the transposed workspace coalesced.  The norm is deterministic: each warp of a
// unit writes one partial sum (fixed shuffle tree), and a second small kernel adds a
// matrix's partials in a fixed order.
#include "muon_internal.h"

namespace muon {
namespace {

constexpr int kThreads = 256;

__device__ __forceinline__ float ld_elem(const void* p, size_t i, bool bf16) {
  return bf16 ? __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(p)[i])
              : reinterpret_cast<const float*>(p)[i];
}

__device__ __forceinline__ void ld8(const void* p, size_t i, bool bf16, float* v) {
  if (bf16) {
    uint4 raw = __ldcs(reinterpret_cast<const uint4*>(reinterpret_cast<const __nv_bfloat16*>(p) + i));
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&raw);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      float2 f = __bfloat1622float2(h[q]);
      v[2 * q] = f.x;
      v[2 * q + 1] = f.y;
    }
  } else {
    const float4* f = reinterpret_cast<const float4*>(reinterpret_cast<const float*>(p) + i);
    float4 a = __ldcs(f), b = __ldcs(f + 1);
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
    v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
  }
}

template <typename T>
__device__ __forceinline__ void st8(T* p, size_t i, const float* v);

template <>
__device__ __forceinline__ void st8<float>(float* p, size_t i, const float* v) {
  float4* f = reinterpret_cast<float4*>(p + i);
  __stcs(f, make_float4(v[0], v[1], v[2], v[3]));
  __stcs(f + 1, make_float4(v[4], v[5], v[6], v[7]));
}

template <>
__device__ __forceinline__ void st8<__nv_bfloat16>(__nv_bfloat16* p, size_t i, const float* v) {
  uint4 raw;
  __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&raw);
#pragma unroll
  for (int q = 0; q < 4; ++q) h[q] = __floats2bfloat162_rn(v[2 * q], v[2 * q + 1]);
  *reinterpret_cast<uint4*>(p + i) = raw;
}

template <typename T>
__device__ __forceinline__ void st1(T* p, size_t i, float v);
template <>
__device__ __forceinline__ void st1<float>(float* p, size_t i, float v) { p[i] = v; }
template <>
__device__ __forceinline__ void st1<__nv_bfloat16>(__nv_bfloat16* p, size_t i, float v) {
  p[i] = __float2bfloat16_rn(v);
}

__device__ __forceinline__ void st1_dyn(void* p, size_t i, float v, bool bf16) {
  if (bf16) reinterpret_cast<__nv_bfloat16*>(p)[i] = __float2bfloat16_rn(v);
  else reinterpret_cast<float*>(p)[i] = v;
}

__device__ __forceinline__ void st8_dyn(void* p, size_t i, const float* v, bool bf16) {
  if (bf16) st8<__nv_bfloat16>(reinterpret_cast<__nv_bfloat16*>(p), i, v);
  else st8<float>(reinterpret_cast<float*>(p), i, v);
}

// Matrix of a launch-wide work unit (binary search over unit_begin).
__device__ __forceinline__ int find_mat(const EwParams& p, int unit) {
  int lo = 0, hi = p.n_mats - 1;
  while (lo < hi) {
    int mid = (lo + hi + 1) >> 1;
    if (p.mats[mid].unit_begin <= unit) lo = mid; else hi = mid - 1;
  }
  return lo;
}

// Loads the 2 x 8 elements a thread owns in a 64 x 64 tile (zeros outside the matrix).
__device__ __forceinline__ void load_tile_rows(const void* src, bool bf16, const EwMat& m, int r0, int c, int tr,
                                               float (*v)[8]) {
#pragma unroll
  for (int pr = 0; pr < 2; ++pr) {
    const int r = r0 + tr + 32 * pr;
    const size_t base = (size_t)r * m.cols + c;
    if (r < m.rows && c + 8 <= m.cols && m.vec_ok) {
      ld8(src, base, bf16, v[pr]);
    } else {
#pragma unroll
      for (int q = 0; q < 8; ++q) v[pr][q] = (r < m.rows && c + q < m.cols) ? ld_elem(src, base + q, bf16) : 0.f;
    }
  }
}

// Momentum + Nesterov + U (workspace) + per-warp sums of U^2.  All loads of a unit are
// issued before any store, so each thread keeps 2 rows of G and M in flight.
template <typename WT>
__global__ void __launch_bounds__(kThreads)
momentum_norm_kernel(const __grid_constant__ EwParams p) {
  __shared__ float tile[kEwTile][kEwTile + 1];
  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const int tr = tid >> 3;        // 0..31
  const int tcol = (tid & 7) * 8; // 0..56

  for (int unit = blockIdx.x; unit < p.total_units; unit += gridDim.x) {
    const int mi = find_mat(p, unit);
    const EwMat& m = p.mats[mi];
    const int u = unit - m.unit_begin;
    const int r0 = (u / m.tiles_c) * kEwTile;
    const int c0 = (u % m.tiles_c) * kEwTile;
    const int c = c0 + tcol;
    WT* work = reinterpret_cast<WT*>(m.work);

    float g[2][8], mo[2][8];
    if (p.use_momentum) {
      load_tile_rows(m.grad, m.grad_bf16, m, r0, c, tr, g);
      load_tile_rows(m.mom, false, m, r0, c, tr, mo);
    } else {
      load_tile_rows(m.param, m.param_bf16, m, r0, c, tr, g);
    }
    float ssq = 0.f;
#pragma unroll
    for (int pr = 0; pr < 2; ++pr) {
      if (p.use_momentum) {
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          const float gq = p.lerp ? __fmul_rn(p.omu, g[pr][q]) : g[pr][q];
          const float mn = __fadd_rn(__fmul_rn(p.mu, mo[pr][q]), gq);
          mo[pr][q] = mn;
          g[pr][q] = p.nesterov ? __fadd_rn(gq, __fmul_rn(p.mu, mn)) : mn;  // g now holds U
        }
      }
#pragma unroll
      for (int q = 0; q < 8; ++q) ssq = fmaf(g[pr][q], g[pr][q], ssq);  // zero outside the matrix
    }
    if (m.transposed) __syncthreads();  // the previous unit's readers are done with `tile`
#pragma unroll
    for (int pr = 0; pr < 2; ++pr) {
      const int r = r0 + tr + 32 * pr;
      const bool in_row = r < m.rows;
      const bool full = in_row && (c + 8 <= m.cols);
      const size_t base = (size_t)r * m.cols + c;
      if (p.use_momentum) {
        if (full && m.vec_ok) {
          st8<float>(m.mom, base, mo[pr]);
        } else {
#pragma unroll
          for (int q = 0; q < 8; ++q)
            if (in_row && c + q < m.cols) m.mom[base + q] = mo[pr][q];
        }
      }
      if (!m.transposed) {
        if (full) {
          st8<WT>(work, (size_t)r * m.ld + c, g[pr]);
        } else {
#pragma unroll
          for (int q = 0; q < 8; ++q)
            if (in_row && c + q < m.cols) st1<WT>(work, (size_t)r * m.ld + c + q, g[pr][q]);
        }
      } else {
#pragma unroll
        for (int q = 0; q < 8; ++q) tile[tr + 32 * pr][tcol + q] = g[pr][q];
      }
    }
    if (m.transposed) {
      __syncthreads();
      // workspace row (c0 + j) holds caller column c0 + j, over caller rows r0..r0+63
#pragma unroll
      for (int pr = 0; pr < 2; ++pr) {
        const int j = tr + 32 * pr;
        const int i0 = tcol;
        const int wr = c0 + j;
        if (wr < m.cols) {
          float v[8];
#pragma unroll
          for (int q = 0; q < 8; ++q) v[q] = tile[i0 + q][j];
          const size_t wb = (size_t)wr * m.ld + r0 + i0;
          if (r0 + i0 + 8 <= m.rows) {
            st8<WT>(work, wb, v);
          } else {
#pragma unroll
            for (int q = 0; q < 8; ++q)
              if (r0 + i0 + q < m.rows) st1<WT>(work, wb + q, v[q]);
          }
        }
      }
    }
    // fixed shuffle tree per warp; one partial per (unit, warp)
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ssq += __shfl_xor_sync(0xffffffffu, ssq, o);
    if (lane == 0) p.partials[(size_t)(m.part_base + u) * kWarpsPerUnit + warp] = ssq;
  }
}

// scale[gid] = 1 / (sqrt(sum of the matrix's partials) + eps): one block per matrix,
// fixed summation order (strided per thread, then a fixed tree), in double.
__global__ void __launch_bounds__(kThreads)
norm_finalize_kernel(const __grid_constant__ EwParams p) {
  __shared__ double red[kThreads / 32];
  const EwMat& m = p.mats[blockIdx.x];
  const size_t b = (size_t)m.part_base * kWarpsPerUnit, n = (size_t)m.n_units * kWarpsPerUnit;
  double acc = 0.0;
  for (size_t k = threadIdx.x; k < n; k += kThreads) acc += (double)p.partials[b + k];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = acc;
  __syncthreads();
  if (threadIdx.x == 0) {
    double t = 0.0;
    for (int w = 0; w < kThreads / 32; ++w) t += red[w];
    p.scale[m.gid] = (float)(1.0 / (sqrt(t) + (double)p.eps));
  }
}

// NorMuon statistics: one warp per row of the wide orientation (s rows of length L):
// q = sum of O^2 / L in a fixed order (lane stride, then a shuffle tree); the caller's
// state v is updated in place; rowsq keeps the sum, rowf the factor 1/(sqrt(v)+eps).
template <typename WT>
__global__ void __launch_bounds__(kThreads)
normuon_rows_kernel(const __grid_constant__ EwParams p, int row_end) {
  const int lane = threadIdx.x & 31;
  const int gw = (blockIdx.x * kThreads + threadIdx.x) >> 5;
  const int nw = (gridDim.x * kThreads) >> 5;
  for (int grow = p.mats[0].row_base + gw; grow < row_end; grow += nw) {
    int lo = 0, hi = p.n_mats - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (p.mats[mid].row_base <= grow) lo = mid; else hi = mid - 1;
    }
    const EwMat& m = p.mats[lo];
    const int i = grow - m.row_base;
    const int L = m.transposed ? m.rows : m.cols;
    const WT* x = reinterpret_cast<const WT*>(m.work) + (size_t)i * m.ld;
    float acc = 0.f;
    for (int l = 8 * lane; l < L; l += 256) {
      float v[8];
      if (l + 8 <= L) {
        ld8(x, l, sizeof(WT) == 2, v);
      } else {
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          float t = 0.f;
          if (l + q < L) {
            if constexpr (sizeof(WT) == 2) t = __bfloat162float(x[l + q]);
            else t = x[l + q];
          }
          v[q] = t;
        }
      }
#pragma unroll
      for (int q = 0; q < 8; ++q) acc = fmaf(v[q], v[q], acc);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if (lane == 0) {
      const float q = __fdiv_rn(acc, (float)L);
      const float vn = __fadd_rn(__fmul_rn(p.nb2, m.nstate[i]), __fmul_rn(__fsub_rn(1.f, p.nb2), q));
      m.nstate[i] = vn;
      p.rowsq[grow] = acc;
      p.rowf[grow] = 1.f / (sqrtf(vn) + p.neps);
    }
  }
}

// Per matrix: r = sqrt(sum q_i / sum q_i f_i^2) in double, fixed order; then
// rowsq[i] <- fl32(f_i * r), the factor the apply pass multiplies O by.
__global__ void __launch_bounds__(kThreads)
normuon_matrix_kernel(const __grid_constant__ EwParams p) {
  __shared__ double red[2][kThreads / 32];
  __shared__ float rr;
  const EwMat& m = p.mats[blockIdx.x];
  const int s = m.transposed ? m.cols : m.rows;
  double a = 0.0, b = 0.0;
  for (int i = threadIdx.x; i < s; i += kThreads) {
    const double q = p.rowsq[m.row_base + i], f = p.rowf[m.row_base + i];
    a += q;
    b += q * f * f;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    a += __shfl_xor_sync(0xffffffffu, a, o);
    b += __shfl_xor_sync(0xffffffffu, b, o);
  }
  if ((threadIdx.x & 31) == 0) {
    red[0][threadIdx.x >> 5] = a;
    red[1][threadIdx.x >> 5] = b;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    double ta = 0.0, tb = 0.0;
    for (int w = 0; w < kThreads / 32; ++w) {
      ta += red[0][w];
      tb += red[1][w];
    }
    rr = (tb > 0.0) ? (float)sqrt(ta / tb) : 1.f;
  }
  __syncthreads();
  for (int i = threadIdx.x; i < s; i += kThreads)
    p.rowsq[m.row_base + i] = __fmul_rn(p.rowf[m.row_base + i], rr);
}

template <typename WT>
__global__ void __launch_bounds__(kThreads)
apply_kernel(const __grid_constant__ EwParams p, int out_kind) {
  __shared__ float tile[kEwTile][kEwTile + 1];
  const int tid = threadIdx.x;
  const int tr = tid >> 3;
  const int tcol = (tid & 7) * 8;

  for (int unit = blockIdx.x; unit < p.total_units; unit += gridDim.x) {
    const int mi = find_mat(p, unit);
    const EwMat& m = p.mats[mi];
    const int u = unit - m.unit_begin;
    const int r0 = (u / m.tiles_c) * kEwTile;
    const int c0 = (u % m.tiles_c) * kEwTile;
    const int c = c0 + tcol;
    const WT* work = reinterpret_cast<const WT*>(m.work);

    float w[2][8], o[2][8];
    if (out_kind == kEwApply) load_tile_rows(m.param, m.param_bf16, m, r0, c, tr, w);
    if (m.transposed) {
      __syncthreads();
      // stage workspace rows c0..c0+63 (caller columns), entries r0..r0+63 (caller rows)
#pragma unroll
      for (int pr = 0; pr < 2; ++pr) {
        const int j = tr + 32 * pr;
        const int wr = c0 + j;
        float v[8];
        const size_t wb = (size_t)wr * m.ld + r0 + tcol;
        if (wr < m.cols && r0 + tcol + 8 <= m.rows) {
          ld8(work, wb, sizeof(WT) == 2, v);
        } else {
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            float x = 0.f;
            if (wr < m.cols && r0 + tcol + q < m.rows) {
              if constexpr (sizeof(WT) == 2) x = __bfloat162float(work[wb + q]);
              else x = work[wb + q];
            }
            v[q] = x;
          }
        }
#pragma unroll
        for (int q = 0; q < 8; ++q) tile[tcol + q][j] = v[q];
      }
      __syncthreads();
#pragma unroll
      for (int pr = 0; pr < 2; ++pr)
#pragma unroll
        for (int q = 0; q < 8; ++q) o[pr][q] = tile[tr + 32 * pr][tcol + q];
    } else {
#pragma unroll
      for (int pr = 0; pr < 2; ++pr) {
        const int r = r0 + tr + 32 * pr;
        if (r < m.rows && c + 8 <= m.cols) {
          ld8(work, (size_t)r * m.ld + c, sizeof(WT) == 2, o[pr]);
        } else {
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            float x = 0.f;
            if (r < m.rows && c + q < m.cols) {
              if constexpr (sizeof(WT) == 2) x = __bfloat162float(work[(size_t)r * m.ld + c + q]);
              else x = work[(size_t)r * m.ld + c + q];
            }
            o[pr][q] = x;
          }
        }
      }
    }
#pragma unroll
    for (int pr = 0; pr < 2; ++pr) {
      const int r = r0 + tr + 32 * pr;
      if (r >= m.rows) continue;
      const bool full = c + 8 <= m.cols;
      const size_t base = (size_t)r * m.cols + c;
      if (p.normuon) {
        // per-row factor of the wide orientation: caller row (wide) or column (tall)
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          const int wi = m.transposed ? (c + q < m.cols ? c + q : 0) : r;
          o[pr][q] = __fmul_rn(p.rowsq[m.row_base + wi], o[pr][q]);
        }
      }
      if (out_kind == kEwApply) {
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          const float w0 = w[pr][q], oq = o[pr][q];
          float wn = __fsub_rn(w0, __fmul_rn(m.lrs, oq));
          const bool agree = (oq >= 0.f && w0 >= 0.f) || (oq <= 0.f && w0 <= 0.f);
          if (m.lrwd != 0.f && (!p.cautious || agree)) wn = __fsub_rn(wn, __fmul_rn(m.lrwd, w0));
          w[pr][q] = wn;
        }
      } else {
#pragma unroll
        for (int q = 0; q < 8; ++q) w[pr][q] = o[pr][q];
      }
      if (full && m.vec_ok) {
        st8_dyn(m.param, base, w[pr], m.param_bf16);
      } else {
#pragma unroll
        for (int q = 0; q < 8; ++q)
          if (c + q < m.cols) st1_dyn(m.param, base + q, w[pr][q], m.param_bf16);
      }
    }
  }
}

}  // namespace

cudaError_t launch_momentum_norm(const EwParams& p, bool work_f32, int grid, cudaStream_t st) {
  if (p.total_units == 0) return cudaSuccess;
  if (work_f32) momentum_norm_kernel<float><<<grid, kThreads, 0, st>>>(p);
  else momentum_norm_kernel<__nv_bfloat16><<<grid, kThreads, 0, st>>>(p);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  norm_finalize_kernel<<<p.n_mats, kThreads, 0, st>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_normuon(const EwParams& p, bool work_f32, int grid, cudaStream_t st) {
  if (p.n_mats == 0) return cudaSuccess;
  const EwMat& last = p.mats[p.n_mats - 1];
  const int row_end = last.row_base + (last.transposed ? last.cols : last.rows);
  if (work_f32) normuon_rows_kernel<float><<<grid, kThreads, 0, st>>>(p, row_end);
  else normuon_rows_kernel<__nv_bfloat16><<<grid, kThreads, 0, st>>>(p, row_end);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  normuon_matrix_kernel<<<p.n_mats, kThreads, 0, st>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_apply(const EwParams& p, bool work_f32, int out_kind, int grid, cudaStream_t st) {
  if (p.total_units == 0) return cudaSuccess;
  if (work_f32) apply_kernel<float><<<grid, kThreads, 0, st>>>(p, out_kind);
  else apply_kernel<__nv_bfloat16><<<grid, kThreads, 0, st>>>(p, out_kind);
  return cudaGetLastError();
}

}  // namespace muon
