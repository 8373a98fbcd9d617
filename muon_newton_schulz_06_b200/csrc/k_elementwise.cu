// Elementwise passes of the Muon step (HBM-bound):
//
//  * momentum_norm: M <- fl32(fl32(mu*M) + G), U <- fl32(G + fl32(mu*M)) (Nesterov) or
//    M, written to the workspace in wide orientation (transposed for tall matrices),
//    with a deterministic per-matrix sum of U^2 that ends in the scale
//    1/(||U||_F + eps).  Autoresearch train.py review, MuonAdamW paragraph: Muon
//    applies Nesterov momentum to the gradient with a buffer of the parameter's shape;
//    the Frobenius normalisation is the benchmark spec's.
//  * apply: W <- fl32(W - lrs*O) rounded to the parameter dtype, O read back from the
//    workspace (transposed for tall matrices); or export O into a caller buffer.
//
// One work unit is a 64 x 64 tile of the caller matrix; 256 threads each own 2 rows x 8
// consecutive columns, so rows move as 16-byte vectors.  Tall matrices go through a
// shared-memory tile to write / read the transposed workspace coalesced.
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
    uint4 raw = *reinterpret_cast<const uint4*>(reinterpret_cast<const __nv_bfloat16*>(p) + i);
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&raw);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      float2 f = __bfloat1622float2(h[q]);
      v[2 * q] = f.x;
      v[2 * q + 1] = f.y;
    }
  } else {
    const float4* f = reinterpret_cast<const float4*>(reinterpret_cast<const float*>(p) + i);
    float4 a = f[0], b = f[1];
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
    v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
  }
}

template <typename T>
__device__ __forceinline__ void st8(T* p, size_t i, const float* v);

template <>
__device__ __forceinline__ void st8<float>(float* p, size_t i, const float* v) {
  float4* f = reinterpret_cast<float4*>(p + i);
  f[0] = make_float4(v[0], v[1], v[2], v[3]);
  f[1] = make_float4(v[4], v[5], v[6], v[7]);
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

// Fixed-order block sum (deterministic for a fixed thread -> value mapping).
__device__ __forceinline__ double block_sum(double v, double* red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  __syncthreads();
  if (lane == 0) red[warp] = v;
  __syncthreads();
  double t = 0.0;
  if (threadIdx.x == 0) {
    for (int w = 0; w < kThreads / 32; ++w) t += red[w];
  }
  return t;  // valid in thread 0
}

template <typename WT>
__global__ void __launch_bounds__(kThreads)
momentum_norm_kernel(const __grid_constant__ EwParams p) {
  __shared__ float tile[kEwTile][kEwTile + 1];
  __shared__ double red[kThreads / 32];
  __shared__ int is_last;
  const int tid = threadIdx.x;
  const int tr = tid >> 3;        // 0..31
  const int tcol = (tid & 7) * 8; // 0..56

  for (int unit = blockIdx.x; unit < p.total_units; unit += gridDim.x) {
    const int mi = find_mat(p, unit);
    const EwMat& m = p.mats[mi];
    const int u = unit - m.unit_begin;
    const int r0 = (u / m.tiles_c) * kEwTile;
    const int c0 = (u % m.tiles_c) * kEwTile;
    WT* work = reinterpret_cast<WT*>(m.work);
    float ssq = 0.f;

#pragma unroll
    for (int pr = 0; pr < 2; ++pr) {
      const int r = r0 + tr + 32 * pr;
      const int c = c0 + tcol;
      float g[8], mo[8], uu[8];
      const bool in_row = r < m.rows;
      const bool full = in_row && (c + 8 <= m.cols);
      const size_t base = (size_t)r * m.cols + c;
      if (full && m.vec_ok) {
        if (p.use_momentum) {
          ld8(m.grad, base, m.grad_bf16, g);
          ld8(m.mom, base, false, mo);
        } else {
          ld8(m.param, base, m.param_bf16, g);
        }
      } else {
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          const bool ok = in_row && (c + q < m.cols);
          if (p.use_momentum) {
            g[q] = ok ? ld_elem(m.grad, base + q, m.grad_bf16) : 0.f;
            mo[q] = ok ? m.mom[base + q] : 0.f;
          } else {
            g[q] = ok ? ld_elem(m.param, base + q, m.param_bf16) : 0.f;
          }
        }
      }
      if (p.use_momentum) {
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          const float mn = __fadd_rn(__fmul_rn(p.mu, mo[q]), g[q]);
          mo[q] = mn;
          uu[q] = p.nesterov ? __fadd_rn(g[q], __fmul_rn(p.mu, mn)) : mn;
        }
        if (full && m.vec_ok) {
          st8<float>(m.mom, base, mo);
        } else {
#pragma unroll
          for (int q = 0; q < 8; ++q)
            if (in_row && c + q < m.cols) m.mom[base + q] = mo[q];
        }
      } else {
#pragma unroll
        for (int q = 0; q < 8; ++q) uu[q] = g[q];
      }
#pragma unroll
      for (int q = 0; q < 8; ++q) ssq = fmaf(uu[q], uu[q], ssq);  // zero outside the matrix

      if (!m.transposed) {
        // workspace row r holds caller row r
        if (full) {
          st8<WT>(work, (size_t)r * m.ld + c, uu);
        } else {
#pragma unroll
          for (int q = 0; q < 8; ++q)
            if (in_row && c + q < m.cols) st1<WT>(work, (size_t)r * m.ld + c + q, uu[q]);
        }
      } else {
#pragma unroll
        for (int q = 0; q < 8; ++q) tile[tr + 32 * pr][tcol + q] = uu[q];
      }
    }

    if (m.transposed) {
      __syncthreads();
      // workspace row (c0 + j) holds caller column c0 + j, over caller rows r0..r0+63
#pragma unroll
      for (int pr = 0; pr < 2; ++pr) {
        const int j = tr + 32 * pr;          // caller column offset
        const int i0 = tcol;                 // caller row offset
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

    const double tot = block_sum((double)ssq, red);
    if (tid == 0) {
      p.partials[m.part_base + u] = (float)tot;
      __threadfence();
      const unsigned prev = atomicAdd(&p.counters[m.gid], 1u);
      is_last = (prev == (unsigned)(m.n_units - 1));
    }
    __syncthreads();
    if (is_last) {
      __threadfence();
      double acc = 0.0;
      for (int k = tid; k < m.n_units; k += kThreads) acc += (double)__ldcg(p.partials + m.part_base + k);
      const double all = block_sum(acc, red);
      if (tid == 0) {
        p.scale[m.gid] = (float)(1.0 / (sqrt(all) + (double)p.eps));
        p.counters[m.gid] = 0u;
      }
    }
    __syncthreads();
  }
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
    const WT* work = reinterpret_cast<const WT*>(m.work);

    if (m.transposed) {
      __syncthreads();
      // stage workspace rows c0..c0+63 (caller columns), entries r0..r0+63 (caller rows)
#pragma unroll
      for (int pr = 0; pr < 2; ++pr) {
        const int j = tr + 32 * pr;
        const int wr = c0 + j;
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          const int i = r0 + tcol + q;
          float v = 0.f;
          if (wr < m.cols && i < m.rows) {
            if constexpr (sizeof(WT) == 2) v = __bfloat162float(work[(size_t)wr * m.ld + i]);
            else v = work[(size_t)wr * m.ld + i];
          }
          tile[tcol + q][j] = v;
        }
      }
      __syncthreads();
    }

#pragma unroll
    for (int pr = 0; pr < 2; ++pr) {
      const int r = r0 + tr + 32 * pr;
      const int c = c0 + tcol;
      const bool in_row = r < m.rows;
      if (!in_row) continue;
      const bool full = c + 8 <= m.cols;
      float o[8];
      if (m.transposed) {
#pragma unroll
        for (int q = 0; q < 8; ++q) o[q] = tile[tr + 32 * pr][tcol + q];
      } else if (full) {
        ld8(work, (size_t)r * m.ld + c, sizeof(WT) == 2, o);
      } else {
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          float v = 0.f;
          if (c + q < m.cols) {
            if constexpr (sizeof(WT) == 2) v = __bfloat162float(work[(size_t)r * m.ld + c + q]);
            else v = work[(size_t)r * m.ld + c + q];
          }
          o[q] = v;
        }
      }
      const size_t base = (size_t)r * m.cols + c;
      float w[8];
      if (out_kind == kEwApply) {
        if (full && m.vec_ok) {
          ld8(m.param, base, m.param_bf16, w);
        } else {
#pragma unroll
          for (int q = 0; q < 8; ++q) w[q] = (c + q < m.cols) ? ld_elem(m.param, base + q, m.param_bf16) : 0.f;
        }
#pragma unroll
        for (int q = 0; q < 8; ++q) w[q] = __fsub_rn(w[q], __fmul_rn(m.lrs, o[q]));
      } else {
#pragma unroll
        for (int q = 0; q < 8; ++q) w[q] = o[q];
      }
      if (full && m.vec_ok) {
        st8_dyn(m.param, base, w, m.param_bf16);
      } else {
#pragma unroll
        for (int q = 0; q < 8; ++q)
          if (c + q < m.cols) st1_dyn(m.param, base + q, w[q], m.param_bf16);
      }
    }
  }
}

}  // namespace

cudaError_t launch_momentum_norm(const EwParams& p, bool work_f32, int grid, cudaStream_t st) {
  if (p.total_units == 0) return cudaSuccess;
  if (work_f32) momentum_norm_kernel<float><<<grid, kThreads, 0, st>>>(p);
  else momentum_norm_kernel<__nv_bfloat16><<<grid, kThreads, 0, st>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_apply(const EwParams& p, bool work_f32, int out_kind, int grid, cudaStream_t st) {
  if (p.total_units == 0) return cudaSuccess;
  if (work_f32) apply_kernel<float><<<grid, kThreads, 0, st>>>(p, out_kind);
  else apply_kernel<__nv_bfloat16><<<grid, kThreads, 0, st>>>(p, out_kind);
  return cudaGetLastError();
}

}  // namespace muon
