// fp32 validation path of the Newton-Schulz steps: the same three products as the
// tensor-core engine (Gram, polynomial, update on the wide-orientation X), in fp32
// storage with fp32 fused multiply-adds on CUDA cores.  No TF32: its 10-bit mantissa
// would not resolve the 1e-4 comparison this mode exists for.
//
// One kernel computes out[i][j] = alpha_add*addend[i][j] + beta*sum_k P[i][k] Q(k, j),
// with Q(k, j) = Q[j][k] (both operands row blocks, Gram / polynomial) or Q[k][j]
// (update).  64 x 64 output tile per 256-thread block, 4 x 4 outputs per thread, k-slabs
// of 16 staged in shared memory.  Every output is a plain k-ordered FMA chain, so
// Gram / polynomial results are symmetric bit for bit.
#include "muon_internal.h"

namespace muon {
namespace {

constexpr int kT = 64;
constexpr int kKs = 16;

template <bool kQRows>
__global__ void __launch_bounds__(256)
sgemm_kernel(const float* __restrict__ P, int ldp, const float* __restrict__ Q, int ldq, int M, int N, int K,
             float* __restrict__ out, int ldo, const float* __restrict__ addend, int lda, float alpha_add,
             float beta, const float* __restrict__ scale, int gid, int scale_mode) {
  __shared__ float sp[kKs][kT + 1];
  __shared__ float sq[kKs][kT + 1];
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  const int i0 = blockIdx.y * kT, j0 = blockIdx.x * kT;
  float acc[4][4] = {};
  for (int k0 = 0; k0 < K; k0 += kKs) {
    for (int e = threadIdx.x; e < kT * kKs; e += 256) {
      const int r = e / kKs, k = e % kKs;
      const int gi = i0 + r, gk = k0 + k;
      sp[k][r] = (gi < M && gk < K) ? P[(size_t)gi * ldp + gk] : 0.f;
      if (kQRows) {
        const int gj = j0 + r;
        sq[k][r] = (gj < N && gk < K) ? Q[(size_t)gj * ldq + gk] : 0.f;
      }
    }
    if (!kQRows) {
      for (int e = threadIdx.x; e < kT * kKs; e += 256) {
        const int k = e / kT, c = e % kT;
        const int gk = k0 + k, gj = j0 + c;
        sq[k][c] = (gk < K && gj < N) ? Q[(size_t)gk * ldq + gj] : 0.f;
      }
    }
    __syncthreads();
#pragma unroll
    for (int k = 0; k < kKs; ++k) {
      float a[4], b[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        a[q] = sp[k][ty + 16 * q];
        b[q] = sq[k][tx + 16 * q];
      }
#pragma unroll
      for (int x = 0; x < 4; ++x)
#pragma unroll
        for (int y = 0; y < 4; ++y) acc[x][y] = fmaf(a[x], b[y], acc[x][y]);
    }
    __syncthreads();
  }
  // scale_mode 0: as given; 1: beta *= s^2 (Gram); 2: alpha_add *= s, beta *= s (update)
  float sc = 1.f;
  if (scale_mode != 0) sc = scale[gid];
  if (scale_mode == 1) beta *= sc * sc;
  if (scale_mode == 2) { alpha_add *= sc; beta *= sc; }
#pragma unroll
  for (int x = 0; x < 4; ++x) {
    const int i = i0 + ty + 16 * x;
    if (i >= M) continue;
#pragma unroll
    for (int y = 0; y < 4; ++y) {
      const int j = j0 + tx + 16 * y;
      if (j >= N) continue;
      float v = beta * acc[x][y];
      if (addend) v = fmaf(alpha_add, addend[(size_t)i * lda + j], v);
      out[(size_t)i * ldo + j] = v;
    }
  }
}

dim3 grid_for(int M, int N) { return dim3((N + kT - 1) / kT, (M + kT - 1) / kT, 1); }

}  // namespace

cudaError_t launch_f32_gram(const F32Mat& m, int first_iter, const float* scale, cudaStream_t st) {
  sgemm_kernel<true><<<grid_for(m.s, m.s), 256, 0, st>>>(m.x_cur, m.ld_x, m.x_cur, m.ld_x, m.s, m.s, m.L,
                                                         m.gram, m.ld_s, nullptr, 0, 0.f, 1.f, scale, m.gid,
                                                         first_iter ? 1 : 0);
  return cudaGetLastError();
}

cudaError_t launch_f32_poly(const F32Mat& m, float cb, float cc, cudaStream_t st) {
  sgemm_kernel<true><<<grid_for(m.s, m.s), 256, 0, st>>>(m.gram, m.ld_s, m.gram, m.ld_s, m.s, m.s, m.s,
                                                         m.poly, m.ld_s, m.gram, m.ld_s, cb, cc, nullptr, 0,
                                                         0);
  return cudaGetLastError();
}

cudaError_t launch_f32_update(const F32Mat& m, int first_iter, const float* scale, float ca, cudaStream_t st) {
  sgemm_kernel<false><<<grid_for(m.s, m.L), 256, 0, st>>>(m.poly, m.ld_s, m.x_cur, m.ld_x, m.s, m.L, m.s,
                                                          m.x_next, m.ld_x, m.x_cur, m.ld_x, ca, 1.f, scale,
                                                          m.gid, first_iter ? 2 : 0);
  return cudaGetLastError();
}

}  // namespace muon
