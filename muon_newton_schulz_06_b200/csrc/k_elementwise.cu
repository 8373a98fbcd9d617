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
// byte is touched once per pass), and every load of a unit is issued before its stores.
// Tall matrices go through a shared-memory tile to write / read the transposed
// workspace coalesced.  The norm is deterministic: each warp of a unit writes one
// partial sum (fixed shuffle tree), and a second small kernel adds a matrix's partials
// in a fixed order.
//
// In bf16 mode the momentum pass and the weight update move data with the copy engine
// instead: wide matrices (workspace copy in the caller's layout) in contiguous units
// through cp.async.bulk (4096 elements for the momentum pass, 8192 for the update), tall
// ones in 64 x 64 tiles through tensor maps (cp.async.bulk.tensor, 128-byte swizzle,
// transposed in shared memory), each through a 3-stage ring per CTA.  The bytes in
// flight are then bounded by shared memory rather than by registers, and the passes
// keep HBM busy at the reduced SM clock of a power-capped step (the register tile
// kernels are bound by load latency there).  Matrices that fit neither (fp32 gradients
// or weights, unaligned rows) keep the register tile kernels.
#include <algorithm>

#include "muon_internal.h"

namespace muon {
namespace {

constexpr int kThreads = 256;

// ---- copy-engine helpers (bulk-copy and tensor-map kernels)
__device__ __forceinline__ uint32_t su32(const void* p) { return (uint32_t)__cvta_generic_to_shared(p); }
__device__ __forceinline__ uint64_t gtimer() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
__device__ __forceinline__ void bar_init(uint64_t* b, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(su32(b)), "r"(count) : "memory");
}
__device__ __forceinline__ void bar_arrive_tx(uint64_t* b, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(su32(b)), "r"(bytes) : "memory");
}
__device__ __forceinline__ void bar_arrive(uint64_t* b) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(su32(b)) : "memory");
}
__device__ __forceinline__ bool bar_try_wait(uint64_t* b, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}\n"
      : "=r"(ok)
      : "r"(su32(b)), "r"(parity)
      : "memory");
  return ok != 0;
}
constexpr unsigned long long kFlatWaitNs = 2000000000ull;  // 2 s per wait
// Bounded wait: false after kFlatWaitNs (the caller records a time-out and stops).
__device__ __noinline__ bool bar_wait(uint64_t* b, uint32_t parity) {
  if (bar_try_wait(b, parity)) return true;
  const uint64_t t0 = gtimer();
  while (!bar_try_wait(b, parity))
    if (gtimer() - t0 > kFlatWaitNs) return false;
  return true;
}
__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                   su32(dst)),
               "l"(src), "r"(bytes), "r"(su32(bar))
               : "memory");
}
__device__ __forceinline__ void bulk_store(void* dst, const void* src, uint32_t bytes) {
  asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(dst), "r"(su32(src)), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, int x, int y, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::
          "r"(su32(dst)),
      "l"(map), "r"(x), "r"(y), "r"(su32(bar))
      : "memory");
}
__device__ __forceinline__ void tma_store_2d(const CUtensorMap* map, const void* src, int x, int y) {
  asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%1, %2}], [%3];" ::"l"(map), "r"(x),
               "r"(y), "r"(su32(src))
               : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_read1() { asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

constexpr int kFlatStages = 3;
constexpr int kFlatCompute = 128;                 // compute threads (warps 1..4)
constexpr int kFlatThreads = 32 + kFlatCompute;   // warp 0: copy producer
constexpr uint32_t kFlatGBytes = kFlatUnit * 2;   // bf16 gradients, then U, per stage
constexpr uint32_t kFlatMBytes = kFlatUnit * 4;   // fp32 momentum per stage
constexpr size_t kFlatSmem = kFlatStages * (kFlatGBytes + kFlatMBytes) + 2 * kFlatStages * sizeof(uint64_t);
// TMA tile pass: per stage a gradient tile (8 KB), a momentum tile (two 32-column halves,
// 16 KB) and the transposed U tile (8 KB), each 1024-byte aligned for the swizzle.
constexpr uint32_t kTileStageBytes = kFlatGBytes + kFlatMBytes + kFlatGBytes;
constexpr size_t kTileSmem = 1024 + kFlatStages * kTileStageBytes + 2 * kFlatStages * sizeof(uint64_t);

// Byte offset of the 16-byte chunk q of row r in a tile with 128-byte rows and the
// 128-byte swizzle (chunk index XOR row mod 8), as the tensor maps lay it out.
__device__ __forceinline__ uint32_t swz128(int r, int q) { return (uint32_t)(r * 128 + ((q ^ (r & 7)) << 4)); }

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
template <typename P>
__device__ __forceinline__ int find_mat(const P& p, int unit) {
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

// Bulk-copy momentum pass (matrices listed in p, all with the caller's layout in the
// workspace).  Unit u of matrix m covers elements [u*4096, min((u+1)*4096, rows*cols)).
// Warp 0, lane 0 copies a unit's gradients and momentum into a ring stage; the 128
// compute threads each take 8-element chunks ct, ct+128, ... of it, update M and write
// U in place (U over the gradients), then one thread stores both back with bulk copies
// and frees the stage once the copy engine has read it.  Each compute warp writes one
// norm partial per unit (slots 0..3; slots 4..7 are written as zero).
__global__ void __launch_bounds__(kFlatThreads)
momentum_flat_kernel(const __grid_constant__ EwParams p) {
  extern __shared__ __align__(128) uint8_t fsm[];
  uint8_t* sg = fsm;                                 // [kFlatStages][kFlatGBytes]
  uint8_t* smo = fsm + kFlatStages * kFlatGBytes;     // [kFlatStages][kFlatMBytes]
  uint64_t* full = reinterpret_cast<uint64_t*>(smo + kFlatStages * kFlatMBytes);
  uint64_t* empty = full + kFlatStages;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (tid == 0) {
    for (int s = 0; s < kFlatStages; ++s) {
      bar_init(&full[s], 1);
      bar_init(&empty[s], 1);
    }
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();

  if (warp == 0) {
    if (lane == 0) {
      int s = 0;
      uint32_t ph = 0;
      bool ok = true;
      for (int unit = blockIdx.x; unit < p.total_units; unit += gridDim.x) {
        const EwMat& m = p.mats[find_mat(p, unit)];
        const size_t off = (size_t)(unit - m.unit_begin) * kFlatUnit;
        const size_t numel = (size_t)m.rows * m.cols;
        const uint32_t cnt = (uint32_t)(numel - off < (size_t)kFlatUnit ? numel - off : (size_t)kFlatUnit);
        if (!bar_wait(&empty[s], ph ^ 1u)) { ok = false; break; }
        bar_arrive_tx(&full[s], cnt * 6u);
        bulk_load(sg + s * kFlatGBytes, reinterpret_cast<const __nv_bfloat16*>(m.grad) + off, cnt * 2u, &full[s]);
        bulk_load(smo + s * kFlatMBytes, m.mom + off, cnt * 4u, &full[s]);
        if (++s == kFlatStages) { s = 0; ph ^= 1u; }
      }
      if (!ok) {
        atomicExch(p.status, kDevTimeout);
        const uint64_t t0 = gtimer();  // copies already issued land within microseconds
        while (gtimer() - t0 < 1000000ull) {
        }
      }
    }
    return;
  }

  const int ct = tid - 32;  // 0..127
  int s = 0, prev = -1;
  uint32_t ph = 0;
  bool ok = true;
  for (int unit = blockIdx.x; unit < p.total_units; unit += gridDim.x) {
    const EwMat& m = p.mats[find_mat(p, unit)];
    const int u = unit - m.unit_begin;
    const size_t off = (size_t)u * kFlatUnit;
    const size_t numel = (size_t)m.rows * m.cols;
    const uint32_t cnt = (uint32_t)(numel - off < (size_t)kFlatUnit ? numel - off : (size_t)kFlatUnit);
    if (!bar_wait(&full[s], ph)) { ok = false; break; }
    uint4* gs = reinterpret_cast<uint4*>(sg + s * kFlatGBytes);
    float4* ms = reinterpret_cast<float4*>(smo + s * kFlatMBytes);
    float ssq = 0.f;
#pragma unroll
    for (int j = 0; j < kFlatUnit / 8 / kFlatCompute; ++j) {
      const int k = ct + j * kFlatCompute;  // chunk of 8 elements
      if ((uint32_t)k * 8u >= cnt) break;
      const uint4 graw = gs[k];
      const float4 m0 = ms[2 * k], m1 = ms[2 * k + 1];
      const __nv_bfloat162* gh = reinterpret_cast<const __nv_bfloat162*>(&graw);
      float g[8], mo[8] = {m0.x, m0.y, m0.z, m0.w, m1.x, m1.y, m1.z, m1.w};
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const float2 f = __bfloat1622float2(gh[q]);
        g[2 * q] = f.x;
        g[2 * q + 1] = f.y;
      }
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        const float gq = p.lerp ? __fmul_rn(p.omu, g[q]) : g[q];
        const float mn = __fadd_rn(__fmul_rn(p.mu, mo[q]), gq);
        mo[q] = mn;
        g[q] = p.nesterov ? __fadd_rn(gq, __fmul_rn(p.mu, mn)) : mn;  // g now holds U
        ssq = fmaf(g[q], g[q], ssq);
      }
      ms[2 * k] = make_float4(mo[0], mo[1], mo[2], mo[3]);
      ms[2 * k + 1] = make_float4(mo[4], mo[5], mo[6], mo[7]);
      uint4 ur;
      __nv_bfloat162* uh = reinterpret_cast<__nv_bfloat162*>(&ur);
#pragma unroll
      for (int q = 0; q < 4; ++q) uh[q] = __floats2bfloat162_rn(g[2 * q], g[2 * q + 1]);
      gs[k] = ur;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ssq += __shfl_xor_sync(0xffffffffu, ssq, o);
    if (lane == 0) {
      float* part = p.partials + (size_t)(m.part_base + u) * kWarpsPerUnit;
      part[warp - 1] = ssq;
      part[warp - 1 + 4] = 0.f;
    }
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");  // smem writes -> bulk store
    asm volatile("bar.sync 1, %0;" ::"n"(kFlatCompute) : "memory");
    if (ct == 0) {
      bulk_store(m.mom + off, smo + s * kFlatMBytes, cnt * 4u);
      bulk_store(reinterpret_cast<__nv_bfloat16*>(m.work) + off, sg + s * kFlatGBytes, cnt * 2u);
      bulk_commit();
      bulk_wait_read1();  // the previous unit's stores have read their stage
      if (prev >= 0) bar_arrive(&empty[prev]);
    }
    prev = s;
    if (++s == kFlatStages) { s = 0; ph ^= 1u; }
  }
  if (ct == 0) bulk_wait_all();
  if (!ok && ct == 0) atomicExch(p.status, kDevTimeout);
}

// TMA momentum pass of tall matrices (p lists them; unit u of matrix m is the 64 x 64 tile
// (u / tiles_c, u % tiles_c) of the caller matrix).  Warp 0, lane 0 loads the gradient
// and momentum tiles through the matrix's tensor maps (out-of-range parts read as
// zero); compute thread ct owns row ct mod 64 of the tile, columns 32*(ct/64) ..+31:
// it updates M in place and writes U transposed into the U tile (U^T row c, column r),
// then one thread stores M and U^T through the maps (clipped at the matrix edge).
// 128-byte swizzled tiles keep both the row reads and the transposed writes free of
// bank conflicts.  Norm partials as in momentum_flat_kernel.
__global__ void __launch_bounds__(kFlatThreads)
momentum_tile_tma_kernel(const __grid_constant__ EwTiledParams p) {
  extern __shared__ uint8_t tsm_raw[];
  uint8_t* tsm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(tsm_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(tsm + kFlatStages * kTileStageBytes);
  uint64_t* empty = full + kFlatStages;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (tid == 0) {
    for (int s = 0; s < kFlatStages; ++s) {
      bar_init(&full[s], 1);
      bar_init(&empty[s], 1);
    }
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();
  auto g_tile = [&](int s) { return tsm + s * kTileStageBytes; };
  auto m_tile = [&](int s) { return tsm + s * kTileStageBytes + kFlatGBytes; };  // [2][64 rows][128 B]
  auto u_tile = [&](int s) { return tsm + s * kTileStageBytes + kFlatGBytes + kFlatMBytes; };

  if (warp == 0) {
    if (lane == 0) {
      int s = 0;
      uint32_t ph = 0;
      bool ok = true;
      for (int unit = blockIdx.x; unit < p.total_units; unit += gridDim.x) {
        const EwMat& m = p.mats[find_mat(p, unit)];
        const int u = unit - m.unit_begin;
        const int r0 = (u / m.tiles_c) * kEwTile, c0 = (u % m.tiles_c) * kEwTile;
        const CUtensorMap* maps = &p.maps[kEwMapsPerMat * find_mat(p, unit)];
        if (!bar_wait(&empty[s], ph ^ 1u)) { ok = false; break; }
        bar_arrive_tx(&full[s], kFlatGBytes + kFlatMBytes);
        tma_load_2d(g_tile(s), &maps[0], c0, r0, &full[s]);
        tma_load_2d(m_tile(s), &maps[1], c0, r0, &full[s]);
        tma_load_2d(m_tile(s) + kFlatMBytes / 2, &maps[1], c0 + 32, r0, &full[s]);
        if (++s == kFlatStages) { s = 0; ph ^= 1u; }
      }
      if (!ok) {
        atomicExch(p.status, kDevTimeout);
        const uint64_t t0 = gtimer();  // copies already issued land within microseconds
        while (gtimer() - t0 < 1000000ull) {
        }
      }
    }
    return;
  }

  const int ct = tid - 32;   // 0..127
  const int r = ct & 63;     // tile row of this thread
  const int h = ct >> 6;     // column half: columns 32h .. 32h+31
  int s = 0, prev = -1;
  uint32_t ph = 0;
  bool ok = true;
  for (int unit = blockIdx.x; unit < p.total_units; unit += gridDim.x) {
    const EwMat& m = p.mats[find_mat(p, unit)];
    const int u = unit - m.unit_begin;
    const int r0 = (u / m.tiles_c) * kEwTile, c0 = (u % m.tiles_c) * kEwTile;
    if (!bar_wait(&full[s], ph)) { ok = false; break; }
    uint8_t* gt = g_tile(s);
    uint8_t* mt = m_tile(s) + h * (kFlatMBytes / 2);
    uint8_t* ut = u_tile(s);
    float ssq = 0.f;
#pragma unroll
    for (int i = 0; i < 4; ++i) {  // 8 columns 32h + 8i .. +7
      const uint4 graw = *reinterpret_cast<const uint4*>(gt + swz128(r, 4 * h + i));
      float4* mp0 = reinterpret_cast<float4*>(mt + swz128(r, 2 * i));
      float4* mp1 = reinterpret_cast<float4*>(mt + swz128(r, 2 * i + 1));
      const float4 m0 = *mp0, m1 = *mp1;
      const __nv_bfloat162* gh = reinterpret_cast<const __nv_bfloat162*>(&graw);
      float g[8], mo[8] = {m0.x, m0.y, m0.z, m0.w, m1.x, m1.y, m1.z, m1.w};
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const float2 f = __bfloat1622float2(gh[q]);
        g[2 * q] = f.x;
        g[2 * q + 1] = f.y;
      }
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        const float gq = p.lerp ? __fmul_rn(p.omu, g[q]) : g[q];
        const float mn = __fadd_rn(__fmul_rn(p.mu, mo[q]), gq);
        mo[q] = mn;
        g[q] = p.nesterov ? __fadd_rn(gq, __fmul_rn(p.mu, mn)) : mn;  // g now holds U
        ssq = fmaf(g[q], g[q], ssq);
      }
      *mp0 = make_float4(mo[0], mo[1], mo[2], mo[3]);
      *mp1 = make_float4(mo[4], mo[5], mo[6], mo[7]);
#pragma unroll
      for (int q = 0; q < 8; ++q) {  // U^T row c = 32h + 8i + q, column r
        const int c = 32 * h + 8 * i + q;
        *reinterpret_cast<__nv_bfloat16*>(ut + swz128(c, r >> 3) + ((r & 7) << 1)) = __float2bfloat16_rn(g[q]);
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ssq += __shfl_xor_sync(0xffffffffu, ssq, o);
    if (lane == 0) {
      float* part = p.partials + (size_t)(m.part_base + u) * kWarpsPerUnit;
      part[warp - 1] = ssq;
      part[warp - 1 + 4] = 0.f;
    }
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");  // smem writes -> tensor store
    asm volatile("bar.sync 1, %0;" ::"n"(kFlatCompute) : "memory");
    if (ct == 0) {
      const CUtensorMap* maps = &p.maps[kEwMapsPerMat * find_mat(p, unit)];
      tma_store_2d(&maps[1], m_tile(s), c0, r0);
      tma_store_2d(&maps[1], m_tile(s) + kFlatMBytes / 2, c0 + 32, r0);
      tma_store_2d(&maps[2], ut, r0, c0);
      bulk_commit();
      bulk_wait_read1();  // the previous unit's stores have read their stage
      if (prev >= 0) bar_arrive(&empty[prev]);
    }
    prev = s;
    if (++s == kFlatStages) { s = 0; ph ^= 1u; }
  }
  if (ct == 0) bulk_wait_all();
  if (!ok && ct == 0) atomicExch(p.status, kDevTimeout);
}

// One weight of the update pass: W - fl32(lrs*O), then the decoupled decay where it
// applies (every entry, or only where O and the old weight agree in sign).
__device__ __forceinline__ float apply_elem(float w0, float o, float lrs, float lrwd, int cautious) {
  float wn = __fsub_rn(w0, __fmul_rn(lrs, o));
  const bool agree = (o >= 0.f && w0 >= 0.f) || (o <= 0.f && w0 <= 0.f);
  if (lrwd != 0.f && (!cautious || agree)) wn = __fsub_rn(wn, __fmul_rn(lrwd, w0));
  return wn;
}

__device__ __forceinline__ void bf16x8_to_f32(const uint4& raw, float* v) {
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&raw);
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const float2 f = __bfloat1622float2(h[q]);
    v[2 * q] = f.x;
    v[2 * q + 1] = f.y;
  }
}

__device__ __forceinline__ uint4 f32x8_to_bf16(const float* v) {
  uint4 raw;
  __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&raw);
#pragma unroll
  for (int q = 0; q < 4; ++q) h[q] = __floats2bfloat162_rn(v[2 * q], v[2 * q + 1]);
  return raw;
}

// The weight update moves half the bytes per element of the momentum pass, so its bulk
// units are twice as long (8192 elements, 16 KB of O and 16 KB of W per stage).
constexpr uint32_t kApplyStageBytes = kApplyUnit * 2;  // one bf16 operand of a unit
constexpr size_t kApplyFlatSmem = kFlatStages * 2 * kApplyStageBytes + 2 * kFlatStages * sizeof(uint64_t);
constexpr size_t kApplyTileSmem = 1024 + kFlatStages * 2 * kFlatGBytes + 2 * kFlatStages * sizeof(uint64_t);

// Bulk-copy weight update of wide matrices (bf16 weights, workspace in the caller's
// layout): unit u covers elements [u*8192, ...) of W and of O; the structure follows
// momentum_flat_kernel.  With NorMuon, O is first scaled by its row's factor
// (rowsq[row_base + row], one load per 8-element chunk).
__global__ void __launch_bounds__(kFlatThreads)
apply_flat_kernel(const __grid_constant__ EwParams p) {
  extern __shared__ __align__(128) uint8_t asm_[];
  uint8_t* so = asm_;                                       // [kFlatStages][16 KB] O
  uint8_t* sw = asm_ + kFlatStages * kApplyStageBytes;      // [kFlatStages][16 KB] W, then W'
  uint64_t* full = reinterpret_cast<uint64_t*>(asm_ + 2 * kFlatStages * kApplyStageBytes);
  uint64_t* empty = full + kFlatStages;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (tid == 0) {
    for (int s = 0; s < kFlatStages; ++s) {
      bar_init(&full[s], 1);
      bar_init(&empty[s], 1);
    }
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();
  if (warp == 0) {
    if (lane == 0) {
      int s = 0;
      uint32_t ph = 0;
      bool ok = true;
      for (int unit = blockIdx.x; unit < p.total_units; unit += gridDim.x) {
        const EwMat& m = p.mats[find_mat(p, unit)];
        const size_t off = (size_t)(unit - m.unit_begin) * kApplyUnit;
        const size_t numel = (size_t)m.rows * m.cols;
        const uint32_t cnt = (uint32_t)(numel - off < (size_t)kApplyUnit ? numel - off : (size_t)kApplyUnit);
        if (!bar_wait(&empty[s], ph ^ 1u)) { ok = false; break; }
        bar_arrive_tx(&full[s], cnt * 4u);
        bulk_load(so + s * kApplyStageBytes, reinterpret_cast<const __nv_bfloat16*>(m.work) + off, cnt * 2u, &full[s]);
        bulk_load(sw + s * kApplyStageBytes, reinterpret_cast<const __nv_bfloat16*>(m.param) + off, cnt * 2u, &full[s]);
        if (++s == kFlatStages) { s = 0; ph ^= 1u; }
      }
      if (!ok) {
        atomicExch(p.status, kDevTimeout);
        const uint64_t t0 = gtimer();  // copies already issued land within microseconds
        while (gtimer() - t0 < 1000000ull) {
        }
      }
    }
    return;
  }
  const int ct = tid - 32;
  int s = 0, prev = -1;
  uint32_t ph = 0;
  bool ok = true;
  for (int unit = blockIdx.x; unit < p.total_units; unit += gridDim.x) {
    const EwMat& m = p.mats[find_mat(p, unit)];
    const size_t off = (size_t)(unit - m.unit_begin) * kApplyUnit;
    const size_t numel = (size_t)m.rows * m.cols;
    const uint32_t cnt = (uint32_t)(numel - off < (size_t)kApplyUnit ? numel - off : (size_t)kApplyUnit);
    float fac[kApplyUnit / 8 / kFlatCompute];  // NorMuon factor of each chunk's row (read while
    if (p.normuon) {                           // the unit's copies are still landing)
      const size_t r_first = off / (size_t)m.cols;  // row of the unit's first element
      const uint32_t rem = (uint32_t)(off - r_first * (size_t)m.cols);
#pragma unroll
      for (int j = 0; j < kApplyUnit / 8 / kFlatCompute; ++j) {
        const uint32_t k = (uint32_t)(ct + j * kFlatCompute);
        fac[j] = k * 8u < cnt ? __ldg(p.rowsq + m.row_base + (int)(r_first + (rem + 8u * k) / (uint32_t)m.cols))
                              : 0.f;
      }
    }
    if (!bar_wait(&full[s], ph)) { ok = false; break; }
    const uint4* os = reinterpret_cast<const uint4*>(so + s * kApplyStageBytes);
    uint4* ws = reinterpret_cast<uint4*>(sw + s * kApplyStageBytes);
#pragma unroll
    for (int j = 0; j < kApplyUnit / 8 / kFlatCompute; ++j) {
      const int k = ct + j * kFlatCompute;
      if ((uint32_t)k * 8u >= cnt) break;
      float o[8], w[8];
      bf16x8_to_f32(os[k], o);
      bf16x8_to_f32(ws[k], w);
      if (p.normuon) {
#pragma unroll
        for (int q = 0; q < 8; ++q) o[q] = __fmul_rn(fac[j], o[q]);
      }
#pragma unroll
      for (int q = 0; q < 8; ++q) w[q] = apply_elem(w[q], o[q], m.lrs, m.lrwd, p.cautious);
      ws[k] = f32x8_to_bf16(w);
    }
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    asm volatile("bar.sync 1, %0;" ::"n"(kFlatCompute) : "memory");
    if (ct == 0) {
      bulk_store(reinterpret_cast<__nv_bfloat16*>(m.param) + off, sw + s * kApplyStageBytes, cnt * 2u);
      bulk_commit();
      bulk_wait_read1();
      if (prev >= 0) bar_arrive(&empty[prev]);
    }
    prev = s;
    if (++s == kFlatStages) { s = 0; ph ^= 1u; }
  }
  if (ct == 0) bulk_wait_all();
  if (!ok && ct == 0) atomicExch(p.status, kDevTimeout);
}

// TMA weight update of tall matrices (bf16 weights): unit u is the 64 x 64 tile
// (u / tiles_c, u % tiles_c) of W; the producer loads the W tile and the matching
// transposed tile of the workspace X through the matrix's maps (128-byte swizzle);
// thread ct owns row ct mod 64 of the tile, columns 32*(ct/64) ..+31, reads O = X^T
// from the transposed tile, updates W in place and one thread stores the tile.  With
// NorMuon, O is scaled by its column's factor (rowsq[row_base + column]).
__global__ void __launch_bounds__(kFlatThreads)
apply_tile_tma_kernel(const __grid_constant__ EwTiledParams p) {
  extern __shared__ uint8_t atsm_raw[];
  uint8_t* tsm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(atsm_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(tsm + kFlatStages * 2 * kFlatGBytes);
  uint64_t* empty = full + kFlatStages;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (tid == 0) {
    for (int s = 0; s < kFlatStages; ++s) {
      bar_init(&full[s], 1);
      bar_init(&empty[s], 1);
    }
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();
  auto w_tile = [&](int s) { return tsm + s * 2 * kFlatGBytes; };
  auto x_tile = [&](int s) { return tsm + s * 2 * kFlatGBytes + kFlatGBytes; };
  if (warp == 0) {
    if (lane == 0) {
      int s = 0;
      uint32_t ph = 0;
      bool ok = true;
      for (int unit = blockIdx.x; unit < p.total_units; unit += gridDim.x) {
        const int mi = find_mat(p, unit);
        const EwMat& m = p.mats[mi];
        const int u = unit - m.unit_begin;
        const int r0 = (u / m.tiles_c) * kEwTile, c0 = (u % m.tiles_c) * kEwTile;
        const CUtensorMap* maps = &p.maps[kEwMapsPerMat * mi];
        if (!bar_wait(&empty[s], ph ^ 1u)) { ok = false; break; }
        bar_arrive_tx(&full[s], 2 * kFlatGBytes);
        tma_load_2d(w_tile(s), &maps[0], c0, r0, &full[s]);
        tma_load_2d(x_tile(s), &maps[1], r0, c0, &full[s]);
        if (++s == kFlatStages) { s = 0; ph ^= 1u; }
      }
      if (!ok) {
        atomicExch(p.status, kDevTimeout);
        const uint64_t t0 = gtimer();
        while (gtimer() - t0 < 1000000ull) {
        }
      }
    }
    return;
  }
  const int ct = tid - 32;
  const int r = ct & 63, h = ct >> 6;
  int s = 0, prev = -1;
  uint32_t ph = 0;
  bool ok = true;
  for (int unit = blockIdx.x; unit < p.total_units; unit += gridDim.x) {
    const int mi = find_mat(p, unit);
    const EwMat& m = p.mats[mi];
    const int u = unit - m.unit_begin;
    const int r0 = (u / m.tiles_c) * kEwTile, c0 = (u % m.tiles_c) * kEwTile;
    // NorMuon factor of column 32h + lane (all lanes of a warp share h), broadcast below;
    // read while the tile's copies are still landing
    float fac_lane = 0.f;
    if (p.normuon && c0 + 32 * h + lane < m.cols) fac_lane = __ldg(p.rowsq + m.row_base + c0 + 32 * h + lane);
    if (!bar_wait(&full[s], ph)) { ok = false; break; }
    uint8_t* wt = w_tile(s);
    const uint8_t* xt = x_tile(s);
#pragma unroll
    for (int i = 0; i < 4; ++i) {  // columns 32h + 8i .. +7
      uint4* wp = reinterpret_cast<uint4*>(wt + swz128(r, 4 * h + i));
      float w[8], o[8];
      bf16x8_to_f32(*wp, w);
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        const int c = 32 * h + 8 * i + q;  // X row c, column r
        o[q] = __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(xt + swz128(c, r >> 3) + ((r & 7) << 1)));
        if (p.normuon) o[q] = __fmul_rn(__shfl_sync(0xffffffffu, fac_lane, 8 * i + q), o[q]);
      }
#pragma unroll
      for (int q = 0; q < 8; ++q) w[q] = apply_elem(w[q], o[q], m.lrs, m.lrwd, p.cautious);
      *wp = f32x8_to_bf16(w);
    }
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    asm volatile("bar.sync 1, %0;" ::"n"(kFlatCompute) : "memory");
    if (ct == 0) {
      tma_store_2d(&p.maps[kEwMapsPerMat * mi], wt, c0, r0);
      bulk_commit();
      bulk_wait_read1();
      if (prev >= 0) bar_arrive(&empty[prev]);
    }
    prev = s;
    if (++s == kFlatStages) { s = 0; ph ^= 1u; }
  }
  if (ct == 0) bulk_wait_all();
  if (!ok && ct == 0) atomicExch(p.status, kDevTimeout);
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

cudaError_t launch_momentum_split(const EwParams& flat, const EwTiledParams* tiled, int n_tiled, const EwParams& rest,
                                  const EwParams& all, int sm_count, int* launches, cudaStream_t st) {
  *launches = 0;
  static bool smem_set[64] = {};  // per device
  int dev = 0;
  cudaError_t e0 = cudaGetDevice(&dev);
  if (e0 != cudaSuccess) return e0;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (!smem_set[dev]) {
    cudaError_t e = cudaFuncSetAttribute(momentum_flat_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)kFlatSmem);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(momentum_tile_tma_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               (int)kTileSmem);
    if (e != cudaSuccess) return e;
    smem_set[dev] = true;
  }
  for (int t = 0; t < n_tiled; ++t) {
    if (tiled[t].n_mats == 0 || tiled[t].total_units == 0) continue;
    const int grid = std::max(1, std::min(tiled[t].total_units, 2 * sm_count));
    momentum_tile_tma_kernel<<<grid, kFlatThreads, kTileSmem, st>>>(tiled[t]);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    ++*launches;
  }
  if (flat.n_mats > 0 && flat.total_units > 0) {
    const int grid = std::max(1, std::min(flat.total_units, 2 * sm_count));
    momentum_flat_kernel<<<grid, kFlatThreads, kFlatSmem, st>>>(flat);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    ++*launches;
  }
  if (rest.n_mats > 0 && rest.total_units > 0) {
    const int grid = std::max(1, std::min(rest.total_units, sm_count * 8));
    momentum_norm_kernel<__nv_bfloat16><<<grid, kThreads, 0, st>>>(rest);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    ++*launches;
  }
  if (all.n_mats > 0) {
    norm_finalize_kernel<<<all.n_mats, kThreads, 0, st>>>(all);
    ++*launches;
    return cudaGetLastError();
  }
  return cudaSuccess;
}

cudaError_t launch_apply_split(const EwParams& flat, const EwTiledParams* tiled, int n_tiled, const EwParams& rest,
                               int sm_count, int* launches, cudaStream_t st) {
  *launches = 0;
  static bool smem_set[64] = {};  // per device
  int dev = 0;
  cudaError_t e0 = cudaGetDevice(&dev);
  if (e0 != cudaSuccess) return e0;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (!smem_set[dev]) {
    cudaError_t e = cudaFuncSetAttribute(apply_flat_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)kApplyFlatSmem);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(apply_tile_tma_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               (int)kApplyTileSmem);
    if (e != cudaSuccess) return e;
    smem_set[dev] = true;
  }
  for (int t = 0; t < n_tiled; ++t) {
    if (tiled[t].n_mats == 0 || tiled[t].total_units == 0) continue;
    const int grid = std::max(1, std::min(tiled[t].total_units, 2 * sm_count));
    apply_tile_tma_kernel<<<grid, kFlatThreads, kApplyTileSmem, st>>>(tiled[t]);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    ++*launches;
  }
  if (flat.n_mats > 0 && flat.total_units > 0) {
    const int grid = std::max(1, std::min(flat.total_units, 2 * sm_count));
    apply_flat_kernel<<<grid, kFlatThreads, kApplyFlatSmem, st>>>(flat);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    ++*launches;
  }
  if (rest.n_mats > 0 && rest.total_units > 0) {
    const int grid = std::max(1, std::min(rest.total_units, sm_count * 8));
    apply_kernel<__nv_bfloat16><<<grid, kThreads, 0, st>>>(rest, kEwApply);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    ++*launches;
  }
  return cudaSuccess;
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
