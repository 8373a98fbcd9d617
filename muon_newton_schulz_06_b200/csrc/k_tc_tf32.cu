// fp32 validation mode of the Newton-Schulz steps on tcgen05 tensor cores, 3xTF32.
//
// The same three products as the bf16 engine (k_tc_gemm.cu), in fp32 storage:
//
//   Gram    A  = alpha * X X^T      Poly    B  = b A + c A A^T      Update  X' = a' X + beta * B X
//
// A TF32 operand keeps 11 significant bits of an fp32 value, too few for the 1e-4
// comparison this mode exists for; the products therefore use the split x ~ hi + lo with
// hi = tf32(x) and lo = tf32(x - hi), both rounded to nearest, and accumulate
// hi*hi + hi*lo + lo*hi in fp32 in tensor memory.  hi + lo carries 22 significant bits of
// x (|x - hi - lo| <= 2^-22 |x|, unbiased) and the dropped lo*lo term is below 2^-22 of
// the product.  Every value is stored in the workspace as its two parts, written by the
// epilogue that produces it; an epilogue that needs a value back reads hi + lo.
//
// Tiles, tile lists and the roles are those of the bf16 engine: a pair of CTAs (2-CTA
// cluster) per 256 x 256 tile with tcgen05.mma.cta_group::2.kind::tf32 (M = N = 256,
// K = 8), CTA r holding rows [128r, 128r+128) of A and of B (or B's columns for the
// MN-major X of Update), persistent over the cluster's share of the tile list:
//   warp 0      TMA producer (one thread): 3-stage ring; a stage holds the hi and lo
//               parts of this CTA's A rows and B rows / columns, 32 fp32 (one 128-byte
//               swizzle row) deep, 64 KB; no multicast.  K-major tiles use the 128-byte
//               swizzle; the MN-major X of Update the 128-byte swizzle with a 32-byte
//               base, the tensor cores' layout for MN-major 32-bit operands
//   warp 1      TMEM owner; in the leader CTA the MMA issuer: three MMAs per 8-deep
//               k-step, hi*hi into one 256-column accumulator and hi*lo, lo*hi into a
//               second one (the epilogue adds the two, rounding to nearest).  The
//               tensor cores' fp32 accumulation does not round to nearest and its error
//               grows with the number of accumulations into the large sum; keeping the
//               cross terms (2^-11 of it) apart leaves one accumulation per k-step in
//               the large sum instead of three.  Both accumulators serve one tile, so
//               the epilogue of a tile does not overlap the next tile's products
//   warps 2..5  epilogue of this CTA's 128 x 256 half: tcgen05.ld 32 lanes x 32
//               columns, the phase's arithmetic in fp32, then the hi and lo parts (and,
//               for Gram / Poly, their mirror below the diagonal) straight to global
//               memory; a thread holds one row, so row stores are 128-byte runs per
//               thread and mirror stores are 128-byte runs per warp
// Every wait is bounded, with the bf16 engine's abort protocol.
#include <algorithm>
#include <atomic>
#include <mutex>

#include "muon_internal.h"
#include "tc_primitives.cuh"

namespace muon {
namespace {

constexpr int kStages32 = 3;
constexpr int kEpi32 = 4;
constexpr int kThreads32 = 64 + 32 * kEpi32;
constexpr int kBK32 = 32;                               // fp32 per 128-byte swizzle row
constexpr uint32_t kPart32 = kHalf * kBK32 * 4;         // 16 KB: 128 rows (or columns) x 32 fp32
constexpr uint32_t kStage32 = 4 * kPart32;              // A hi, A lo, B hi, B lo
constexpr uint32_t kPairTx32 = 2 * kStage32;
constexpr uint32_t kTmemCols32 = 2 * kTile;
constexpr uint32_t kBarrier32 = 256;
constexpr uint32_t kSmem32 = kStages32 * kStage32 + kBarrier32 + 1024;
static_assert(kSmem32 <= 232448, "shared memory per CTA (3xTF32 engine)");

// tcgen05 instruction descriptor, kind::tf32: D f32, A/B TF32, A K-major, M = N = 256.
__host__ __device__ constexpr uint32_t make_idesc_tf32(bool b_mn_major) {
  return (1u << 4) | (2u << 7) | (2u << 10) | ((b_mn_major ? 1u : 0u) << 16) | ((uint32_t)(kTile >> 3) << 17) |
         ((uint32_t)(kTile >> 4) << 24);
}

__device__ __forceinline__ void umma_pair_tf32(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                               uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::tf32 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate));
}

// Shared-memory matrix descriptor for an MN-major 32-bit operand: the only layout the
// tensor cores take for it is the 128-byte swizzle with a 32-byte base (32-byte chunks
// of each 128-byte row XOR-ed with the row index modulo 4; the TMA mode
// CU_TENSOR_MAP_SWIZZLE_128B_ATOM_32B writes it).  Leading offset: bytes between
// consecutive 32-element MN atoms; stride offset: bytes between consecutive groups of
// 4 K-rows.
__device__ __forceinline__ uint64_t sdesc_mn32(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
  d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
  d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;
  d |= (uint64_t)1 << 46;
  d |= (uint64_t)1 << 61;
  return d;
}

// Round to the nearest TF32 value (ties away from zero), as an fp32 bit pattern.
__device__ __forceinline__ float tf32_hi(float x) {
  uint32_t r;
  asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
  return __uint_as_float(r);
}

// 32 consecutive fp32 of one row: hi + lo, columns at or beyond `lim` read as 0.
__device__ __forceinline__ void load_row32(const float* hi, const float* lo, int col0, int lim, float* v) {
  if (col0 + 32 <= lim) {
    const float4* h4 = reinterpret_cast<const float4*>(hi + col0);
    const float4* l4 = reinterpret_cast<const float4*>(lo + col0);
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const float4 a = h4[q], b = l4[q];
      v[4 * q] = __fadd_rn(a.x, b.x);
      v[4 * q + 1] = __fadd_rn(a.y, b.y);
      v[4 * q + 2] = __fadd_rn(a.z, b.z);
      v[4 * q + 3] = __fadd_rn(a.w, b.w);
    }
    return;
  }
#pragma unroll
  for (int j = 0; j < 32; ++j) v[j] = (col0 + j < lim) ? __fadd_rn(hi[col0 + j], lo[col0 + j]) : 0.f;
}

// Stores value v at (hi, lo), split, or unsplit into hi alone.
__device__ __forceinline__ void put(float* hi, float* lo, size_t i, float v, bool plain) {
  if (plain) {
    hi[i] = v;
    return;
  }
  const float h = tf32_hi(v);
  hi[i] = h;
  lo[i] = tf32_hi(__fsub_rn(v, h));
}

// 32 consecutive values of one row, columns below `lim`.
__device__ __forceinline__ void store_row32(float* hi, float* lo, int col0, int lim, const float* v, bool plain) {
  if (col0 + 32 <= lim) {
    float4* h4 = reinterpret_cast<float4*>(hi + col0);
    float4* l4 = reinterpret_cast<float4*>(lo + col0);
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      if (plain) {
        h4[q] = make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
      } else {
        float h[4], l[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          h[e] = tf32_hi(v[4 * q + e]);
          l[e] = tf32_hi(__fsub_rn(v[4 * q + e], h[e]));
        }
        h4[q] = make_float4(h[0], h[1], h[2], h[3]);
        l4[q] = make_float4(l[0], l[1], l[2], l[3]);
      }
    }
    return;
  }
#pragma unroll
  for (int j = 0; j < 32; ++j)
    if (col0 + j < lim) put(hi, lo, (size_t)(col0 + j), v[j], plain);
}

__global__ void tf32_split_kernel(float* __restrict__ hi, float* __restrict__ lo, size_t n) {
  for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (size_t)gridDim.x * blockDim.x) {
    const float x = hi[i];
    const float h = tf32_hi(x);
    hi[i] = h;
    lo[i] = tf32_hi(__fsub_rn(x, h));
  }
}

template <int PHASE>
__global__ void __launch_bounds__(kThreads32, 1) tc32_kernel(const __grid_constant__ Tc32Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kStages32 * kStage32);
  uint64_t* empty = full + kStages32;
  uint64_t* tfull = empty + kStages32;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank();
  const int cluster = blockIdx.x >> 1;
  const int n_clusters = gridDim.x >> 1;
  constexpr bool kSyrk = PHASE != kPhaseUpdate;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages32; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], 2 * kEpi32);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                 "r"(kTmemCols32)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  cluster_sync_all();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const uint32_t peer_abort = peer_addr(smem_u32((const void*)abort_flag), rank ^ 1u);
  auto give_up = [&]() {
    atomicExch(p.status, kDevTimeout);
    *abort_flag = 1;
    remote_store_flag(peer_abort, 1);
  };

  if (warp == 0) {
    // ------------------------------------------------------------------ TMA producer (both CTAs)
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int t = cluster; t < p.n_tiles && ok; t += n_clusters) {
        const TcTile tile = p.tiles[t];
        const Tc32Group& g = p.g[tile.group];
        const int K = (PHASE == kPhaseGram) ? g.L : g.s;
        const int nk = (K + kBK32 - 1) / kBK32;
        const int row_a = tile.bi * kTile + (int)rank * kHalf;
        const int col_b = tile.bj * kTile + (int)rank * kHalf;
        for (int kb = 0; kb < nk; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1u, abort_flag)) { ok = false; break; }
          if (rank == 0) mbar_arrive_expect_tx(&full[stage], kPairTx32);
          const uint32_t base = smem_u32(smem + stage * kStage32);
          const uint32_t bar = peer_addr(smem_u32(&full[stage]), 0);
          const int k0 = kb * kBK32;
          tma_load_3d_pair(base, &p.a_hi[tile.group], bar, k0, row_a, tile.mat);
          tma_load_3d_pair(base + kPart32, &p.a_lo[tile.group], bar, k0, row_a, tile.mat);
          if (kSyrk) {
            tma_load_3d_pair(base + 2 * kPart32, &p.a_hi[tile.group], bar, k0, col_b, tile.mat);
            tma_load_3d_pair(base + 3 * kPart32, &p.a_lo[tile.group], bar, k0, col_b, tile.mat);
          } else {
#pragma unroll
            for (int q = 0; q < kHalf / 32; ++q) {
              tma_load_3d_pair(base + 2 * kPart32 + q * (32 * kBK32 * 4), &p.b_hi[tile.group], bar, col_b + 32 * q,
                               k0, tile.mat);
              tma_load_3d_pair(base + 3 * kPart32 + q * (32 * kBK32 * 4), &p.b_lo[tile.group], bar, col_b + 32 * q,
                               k0, tile.mat);
            }
          }
          if (++stage == kStages32) { stage = 0; phase ^= 1u; }
        }
      }
      if (!ok || *abort_flag) {
        give_up();
        spin_ns(kAbortGraceNs);
      } else if (rank == 0) {
        for (int s = 0; s < kStages32; ++s) {
          const uint32_t par = (s < stage) ? phase : (phase ^ 1u);
          (void)mbar_wait(&full[s], par, nullptr);
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer (leader CTA)
    if (lane == 0 && rank == 0) {
      constexpr uint32_t idesc = make_idesc_tf32(!kSyrk);
      int stage = 0;
      uint32_t phase = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      for (int t = cluster; t < p.n_tiles && ok; t += n_clusters) {
        const TcTile tile = p.tiles[t];
        const Tc32Group& g = p.g[tile.group];
        const int K = (PHASE == kPhaseGram) ? g.L : g.s;
        const int nk = (K + kBK32 - 1) / kBK32;
        if (!mbar_wait(&tempty[0], acc_phase ^ 1u, abort_flag)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d_big = tmem_base, d_small = tmem_base + (uint32_t)kTile;
        for (int kb = 0; kb < nk; ++kb) {
          if (!mbar_wait(&full[stage], phase, abort_flag)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a_hi = smem_u32(smem + stage * kStage32);
          const uint32_t a_lo = a_hi + kPart32, b_hi = a_hi + 2 * kPart32, b_lo = a_hi + 3 * kPart32;
#pragma unroll
          for (int k = 0; k < kBK32 / 8; ++k) {
            const uint64_t ah = sdesc(a_hi + k * 32, 16, 1024), al = sdesc(a_lo + k * 32, 16, 1024);
            const uint64_t bh = kSyrk ? sdesc(b_hi + k * 32, 16, 1024) : sdesc_mn32(b_hi + k * 1024, 32 * kBK32 * 4, 512);
            const uint64_t bl = kSyrk ? sdesc(b_lo + k * 32, 16, 1024) : sdesc_mn32(b_lo + k * 1024, 32 * kBK32 * 4, 512);
            const uint32_t accum = (kb > 0 || k > 0) ? 1u : 0u;
            umma_pair_tf32(d_big, ah, bh, idesc, accum);
            umma_pair_tf32(d_small, ah, bl, idesc, accum);
            umma_pair_tf32(d_small, al, bh, idesc, 1u);
          }
          umma_commit_both(&empty[stage]);
          if (++stage == kStages32) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        umma_commit_both(&tfull[0]);
        acc_phase ^= 1u;
      }
      if (!ok) give_up();
      umma_commit_local(drain);
      (void)mbar_wait(drain, 0, nullptr);
    }
  } else {
    // ------------------------------------------------------------------ epilogue (both CTAs)
    const int quad = warp & 3;
    const uint32_t leader_tempty0 = peer_addr(smem_u32(&tempty[0]), 0);
    uint32_t acc_phase = 0;
    bool ok = true;
    for (int t = cluster; t < p.n_tiles && ok; t += n_clusters) {
      const TcTile tile = p.tiles[t];
      const Tc32Group& g = p.g[tile.group];
      if (!mbar_wait(&tfull[0], acc_phase, abort_flag)) { ok = false; break; }
      tc_fence_after();
      const int s = g.s;
      const int lim = kSyrk ? g.s : g.L;
      const int row0 = tile.bi * kTile + (int)rank * kHalf + 32 * quad;
      const int row = row0 + lane;
      const float sc = p.first_iter ? p.scale[g.gid_base + tile.mat] : 1.f;
      const uint32_t tbase = tmem_base + ((uint32_t)(32 * quad) << 16);
      const float* in_hi = (PHASE == kPhaseGram) ? nullptr : g.in_hi + tile.mat * g.in_stride + (size_t)row * g.ld_in;
      const float* in_lo = (PHASE == kPhaseGram) ? nullptr : g.in_lo + tile.mat * g.in_stride + (size_t)row * g.ld_in;
      float* out_hi = g.out_hi + tile.mat * g.out_stride;
      float* out_lo = g.out_lo + tile.mat * g.out_stride;
      const bool plain = PHASE == kPhaseUpdate && p.plain_out;
      // valid chunks: inside the result and, for Gram / Poly, not below the diagonal
      int c_lo = 0, c_hi = kTile / 32;
      if (row0 >= s) c_hi = c_lo;
      while (c_hi > c_lo && tile.bj * kTile + 32 * (c_hi - 1) >= lim) --c_hi;
      if (kSyrk)
        while (c_lo < c_hi && tile.bj * kTile + 32 * c_lo + 31 < row0) ++c_lo;
      for (int c = c_lo; c < c_hi; ++c) {
        const int col0 = tile.bj * kTile + 32 * c;
        float v[32], vs[32];
        tmem_ld32(tbase + (uint32_t)(32 * c), v);                      // hi*hi
        tmem_ld32(tbase + (uint32_t)kTile + (uint32_t)(32 * c), vs);  // hi*lo + lo*hi
#pragma unroll
        for (int j = 0; j < 32; ++j) v[j] = __fadd_rn(v[j], vs[j]);
        if (PHASE == kPhaseGram) {
          const float alpha = sc * sc;
#pragma unroll
          for (int j = 0; j < 32; ++j) v[j] *= alpha;
        } else {
          float in_v[32];
          if (row < s) {
            load_row32(in_hi, in_lo, col0, lim, in_v);
          } else {
#pragma unroll
            for (int j = 0; j < 32; ++j) in_v[j] = 0.f;
          }
          if (PHASE == kPhasePoly) {
#pragma unroll
            for (int j = 0; j < 32; ++j) v[j] = fmaf(p.cb, in_v[j], p.cc * v[j]);
          } else {
            const float alpha = p.ca * sc;
#pragma unroll
            for (int j = 0; j < 32; ++j) v[j] = fmaf(alpha, in_v[j], sc * v[j]);
          }
        }
        if (!kSyrk) {
          if (row < s) store_row32(out_hi + (size_t)row * g.ld_out, out_lo + (size_t)row * g.ld_out, col0, lim, v,
                                   plain);
          continue;
        }
        // symmetric store: the block (row0.., col0..) and its mirror, both from the upper
        // triangle's values, so the result is exactly symmetric
        if (row < s) {
          if (col0 >= row0 + 32) {
            store_row32(out_hi + (size_t)row * g.ld_out, out_lo + (size_t)row * g.ld_out, col0, lim, v, false);
#pragma unroll
            for (int j = 0; j < 32; ++j)
              if (col0 + j < s) put(out_hi, out_lo, (size_t)(col0 + j) * g.ld_out + row, v[j], false);
          } else {
            // diagonal block (col0 == row0): element (lane, j) for j >= lane, mirrored below
#pragma unroll
            for (int j = 0; j < 32; ++j) {
              if (j >= lane && col0 + j < s) {
                put(out_hi, out_lo, (size_t)row * g.ld_out + col0 + j, v[j], false);
                if (j > lane) put(out_hi, out_lo, (size_t)(col0 + j) * g.ld_out + row, v[j], false);
              }
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) remote_arrive(leader_tempty0);
      acc_phase ^= 1u;
    }
    if (!ok && lane == 0) give_up();
  }

  __syncwarp();
  tc_fence_before();
  cluster_sync_all();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(kTmemCols32)
                 : "memory");
  }
}

struct Dev32Info {
  std::atomic<bool> ready{false};
  int clusters = 0;
};
Dev32Info g_dev32[64];
std::mutex g_dev32_mutex;

cudaError_t device_setup32(int dev) {
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  Dev32Info& d = g_dev32[dev];
  if (d.ready.load(std::memory_order_acquire)) return cudaSuccess;
  std::lock_guard<std::mutex> lock(g_dev32_mutex);
  if (d.ready.load(std::memory_order_relaxed)) return cudaSuccess;
  cudaError_t e = cudaFuncSetAttribute(tc32_kernel<kPhaseGram>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmem32);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(tc32_kernel<kPhasePoly>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmem32);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(tc32_kernel<kPhaseUpdate>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmem32);
  if (e != cudaSuccess) return e;
  int sms = 0;
  e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(sms & ~1), 1, 1);
  cfg.blockDim = dim3(kThreads32, 1, 1);
  cfg.dynamicSmemBytes = kSmem32;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  e = cudaOccupancyMaxActiveClusters(&n, tc32_kernel<kPhaseUpdate>, &cfg);
  if (e != cudaSuccess || n <= 0) {
    cudaGetLastError();
    n = sms / 2;
  }
  d.clusters = n;
  d.ready.store(true, std::memory_order_release);
  return cudaSuccess;
}

template <int PHASE>
cudaError_t launch32(const Tc32Params& p, int clusters, cudaStream_t st) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(2 * clusters), 1, 1);
  cfg.blockDim = dim3(kThreads32, 1, 1);
  cfg.dynamicSmemBytes = kSmem32;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, tc32_kernel<PHASE>, p);
}

}  // namespace

cudaError_t launch_tc32(int phase, const Tc32Params& p, cudaStream_t st) {
  if (p.n_tiles == 0) return cudaSuccess;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e == cudaSuccess) e = device_setup32(dev);
  if (e != cudaSuccess) return e;
  const int clusters = std::max(1, std::min(g_dev32[dev].clusters, p.n_tiles));
  switch (phase) {
    case kPhaseGram: return launch32<kPhaseGram>(p, clusters, st);
    case kPhasePoly: return launch32<kPhasePoly>(p, clusters, st);
    case kPhaseUpdate: return launch32<kPhaseUpdate>(p, clusters, st);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_tf32_split(float* hi, float* lo, size_t n, cudaStream_t st) {
  if (n == 0) return cudaSuccess;
  const size_t blocks = std::min<size_t>((n + 255) / 256, 148 * 16);
  tf32_split_kernel<<<(unsigned)blocks, 256, 0, st>>>(hi, lo, n);
  return cudaGetLastError();
}

}  // namespace muon
