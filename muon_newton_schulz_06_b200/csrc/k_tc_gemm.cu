// Grouped, persistent tcgen05 GEMM engine for the Newton-Schulz steps (bf16 operands,
// fp32 accumulation in tensor memory).
//
// Every matrix is held in wide orientation X (s x L, s <= L; tall matrices are
// transposed by the momentum pass), so one step of the page's iteration is, for both
// the tall and the wide rule (autoresearch train.py review, MuonAdamW paragraph):
//
//   Gram    A  = alpha * X X^T            (s x s, contraction over L)
//   Poly    B  = b A + c A A^T            (s x s, contraction over s; A symmetric)
//   Update  X' = a' X + beta * B X        (s x L, contraction over s)
//
// with alpha = scale^2, a' = a*scale, beta = scale on the first step (the Frobenius
// normalisation folded in) and 1 afterwards.  Gram and Poly are SYRK-shaped: both
// operands are row blocks of one K-major matrix, only tiles that touch the upper
// triangle are computed, and the epilogue writes each upper element and its mirror.
// Update reads X as an MN-major operand.
//
// CTA layout (192 threads, one CTA per SM, persistent over a cost-sorted tile list):
//   warp 0      TMA producer (one thread): 4-stage ring of A (128 x 64) and
//               B (256 x 64) tiles, 128-byte swizzle
//   warp 1      TMEM owner and MMA issuer (one thread): tcgen05.mma M=128 N=256 K=16
//   warps 2..5  epilogue: tcgen05.ld 32 lanes x 32 columns, fused scale / polynomial /
//               update arithmetic, bf16 stores (+ mirrored stores for Gram/Poly)
// Two 256-column accumulators in TMEM let the epilogue of tile t overlap the
// main loop of tile t+1.  Every mbarrier wait is bounded in time; on expiry the
// kernel writes kDevTimeout to the status word, drains its own MMAs and returns.
#include "muon_internal.h"

namespace muon {
namespace {

constexpr int kStages = 4;
constexpr int kThreadsTc = 192;
constexpr uint32_t kABytes = kBM * kBK * 2;   // 16 KB
constexpr uint32_t kBBytes = kBN * kBK * 2;   // 32 KB
constexpr uint32_t kStageBytes = kABytes + kBBytes;
constexpr uint32_t kTmemCols = 2 * kBN;       // two fp32 accumulators of 256 columns
constexpr uint32_t kBarrierBytes = 256;
constexpr uint32_t kSmemBytes = kStages * kStageBytes + kBarrierBytes + 1024;
constexpr unsigned long long kWaitLimitNs = 2000000000ull;  // 2 s per wait

// tcgen05 instruction descriptor, kind::f16: D f32, A/B bf16, A K-major, N=256, M=128.
__host__ __device__ constexpr uint32_t make_idesc(bool b_mn_major) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((b_mn_major ? 1u : 0u) << 16) |
         ((uint32_t)(kBN >> 3) << 17) | ((uint32_t)(kBM >> 4) << 24);
}

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// Shared-memory matrix descriptor (sm_100 format): start, leading / stride byte
// offsets (16-byte units), version 1, 128-byte swizzle.
__device__ __forceinline__ uint64_t sdesc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
  d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
  d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;
  d |= (uint64_t)1 << 46;
  d |= (uint64_t)2 << 61;
  return d;
}

__device__ __forceinline__ uint64_t global_timer() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}\n"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Bounded wait: false on time-out, or (when abort_flag is given) once another role of
// the CTA gave up.
__device__ __noinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_timer();
  uint32_t n = 0;
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((++n & 63u) == 0) {
      if (abort_flag != nullptr && *abort_flag) return false;
      if (global_timer() - t0 > kWaitLimitNs) return false;
    }
  }
}

__device__ __forceinline__ void tma_load_3d(uint32_t dst, const CUtensorMap* map, uint64_t* bar, int x,
                                            int y, int z) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(x), "r"(y), "r"(z)
      : "memory");
}

__device__ __forceinline__ void umma_bf16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                          uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate));
}

__device__ __forceinline__ void umma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   smem_u32(bar))
               : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// 32 lanes x 32 consecutive fp32 columns: thread i gets row (lane base + i).
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float* v) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
        "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
        "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

__device__ __forceinline__ void load_bf16x32(const __nv_bfloat16* src, float* v) {
  const uint4* s4 = reinterpret_cast<const uint4*>(src);
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    uint4 raw = s4[q];
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&raw);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      float2 f = __bfloat1622float2(h[e]);
      v[8 * q + 2 * e] = f.x;
      v[8 * q + 2 * e + 1] = f.y;
    }
  }
}

__device__ __forceinline__ void store_bf16x32(__nv_bfloat16* dst, const float* v) {
  uint4* d4 = reinterpret_cast<uint4*>(dst);
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    uint4 raw;
    __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&raw);
#pragma unroll
    for (int e = 0; e < 4; ++e) h[e] = __floats2bfloat162_rn(v[8 * q + 2 * e], v[8 * q + 2 * e + 1]);
    d4[q] = raw;
  }
}

template <int PHASE>
__global__ void __launch_bounds__(kThreadsTc, 1) tc_kernel(const __grid_constant__ TcParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kStages * kStageBytes);
  uint64_t* empty = full + kStages;
  uint64_t* tfull = empty + kStages;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], 4);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                 "r"(kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  constexpr bool kSyrk = (PHASE != kPhaseUpdate);

  if (warp == 0) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < p.n_tiles && ok; t += gridDim.x) {
        const TcTile tile = p.tiles[t];
        const TcGroup& g = p.g[tile.group];
        const int K = (PHASE == kPhaseGram) ? g.L : g.s;
        const int nk = (K + kBK - 1) / kBK;
        const CUtensorMap* ma = &p.map_a[tile.group];
        const CUtensorMap* mb = &p.map_b[tile.group];
        const int row_a = tile.bi * kBM;
        const int col_b = tile.bj * kBN;
        for (int kb = 0; kb < nk; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1u, abort_flag)) { ok = false; break; }
          mbar_arrive_expect_tx(&full[stage], kStageBytes);
          const uint32_t a_dst = smem_u32(smem + stage * kStageBytes);
          const uint32_t b_dst = a_dst + kABytes;
          const int k0 = kb * kBK;
          tma_load_3d(a_dst, ma, &full[stage], k0, row_a, tile.mat);
          if (kSyrk) {
            tma_load_3d(b_dst, ma, &full[stage], k0, col_b, tile.mat);
            tma_load_3d(b_dst + kABytes, ma, &full[stage], k0, col_b + kBM, tile.mat);
          } else {
#pragma unroll
            for (int q = 0; q < kBN / 64; ++q)
              tma_load_3d(b_dst + q * (64 * kBK * 2), mb, &full[stage], col_b + 64 * q, k0, tile.mat);
          }
          if (++stage == kStages) { stage = 0; phase ^= 1u; }
        }
      }
      if (!ok) {
        atomicExch(p.status, kDevTimeout);
        *abort_flag = 1;
      }
      // let every copy this thread armed land before the CTA can exit
      for (int s = 0; s < kStages; ++s) {
        // the most recent arm of stage s used parity (phase of that pass)
        const int passes_back = (s < stage) ? 0 : 1;
        const uint32_t par = passes_back ? (phase ^ 1u) : phase;
        (void)mbar_wait(&full[s], par, nullptr);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = make_idesc(!kSyrk);
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < p.n_tiles && ok; t += gridDim.x) {
        const TcTile tile = p.tiles[t];
        const TcGroup& g = p.g[tile.group];
        const int K = (PHASE == kPhaseGram) ? g.L : g.s;
        const int nk = (K + kBK - 1) / kBK;
        if (!mbar_wait(&tempty[acc], acc_phase ^ 1u, abort_flag)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + (uint32_t)(acc * kBN);
        for (int kb = 0; kb < nk; ++kb) {
          if (!mbar_wait(&full[stage], phase, abort_flag)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a_addr = smem_u32(smem + stage * kStageBytes);
          const uint32_t b_addr = a_addr + kABytes;
#pragma unroll
          for (int k = 0; k < kBK / 16; ++k) {
            const uint64_t ad = sdesc(a_addr + k * 32, 16, 1024);
            const uint64_t bd = kSyrk ? sdesc(b_addr + k * 32, 16, 1024)
                                      : sdesc(b_addr + k * 2048, 64 * kBK * 2, 1024);
            umma_bf16(d_tmem, ad, bd, idesc, (kb > 0 || k > 0) ? 1u : 0u);
          }
          umma_commit(&empty[stage]);
          if (++stage == kStages) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        umma_commit(&tfull[acc]);
        if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
      }
      if (!ok) {
        atomicExch(p.status, kDevTimeout);
        *abort_flag = 1;
      }
      // all MMAs issued by this thread complete before TMEM is released
      umma_commit(drain);
      (void)mbar_wait(drain, 0, nullptr);
    }
  } else {
    // ------------------------------------------------------------------ epilogue
    const int quad = warp & 3;  // TMEM lane quadrant this warp may access
    int acc = 0;
    uint32_t acc_phase = 0;
    bool ok = true;
    for (int t = blockIdx.x; t < p.n_tiles; t += gridDim.x) {
      const TcTile tile = p.tiles[t];
      const TcGroup& g = p.g[tile.group];
      if (!mbar_wait(&tfull[acc], acc_phase, abort_flag)) { ok = false; break; }
      tc_fence_after();

      const int s = g.s;
      const int row0 = tile.bi * kBM + 32 * quad;  // first row of this warp
      const int row = row0 + lane;
      const float sc = p.first_iter ? p.scale[g.gid_base + tile.mat] : 1.f;
      const uint32_t tbase = tmem_base + ((uint32_t)(32 * quad) << 16) + (uint32_t)(acc * kBN);

      if (row0 < s) {
        for (int c = 0; c < kBN / 32; ++c) {
          const int col0 = tile.bj * kBN + 32 * c;
          if (kSyrk) {
            if (col0 >= s || col0 + 31 < row0) continue;  // outside / strictly lower block
          } else {
            if (col0 >= g.L) continue;
          }
          float v[32];
          tmem_ld32(tbase + (uint32_t)(32 * c), v);
          if (PHASE == kPhaseGram) {
            const float alpha = sc * sc;
#pragma unroll
            for (int j = 0; j < 32; ++j) v[j] *= alpha;
          } else if (PHASE == kPhasePoly) {
            const __nv_bfloat16* a = g.gram + (size_t)tile.mat * s * g.ld_s;
            if (row < s) {
              float av[32];
              if (col0 + 32 <= s) {
                load_bf16x32(a + (size_t)row * g.ld_s + col0, av);
              } else {
#pragma unroll
                for (int j = 0; j < 32; ++j)
                  av[j] = (col0 + j < s) ? __bfloat162float(a[(size_t)row * g.ld_s + col0 + j]) : 0.f;
              }
#pragma unroll
              for (int j = 0; j < 32; ++j) v[j] = fmaf(p.cb, av[j], p.cc * v[j]);
            }
          } else {
            const size_t moff = (size_t)tile.mat * s * g.ld_x;
            const __nv_bfloat16* x = g.x_cur + moff;
            __nv_bfloat16* xn = g.x_next + moff;
            const float alpha = p.ca * sc;
            if (row < s) {
              float xv[32];
              if (col0 + 32 <= g.L) {
                load_bf16x32(x + (size_t)row * g.ld_x + col0, xv);
#pragma unroll
                for (int j = 0; j < 32; ++j) xv[j] = fmaf(alpha, xv[j], sc * v[j]);
                store_bf16x32(xn + (size_t)row * g.ld_x + col0, xv);
              } else {
#pragma unroll
                for (int j = 0; j < 32; ++j) {
                  if (col0 + j < g.L) {
                    const size_t o = (size_t)row * g.ld_x + col0 + j;
                    xn[o] = __float2bfloat16_rn(fmaf(alpha, __bfloat162float(x[o]), sc * v[j]));
                  }
                }
              }
            }
            continue;
          }
          // symmetric store: upper element (row, col) and its mirror (col, row)
          __nv_bfloat16* out = (PHASE == kPhaseGram ? g.gram : g.poly) + (size_t)tile.mat * s * g.ld_s;
          if (row < s) {
            if (col0 >= row0 + 32) {
              if (col0 + 32 <= s) {
                store_bf16x32(out + (size_t)row * g.ld_s + col0, v);
              } else {
#pragma unroll
                for (int j = 0; j < 32; ++j)
                  if (col0 + j < s) out[(size_t)row * g.ld_s + col0 + j] = __float2bfloat16_rn(v[j]);
              }
#pragma unroll
              for (int j = 0; j < 32; ++j)
                if (col0 + j < s) out[(size_t)(col0 + j) * g.ld_s + row] = __float2bfloat16_rn(v[j]);
            } else {
              // diagonal 32 x 32 block (col0 == row0)
#pragma unroll
              for (int j = 0; j < 32; ++j) {
                const int col = col0 + j;
                if (col < s && col >= row) {
                  const __nv_bfloat16 b = __float2bfloat16_rn(v[j]);
                  out[(size_t)row * g.ld_s + col] = b;
                  if (col > row) out[(size_t)col * g.ld_s + row] = b;
                }
              }
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty[acc]);
      if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
    }
    if (!ok && lane == 0) {
      atomicExch(p.status, kDevTimeout);
      *abort_flag = 1;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(kTmemCols)
                 : "memory");
  }
}

template <int PHASE>
cudaError_t launch_phase(const TcParams& p, int grid, cudaStream_t st) {
  static uint64_t configured = 0;  // one bit per device: the attribute is set per device
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const uint64_t bit = (dev < 64) ? (uint64_t(1) << dev) : 0;
  if (!(configured & bit)) {
    e = cudaFuncSetAttribute(tc_kernel<PHASE>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemBytes);
    if (e != cudaSuccess) return e;
    configured |= bit;
  }
  tc_kernel<PHASE><<<grid, kThreadsTc, kSmemBytes, st>>>(p);
  return cudaGetLastError();
}

}  // namespace

int tc_smem_bytes() { return (int)kSmemBytes; }

cudaError_t launch_tc(int phase, const TcParams& p, int grid, cudaStream_t st) {
  if (p.n_tiles == 0) return cudaSuccess;
  switch (phase) {
    case kPhaseGram: return launch_phase<kPhaseGram>(p, grid, st);
    case kPhasePoly: return launch_phase<kPhasePoly>(p, grid, st);
    case kPhaseUpdate: return launch_phase<kPhaseUpdate>(p, grid, st);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace muon
