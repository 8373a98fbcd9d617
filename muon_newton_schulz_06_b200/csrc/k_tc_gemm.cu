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
// A pair of CTAs (2-CTA cluster, one CTA per SM) computes each 256 x 256 tile with
// tcgen05.mma.cta_group::2 (M = N = 256, K = 16): CTA r holds rows [128r, 128r+128) of
// the A operand and rows / columns [128r, 128r+128) of the B operand, so each SM
// stages only half of B and its shared memory serves 64 B/clk of operands instead of
// 96 (the limit of the single-CTA form).  Per CTA (192 threads, persistent over the
// cluster's share of a cost-sorted tile list):
//   warp 0      TMA producer (one thread): 6-stage ring of 128 x 64 A and 128 x 64 B
//               tiles, 128-byte swizzle; both CTAs' copies complete on the leader
//               CTA's barrier (cta_group::2 form of the bulk tensor copy, no multicast)
//   warp 1      TMEM owner; in the leader CTA also the MMA issuer (one thread), whose
//               commits arrive on both CTAs' barriers
//   warps 2..5  epilogue of this CTA's 128 x 256 half (one warp per TMEM lane
//               quadrant): tcgen05.ld 32 lanes x 32 columns, fused scale / polynomial /
//               update arithmetic; each 32 x 32 bf16 block (and, for Gram/Poly, its
//               mirror) is staged in shared memory and written by a TMA store
// Two 256-column accumulators in TMEM let the epilogue of tile t overlap the main loop
// of tile t+1.  Every mbarrier wait is bounded in time; on expiry the kernel writes
// kDevTimeout to the status word, tells the peer CTA, lets its own copies and MMAs
// drain, frees TMEM and returns.
#include <algorithm>
#include <atomic>
#include <mutex>

#include "muon_internal.h"
#include "tc_primitives.cuh"

namespace muon {
namespace {

// Stage ring depth per phase (Poly keeps one stage less to fit its larger staging area).
__host__ __device__ constexpr int stages_for(int phase) { return phase == 1 ? 5 : 6; }
constexpr int kEpiWarps = 4;  // one per TMEM lane quadrant
constexpr int kThreadsTc = 64 + 32 * kEpiWarps;
constexpr uint32_t kABytes = kHalf * kBK * 2;   // 16 KB: this CTA's 128 rows of A
constexpr uint32_t kBBytes = kHalf * kBK * 2;   // 16 KB: this CTA's half of B
constexpr uint32_t kStageBytes = kABytes + kBBytes;
constexpr uint32_t kPairTxBytes = 2 * kStageBytes;  // both CTAs' copies land on the leader's barrier
constexpr uint32_t kTmemCols = 2 * kTile;        // two fp32 accumulators of 256 columns
constexpr uint32_t kBarrierBytes = 256;
// Epilogue staging per warp (32 x 32 bf16 blocks of 2 KB, 64-byte swizzle), double
// buffered: output blocks for the TMA stores (Gram/Poly: block + mirror; Update: block)
// and, for Poly and Update, the prefetched input block (A, or X) of the next chunk.
constexpr uint32_t kOutBlockBytes = kOutBox * kOutBox * 2;
__host__ __device__ constexpr uint32_t out_bytes_for(int phase) { return 2u * (phase == 2 ? 1u : 2u) * kOutBlockBytes; }
__host__ __device__ constexpr uint32_t in_bytes_for(int phase) { return phase == 0 ? 0u : 2u * kOutBlockBytes; }
__host__ __device__ constexpr uint32_t warp_stage_bytes_for(int phase) { return out_bytes_for(phase) + in_bytes_for(phase); }
__host__ __device__ constexpr uint32_t smem_bytes_for(int phase) {
  return (uint32_t)stages_for(phase) * kStageBytes + kEpiWarps * warp_stage_bytes_for(phase) + kBarrierBytes + 1024;
}
static_assert(smem_bytes_for(0) <= 232448 && smem_bytes_for(1) <= 232448 && smem_bytes_for(2) <= 232448,
              "shared memory per CTA");

// tcgen05 instruction descriptor, kind::f16: D f32, A/B bf16, A K-major, M = N = 256.
__host__ __device__ constexpr uint32_t make_idesc(bool b_mn_major) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((b_mn_major ? 1u : 0u) << 16) |
         ((uint32_t)(kTile >> 3) << 17) | ((uint32_t)(kTile >> 4) << 24);
}

// Diagnostic: one thread waits, with the same bounded wait as the engine, on a barrier
// that nothing ever completes, and records the time-out in the status word.
__global__ void wait_selftest_kernel(int* status, unsigned long long limit_ns) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    if (!mbar_wait(&bar, 0, nullptr, limit_ns)) atomicExch(status, kDevTimeout);
  }
}

__device__ __forceinline__ void umma_pair_bf16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                               uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate));
}

// Thread `r` reads row r of a staged 32 x 32 bf16 block (4 x 16-byte loads).
__device__ __forceinline__ void unstage_row(const uint8_t* blk, int r, float* v) {
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const uint4 raw = *reinterpret_cast<const uint4*>(blk + r * 64 + (((q ^ (r >> 1)) & 3) << 4));
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&raw);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 f = __bfloat1622float2(h[e]);
      v[8 * q + 2 * e] = f.x;
      v[8 * q + 2 * e + 1] = f.y;
    }
  }
}

// Byte offset of element (r, c) in a 32 x 32 bf16 block with 64-byte rows under the
// 64-byte swizzle: the 16-byte chunk index is XORed with bits 1..2 of the row.
__device__ __forceinline__ uint32_t swz64(int r, int c) {
  return (uint32_t)(r * 64 + ((((c >> 3) ^ (r >> 1)) & 3) << 4) + (c & 7) * 2);
}

// Thread `r` writes its 32 values as row r of the block (4 x 16-byte stores).
__device__ __forceinline__ void stage_row(uint8_t* blk, int r, const float* v) {
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    uint4 raw;
    __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&raw);
#pragma unroll
    for (int e = 0; e < 4; ++e) h[e] = __floats2bfloat162_rn(v[8 * q + 2 * e], v[8 * q + 2 * e + 1]);
    *reinterpret_cast<uint4*>(blk + r * 64 + (((q ^ (r >> 1)) & 3) << 4)) = raw;
  }
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

struct TcNoApply {
  int unused;
};

// Weight update of one 32-column chunk of a fused epilogue (see TcApply).  xv holds
// X_K in fp32; O is its bf16 rounding, as the workspace copy would hold it.  All 32
// weight loads of the chunk are issued before any store.
// New weight of one entry: fl32(W - lrs*O), then weight decay where it applies.
__device__ __forceinline__ float apply_one(float w0, float o, float lrs, float lrwd, bool cautious) {
  float wn = __fsub_rn(w0, __fmul_rn(lrs, o));
  const bool agree = (o >= 0.f && w0 >= 0.f) || (o <= 0.f && w0 <= 0.f);
  if (lrwd != 0.f && (!cautious || agree)) wn = __fsub_rn(wn, __fmul_rn(lrwd, w0));
  return wn;
}

template <typename WT>
__device__ __forceinline__ void fused_apply_chunk_t(WT* w, float lrs, float lrwd, bool cautious, bool transposed,
                                                    bool vec, int s, int L, int row, int col0, float* o) {
  float wv[32];
  // O = bf16(X_K), in place
#pragma unroll
  for (int j = 0; j < 32; ++j) o[j] = __bfloat162float(__float2bfloat16_rn(o[j]));
  if (!transposed && vec && col0 + 32 <= L) {
    // W is s x L: this thread's 32 consecutive entries of row `row`
    WT* p = w + (size_t)row * L + col0;
    if constexpr (sizeof(WT) == 2) {
      load_bf16x32(reinterpret_cast<const __nv_bfloat16*>(p), wv);
    } else {
      const float4* p4 = reinterpret_cast<const float4*>(p);
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        const float4 v = p4[q];
        wv[4 * q] = v.x; wv[4 * q + 1] = v.y; wv[4 * q + 2] = v.z; wv[4 * q + 3] = v.w;
      }
    }
    if (lrwd == 0.f) {
#pragma unroll
      for (int j = 0; j < 32; ++j) wv[j] = __fsub_rn(wv[j], __fmul_rn(lrs, o[j]));
    } else {
#pragma unroll
      for (int j = 0; j < 32; ++j) wv[j] = apply_one(wv[j], o[j], lrs, lrwd, cautious);
    }
    if constexpr (sizeof(WT) == 2) {
      store_bf16x32(reinterpret_cast<__nv_bfloat16*>(p), wv);
    } else {
      float4* p4 = reinterpret_cast<float4*>(p);
#pragma unroll
      for (int q = 0; q < 8; ++q) p4[q] = make_float4(wv[4 * q], wv[4 * q + 1], wv[4 * q + 2], wv[4 * q + 3]);
    }
    return;
  }
  // element-wise: wide rows that are not 16-byte aligned or end inside the chunk, and tall
  // matrices (W is L x s, entry (col0 + j, row); a warp covers 32 consecutive rows, so
  // every access below is a coalesced 32-element run across the warp)
  WT* p0 = transposed ? w + (size_t)col0 * s + row : w + (size_t)row * L + col0;
  const size_t stride = transposed ? (size_t)s : 1;
#pragma unroll
  for (int j = 0; j < 32; ++j) {
    float x = 0.f;
    if (col0 + j < L) {
      if constexpr (sizeof(WT) == 2) x = __bfloat162float(p0[j * stride]);
      else x = p0[j * stride];
    }
    wv[j] = x;
  }
  if (lrwd == 0.f) {
#pragma unroll
    for (int j = 0; j < 32; ++j) wv[j] = __fsub_rn(wv[j], __fmul_rn(lrs, o[j]));
  } else {
#pragma unroll
    for (int j = 0; j < 32; ++j) wv[j] = apply_one(wv[j], o[j], lrs, lrwd, cautious);
  }
#pragma unroll
  for (int j = 0; j < 32; ++j) {
    if (col0 + j < L) {
      const float r = wv[j];
      if constexpr (sizeof(WT) == 2) p0[j * stride] = __float2bfloat16_rn(r);
      else p0[j * stride] = r;
    }
  }
}

// xv: X_K of the chunk in fp32, overwritten with O = bf16(X_K).
__device__ __forceinline__ void fused_apply_chunk(const TcApply& ap, int s, int L, int row, int col0, float* xv) {
  const bool tr = ap.flags & kApplyTransposed, vec = ap.flags & kApplyVec, ca = ap.flags & kApplyCautious;
  if (ap.flags & kApplyBf16)
    fused_apply_chunk_t(reinterpret_cast<__nv_bfloat16*>(ap.w), ap.lrs, ap.lrwd, ca, tr, vec, s, L, row, col0, xv);
  else
    fused_apply_chunk_t(reinterpret_cast<float*>(ap.w), ap.lrs, ap.lrwd, ca, tr, vec, s, L, row, col0, xv);
}

template <int PHASE, typename AppT>
__global__ void __launch_bounds__(kThreadsTc, 1)
tc_kernel(const __grid_constant__ TcParams p, const __grid_constant__ AppT app) {
  constexpr bool kFuse = sizeof(AppT) > sizeof(TcNoApply);
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  constexpr int kStages = stages_for(PHASE);
  constexpr uint32_t kWarpStage = warp_stage_bytes_for(PHASE);
  constexpr uint32_t kOutPart = out_bytes_for(PHASE);
  constexpr bool kHasIn = in_bytes_for(PHASE) > 0;
  uint8_t* out_stage = smem + kStages * kStageBytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kStages * kStageBytes + kEpiWarps * kWarpStage);
  uint64_t* empty = full + kStages;
  uint64_t* tfull = empty + kStages;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint64_t* in_bar = drain + 1;  // [kEpiWarps][2] input-block barriers
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(in_bar + 2 * kEpiWarps);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank();
  const int cluster = blockIdx.x >> 1;
  const int n_clusters = gridDim.x >> 1;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], 2 * kEpiWarps);  // every epilogue warp of both CTAs
    }
    mbar_init(drain, 1);
    for (int b = 0; b < 2 * kEpiWarps; ++b) mbar_init(&in_bar[b], 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                 "r"(kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  cluster_sync_all();  // both CTAs' barriers and TMEM are ready before any remote use
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const uint32_t peer_abort = peer_addr(smem_u32((const void*)abort_flag), rank ^ 1u);

  constexpr bool kSyrk = (PHASE != kPhaseUpdate);
  bool aborted = false;

  if (warp == 0) {
    // ------------------------------------------------------------------ TMA producer (both CTAs)
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int t = cluster; t < p.n_tiles && ok; t += n_clusters) {
        const TcTile tile = p.tiles[t];
        const TcGroup& g = p.g[tile.group];
        const int K = (PHASE == kPhaseGram) ? g.L : g.s;
        const int nk = (K + kBK - 1) / kBK;
        const CUtensorMap* ma = &p.map_a[tile.group];
        const CUtensorMap* mb = &p.map_b[tile.group];
        const int row_a = tile.bi * kTile + (int)rank * kHalf;
        const int col_b = tile.bj * kTile + (int)rank * kHalf;
        for (int kb = 0; kb < nk; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1u, abort_flag)) { ok = false; break; }
          if (rank == 0) mbar_arrive_expect_tx(&full[stage], kPairTxBytes);
          const uint32_t a_dst = smem_u32(smem + stage * kStageBytes);
          const uint32_t b_dst = a_dst + kABytes;
          const uint32_t bar = peer_addr(smem_u32(&full[stage]), 0);
          const int k0 = kb * kBK;
          tma_load_3d_pair(a_dst, ma, bar, k0, row_a, tile.mat);
          if (kSyrk) {
            tma_load_3d_pair(b_dst, ma, bar, k0, col_b, tile.mat);
          } else {
#pragma unroll
            for (int q = 0; q < kHalf / 64; ++q)
              tma_load_3d_pair(b_dst + q * (64 * kBK * 2), mb, bar, col_b + 64 * q, k0, tile.mat);
          }
          if (++stage == kStages) { stage = 0; phase ^= 1u; }
        }
      }
      if (!ok || *abort_flag) {
        aborted = true;
        atomicExch(p.status, kDevTimeout);
        *abort_flag = 1;
        remote_store_flag(peer_abort, 1);
        spin_ns(kAbortGraceNs);  // copies already issued land within microseconds
      } else if (rank == 0) {
        // every copy armed on this barrier set has landed (all were consumed in order)
        for (int s = 0; s < kStages; ++s) {
          const uint32_t par = (s < stage) ? phase : (phase ^ 1u);
          (void)mbar_wait(&full[s], par, nullptr);
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer (leader CTA)
    if (lane == 0 && rank == 0) {
      constexpr uint32_t idesc = make_idesc(!kSyrk);
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      for (int t = cluster; t < p.n_tiles && ok; t += n_clusters) {
        const TcTile tile = p.tiles[t];
        const TcGroup& g = p.g[tile.group];
        const int K = (PHASE == kPhaseGram) ? g.L : g.s;
        const int nk = (K + kBK - 1) / kBK;
        if (!mbar_wait(&tempty[acc], acc_phase ^ 1u, abort_flag)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + (uint32_t)(acc * kTile);
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
            umma_pair_bf16(d_tmem, ad, bd, idesc, (kb > 0 || k > 0) ? 1u : 0u);
          }
          umma_commit_both(&empty[stage]);
          if (++stage == kStages) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        umma_commit_both(&tfull[acc]);
        if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
      }
      if (!ok) {
        aborted = true;
        atomicExch(p.status, kDevTimeout);
        *abort_flag = 1;
        remote_store_flag(peer_abort, 1);
      }
      // every MMA issued by this thread completes before TMEM is released
      umma_commit_local(drain);
      (void)mbar_wait(drain, 0, nullptr);
    }
  } else {
    // ------------------------------------------------------------------ epilogue (both CTAs)
    const int quad = warp & 3;                       // TMEM lane quadrant this warp may access
    const int ew = warp - 2;                         // epilogue warp index
    uint8_t* my_out = out_stage + ew * kWarpStage;   // [2] output buffers
    uint8_t* my_in = my_out + kOutPart;              // [2] input buffers (Poly / Update)
    uint64_t* my_bar = in_bar + 2 * ew;
    constexpr int kChunks = kTile / 32 * 4 / kEpiWarps;
    const int c_begin = (ew / 4) * kChunks;          // first 32-column chunk of this warp
    const uint32_t leader_tempty0 = peer_addr(smem_u32(&tempty[0]), 0);

    // Valid chunks of a tile for this warp form the range [lo, hi): columns inside the
    // result, and for Gram/Poly not strictly below the diagonal.
    auto chunk_range = [&](const TcTile& tl, int& lo, int& hi) {
      const TcGroup& gg = p.g[tl.group];
      const int r0 = tl.bi * kTile + (int)rank * kHalf + 32 * quad;
      lo = c_begin;
      hi = c_begin + kChunks;
      if (r0 >= gg.s) { hi = lo; return; }
      const int lim = kSyrk ? gg.s : gg.L;
      while (hi > lo && tl.bj * kTile + 32 * (hi - 1) >= lim) --hi;
      if (kSyrk)
        while (lo < hi && tl.bj * kTile + 32 * lo + 31 < r0) ++lo;
    };
    // Input prefetch cursor over (tile, chunk) pairs of this warp, in processing order:
    // (pf_t, pf_c) is the next block to request; pf_t >= n_tiles when none is left.
    int pf_t = p.n_tiles, pf_c = 0, pf_hi = 0;
    uint32_t n_req = 0;  // input blocks requested so far (buffer = n & 1)
    auto pf_first_from = [&](int t0) {  // first tile at or after t0 that has chunks for this warp
      pf_t = t0;
      while (pf_t < p.n_tiles) {
        int lo, hi;
        chunk_range(p.tiles[pf_t], lo, hi);
        if (lo < hi) { pf_c = lo; pf_hi = hi; return; }
        pf_t += n_clusters;
      }
    };
    auto pf_issue = [&]() {  // lane 0 requests the cursor's block; every lane advances the cursor
      if (pf_t >= p.n_tiles) return;
      const TcTile tl = p.tiles[pf_t];
      const int b = n_req & 1;
      if (lane == 0) {
        fence_async_smem();
        mbar_arrive_expect_tx(&my_bar[b], kOutBlockBytes);
        tma_load_3d_local(smem_u32(my_in + b * kOutBlockBytes), &p.map_in[tl.group], &my_bar[b],
                          tl.bj * kTile + 32 * pf_c, tl.bi * kTile + (int)rank * kHalf + 32 * quad, tl.mat);
      }
      ++n_req;
      if (++pf_c >= pf_hi) pf_first_from(pf_t + n_clusters);
    };
    if constexpr (kHasIn) {
      pf_first_from(cluster);
      pf_issue();
    }
    uint32_t n_used = 0;  // input blocks consumed so far
    uint32_t n_out = 0;   // staged output blocks so far (buffer parity)

    int acc = 0;
    uint32_t acc_phase = 0;
    bool ok = true;
    for (int t = cluster; t < p.n_tiles && ok; t += n_clusters) {
      const TcTile tile = p.tiles[t];
      const TcGroup& g = p.g[tile.group];
      if (!mbar_wait(&tfull[acc], acc_phase, abort_flag)) { ok = false; break; }
      tc_fence_after();

      const int s = g.s;
      const int row0 = tile.bi * kTile + (int)rank * kHalf + 32 * quad;  // first row of this warp
      const int row = row0 + lane;
      const float sc = p.first_iter ? p.scale[g.gid_base + tile.mat] : 1.f;
      const uint32_t tbase = tmem_base + ((uint32_t)(32 * quad) << 16) + (uint32_t)(acc * kTile);
      int c_lo, c_hi;
      chunk_range(tile, c_lo, c_hi);

      for (int c = c_lo; c < c_hi; ++c) {
        const int col0 = tile.bj * kTile + 32 * c;
        float in_v[32];
        if constexpr (kHasIn) {
          pf_issue();  // next block (this or a later tile) into the other buffer
        }
        float v[32];
        tmem_ld32(tbase + (uint32_t)(32 * c), v);
        if constexpr (kHasIn) {
          const int b = n_used & 1;
          if (!mbar_wait(&my_bar[b], (n_used >> 1) & 1u, abort_flag)) { ok = false; break; }
          unstage_row(my_in + b * kOutBlockBytes, lane, in_v);
          ++n_used;
          __syncwarp();  // every lane has read the block before its buffer is refilled
        }
        if (PHASE == kPhaseGram) {
          const float alpha = sc * sc;
#pragma unroll
          for (int j = 0; j < 32; ++j) v[j] *= alpha;
        } else if (PHASE == kPhasePoly) {
#pragma unroll
          for (int j = 0; j < 32; ++j) v[j] = fmaf(p.cb, in_v[j], p.cc * v[j]);
        } else {
          const float alpha = p.ca * sc;
#pragma unroll
          for (int j = 0; j < 32; ++j) v[j] = fmaf(alpha, in_v[j], sc * v[j]);
          if constexpr (kFuse) {
            if (row < s)
              fused_apply_chunk(reinterpret_cast<const TcApplyTable&>(app).m[g.gid_base + tile.mat -
                                                                              reinterpret_cast<const TcApplyTable&>(app).base],
                                s, g.L, row, col0, v);
            continue;
          }
          uint8_t* blk = my_out + (n_out & 1) * kOutBlockBytes;
          if (lane == 0) bulk_wait_read_1();
          __syncwarp();
          stage_row(blk, lane, v);
          fence_async_smem();
          __syncwarp();
          if (lane == 0) {
            tma_store_3d(&p.map_out[tile.group], smem_u32(blk), col0, row0, tile.mat);
            bulk_commit();
          }
          ++n_out;
          continue;
        }
        // symmetric store: the block (row0.., col0..) and its mirror (col0.., row0..),
        // both built from the upper-triangle values so the result is exactly symmetric
        uint8_t* blk = my_out + (n_out & 1) * 2 * kOutBlockBytes;
        if (lane == 0) bulk_wait_read_1();
        __syncwarp();
        const bool upper = col0 >= row0 + 32;
        if (upper) {
          stage_row(blk, lane, v);
          uint8_t* mir = blk + kOutBlockBytes;
#pragma unroll
          for (int j = 0; j < 32; ++j)
            *reinterpret_cast<__nv_bfloat16*>(mir + swz64(j, lane)) = __float2bfloat16_rn(v[j]);
        } else {
          // diagonal block (col0 == row0): element (lane, j) for j >= lane, mirrored below
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            if (j >= lane) {
              const __nv_bfloat16 bv = __float2bfloat16_rn(v[j]);
              *reinterpret_cast<__nv_bfloat16*>(blk + swz64(lane, j)) = bv;
              if (j > lane) *reinterpret_cast<__nv_bfloat16*>(blk + swz64(j, lane)) = bv;
            }
          }
        }
        fence_async_smem();
        __syncwarp();
        if (lane == 0) {
          tma_store_3d(&p.map_out[tile.group], smem_u32(blk), col0, row0, tile.mat);
          if (upper) tma_store_3d(&p.map_out[tile.group], smem_u32(blk + kOutBlockBytes), row0, col0, tile.mat);
          bulk_commit();
        }
        ++n_out;
      }
      if (!ok) break;
      tc_fence_before();
      __syncwarp();
      if (lane == 0) remote_arrive(leader_tempty0 + (uint32_t)(acc * sizeof(uint64_t)));
      if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
    }
    if (lane == 0) bulk_wait_all();  // this warp's stores are complete and its staging is free
    if (!ok && lane == 0) {
      aborted = true;
      atomicExch(p.status, kDevTimeout);
      *abort_flag = 1;
      remote_store_flag(peer_abort, 1);
    }
    if constexpr (kHasIn) {
      // input blocks requested but not consumed (after an abort) land before exit
      while (n_used < n_req) {
        (void)mbar_wait(&my_bar[n_used & 1], (n_used >> 1) & 1u, nullptr);
        ++n_used;
      }
    }
  }
  (void)aborted;

  // Both CTAs wait here: the leader's MMAs (which write the peer's TMEM) and every copy
  // are complete before either CTA releases TMEM or exits.
  __syncwarp();
  tc_fence_before();
  cluster_sync_all();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(kTmemCols)
                 : "memory");
  }
}

// ---------------------------------------------------------------------- persistent kernel
//
// The whole Newton-Schulz loop of one chunk of shape groups in one launch (see
// TcPersistParams).  Roles as in tc_kernel; what changes:
//   - work items come from a global counter: the leader's producer takes the next item
//     (atomicAdd), writes it into an 8-slot ring in both CTAs' shared memory and
//     arrives on the slot's "full" barrier in both CTAs; every consumer (the peer's
//     producer, the MMA issuer, the eight epilogue warps) reads the slot and arrives on
//     the leader's "empty" barrier.  Items are handed out in order, so the lowest
//     unfinished item always belongs to a running cluster and has no unfinished
//     dependency: the launch makes progress whatever number of clusters is resident.
//   - before loading an item's operands, each producer waits (acquire, bounded) until
//     the item's matrix has finished the previous phase; the epilogue's lane 0 does
//     the same before its input-block loads.  After its TMA stores of a tile have
//     completed, each epilogue warp adds 1 (release) to the matrix's counter.
//   - the phase is a run-time property of the item: operands, descriptors, epilogue
//     arithmetic and output maps are chosen per item; 4 stages for every phase.
//   - eight epilogue warps, two per TMEM lane quadrant, each with half of the tile's
//     columns, so two warps per scheduler hide each other's latencies; one output
//     staging buffer per warp (the other warp on its scheduler covers the wait for the
//     previous store to leave it).
//   - the epilogue requests all input blocks of its part of a tile (X for Update, A for
//     Poly; 4 blocks of 32 x 32) as soon as it takes the item, and publishes the
//     previous tile's completion only after that, so one memory latency per tile is
//     exposed instead of one per chunk.  When the item's inputs are not ready yet, the
//     previous tile's completion is published first and the wait follows, so no warp
//     ever waits with an unpublished tile.
// Every wait is bounded; on expiry, or when another CTA has already recorded a
// time-out in the status word, the kernel records kDevTimeout, lets its own copies
// and MMAs drain, frees TMEM and returns.
constexpr int kPStages = 4;
constexpr int kPEpi = 8;                                  // epilogue warps: two per TMEM lane quadrant
constexpr int kPThreads = 64 + 32 * kPEpi;
constexpr int kSched = 8;  // slots of the work-item ring
constexpr int kPChunks = kTile / 32 * 4 / kPEpi;          // 32-column chunks per epilogue warp and tile
constexpr uint32_t kPOutPart = 2u * kOutBlockBytes;       // one block + its mirror
constexpr uint32_t kPInPart = kPChunks * kOutBlockBytes;  // every input block of the warp's tile part
constexpr uint32_t kPWarpStage = kPOutPart + kPInPart;
constexpr uint32_t kPBarrierBytes = 512;
constexpr uint32_t kPSmemBytes = kPStages * kStageBytes + kPEpi * kPWarpStage + kPBarrierBytes + 1024;
static_assert(kPSmemBytes <= 232448, "shared memory per CTA (persistent kernel)");
constexpr unsigned kArrivalsPerTile = 2 * kPEpi;
// ring consumers arriving on the leader's empty barrier: the leader's MMA issuer and
// epilogue warps, the peer's producer and epilogue warps
constexpr uint32_t kSchedConsumers = 1 + kPEpi + 1 + kPEpi;

__device__ __forceinline__ unsigned ld_acquire_gpu(const unsigned* p) {
  unsigned v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void red_release_gpu_add(unsigned* p, unsigned v) {
  asm volatile("red.release.gpu.global.add.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
// Every committed store group of this thread has finished reading shared memory.
__device__ __forceinline__ void bulk_wait_read_0() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
// Orders this thread's generic-proxy global accesses with its async-proxy (TMA) ones.
__device__ __forceinline__ void fence_async_global() { asm volatile("fence.proxy.async.global;" ::: "memory"); }

__device__ __forceinline__ bool mbar_try_wait_cluster(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}\n"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Bounded wait with cluster-scope acquire (barriers that the other CTA arrives on and
// whose arrival publishes shared-memory data).
__device__ __noinline__ bool mbar_wait_cluster(uint64_t* bar, uint32_t parity, volatile int* abort_flag) {
  if (mbar_try_wait_cluster(bar, parity)) return true;
  const uint64_t t0 = global_timer();
  uint32_t n = 0;
  while (true) {
    if (mbar_try_wait_cluster(bar, parity)) return true;
    if ((++n & 63u) == 0) {
      if (*abort_flag) return false;
      if (global_timer() - t0 > kWaitLimitNs) return false;
    }
  }
}

__device__ __forceinline__ void mbar_arrive_local(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void st_cluster_u32(uint32_t cluster_addr, uint32_t v) {
  asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(cluster_addr), "r"(v) : "memory");
}

// Counter value at which the item's matrix has finished every earlier phase.
__device__ __forceinline__ unsigned dep_target(const TcGroup& g, int k, int ph) {
  const int nb = (g.s + kTile - 1) / kTile, nbl = (g.L + kTile - 1) / kTile;
  const unsigned n_s = (unsigned)(nb * (nb + 1) / 2), n_u = (unsigned)(nb * nbl);
  const unsigned before = (unsigned)k * (2u * n_s + n_u) + (ph >= kPhasePoly ? n_s : 0u) +
                          (ph >= kPhaseUpdate ? n_s : 0u);
  return kArrivalsPerTile * before;
}

// Waits until *ctr >= target (acquire at GPU scope), bounded; false on time-out, on
// this CTA's abort flag, or when the status word already records a failure.
__device__ __noinline__ bool wait_count(const unsigned* ctr, unsigned target, const int* status,
                                        volatile int* abort_flag, unsigned long long limit_ns = kWaitLimitNs) {
  if (ld_acquire_gpu(ctr) >= target) return true;
  const uint64_t t0 = global_timer();
  uint32_t n = 0;
  while (true) {
    __nanosleep(64);
    if (ld_acquire_gpu(ctr) >= target) return true;
    if ((++n & 15u) == 0) {
      if (*abort_flag) return false;
      if (*reinterpret_cast<const volatile int*>(status) != kDevOk) return false;
      if (global_timer() - t0 > limit_ns) return false;
    }
  }
}

// Dependency of one item: its matrix's counter must reach the returned value (see
// TcPersistParams::stall_ns for the self-test form, whose count is never reached).
__device__ __forceinline__ unsigned item_target(const TcPersistParams& p, const TcGroup& g, int gid, int k, int ph) {
  if (p.stall_ns != 0 && gid == 0 && k == 0 && ph == kPhasePoly) return 0xffffffffu;
  return dep_target(g, k, ph);
}
__device__ __forceinline__ bool item_ready(const TcPersistParams& p, const TcGroup& g, int gid, int k, int ph) {
  return ld_acquire_gpu(p.done + gid) >= item_target(p, g, gid, k, ph);
}
__device__ __forceinline__ bool wait_item_deps(const TcPersistParams& p, const TcGroup& g, int gid, int k, int ph,
                                               volatile int* abort_flag) {
  const unsigned target = item_target(p, g, gid, k, ph);
  const bool stall = p.stall_ns != 0 && target == 0xffffffffu;
  return wait_count(p.done + gid, target, p.status, abort_flag, stall ? p.stall_ns : kWaitLimitNs);
}

// One work item: step k, phase, tile.
struct PItem {
  int k, ph;
  TcTile tile;
};

__device__ __forceinline__ PItem decode_item(const TcPersistParams& p, int item) {
  const int per_iter = 2 * p.n_syrk + p.n_upd;
  PItem it;
  it.k = item / per_iter;
  int r = item - it.k * per_iter;
  if (r < p.n_syrk) {
    it.ph = kPhaseGram;
    it.tile = p.tiles_syrk[r];
  } else if (r < 2 * p.n_syrk) {
    it.ph = kPhasePoly;
    it.tile = p.tiles_syrk[r - p.n_syrk];
  } else {
    it.ph = kPhaseUpdate;
    it.tile = p.tiles_upd[r - 2 * p.n_syrk];
  }
  return it;
}

template <typename AppT>
__global__ void __launch_bounds__(kPThreads, 1)
tc_persistent_kernel(const __grid_constant__ TcPersistParams p, const __grid_constant__ AppT app) {
  constexpr bool kFuse = sizeof(AppT) > sizeof(TcNoApply);
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* out_stage = smem + kPStages * kStageBytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kPStages * kStageBytes + kPEpi * kPWarpStage);
  uint64_t* empty = full + kPStages;
  uint64_t* tfull = empty + kPStages;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint64_t* in_bar = drain + 1;               // [kPEpi] input-block barriers
  uint64_t* sched_full = in_bar + kPEpi;
  uint64_t* sched_empty = sched_full + kSched;  // used in the leader CTA only
  int* sched_item = reinterpret_cast<int*>(sched_empty + kSched);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sched_item + kSched);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank();
  const int n_items = p.ns_steps * (2 * p.n_syrk + p.n_upd);

  if (threadIdx.x == 0) {
    for (int s = 0; s < kPStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], 2 * kPEpi);
    }
    mbar_init(drain, 1);
    for (int b = 0; b < kPEpi; ++b) mbar_init(&in_bar[b], 1);
    for (int q = 0; q < kSched; ++q) {
      mbar_init(&sched_full[q], 1);
      mbar_init(&sched_empty[q], kSchedConsumers);
    }
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                 "r"(kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  cluster_sync_all();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const uint32_t peer_abort = peer_addr(smem_u32((const void*)abort_flag), rank ^ 1u);
  // the leader's empty barriers, as seen from this CTA (consumers arrive there)
  const uint32_t leader_sched_empty = peer_addr(smem_u32(&sched_empty[0]), 0);

  auto give_up = [&]() {
    atomicExch(p.status, kDevTimeout);
    *abort_flag = 1;
    remote_store_flag(peer_abort, 1);
  };
  // Ring consumer: waits for slot j's item, reads it and releases the slot.
  auto take_item = [&](uint32_t j, int& item, bool arrive) -> bool {
    const uint32_t slot = j % kSched, par = (j / kSched) & 1u;
    if (!mbar_wait_cluster(&sched_full[slot], par, abort_flag)) return false;
    item = *reinterpret_cast<volatile int*>(&sched_item[slot]);
    if (arrive) remote_arrive(leader_sched_empty + slot * (uint32_t)sizeof(uint64_t));
    return true;
  };

  if (warp == 0) {
    // ------------------------------------------------------------------ producer (both CTAs)
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      // Item j of this cluster: the leader takes it from the global counter and publishes
      // it; the peer reads it from the ring.
      auto next_item = [&](uint32_t j, int& item) -> bool {
        if (rank != 0) return take_item(j, item, true);
        const uint32_t slot = j % kSched, par = (j / kSched) & 1u;
        if (!mbar_wait_cluster(&sched_empty[slot], par ^ 1u, abort_flag)) return false;
        item = (int)atomicAdd(p.queue, 1u);
        if (item >= n_items) item = -1;
        sched_item[slot] = item;
        st_cluster_u32(peer_addr(smem_u32(&sched_item[slot]), 1), (uint32_t)item);
        mbar_arrive_local(&sched_full[slot]);
        remote_arrive(peer_addr(smem_u32(&sched_full[slot]), 1));
        return true;
      };
      // The next item is taken as soon as the current one's inputs are complete, and its
      // own inputs are polled while the current one's loads wait for free stages, so its
      // first loads go out as soon as a stage frees.
      int cur = -1;
      bool cur_ready = false;  // cur's inputs already seen complete (acquire done)
      if (!next_item(0, cur)) ok = false;
      for (uint32_t j = 0; ok && cur >= 0; ++j) {
        const PItem it = decode_item(p, cur);
        const TcGroup& g = p.g[it.tile.group];
        if (!cur_ready && !wait_item_deps(p, g, g.gid_base + it.tile.mat, it.k, it.ph, abort_flag)) {
          ok = false;
          break;
        }
        fence_async_global();
        int nxt = -1;
        if (!next_item(j + 1, nxt)) { ok = false; break; }
        bool nxt_ready = false;
        const unsigned* nxt_ctr = nullptr;
        unsigned nxt_target = 0;
        if (nxt >= 0) {
          const PItem itn = decode_item(p, nxt);
          const TcGroup& gn = p.g[itn.tile.group];
          nxt_ctr = p.done + gn.gid_base + itn.tile.mat;
          nxt_target = item_target(p, gn, gn.gid_base + itn.tile.mat, itn.k, itn.ph);
        }
        const bool syrk = it.ph != kPhaseUpdate;
        const int K = (it.ph == kPhaseGram) ? g.L : g.s;
        const int nk = (K + kBK - 1) / kBK;
        const int par_x = it.k & 1;
        const CUtensorMap* ma = it.ph == kPhaseGram ? &p.xk[it.tile.group][par_x]
                                : it.ph == kPhasePoly ? &p.gram[it.tile.group] : &p.poly[it.tile.group];
        const CUtensorMap* mb = &p.xmn[it.tile.group][par_x];
        const int row_a = it.tile.bi * kTile + (int)rank * kHalf;
        const int col_b = it.tile.bj * kTile + (int)rank * kHalf;
        for (int kb = 0; kb < nk; ++kb) {
          if (!mbar_try_wait(&empty[stage], phase ^ 1u)) {
            if (nxt_ctr != nullptr && !nxt_ready) nxt_ready = ld_acquire_gpu(nxt_ctr) >= nxt_target;
            if (!mbar_wait(&empty[stage], phase ^ 1u, abort_flag)) { ok = false; break; }
          }
          if (rank == 0) mbar_arrive_expect_tx(&full[stage], kPairTxBytes);
          const uint32_t a_dst = smem_u32(smem + stage * kStageBytes);
          const uint32_t b_dst = a_dst + kABytes;
          const uint32_t bar = peer_addr(smem_u32(&full[stage]), 0);
          const int k0 = kb * kBK;
          tma_load_3d_pair(a_dst, ma, bar, k0, row_a, it.tile.mat);
          if (syrk) {
            tma_load_3d_pair(b_dst, ma, bar, k0, col_b, it.tile.mat);
          } else {
#pragma unroll
            for (int q = 0; q < kHalf / 64; ++q)
              tma_load_3d_pair(b_dst + q * (64 * kBK * 2), mb, bar, col_b + 64 * q, k0, it.tile.mat);
          }
          if (++stage == kPStages) { stage = 0; phase ^= 1u; }
        }
        cur = nxt;
        cur_ready = nxt_ready;
      }
      if (!ok || *abort_flag) {
        give_up();
        spin_ns(kAbortGraceNs);  // copies already issued land within microseconds
      } else if (rank == 0) {
        for (int s = 0; s < kPStages; ++s) {
          const uint32_t par = (s < stage) ? phase : (phase ^ 1u);
          (void)mbar_wait(&full[s], par, nullptr);
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer (leader CTA)
    if (lane == 0 && rank == 0) {
      constexpr uint32_t idesc_k = make_idesc(false), idesc_mn = make_idesc(true);
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      for (uint32_t j = 0; ok; ++j) {
        int item;
        if (!take_item(j, item, true)) { ok = false; break; }
        if (item < 0) break;
        const PItem it = decode_item(p, item);
        const TcGroup& g = p.g[it.tile.group];
        const bool syrk = it.ph != kPhaseUpdate;
        const int K = (it.ph == kPhaseGram) ? g.L : g.s;
        const int nk = (K + kBK - 1) / kBK;
        if (!mbar_wait(&tempty[acc], acc_phase ^ 1u, abort_flag)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + (uint32_t)(acc * kTile);
        const uint32_t idesc = syrk ? idesc_k : idesc_mn;
        for (int kb = 0; kb < nk; ++kb) {
          if (!mbar_wait(&full[stage], phase, abort_flag)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a_addr = smem_u32(smem + stage * kStageBytes);
          const uint32_t b_addr = a_addr + kABytes;
#pragma unroll
          for (int k = 0; k < kBK / 16; ++k) {
            const uint64_t ad = sdesc(a_addr + k * 32, 16, 1024);
            const uint64_t bd = syrk ? sdesc(b_addr + k * 32, 16, 1024) : sdesc(b_addr + k * 2048, 64 * kBK * 2, 1024);
            umma_pair_bf16(d_tmem, ad, bd, idesc, (kb > 0 || k > 0) ? 1u : 0u);
          }
          umma_commit_both(&empty[stage]);
          if (++stage == kPStages) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        umma_commit_both(&tfull[acc]);
        if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
      }
      if (!ok) give_up();
      umma_commit_local(drain);
      (void)mbar_wait(drain, 0, nullptr);
    }
  } else {
    // ------------------------------------------------------------------ epilogue (both CTAs)
    const int quad = warp & 3;
    const int ew = warp - 2;
    uint8_t* my_out = out_stage + ew * kPWarpStage;
    uint8_t* my_in = my_out + kPOutPart;   // kPChunks input blocks
    uint64_t* my_bar = in_bar + ew;
    const int c_begin = (ew / 4) * kPChunks;
    const uint32_t leader_tempty0 = peer_addr(smem_u32(&tempty[0]), 0);
    uint32_t in_phase = 0;     // parity of my_bar
    bool in_pending = false;   // input blocks requested and not yet waited for
    int pend_gid = -1;         // matrix of this warp's last tile, whose completion is unpublished
    int acc = 0;
    uint32_t acc_phase = 0;
    bool ok = true;
    // lane 0: the previous tile's stores have landed -> add 1 to its matrix's counter
    auto publish = [&]() {
      if (pend_gid >= 0 && lane == 0) {
        bulk_wait_all();
        fence_async_global();
        red_release_gpu_add(p.done + pend_gid, 1u);
      }
      pend_gid = -1;
    };
    for (uint32_t j = 0; ok; ++j) {
      int item = -1;
      bool got = true;
      if (lane == 0) got = take_item(j, item, true);
      got = __shfl_sync(0xffffffffu, got ? 1 : 0, 0) != 0;
      item = __shfl_sync(0xffffffffu, item, 0);
      if (!got) { ok = false; break; }
      if (item < 0) break;
      const PItem it = decode_item(p, item);
      const TcGroup& g = p.g[it.tile.group];
      const int grp = it.tile.group;
      const bool syrk = it.ph != kPhaseUpdate;
      const bool last_update = it.ph == kPhaseUpdate && it.k == p.ns_steps - 1;
      const int par_x = it.k & 1;
      const int gid = g.gid_base + it.tile.mat;
      const int row0 = it.tile.bi * kTile + (int)rank * kHalf + 32 * quad;
      const int row = row0 + lane;
      // valid 32-column chunks of this warp: inside the result and, for Gram/Poly, not
      // strictly below the diagonal
      int lo = c_begin, hi = c_begin + kPChunks;
      if (row0 >= g.s) {
        hi = lo;
      } else {
        const int lim = syrk ? g.s : g.L;
        while (hi > lo && it.tile.bj * kTile + 32 * (hi - 1) >= lim) --hi;
        if (syrk)
          while (lo < hi && it.tile.bj * kTile + 32 * lo + 31 < row0) ++lo;
      }
      const bool has_in = it.ph != kPhaseGram && lo < hi;
      const CUtensorMap* map_in = it.ph == kPhasePoly ? &p.gram_out[grp] : &p.xout[grp][par_x];
      const CUtensorMap* map_out = it.ph == kPhaseGram ? &p.gram_out[grp]
                                   : it.ph == kPhasePoly ? &p.poly_out[grp] : &p.xout[grp][par_x ^ 1];
      auto request_all = [&]() {  // lane 0: every input block of chunks [lo, hi), one barrier
        fence_async_smem();
        mbar_arrive_expect_tx(my_bar, (uint32_t)(hi - lo) * kOutBlockBytes);
        for (int c = lo; c < hi; ++c)
          tma_load_3d_local(smem_u32(my_in + (c - c_begin) * kOutBlockBytes), map_in, my_bar,
                            it.tile.bj * kTile + 32 * c, row0, it.tile.mat);
      };
      if (has_in) {
        // inputs already complete: request them before publishing the previous tile, so
        // the two latencies overlap; otherwise publish first, then wait (bounded)
        int issued = 0;
        if (lane == 0 && item_ready(p, g, gid, it.k, it.ph)) {
          fence_async_global();
          request_all();
          issued = 1;
        }
        issued = __shfl_sync(0xffffffffu, issued, 0);
        publish();
        if (!issued) {
          int dep = 1;
          if (lane == 0) {
            dep = wait_item_deps(p, g, gid, it.k, it.ph, abort_flag) ? 1 : 0;
            if (dep) {
              fence_async_global();
              request_all();
            }
          }
          if (__shfl_sync(0xffffffffu, dep, 0) == 0) { ok = false; break; }
        }
        in_pending = true;
      } else {
        publish();
      }
      if (!mbar_wait(&tfull[acc], acc_phase, abort_flag)) { ok = false; break; }
      tc_fence_after();
      if (has_in) {
        if (!mbar_wait(my_bar, in_phase, abort_flag)) { ok = false; break; }
        in_phase ^= 1u;
        in_pending = false;
      }
      const float sc = it.k == 0 ? p.scale[gid] : 1.f;
      const uint32_t tbase = tmem_base + ((uint32_t)(32 * quad) << 16) + (uint32_t)(acc * kTile);
      for (int c = lo; c < hi; ++c) {
        const int col0 = it.tile.bj * kTile + 32 * c;
        float in_v[32];
        float v[32];
        tmem_ld32(tbase + (uint32_t)(32 * c), v);
        if (it.ph == kPhaseGram) {
          const float alpha = sc * sc;
#pragma unroll
          for (int q = 0; q < 32; ++q) v[q] *= alpha;
        } else if (it.ph == kPhasePoly) {
          unstage_row(my_in + (c - c_begin) * kOutBlockBytes, lane, in_v);
          const float cb = p.cb[it.k], cc = p.cc[it.k];
#pragma unroll
          for (int q = 0; q < 32; ++q) v[q] = fmaf(cb, in_v[q], cc * v[q]);
        } else {
          unstage_row(my_in + (c - c_begin) * kOutBlockBytes, lane, in_v);
          const float alpha = p.ca[it.k] * sc;
#pragma unroll
          for (int q = 0; q < 32; ++q) v[q] = fmaf(alpha, in_v[q], sc * v[q]);
        }
        if (!syrk) {
          if constexpr (kFuse) {
            if (last_update) {
              if (row < g.s) {
                const TcApplyTable& at = reinterpret_cast<const TcApplyTable&>(app);
                fused_apply_chunk(at.m[gid - at.base], g.s, g.L, row, col0, v);
              }
              continue;
            }
          }
          uint8_t* blk = my_out;  // single staging buffer: the previous store has read it
          if (lane == 0) bulk_wait_read_0();
          __syncwarp();
          stage_row(blk, lane, v);
          fence_async_smem();
          __syncwarp();
          if (lane == 0) {
            tma_store_3d(map_out, smem_u32(blk), col0, row0, it.tile.mat);
            bulk_commit();
          }
          continue;
        }
        uint8_t* blk = my_out;
        if (lane == 0) bulk_wait_read_0();
        __syncwarp();
        const bool upper = col0 >= row0 + 32;
        if (upper) {
          stage_row(blk, lane, v);
          uint8_t* mir = blk + kOutBlockBytes;
#pragma unroll
          for (int q = 0; q < 32; ++q)
            *reinterpret_cast<__nv_bfloat16*>(mir + swz64(q, lane)) = __float2bfloat16_rn(v[q]);
        } else {
#pragma unroll
          for (int q = 0; q < 32; ++q) {
            if (q >= lane) {
              const __nv_bfloat16 bv = __float2bfloat16_rn(v[q]);
              *reinterpret_cast<__nv_bfloat16*>(blk + swz64(lane, q)) = bv;
              if (q > lane) *reinterpret_cast<__nv_bfloat16*>(blk + swz64(q, lane)) = bv;
            }
          }
        }
        fence_async_smem();
        __syncwarp();
        if (lane == 0) {
          tma_store_3d(map_out, smem_u32(blk), col0, row0, it.tile.mat);
          if (upper) tma_store_3d(map_out, smem_u32(blk + kOutBlockBytes), row0, col0, it.tile.mat);
          bulk_commit();
        }
      }
      tc_fence_before();
      __syncwarp();  // every lane has read its input rows before the buffer is refilled
      if (lane == 0) remote_arrive(leader_tempty0 + (uint32_t)(acc * sizeof(uint64_t)));
      if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
      // the last Update's outputs are read by no later item
      pend_gid = last_update ? -1 : gid;
    }
    if (ok) publish();
    if (lane == 0) bulk_wait_all();
    if (!ok && lane == 0) give_up();
    if (in_pending) (void)mbar_wait(my_bar, in_phase, nullptr);  // requested blocks land before exit
  }

  __syncwarp();
  tc_fence_before();
  cluster_sync_all();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(kTmemCols)
                 : "memory");
  }
}

template <int PHASE, typename AppT>
cudaError_t set_smem_attr() {
  return cudaFuncSetAttribute(tc_kernel<PHASE, AppT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              (int)smem_bytes_for(PHASE));
}

struct DeviceInfo {
  std::atomic<bool> ready{false};
  int clusters = 0;
  int persistent_clusters = 0;
};
DeviceInfo g_dev_info[64];
// Serialises the first set-up of a device between host threads (several handles, or
// the allocation-free entry point, may reach it at once); later calls only read
// `ready` (acquire) and the values published before it.
std::mutex g_dev_setup_mutex;

// Sets the shared-memory attribute of every phase on the current device and finds how
// many 2-CTA clusters of this kernel fit at once.
cudaError_t device_setup(int dev) {
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  DeviceInfo& d = g_dev_info[dev];
  if (d.ready.load(std::memory_order_acquire)) return cudaSuccess;
  std::lock_guard<std::mutex> lock(g_dev_setup_mutex);
  if (d.ready.load(std::memory_order_relaxed)) return cudaSuccess;
  cudaError_t e = set_smem_attr<kPhaseGram, TcNoApply>();
  if (e == cudaSuccess) e = set_smem_attr<kPhasePoly, TcNoApply>();
  if (e == cudaSuccess) e = set_smem_attr<kPhaseUpdate, TcNoApply>();
  if (e == cudaSuccess) e = set_smem_attr<kPhaseUpdate, TcApplyTable>();
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(tc_persistent_kernel<TcNoApply>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)kPSmemBytes);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(tc_persistent_kernel<TcApplyTable>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)kPSmemBytes);
  if (e != cudaSuccess) return e;
  int sms = 0;
  e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(sms & ~1), 1, 1);
  cfg.blockDim = dim3(kThreadsTc, 1, 1);
  cfg.dynamicSmemBytes = smem_bytes_for(kPhaseUpdate);
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  e = cudaOccupancyMaxActiveClusters(&n, tc_kernel<kPhaseUpdate, TcNoApply>, &cfg);
  if (e != cudaSuccess || n <= 0) {
    cudaGetLastError();
    n = sms / 2;
  }
  d.clusters = n;
  cfg.blockDim = dim3(kPThreads, 1, 1);
  cfg.dynamicSmemBytes = kPSmemBytes;
  int np = 0;
  e = cudaOccupancyMaxActiveClusters(&np, tc_persistent_kernel<TcApplyTable>, &cfg);
  if (e != cudaSuccess || np <= 0) {
    cudaGetLastError();
    np = n;
  }
  d.persistent_clusters = np;
  d.ready.store(true, std::memory_order_release);
  return cudaSuccess;
}

template <int PHASE, typename AppT>
cudaError_t launch_phase(const TcParams& p, const AppT& app, int clusters, cudaStream_t st) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(2 * clusters), 1, 1);
  cfg.blockDim = dim3(kThreadsTc, 1, 1);
  cfg.dynamicSmemBytes = smem_bytes_for(PHASE);
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, tc_kernel<PHASE, AppT>, p, app);
}

}  // namespace

int tc_grid_clusters(int n_tiles) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || device_setup(dev) != cudaSuccess) return 1;
  int c = g_dev_info[dev].clusters;
  if (n_tiles < c) c = n_tiles;
  return c < 1 ? 1 : c;
}

cudaError_t launch_tc(int phase, const TcParams& p, int clusters, cudaStream_t st) {
  if (p.n_tiles == 0) return cudaSuccess;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e == cudaSuccess) e = device_setup(dev);
  if (e != cudaSuccess) return e;
  const TcNoApply none{0};
  switch (phase) {
    case kPhaseGram: return launch_phase<kPhaseGram>(p, none, clusters, st);
    case kPhasePoly: return launch_phase<kPhasePoly>(p, none, clusters, st);
    case kPhaseUpdate: return launch_phase<kPhaseUpdate>(p, none, clusters, st);
    default: return cudaErrorInvalidValue;
  }
}

int tc_persistent_clusters() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || device_setup(dev) != cudaSuccess) return 1;
  return std::max(1, g_dev_info[dev].persistent_clusters);
}

cudaError_t launch_tc_persistent(const TcPersistParams& p, const TcApplyTable* app, int clusters, cudaStream_t st) {
  if (p.n_syrk + p.n_upd == 0 || p.ns_steps == 0) return cudaSuccess;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e == cudaSuccess) e = device_setup(dev);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(2 * clusters), 1, 1);
  cfg.blockDim = dim3(kPThreads, 1, 1);
  cfg.dynamicSmemBytes = kPSmemBytes;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (app) return cudaLaunchKernelEx(&cfg, tc_persistent_kernel<TcApplyTable>, p, *app);
  const TcNoApply none{0};
  return cudaLaunchKernelEx(&cfg, tc_persistent_kernel<TcNoApply>, p, none);
}

cudaError_t launch_wait_selftest(int* status, unsigned long long limit_ns, cudaStream_t st) {
  wait_selftest_kernel<<<1, 32, 0, st>>>(status, limit_ns);
  return cudaGetLastError();
}

cudaError_t launch_tc_update_apply(const TcParams& p, const TcApplyTable& a, int clusters, cudaStream_t st) {
  if (p.n_tiles == 0) return cudaSuccess;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e == cudaSuccess) e = device_setup(dev);
  if (e != cudaSuccess) return e;
  return launch_phase<kPhaseUpdate>(p, a, clusters, st);
}

}  // namespace muon
