// Internal structures shared by the host driver (muon_api.cu) and the kernels.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace muon {

// Device-side status codes written into the handle's status word.
enum DevStatus : int {
  kDevOk = 0,
  kDevTimeout = 1,
};

// ----------------------------------------------------------------- elementwise passes

// Max matrices handled by one elementwise launch (they travel as kernel
// parameters; larger lists are split into several launches).
constexpr int kMaxMatsPerLaunch = 192;

// Square tile of one elementwise work unit, and the norm partials it writes (one per warp).
constexpr int kEwTile = 64;
constexpr int kWarpsPerUnit = 8;
// Unit of the bulk-copy momentum pass: a contiguous run of elements of a matrix whose
// workspace copy has the caller's layout (wide, row length a multiple of 8).  It holds
// as many elements as a 64 x 64 tile, so a matrix never has more of these units than
// tiles and the partials array sized for tiles holds them.
constexpr int kFlatUnit = kEwTile * kEwTile;
// Unit of the bulk-copy weight-update pass (no partials, so not tied to the tile count).
constexpr int kApplyUnit = 2 * kFlatUnit;

struct EwMat {
  void* param;          // caller matrix: param (apply), or x_in (normalise-only)
  const void* grad;     // caller gradient (momentum pass) / unused
  float* mom;           // caller momentum buffer (momentum pass) / unused
  void* work;           // workspace matrix in wide orientation, s x ld
  int32_t rows, cols;   // caller shape
  int32_t ld;           // leading dimension of the workspace matrix (elements)
  int32_t tiles_c;      // number of 64-wide tile columns of the caller matrix
  int32_t unit_begin;   // first work unit of this matrix inside the launch
  int32_t gid;          // global matrix index (partials, counters, scales)
  int32_t part_base;    // first work unit of this matrix in the partials array
  int32_t n_units;      // work units of this matrix (kWarpsPerUnit partials each)
  uint8_t transposed;   // rows > cols: the workspace holds the transpose
  uint8_t vec_ok;       // caller rows are 16-byte aligned: vector path allowed
  uint8_t param_bf16;   // dtype of `param` (apply / export / normalise input)
  uint8_t grad_bf16;    // dtype of `grad`
  float lrs;            // fl32(lr * sqrt(max(1, rows/cols))) (apply)
  float lrwd;           // fl32(lr * weight_decay) (apply; 0 = no decay)
  float* nstate;        // NorMuon second moments (s floats) or null
  int32_t row_base;     // first entry of this matrix in the NorMuon row arrays
};

struct EwParams {
  EwMat mats[kMaxMatsPerLaunch];
  int n_mats;
  int total_units;
  float mu;
  int nesterov;
  int use_momentum;     // 0: U = x_in (Newton-Schulz entry point)
  int lerp;             // interpolation-form momentum
  float omu;            // fl32(1 - mu)
  int cautious;         // decay only where O * W >= 0
  int normuon;          // apply: scale O by the per-row NorMuon factor
  float nb2, neps;      // NorMuon beta2, eps
  float* rowsq;         // NorMuon: per-row sum of O^2, then per-row factor f_i * r
  float* rowf;          // NorMuon: per-row 1/(sqrt(v)+eps)
  float eps;
  float* partials;      // per (unit, warp) sum of squares
  float* scale;         // per-matrix 1/(||U||_F + eps)
  int* status;          // device status word (bounded waits record a time-out here)
};
static_assert(sizeof(EwParams) <= 32764, "elementwise parameters must fit the kernel parameter space");

// TMA momentum pass of tall matrices (rows > cols): per matrix three tensor maps, passed
// by value with the launch: gradient (bf16, 64 x 64 boxes), momentum (fp32, 32 x 64
// boxes) and workspace X = U^T (bf16, 64 x 64 boxes), all with the 128-byte swizzle.
constexpr int kEwMapsPerMat = 3;
constexpr int kMaxTiledPerLaunch = 32;
struct __align__(64) EwTiledParams {
  CUtensorMap maps[kMaxTiledPerLaunch * kEwMapsPerMat];
  EwMat mats[kMaxTiledPerLaunch];
  int n_mats;
  int total_units;
  float mu;
  int nesterov;
  int lerp;
  float omu;
  float* partials;
  int* status;
  // apply pass of tall matrices (maps per matrix: weights, final workspace X)
  int cautious;
  int normuon;
  const float* rowsq;   // NorMuon per-row factors (indexed by row_base + caller column)
};
static_assert(sizeof(EwTiledParams) <= 32764, "tiled momentum parameters must fit the kernel parameter space");

enum EwOut : int { kEwApply = 0, kEwExport = 1 };

// NorMuon passes (k_elementwise.cu): per-row statistics and state update, then the
// per-matrix norm-preserving factor; the apply pass reads the factors.
cudaError_t launch_normuon(const EwParams& p, bool work_f32, int grid, cudaStream_t st);

// Launchers (k_elementwise.cu).  work_f32 selects the workspace element type.
// launch_momentum_norm enqueues two kernels: the pass and the per-matrix norm finalize.
cudaError_t launch_momentum_norm(const EwParams& p, bool work_f32, int grid, cudaStream_t st);
// Momentum pass split by matrix kind (bf16 workspace): `flat` lists the wide matrices run
// by the bulk-copy kernel (units of kFlatUnit contiguous elements), `tiled[0..n_tiled)`
// the tall ones run by the TMA tile kernel (64 x 64 tiles through tensor maps,
// transposed in shared memory; one launch per entry), `rest` those run by the register
// tile kernel; `all` lists every matrix with its unit count for the norm finalize.
// Empty lists are skipped.  Returns the number of kernels enqueued in *launches.
cudaError_t launch_momentum_split(const EwParams& flat, const EwTiledParams* tiled, int n_tiled, const EwParams& rest,
                                  const EwParams& all, int sm_count, int* launches, cudaStream_t st);
cudaError_t launch_apply(const EwParams& p, bool work_f32, int out_kind, int grid, cudaStream_t st);
// Weight-update pass split like the momentum pass (bf16 weights and workspace): `flat`
// wide matrices through bulk copies, `tiled[0..n_tiled)` tall ones through tensor maps
// (maps[0] = weights, maps[1] = workspace X), `rest` through the register tile kernel.
cudaError_t launch_apply_split(const EwParams& flat, const EwTiledParams* tiled, int n_tiled, const EwParams& rest,
                               int sm_count, int* launches, cudaStream_t st);

// ----------------------------------------------------------------- tensor-core engine

// Shape groups per tensor-core launch (tensor maps travel as kernel parameters).
constexpr int kMaxGroups = 12;

// A tile is 256 x 256 outputs computed by a pair of CTAs (a 2-CTA cluster): each CTA
// holds 128 rows of the A operand and 128 rows (K-major) or columns (MN-major) of the
// B operand, and accumulates its 128 x 256 half of the tile in its own TMEM.
constexpr int kTile = 256;  // tile rows = tile cols (UMMA M = N = 256 across the pair)
constexpr int kHalf = 128;  // rows of A / of B each CTA loads (TMA box rows)
constexpr int kBK = 64;     // k-block (one 128-byte swizzle row of bf16)

enum TcPhase : int { kPhaseGram = 0, kPhasePoly = 1, kPhaseUpdate = 2 };

struct TcTile {
  uint16_t group;
  uint16_t mat;   // index inside the group
  uint16_t bi;    // 256-row block
  uint16_t bj;    // 256-col block
};

struct TcGroup {
  int s, L;              // matrix in wide orientation: s x L
  int ld_x;              // leading dimension of X buffers (elements)
  int ld_s;              // leading dimension of the s x s buffers
  int gid_base;          // global index of matrix 0 of the group
  __nv_bfloat16* x_cur;  // [n][s][ld_x]
  __nv_bfloat16* x_next; // [n][s][ld_x]
  __nv_bfloat16* gram;   // [n][s][ld_s]
  __nv_bfloat16* poly;   // [n][s][ld_s]
};

// Output blocks are written by TMA bulk-tensor stores of 32 x 32 bf16 blocks staged in
// shared memory with the 64-byte swizzle.
constexpr int kOutBox = 32;

struct __align__(64) TcParams {
  CUtensorMap map_a[kMaxGroups];    // A operand (K-major, box 64 x 128)
  CUtensorMap map_b[kMaxGroups];    // B operand (K-major box 64 x 128, or MN-major box 64 x 64)
  CUtensorMap map_out[kMaxGroups];  // output (X_next / Gram / Poly), box 32 x 32, 64-byte swizzle
  CUtensorMap map_in[kMaxGroups];   // epilogue input (X_cur for Update, Gram for Poly), same boxes
  TcGroup g[kMaxGroups];
  const TcTile* tiles;
  int n_tiles;
  int first_iter;                 // fold the Frobenius scale into this pass
  float ca, cb, cc;               // coefficient triple of this step
  const float* scale;             // per-matrix 1/(||U||_F + eps)
  int* status;                    // device status word
};

// Weight update fused into the last Update pass: W <- RNE(fl32(W - fl32(lrs * O))) with
// O = bf16(X_K), exactly what the separate apply pass computes; X_K itself is not stored.
constexpr int kMaxFusedApply = 768;
enum : uint16_t { kApplyBf16 = 1, kApplyTransposed = 2, kApplyVec = 4, kApplyCautious = 8 };
struct TcApply {
  void* w;         // caller weight, rows x cols row-major
  float lrs;       // fl32(lr * sqrt(max(1, rows/cols)))
  float lrwd;      // fl32(lr * weight_decay), 0 = no decay
  uint16_t flags;  // kApplyBf16 | kApplyTransposed (rows > cols) | kApplyVec (16-byte rows) | kApplyCautious
  uint16_t pad;
  uint32_t pad2;
};
struct __align__(16) TcApplyTable {
  int base;        // global index of entry 0
  int n;
  TcApply m[kMaxFusedApply];
};

// Whole Newton-Schulz loop in one persistent launch (tc_persistent_kernel): every
// (step k, phase, tile) item of one chunk of shape groups, in the order
//   k = 0: Gram tiles, Poly tiles, Update tiles; k = 1: ...
// is taken from a global work counter by the pair's leader CTA and broadcast to both
// CTAs' roles.  An item waits until its matrix has finished the previous phase: every
// epilogue warp of a pair adds 1 to the matrix's counter once its part of a tile is
// stored, so phase p of step k of a matrix with nS symmetric and nU update tiles may
// start once the counter reaches kArrivalsPerTile * (k*(2 nS + nU) + [p >= 1] nS +
// [p >= 2] nS).  The tiles are those of the per-phase launches (listed in one matrix
// priority for every phase, larger L first), and each tile's products and epilogue
// arithmetic are the same, so results are bit-identical to launch_tc's.
constexpr int kMaxNsStepsDev = 16;
// Shape groups of one persistent launch (ten tensor maps per group travel with it).
constexpr int kMaxGroupsPersist = 8;
struct __align__(64) TcPersistParams {
  CUtensorMap xk[kMaxGroupsPersist][2];   // X (ping, pong) K-major, box 64 x 128: Gram operands
  CUtensorMap xmn[kMaxGroupsPersist][2];  // X MN-major, box 64 x 64: Update B operand
  CUtensorMap xout[kMaxGroupsPersist][2]; // X 32 x 32 blocks: Update output and epilogue input
  CUtensorMap gram[kMaxGroupsPersist];    // Gram K-major: Poly operands
  CUtensorMap gram_out[kMaxGroupsPersist];// Gram 32 x 32 blocks: Gram output, Poly epilogue input
  CUtensorMap poly[kMaxGroupsPersist];    // Poly K-major: Update A operand
  CUtensorMap poly_out[kMaxGroupsPersist];// Poly 32 x 32 blocks: Poly output
  TcGroup g[kMaxGroupsPersist];    // x_cur / x_next: the X buffers of even / odd steps
  const TcTile* tiles_syrk;        // Gram and Poly tiles (cost-sorted), n_syrk entries
  const TcTile* tiles_upd;         // Update tiles (cost-sorted), n_upd entries
  int n_syrk, n_upd;
  int ns_steps;
  float ca[kMaxNsStepsDev], cb[kMaxNsStepsDev], cc[kMaxNsStepsDev];
  const float* scale;              // per-matrix 1/(||U||_F + eps)
  int* status;                     // device status word
  unsigned* queue;                 // work counter, zero at launch
  unsigned* done;                  // per-matrix tile arrivals (indexed by gid), zero at launch
  // self-test of the abort path: when nonzero, the first polynomial item of matrix 0
  // waits for a count that is never reached, with this limit instead of the usual one
  unsigned long long stall_ns;
};
static_assert(sizeof(TcPersistParams) + sizeof(TcApplyTable) <= 32764,
              "persistent-kernel parameters must fit the kernel parameter space");

// Launches the persistent kernel with `clusters` 2-CTA clusters (at most the number that
// fit at once; more items than clusters are fine).  `app` non-null: the last Update
// applies the weight update in its epilogue instead of storing X_K.
cudaError_t launch_tc_persistent(const TcPersistParams& p, const TcApplyTable* app, int clusters, cudaStream_t st);
// Clusters of the persistent kernel that fit on the current device at once.
int tc_persistent_clusters();

// Number of 2-CTA clusters to launch for n_tiles tiles on the current device.
int tc_grid_clusters(int n_tiles);
// Launches 2 * clusters CTAs (one cluster per tile at a time, persistent).
cudaError_t launch_tc(int phase, const TcParams& p, int clusters, cudaStream_t st);
// Diagnostic kernel: a bounded wait on a barrier that nothing completes (k_tc_gemm.cu).
cudaError_t launch_wait_selftest(int* status, unsigned long long limit_ns, cudaStream_t st);
// The last Update pass with the weight update fused into its epilogue.
cudaError_t launch_tc_update_apply(const TcParams& p, const TcApplyTable& a, int clusters, cudaStream_t st);

// Tile lists of one matrix.  Symmetric products: 256 x 256 blocks (bi <= bj) of the
// s x s result, row-block major.  Update: every 256 x 256 block of the s x L result,
// column-block major, so that the CTAs running at one time share X's column blocks
// and the whole polynomial matrix in L2.  Returns the count; writes when out != null.
inline int tc_syrk_tiles(int s, uint16_t group, uint16_t mat, TcTile* out) {
  const int nb = (s + kTile - 1) / kTile;
  int n = 0;
  for (int bi = 0; bi < nb; ++bi)
    for (int bj = bi; bj < nb; ++bj) {
      if (out) out[n] = TcTile{group, mat, (uint16_t)bi, (uint16_t)bj};
      ++n;
    }
  return n;
}

inline int tc_update_tiles(int s, int L, uint16_t group, uint16_t mat, TcTile* out) {
  const int mb = (s + kTile - 1) / kTile, nb = (L + kTile - 1) / kTile;
  int n = 0;
  for (int bj = 0; bj < nb; ++bj)
    for (int bi = 0; bi < mb; ++bi) {
      if (out) out[n] = TcTile{group, mat, (uint16_t)bi, (uint16_t)bj};
      ++n;
    }
  return n;
}

// ----------------------------------------------------------------- fp32 validation, tensor cores
//
// fp32 storage and 3xTF32 products on tcgen05 (kind::tf32): every fp32 value x of X, the
// Gram matrix and the polynomial matrix is kept as hi = tf32(x) and lo = tf32(x - hi)
// (both rounded to nearest; hi + lo holds 22 significant bits of x), and each product
// accumulates hi*hi + hi*lo + lo*hi in fp32 in tensor memory.  Tile lists, tile shapes and the operand layouts in shared
// memory are those of the bf16 engine, with 32 fp32 (one 128-byte swizzle row) per
// k-block.  The last Update stores its value unsplit, for the weight-update / export
// pass.
struct Tc32Group {
  int s, L;              // matrix in wide orientation: s x L
  int gid_base;          // global index of matrix 0 of the group
  int ld_in, ld_out;     // leading dimensions (elements) of the epilogue input and output
  size_t in_stride, out_stride;  // elements between consecutive matrices of the group
  const float* in_hi;    // epilogue input: Gram (Poly) or X_cur (Update), hi and lo parts
  const float* in_lo;
  float* out_hi;         // output: Gram, Poly or X_next, hi and lo parts
  float* out_lo;
};

struct __align__(64) Tc32Params {
  CUtensorMap a_hi[kMaxGroups];  // A operand, K-major, box 32 x 128 (Gram: X; Poly: Gram; Update: Poly)
  CUtensorMap a_lo[kMaxGroups];
  CUtensorMap b_hi[kMaxGroups];  // Update B operand: X, MN-major, box 32 x 32
  CUtensorMap b_lo[kMaxGroups];
  Tc32Group g[kMaxGroups];
  const TcTile* tiles;
  int n_tiles;
  int first_iter;                // fold the Frobenius scale into this pass
  int plain_out;                 // last Update: store the value unsplit into out_hi
  float ca, cb, cc;
  const float* scale;
  int* status;
};
static_assert(sizeof(Tc32Params) <= 32764, "3xTF32 parameters must fit the kernel parameter space");

// One grouped launch of one phase (k_tc_tf32.cu).
cudaError_t launch_tc32(int phase, const Tc32Params& p, cudaStream_t st);
// In place hi = tf32(x), and lo = tf32(x - hi), over n floats (the momentum pass's X0).
cudaError_t launch_tf32_split(float* hi, float* lo, size_t n, cudaStream_t st);

// ----------------------------------------------------------------- fp32 validation, CUDA cores

struct F32Mat {
  float* x_cur;
  float* x_next;
  float* gram;
  float* poly;
  int s, L, ld_x, ld_s, gid;
};

cudaError_t launch_f32_gram(const F32Mat& m, int first_iter, const float* scale, cudaStream_t st);
cudaError_t launch_f32_poly(const F32Mat& m, float cb, float cc, cudaStream_t st);
cudaError_t launch_f32_update(const F32Mat& m, int first_iter, const float* scale, float ca,
                              cudaStream_t st);

}  // namespace muon
