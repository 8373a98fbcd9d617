// Allocation-free Newton-Schulz for one matrix (muon_newton_schulz_noalloc).
//
// Who needs it: callers that are not allowed to allocate device memory when they
// want the orthogonalised update -- runtimes that reserve all device memory for their
// own pool up front, engines that forbid allocation after start-up, or latency-bound
// loops where a cudaMalloc (which may synchronise the device) is not acceptable.
// muon_newton_schulz allocates its workspace on first use; this entry point keeps its
// whole scratch (wide-orientation X ping/pong, Gram and polynomial matrices, norm
// partials, tile lists) in one fixed array compiled into the library and calls no
// cudaMalloc, cudaFree or other allocating routine.  It runs the same kernels as the
// handle-based path in MUON_MODE_BF16.
//
// The array is a file-scope __device__ variable.  Host code cannot use its name as a
// device address (on the host it names a stand-in object); the first call on each
// device, with that device current, asks the runtime for the real address with
// cudaGetSymbolAddress and caches it.  Every call shares the array and leaves its
// contents behind, so each call re-zeroes what must start at zero (the internal status
// word; every other region is fully written before it is read), and calls that overlap
// on the GPU race.  The tile lists are written into the array by a small kernel on the
// caller's stream, so a call makes no host-to-device copy.
#include <algorithm>
#include <cmath>
#include <cstring>
#include <mutex>

#include "muon.h"
#include "muon_internal.h"

using namespace muon;

namespace {

constexpr size_t kScratchBytes = size_t(32) << 20;  // 32 MiB per device
constexpr int kMaxTiles = 16384;                     // tile-list entries kept in the scratch
constexpr int kMaxDevices = 64;
constexpr float kDefaultTriple[3] = {3.4445f, -4.7750f, 2.0315f};

static __device__ __align__(256) unsigned char g_scratch[kScratchBytes];

typedef CUresult (*EncodeFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                             const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                             CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// Host-side state: no heap use.  Device address of g_scratch per device (null until
// the first call on that device), the tensor-map encoder, and the parameter blocks.
char* g_scratch_addr[kMaxDevices] = {};
EncodeFn g_encode = nullptr;
EwParams g_ew;
TcParams g_tc;

std::mutex g_setup_mutex;  // first call on a device from several host threads

size_t up(size_t v, size_t a) { return (v + a - 1) / a * a; }

// Tile lists of one s x L (wide orientation) matrix, in the order of tc_syrk_tiles and
// tc_update_tiles: entries [0, n_syrk) are the 256 x 256 blocks (bi <= bj) of the
// symmetric products, row-block major; entries [n_syrk, n_syrk + n_upd) the blocks of
// the update, column-block major.  One thread per entry.
__global__ void noalloc_tiles_kernel(TcTile* out, int s, int L, int n_syrk, int n_upd) {
  const int t = blockIdx.x * blockDim.x + threadIdx.x;
  if (t >= n_syrk + n_upd) return;
  const int nb = (s + kTile - 1) / kTile;
  if (t < n_syrk) {
    int bi = 0, first = 0;  // first = index of tile (bi, bi)
    while (first + (nb - bi) <= t) {
      first += nb - bi;
      ++bi;
    }
    out[t] = TcTile{0, 0, (uint16_t)bi, (uint16_t)(bi + (t - first))};
  } else {
    const int u = t - n_syrk, mb = nb;
    out[t] = TcTile{0, 0, (uint16_t)(u % mb), (uint16_t)(u / mb)};
  }
}

// True when p is device memory of device `dev` (plain or managed allocation).
bool on_device(const void* p, int dev) {
  cudaPointerAttributes a;
  if (cudaPointerGetAttributes(&a, p) != cudaSuccess) {
    cudaGetLastError();
    return false;
  }
  return (a.type == cudaMemoryTypeDevice || a.type == cudaMemoryTypeManaged) && a.device == dev;
}

bool encode(CUtensorMap* map, void* base, int inner, int rows, int ld, int box_inner, int box_rows,
            CUtensorMapSwizzle swizzle = CU_TENSOR_MAP_SWIZZLE_128B) {
  cuuint64_t dims[3] = {(cuuint64_t)inner, (cuuint64_t)rows, 1};
  cuuint64_t strides[2] = {(cuuint64_t)ld * 2, (cuuint64_t)ld * 2 * (cuuint64_t)rows};
  cuuint32_t box[3] = {(cuuint32_t)box_inner, (cuuint32_t)box_rows, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  return g_encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, base, dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

extern "C" MUON_API muon_status muon_newton_schulz_noalloc(const void* x_in, void* o_out, int64_t rows,
                                                           int64_t cols, muon_dtype dtype, const float* coeffs,
                                                           int ns_steps, float eps, int* status,
                                                           void* cuda_stream) {
  // ---- arguments (host only, nothing enqueued on failure)
  if (!x_in || !o_out) return MUON_ERR_INVALID_ARG;
  if (rows < 1 || cols < 1 || rows > (int64_t(1) << 24) || cols > (int64_t(1) << 24)) return MUON_ERR_INVALID_ARG;
  if (dtype != MUON_F32 && dtype != MUON_BF16) return MUON_ERR_INVALID_ARG;
  if (ns_steps < 1 || ns_steps > 16) return MUON_ERR_INVALID_ARG;
  if (!std::isfinite(eps) || eps < 0.f) return MUON_ERR_INVALID_ARG;
  if (coeffs)
    for (int i = 0; i < 3 * ns_steps; ++i)
      if (!std::isfinite(coeffs[i])) return MUON_ERR_INVALID_ARG;
  if (((uintptr_t)x_in | (uintptr_t)o_out | (uintptr_t)status) & 3u) return MUON_ERR_INVALID_ARG;
  if (((uintptr_t)x_in | (uintptr_t)o_out) & 15u) return MUON_ERR_INVALID_ARG;
  const size_t esz = dtype == MUON_BF16 ? 2 : 4;
  const size_t bytes = (size_t)rows * (size_t)cols * esz;
  if ((uintptr_t)x_in < (uintptr_t)o_out + bytes && (uintptr_t)o_out < (uintptr_t)x_in + bytes)
    return MUON_ERR_INVALID_ARG;

  // ---- layout inside the fixed scratch
  const int s = (int)std::min(rows, cols), L = (int)std::max(rows, cols);
  const int ld_x = (L + 7) / 8 * 8, ld_s = (s + 7) / 8 * 8;
  const int tiles_c = (int)((cols + kEwTile - 1) / kEwTile);
  const int n_units = (int)((rows + kEwTile - 1) / kEwTile) * tiles_c;
  const int n_syrk = tc_syrk_tiles(s, 0, 0, nullptr);
  const int n_upd = tc_update_tiles(s, L, 0, 0, nullptr);
  if ((int64_t)n_syrk + n_upd > kMaxTiles) return MUON_ERR_TOO_LARGE;
  size_t off = 0;
  const size_t off_x0 = off; off = up(off + (size_t)s * ld_x * 2, 1024);
  const size_t off_x1 = off; off = up(off + (size_t)s * ld_x * 2, 1024);
  const size_t off_gram = off; off = up(off + (size_t)s * ld_s * 2, 1024);
  const size_t off_poly = off; off = up(off + (size_t)s * ld_s * 2, 1024);
  const size_t off_part = off; off = up(off + (size_t)n_units * kWarpsPerUnit * 4, 256);
  const size_t off_scale = off; off += 4;
  const size_t off_status = off; off = up(off + 4, 256);
  const size_t off_tiles = off; off += (size_t)(n_syrk + n_upd) * sizeof(TcTile);
  if (off > kScratchBytes) return MUON_ERR_TOO_LARGE;

  // ---- per-device set-up (first call on a device; must precede any stream capture)
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return MUON_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return MUON_ERR_UNSUPPORTED;
  if (!on_device(x_in, dev) || !on_device(o_out, dev) || (status && !on_device(status, dev)))
    return MUON_ERR_INVALID_ARG;
  if (!g_scratch_addr[dev]) {
    std::lock_guard<std::mutex> lock(g_setup_mutex);
    int major = 0, minor = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
      return MUON_ERR_CUDA;
    if (major != 10 || minor != 0) return MUON_ERR_UNSUPPORTED;
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_scratch) != cudaSuccess || p == nullptr) {
      cudaGetLastError();
      return MUON_ERR_CUDA;
    }
    g_scratch_addr[dev] = static_cast<char*>(p);
  }
  if (!g_encode) {
    std::lock_guard<std::mutex> lock(g_setup_mutex);
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess || !fn)
      return MUON_ERR_CUDA;
    g_encode = reinterpret_cast<EncodeFn>(fn);
  }
  int sms = 148;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return MUON_ERR_CUDA;
  char* scr = g_scratch_addr[dev];
  cudaStream_t st = static_cast<cudaStream_t>(cuda_stream);

  // ---- tile lists (Gram and Poly share the triangle list) and zeroed words
  const int n_tiles = n_syrk + n_upd;
  noalloc_tiles_kernel<<<(n_tiles + 255) / 256, 256, 0, st>>>(reinterpret_cast<TcTile*>(scr + off_tiles), s, L,
                                                             n_syrk, n_upd);
  if (cudaGetLastError() != cudaSuccess) return MUON_ERR_CUDA;
  if (cudaMemsetAsync(scr + off_status, 0, 4, st) != cudaSuccess) return MUON_ERR_CUDA;
  int* stat = status ? status : reinterpret_cast<int*>(scr + off_status);

  // ---- norm pass: U (wide orientation) and 1/(||U||_F + eps)
  std::memset(&g_ew, 0, sizeof(g_ew));
  g_ew.n_mats = 1;
  g_ew.total_units = n_units;
  g_ew.use_momentum = 0;
  g_ew.lerp = 0;
  g_ew.cautious = 0;
  g_ew.eps = eps;
  g_ew.partials = reinterpret_cast<float*>(scr + off_part);
  g_ew.scale = reinterpret_cast<float*>(scr + off_scale);
  EwMat& m = g_ew.mats[0];
  m.param = const_cast<void*>(x_in);
  m.work = scr + off_x0;
  m.rows = (int32_t)rows;
  m.cols = (int32_t)cols;
  m.ld = ld_x;
  m.tiles_c = tiles_c;
  m.n_units = n_units;
  m.transposed = rows > cols ? 1 : 0;
  m.vec_ok = (cols % 8 == 0) ? 1 : 0;
  m.param_bf16 = dtype == MUON_BF16 ? 1 : 0;
  const int ew_grid = std::max(1, std::min(n_units, sms * 8));
  if (launch_momentum_norm(g_ew, false, ew_grid, st) != cudaSuccess) return MUON_ERR_CUDA;

  // ---- Newton-Schulz steps on the tensor cores
  CUtensorMap xk[2], xmn[2], xout[2], gram_map, poly_map, gram_out, poly_out;
  for (int b = 0; b < 2; ++b) {
    char* xb = scr + (b == 0 ? off_x0 : off_x1);
    if (!encode(&xk[b], xb, L, s, ld_x, kBK, kHalf) || !encode(&xmn[b], xb, L, s, ld_x, 64, kBK) ||
        !encode(&xout[b], xb, L, s, ld_x, kOutBox, kOutBox, CU_TENSOR_MAP_SWIZZLE_64B))
      return MUON_ERR_CUDA;
  }
  if (!encode(&gram_map, scr + off_gram, s, s, ld_s, kBK, kHalf) ||
      !encode(&poly_map, scr + off_poly, s, s, ld_s, kBK, kHalf) ||
      !encode(&gram_out, scr + off_gram, s, s, ld_s, kOutBox, kOutBox, CU_TENSOR_MAP_SWIZZLE_64B) ||
      !encode(&poly_out, scr + off_poly, s, s, ld_s, kOutBox, kOutBox, CU_TENSOR_MAP_SWIZZLE_64B))
    return MUON_ERR_CUDA;
  const TcTile* dev_tiles = reinterpret_cast<const TcTile*>(scr + off_tiles);
  for (int k = 0; k < ns_steps; ++k) {
    const int cur = k & 1;
    const float* c = coeffs ? coeffs + 3 * k : kDefaultTriple;
    for (int ph = 0; ph < 3; ++ph) {
      std::memset(&g_tc, 0, sizeof(g_tc));
      TcGroup& g = g_tc.g[0];
      g.s = s;
      g.L = L;
      g.ld_x = ld_x;
      g.ld_s = ld_s;
      g.gid_base = 0;
      g.x_cur = reinterpret_cast<__nv_bfloat16*>(scr + (cur == 0 ? off_x0 : off_x1));
      g.x_next = reinterpret_cast<__nv_bfloat16*>(scr + (cur == 0 ? off_x1 : off_x0));
      g.gram = reinterpret_cast<__nv_bfloat16*>(scr + off_gram);
      g.poly = reinterpret_cast<__nv_bfloat16*>(scr + off_poly);
      if (ph == kPhaseGram) {
        g_tc.map_a[0] = xk[cur];
        g_tc.map_out[0] = gram_out;
      } else if (ph == kPhasePoly) {
        g_tc.map_a[0] = gram_map;
        g_tc.map_out[0] = poly_out;
        g_tc.map_in[0] = gram_out;
      } else {
        g_tc.map_a[0] = poly_map;
        g_tc.map_b[0] = xmn[cur];
        g_tc.map_out[0] = xout[cur ^ 1];
        g_tc.map_in[0] = xout[cur];
      }
      g_tc.tiles = ph == kPhaseUpdate ? dev_tiles + n_syrk : dev_tiles;
      g_tc.n_tiles = ph == kPhaseUpdate ? n_upd : n_syrk;
      g_tc.first_iter = k == 0 ? 1 : 0;
      g_tc.ca = c[0];
      g_tc.cb = c[1];
      g_tc.cc = c[2];
      g_tc.scale = reinterpret_cast<const float*>(scr + off_scale);
      g_tc.status = stat;
      if (launch_tc(ph, g_tc, tc_grid_clusters(g_tc.n_tiles), st) != cudaSuccess) return MUON_ERR_CUDA;
    }
  }

  // ---- export O (transposed back for tall matrices) into the caller's buffer
  m.param = o_out;
  m.work = scr + ((ns_steps & 1) ? off_x1 : off_x0);
  if (launch_apply(g_ew, false, kEwExport, ew_grid, st) != cudaSuccess) return MUON_ERR_CUDA;
  return MUON_OK;
}
