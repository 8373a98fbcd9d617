// Host side of the Muon C ABI: argument checks, the plan (shape groups, workspace
// layout, tile lists, TMA tensor maps) and the stream-ordered launch sequence
//
//   momentum pass + norm finalize -> { Gram -> Poly -> Update } x ns_steps
//
// where the last Update also applies W -= lr*scale*O in its epilogue (bf16 mode; in fp32
// mode, and for the Newton-Schulz entry point, a separate apply / export pass follows).
// In bf16 mode the momentum pass is a bulk-copy kernel for wide matrices and a TMA tile
// kernel for tall ones (register tile kernel otherwise): 18 launches for five steps
// when a set has both orientations and the shapes fit one launch per phase.  Matrices
// of equal wide-orientation shape (s, L) = (min(r,c), max(r,c)) are stacked into one
// group, the device analogue of the per-shape-group stacking of the momentum
// buffers that the autoresearch train.py review describes for MuonAdamW.
#include <algorithm>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <string>
#include <vector>

#include <nvtx3/nvToolsExt.h>

#include "muon.h"
#include "muon_internal.h"

using namespace muon;

namespace {

constexpr float kDefaultCoeffs[3] = {3.4445f, -4.7750f, 2.0315f};
constexpr int64_t kMaxDim = int64_t(1) << 24;
constexpr int kMaxNsSteps = 16;
constexpr int kMaxMatrices = 65535;
// MUON_LAUNCH_AUTO takes the persistent launch below this algorithmic work of one
// Newton-Schulz step over all of a call's matrices.
constexpr double kPersistentMaxFlops = 1e12;
// MUON_MODE_FP32_VALIDATE runs 3xTF32 on the tensor cores only while every contraction is
// at most this long: the tensor cores' fp32 accumulation error grows with the number of
// accumulations (measured on one B200: ~4e-5 relative error of O at 8192, ~9e-5 at
// 16384, ~1.9e-4 at 32768, against 2-7e-6 on CUDA cores); longer ones run on CUDA cores.
constexpr int64_t kTf32MaxContraction = 8192;

// The fp32 validation form a call runs in: 3xTF32 unless a matrix is too long for it.
muon_mode fp32_form(muon_mode mode, const int64_t* rows, const int64_t* cols, int n) {
  if (mode != MUON_MODE_FP32_VALIDATE) return mode;
  for (int i = 0; i < n; ++i)
    if (std::max(rows[i], cols[i]) > kTf32MaxContraction) return MUON_MODE_FP32_SIMT;
  return mode;
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }
int round8(int v) { return (v + 7) / 8 * 8; }

struct GroupPlan {
  int s = 0, L = 0, n = 0;
  int ld_x = 0, ld_s = 0;
  int gid_base = 0;
  size_t off_x[2] = {0, 0};
  size_t off_gram = 0, off_poly = 0;
  // 3xTF32 mode: the lo parts (the arrays above hold the hi parts)
  size_t off_xlo[2] = {0, 0};
  size_t off_gram_lo = 0, off_poly_lo = 0;
};

struct MatPlan {
  int group = 0, idx = 0, gid = 0;
  int row_base = 0;  // first entry in the NorMuon row arrays (prefix of min(rows, cols))
  int64_t rows = 0, cols = 0;
  bool transposed = false;
  int n_units = 0, part_base = 0, tiles_c = 0;
};

struct ChunkPlan {
  int g_begin = 0, g_end = 0;
  size_t off_tiles[3] = {0, 0, 0};
  // the persistent launch's lists (symmetric products, update): every phase in one
  // matrix priority, larger L first, so a matrix's next phase follows its previous one
  size_t off_ptiles[2] = {0, 0};
  int n_tiles[3] = {0, 0, 0};
};

struct Plan {
  bool valid = false;
  muon_mode mode = MUON_MODE_BF16;
  std::vector<int64_t> sig;  // rows, cols pairs
  std::vector<GroupPlan> groups;
  std::vector<MatPlan> mats;
  std::vector<int> mat_of_gid;  // caller index of each global (group-major) index
  std::vector<ChunkPlan> chunks;
  std::vector<TcTile> tiles;  // host copy of every chunk's tile lists
  size_t off_partials = 0, off_scale = 0, off_tiles = 0, off_rowsq = 0, off_rowf = 0, off_sched = 0, bytes = 0;
  int total_rows = 0;
  int total_units = 0;
  // TMA maps per group (bf16 mode): X K-major (ping/pong), X MN-major (ping/pong), Gram, Poly
  std::vector<CUtensorMap> map_xk[2], map_xmn[2], map_gram, map_poly;
  // output maps (32 x 32 boxes, 64-byte swizzle) for the epilogue's TMA stores
  std::vector<CUtensorMap> map_xout[2], map_gram_out, map_poly_out;
  // 3xTF32 mode (fp32): X K-major and MN-major, Gram, Poly; hi and lo parts
  std::vector<CUtensorMap> t_xk[2][2], t_xmn[2][2], t_gram[2], t_poly[2];
  // debug mode: guard bands after every workspace region (offset, region name), their
  // offsets on the device, and the check's result words
  std::vector<std::pair<size_t, const char*>> guards;
  size_t off_guard_table = 0, off_guard_result = 0;
};

}  // namespace

struct muon_handle {
  int device = 0;
  int sm_count = 148;
  std::string err;
  int last_launches = 0;
  EncodeTiledFn encode = nullptr;
  char* ws = nullptr;
  size_t ws_bytes = 0;
  int* dev_status = nullptr;
  int* host_status = nullptr;
  cudaEvent_t status_event = nullptr;
  bool status_pending = false;
  Plan plan;
  TcApplyTable* apply_table = nullptr;  // host staging of the fused weight-update table
  // TMA momentum pass of tall matrices: the tensor maps of each caller matrix and the
  // pointers they were encoded for (grad, momentum, workspace); cleared with the plan
  std::vector<CUtensorMap> ewmap;
  std::vector<const void*> ewmap_key;
  // the same for the weight-update pass (weights, final workspace X)
  std::vector<CUtensorMap> ewmap_apply;
  std::vector<const void*> ewmap_apply_key;
  // per-launch timing (muon_profile_enable)
  bool profiling = false;
  std::vector<cudaEvent_t> ev_free;
  struct Pending {
    int kind;
    cudaEvent_t a, b;
  };
  std::vector<Pending> ev_pending;
  cudaEvent_t ev_open = nullptr;
  double prof_ms[MUON_KIND_COUNT] = {};
  int64_t prof_launches[MUON_KIND_COUNT] = {};
  // muon_selftest_fail_next_alloc: the next workspace allocation reports failure
  bool fail_next_alloc = false;
  // muon_set_launch_mode
  int launch_mode = MUON_LAUNCH_AUTO;
  unsigned long long stall_ns = 0;  // muon_selftest_stall_persistent (next persistent launch)
  TcPersistParams* persist = nullptr;  // host staging of the persistent launch's parameters
  // MUON_LOG set (and not "0") at muon_init: plan summaries and errors go to stderr
  bool log = false;
  // MUON_DEBUG set (and not "0") at muon_init: guard bands around workspace regions,
  // checked after every call
  bool debug = false;
  // MUON_NVTX set (and not "0") at muon_init: an NVTX range around every call and every
  // kernel launch, for timeline profilers
  bool nvtx = false;
  // the pointer lists of the last two calls that were found to be device memory of
  // `device` (a call with one of them is not checked again; loops often alternate
  // between two sets of buffers)
  std::vector<const void*> checked_ptrs[2];
  int checked_next = 0;
};

namespace {

muon_status fail(muon_handle* h, muon_status st, const char* fmt, ...) {
  if (h) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof(buf), fmt, ap);
    va_end(ap);
    h->err = buf;
    if (h->log) fprintf(stderr, "muon: %s: %s\n", muon_status_string(st), buf);
  }
  return st;
}

muon_status cuda_fail(muon_handle* h, cudaError_t e, const char* what) {
  return fail(h, MUON_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

cudaEvent_t take_event(muon_handle* h) {
  if (!h->ev_free.empty()) {
    cudaEvent_t e = h->ev_free.back();
    h->ev_free.pop_back();
    return e;
  }
  cudaEvent_t e = nullptr;
  if (cudaEventCreate(&e) != cudaSuccess) {
    cudaGetLastError();
    return nullptr;
  }
  return e;
}

// Brackets one launch with events on its stream while profiling is on.
// Name of a kernel kind in the NVTX ranges (muon_kernel_kind order).
const char* kind_name(int kind) {
  static const char* const names[MUON_KIND_COUNT] = {"muon momentum/norm", "muon Gram",   "muon polynomial",
                                                     "muon update",        "muon apply",  "muon update+apply",
                                                     "muon persistent Newton-Schulz"};
  return kind >= 0 && kind < MUON_KIND_COUNT ? names[kind] : "muon";
}

void prof_begin(muon_handle* h, cudaStream_t st, int kind) {
  if (h->nvtx) nvtxRangePushA(kind_name(kind));
  if (!h->profiling) return;
  h->ev_open = take_event(h);
  if (h->ev_open) cudaEventRecord(h->ev_open, st);
}

void prof_end(muon_handle* h, int kind, cudaStream_t st) {
  if (h->nvtx) nvtxRangePop();
  if (!h->profiling || !h->ev_open) return;
  cudaEvent_t b = take_event(h);
  if (!b) return;
  cudaEventRecord(b, st);
  h->ev_pending.push_back({kind, h->ev_open, b});
  h->ev_open = nullptr;
}

// Restores the caller's current device on scope exit.
struct DeviceGuard {
  int prev = -1;
  bool ok = false;
  explicit DeviceGuard(int dev) {
    if (cudaGetDevice(&prev) != cudaSuccess) prev = -1;
    ok = cudaSetDevice(dev) == cudaSuccess;
  }
  ~DeviceGuard() {
    if (prev >= 0) cudaSetDevice(prev);
  }
};

bool finite(float v) { return std::isfinite(v); }

struct Range {
  uintptr_t lo, hi;
  int mat;
};

muon_status check_overlaps(muon_handle* h, std::vector<Range>& rs) {
  std::sort(rs.begin(), rs.end(), [](const Range& a, const Range& b) { return a.lo < b.lo; });
  for (size_t i = 1; i < rs.size(); ++i)
    if (rs[i].lo < rs[i - 1].hi)
      return fail(h, MUON_ERR_INVALID_ARG, "buffers of matrices %d and %d overlap", rs[i - 1].mat, rs[i].mat);
  return MUON_OK;
}

// Every pointer must be device memory (plain or managed) of the handle's device: host
// memory, or another GPU's, would be read and written by the kernels.  The last two lists
// that passed are remembered, so a loop over the same buffers pays one comparison each.
muon_status check_device_pointers(muon_handle* h, const std::vector<const void*>& ptrs) {
  if (ptrs == h->checked_ptrs[0] || ptrs == h->checked_ptrs[1]) return MUON_OK;
  for (size_t i = 0; i < ptrs.size(); ++i) {
    if (i > 0 && ptrs[i] == ptrs[i - 1]) continue;
    cudaPointerAttributes a;
    const cudaError_t e = cudaPointerGetAttributes(&a, ptrs[i]);
    if (e != cudaSuccess) cudaGetLastError();
    if (e != cudaSuccess || (a.type != cudaMemoryTypeDevice && a.type != cudaMemoryTypeManaged) ||
        a.device != h->device)
      return fail(h, MUON_ERR_INVALID_ARG, "pointer %zu of the call (%p) is not device memory of device %d", i,
                  ptrs[i], h->device);
  }
  h->checked_ptrs[h->checked_next] = ptrs;
  h->checked_next ^= 1;
  return MUON_OK;
}

muon_status check_coeffs(muon_handle* h, const float* coeffs, int ns_steps) {
  if (ns_steps < 1 || ns_steps > kMaxNsSteps)
    return fail(h, MUON_ERR_INVALID_ARG, "ns_steps %d outside 1..%d", ns_steps, kMaxNsSteps);
  if (coeffs)
    for (int i = 0; i < 3 * ns_steps; ++i)
      if (!finite(coeffs[i])) return fail(h, MUON_ERR_INVALID_ARG, "coefficient %d is not finite", i);
  return MUON_OK;
}

// ------------------------------------------------------------------ plan

// Per-phase launches: each list longest contraction first (Gram by L, Poly and Update by
// s), for the balance of one launch's waves.
void sort_tiles(std::vector<TcTile>& t, const std::vector<GroupPlan>& groups, int phase) {
  auto cost = [&](const TcTile& x) {
    const GroupPlan& g = groups[x.group];
    return (int64_t)(phase == kPhaseGram ? g.L : g.s);
  };
  std::stable_sort(t.begin(), t.end(), [&](const TcTile& a, const TcTile& b) { return cost(a) > cost(b); });
}

// Persistent launch: the same matrix priority in every phase (larger L first, the
// matrices with the longest Gram contraction and the most update tiles), so the items of
// a matrix's next phase come up in the order its previous phase completes.
void sort_tiles_persistent(std::vector<TcTile>& t, const std::vector<GroupPlan>& groups) {
  std::stable_sort(t.begin(), t.end(),
                   [&](const TcTile& a, const TcTile& b) { return groups[a.group].L > groups[b.group].L; });
}

muon_status encode_map(muon_handle* h, CUtensorMap* map, void* base, int inner, int rows, int n, int ld,
                       int box_inner, int box_rows,
                       CUtensorMapSwizzle swizzle = CU_TENSOR_MAP_SWIZZLE_128B, bool f32 = false) {
  const cuuint64_t esz = f32 ? 4 : 2;
  cuuint64_t dims[3] = {(cuuint64_t)inner, (cuuint64_t)rows, (cuuint64_t)n};
  cuuint64_t strides[2] = {(cuuint64_t)ld * esz, (cuuint64_t)ld * esz * (cuuint64_t)rows};
  cuuint32_t box[3] = {(cuuint32_t)box_inner, (cuuint32_t)box_rows, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = h->encode(map, f32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, base,
                         dims, strides, box, estr,
                         CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle,
                         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(h, MUON_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
  return MUON_OK;
}

// ------------------------------------------------------------------ debug mode: guard bands

constexpr size_t kGuardBytes = 256;
constexpr unsigned char kGuardByte = 0xA5;

// One block per guard band: counts the bytes that no longer hold the pattern, and
// records the lowest index of a band that changed.
__global__ void guard_check_kernel(const unsigned char* ws, const uint64_t* offs, int n, unsigned* result) {
  const int gi = blockIdx.x;
  if (gi >= n) return;
  const unsigned char* g = ws + offs[gi];
  unsigned bad = 0;
  for (int i = threadIdx.x; i < (int)kGuardBytes; i += blockDim.x) bad += g[i] != kGuardByte ? 1u : 0u;
  if (bad) {
    atomicAdd(&result[0], bad);
    atomicMin(&result[1], (unsigned)gi);
  }
}

// Fills every guard band with the pattern.
cudaError_t arm_guards(muon_handle* h, cudaStream_t st) {
  for (const auto& g : h->plan.guards) {
    const cudaError_t e = cudaMemsetAsync(h->ws + g.first, kGuardByte, kGuardBytes, st);
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

// Debug mode, after a call's work: waits for it, checks every guard band and reports an
// overwritten one as MUON_ERR_CORRUPT (the bands are then filled again).
muon_status check_guards(muon_handle* h, cudaStream_t st) {
  const Plan& P = h->plan;
  if (!h->debug || P.guards.empty()) return MUON_OK;
  unsigned* res = reinterpret_cast<unsigned*>(h->ws + P.off_guard_result);
  cudaError_t e = cudaMemsetAsync(res, 0, 4, st);
  if (e == cudaSuccess) e = cudaMemsetAsync(res + 1, 0xFF, 4, st);
  if (e == cudaSuccess) {
    guard_check_kernel<<<(unsigned)P.guards.size(), 128, 0, st>>>(
        reinterpret_cast<const unsigned char*>(h->ws), reinterpret_cast<const uint64_t*>(h->ws + P.off_guard_table),
        (int)P.guards.size(), res);
    e = cudaGetLastError();
  }
  unsigned host[2] = {0, 0};
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  if (e == cudaSuccess) e = cudaMemcpy(host, res, sizeof(host), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail(h, e, "guard band check");
  if (host[0] == 0) return MUON_OK;
  const char* what = host[1] < P.guards.size() ? P.guards[host[1]].second : "?";
  if ((e = arm_guards(h, st)) == cudaSuccess) e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return cuda_fail(h, e, "guard band re-arm");
  return fail(h, MUON_ERR_CORRUPT, "%u bytes of the guard bands changed; the first one follows the %s", host[0],
              what);
}

muon_status build_plan(muon_handle* h, const int64_t* rows, const int64_t* cols, int n, muon_mode mode,
                       cudaStream_t st) {
  Plan& P = h->plan;
  P = Plan();
  h->ewmap.clear();  // the momentum-pass tensor maps describe the old plan's buffers
  h->ewmap_key.clear();
  h->ewmap_apply.clear();
  h->ewmap_apply_key.clear();
  P.mode = mode;
  const size_t esz = (mode == MUON_MODE_BF16) ? 2 : 4;
  // every per-call count below must fit the 32-bit fields of the kernels' tables
  {
    int64_t units = 0, rows_total = 0;
    for (int i = 0; i < n; ++i) {
      units += ((rows[i] + kEwTile - 1) / kEwTile) * ((cols[i] + kEwTile - 1) / kEwTile);
      rows_total += std::min(rows[i], cols[i]);
    }
    if (units * kWarpsPerUnit >= (int64_t(1) << 31) || rows_total >= (int64_t(1) << 31))
      return fail(h, MUON_ERR_INVALID_ARG, "the matrices of one call are too large for one workspace");
  }
  P.sig.resize(2 * (size_t)n);
  P.mats.resize(n);
  for (int i = 0; i < n; ++i) {
    P.sig[2 * i] = rows[i];
    P.sig[2 * i + 1] = cols[i];
    const int s = (int)std::min(rows[i], cols[i]);
    const int L = (int)std::max(rows[i], cols[i]);
    int gi = -1;
    for (size_t g = 0; g < P.groups.size(); ++g)
      if (P.groups[g].s == s && P.groups[g].L == L) gi = (int)g;
    if (gi < 0) {
      GroupPlan g;
      g.s = s;
      g.L = L;
      g.ld_x = round8(L);
      g.ld_s = round8(s);
      P.groups.push_back(g);
      gi = (int)P.groups.size() - 1;
    }
    MatPlan& m = P.mats[i];
    m.group = gi;
    m.idx = P.groups[gi].n++;
    m.rows = rows[i];
    m.cols = cols[i];
    m.transposed = rows[i] > cols[i];
    m.tiles_c = (int)((cols[i] + kEwTile - 1) / kEwTile);
    m.n_units = (int)((rows[i] + kEwTile - 1) / kEwTile) * m.tiles_c;
    m.part_base = P.total_units;
    P.total_units += m.n_units;
    m.row_base = P.total_rows;
    P.total_rows += s;
  }
  // global matrix index = group-major order
  int gid = 0;
  for (auto& g : P.groups) {
    g.gid_base = gid;
    gid += g.n;
  }
  P.mat_of_gid.assign(n, 0);
  for (int i = 0; i < n; ++i) {
    P.mats[i].gid = P.groups[P.mats[i].group].gid_base + P.mats[i].idx;
    P.mat_of_gid[P.mats[i].gid] = i;
  }
  // workspace layout
  size_t off = 0;
  const bool tf32x3 = mode == MUON_MODE_FP32_VALIDATE;
  // Places a region of `bytes` at the next multiple of `align`; in debug mode a guard
  // band follows its last byte (at the next 16-byte boundary).
  auto place = [&](size_t bytes, size_t align, const char* what) {
    off = align_up(off, align);
    const size_t o = off;
    off += bytes;
    if (h->debug) {
      off = align_up(off, 16);
      P.guards.push_back({off, what});
      off += kGuardBytes;
    }
    return o;
  };
  for (auto& g : P.groups) {
    const size_t xbytes = (size_t)g.n * g.s * g.ld_x * esz;
    const size_t sbytes = (size_t)g.n * g.s * g.ld_s * esz;
    g.off_x[0] = place(xbytes, 1024, "X (even steps)");
    g.off_x[1] = place(xbytes, 1024, "X (odd steps)");
    g.off_gram = place(sbytes, 1024, "Gram matrices");
    g.off_poly = place(sbytes, 1024, "polynomial matrices");
    if (tf32x3) {
      g.off_xlo[0] = place(xbytes, 1024, "X lo parts (even steps)");
      g.off_xlo[1] = place(xbytes, 1024, "X lo parts (odd steps)");
      g.off_gram_lo = place(sbytes, 1024, "Gram lo parts");
      g.off_poly_lo = place(sbytes, 1024, "polynomial lo parts");
    }
  }
  P.off_partials = place((size_t)P.total_units * kWarpsPerUnit * 4, 1024, "norm partials");
  P.off_scale = place((size_t)n * 4, 256, "norm scales");
  P.off_rowsq = place((size_t)P.total_rows * 4, 256, "NorMuon row sums");
  P.off_rowf = place((size_t)P.total_rows * 4, 256, "NorMuon row factors");
  // persistent launch: work counter + one completed-tile counter per matrix
  P.off_sched = place((size_t)(1 + n) * 4, 256, "persistent-launch counters");
  // tile lists (tensor-core paths)
  if (mode != MUON_MODE_FP32_SIMT) {
    for (int g0 = 0; g0 < (int)P.groups.size(); g0 += kMaxGroups) {
      ChunkPlan c;
      c.g_begin = g0;
      c.g_end = std::min((int)P.groups.size(), g0 + kMaxGroups);
      std::vector<TcTile> syrk, upd;
      for (int gg = c.g_begin; gg < c.g_end; ++gg) {
        const GroupPlan& g = P.groups[gg];
        const uint16_t lg = (uint16_t)(gg - c.g_begin);
        for (int m = 0; m < g.n; ++m) {
          const size_t s0 = syrk.size(), u0 = upd.size();
          syrk.resize(s0 + tc_syrk_tiles(g.s, lg, (uint16_t)m, nullptr));
          tc_syrk_tiles(g.s, lg, (uint16_t)m, syrk.data() + s0);
          upd.resize(u0 + tc_update_tiles(g.s, g.L, lg, (uint16_t)m, nullptr));
          tc_update_tiles(g.s, g.L, lg, (uint16_t)m, upd.data() + u0);
        }
      }
      std::vector<GroupPlan> cg(P.groups.begin() + c.g_begin, P.groups.begin() + c.g_end);
      std::vector<TcTile> lists[3] = {syrk, syrk, upd};
      for (int ph = 0; ph < 3; ++ph) {
        sort_tiles(lists[ph], cg, ph);
        c.off_tiles[ph] = P.tiles.size();
        c.n_tiles[ph] = (int)lists[ph].size();
        P.tiles.insert(P.tiles.end(), lists[ph].begin(), lists[ph].end());
      }
      std::vector<TcTile> plists[2] = {syrk, upd};
      for (int q = 0; q < 2; ++q) {
        sort_tiles_persistent(plists[q], cg);
        c.off_ptiles[q] = P.tiles.size();
        P.tiles.insert(P.tiles.end(), plists[q].begin(), plists[q].end());
      }
      P.chunks.push_back(c);
    }
  }
  P.off_tiles = place(P.tiles.size() * sizeof(TcTile), 256, "tile lists");
  if (h->debug) {
    P.off_guard_table = align_up(off, 256);
    P.off_guard_result = align_up(P.off_guard_table + P.guards.size() * 8, 256);
    off = P.off_guard_result + 256;
  }
  P.bytes = align_up(off, 256);

  // (re)allocate the workspace
  if (P.bytes > h->ws_bytes) {
    if (h->ws) {
      cudaError_t e = cudaStreamSynchronize(st);
      if (e != cudaSuccess) return cuda_fail(h, e, "synchronize before workspace reallocation");
      cudaFree(h->ws);
      h->ws = nullptr;
      h->ws_bytes = 0;
    }
    void* p = nullptr;
    const bool injected = h->fail_next_alloc;
    h->fail_next_alloc = false;
    if (injected || cudaMalloc(&p, P.bytes) != cudaSuccess) {
      cudaGetLastError();
      return fail(h, MUON_ERR_OOM, "workspace allocation of %zu bytes failed%s", P.bytes,
                  injected ? " (injected by muon_selftest_fail_next_alloc)" : "");
    }
    h->ws = static_cast<char*>(p);
    h->ws_bytes = P.bytes;
  }
  cudaError_t e = cudaSuccess;
  if (!P.tiles.empty()) {
    e = cudaMemcpyAsync(h->ws + P.off_tiles, P.tiles.data(), P.tiles.size() * sizeof(TcTile),
                        cudaMemcpyHostToDevice, st);
    if (e != cudaSuccess) return cuda_fail(h, e, "tile list upload");
    e = cudaStreamSynchronize(st);  // the host vector must outlive the copy
    if (e != cudaSuccess) return cuda_fail(h, e, "tile list upload");
  }
  if (h->debug) {
    std::vector<uint64_t> table(P.guards.size());
    for (size_t i = 0; i < P.guards.size(); ++i) table[i] = P.guards[i].first;
    if (!table.empty()) e = cudaMemcpy(h->ws + P.off_guard_table, table.data(), table.size() * 8, cudaMemcpyHostToDevice);
    if (e == cudaSuccess) e = arm_guards(h, st);
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    if (e != cudaSuccess) return cuda_fail(h, e, "guard band set-up");
  }
  if (mode == MUON_MODE_BF16) {
    const size_t ng = P.groups.size();
    for (int b = 0; b < 2; ++b) {
      P.map_xk[b].resize(ng);
      P.map_xmn[b].resize(ng);
      P.map_xout[b].resize(ng);
    }
    P.map_gram.resize(ng);
    P.map_poly.resize(ng);
    P.map_gram_out.resize(ng);
    P.map_poly_out.resize(ng);
    for (size_t gg = 0; gg < ng; ++gg) {
      const GroupPlan& g = P.groups[gg];
      muon_status s;
      for (int b = 0; b < 2; ++b) {
        if ((s = encode_map(h, &P.map_xk[b][gg], h->ws + g.off_x[b], g.L, g.s, g.n, g.ld_x, kBK, kHalf))) return s;
        if ((s = encode_map(h, &P.map_xmn[b][gg], h->ws + g.off_x[b], g.L, g.s, g.n, g.ld_x, 64, kBK))) return s;
        if ((s = encode_map(h, &P.map_xout[b][gg], h->ws + g.off_x[b], g.L, g.s, g.n, g.ld_x, kOutBox, kOutBox,
                            CU_TENSOR_MAP_SWIZZLE_64B)))
          return s;
      }
      if ((s = encode_map(h, &P.map_gram[gg], h->ws + g.off_gram, g.s, g.s, g.n, g.ld_s, kBK, kHalf))) return s;
      if ((s = encode_map(h, &P.map_poly[gg], h->ws + g.off_poly, g.s, g.s, g.n, g.ld_s, kBK, kHalf))) return s;
      if ((s = encode_map(h, &P.map_gram_out[gg], h->ws + g.off_gram, g.s, g.s, g.n, g.ld_s, kOutBox, kOutBox,
                          CU_TENSOR_MAP_SWIZZLE_64B)))
        return s;
      if ((s = encode_map(h, &P.map_poly_out[gg], h->ws + g.off_poly, g.s, g.s, g.n, g.ld_s, kOutBox, kOutBox,
                          CU_TENSOR_MAP_SWIZZLE_64B)))
        return s;
    }
  }
  if (tf32x3) {
    const size_t ng = P.groups.size();
    for (int part = 0; part < 2; ++part) {
      for (int b = 0; b < 2; ++b) {
        P.t_xk[part][b].resize(ng);
        P.t_xmn[part][b].resize(ng);
      }
      P.t_gram[part].resize(ng);
      P.t_poly[part].resize(ng);
    }
    const auto sw = CU_TENSOR_MAP_SWIZZLE_128B;
    for (size_t gg = 0; gg < ng; ++gg) {
      const GroupPlan& g = P.groups[gg];
      muon_status s;
      for (int part = 0; part < 2; ++part) {
        for (int b = 0; b < 2; ++b) {
          char* xb = h->ws + (part == 0 ? g.off_x[b] : g.off_xlo[b]);
          if ((s = encode_map(h, &P.t_xk[part][b][gg], xb, g.L, g.s, g.n, g.ld_x, 32, kHalf, sw, true))) return s;
          if ((s = encode_map(h, &P.t_xmn[part][b][gg], xb, g.L, g.s, g.n, g.ld_x, 32, 32,
                              CU_TENSOR_MAP_SWIZZLE_128B_ATOM_32B, true)))
            return s;
        }
        char* gb = h->ws + (part == 0 ? g.off_gram : g.off_gram_lo);
        char* pb = h->ws + (part == 0 ? g.off_poly : g.off_poly_lo);
        if ((s = encode_map(h, &P.t_gram[part][gg], gb, g.s, g.s, g.n, g.ld_s, 32, kHalf, sw, true))) return s;
        if ((s = encode_map(h, &P.t_poly[part][gg], pb, g.s, g.s, g.n, g.ld_s, 32, kHalf, sw, true))) return s;
      }
    }
  }
  P.valid = true;
  if (h->log) {
    size_t n_tiles[3] = {0, 0, 0};
    for (const ChunkPlan& c : P.chunks)
      for (int ph = 0; ph < 3; ++ph) n_tiles[ph] += (size_t)c.n_tiles[ph];
    fprintf(stderr,
            "muon: plan: %d matrices, %zu shape groups, %zu launch chunks, tiles gram/poly/update %zu/%zu/%zu, "
            "workspace %zu bytes (%s mode)\n",
            n, P.groups.size(), P.chunks.size(), n_tiles[0], n_tiles[1], n_tiles[2], P.bytes,
            mode == MUON_MODE_BF16 ? "bf16" : mode == MUON_MODE_FP32_VALIDATE ? "fp32 3xTF32" : "fp32 CUDA-core");
    for (const GroupPlan& g : P.groups) fprintf(stderr, "muon:   group s=%d L=%d n=%d\n", g.s, g.L, g.n);
  }
  return MUON_OK;
}

bool plan_matches(const Plan& P, const int64_t* rows, const int64_t* cols, int n, muon_mode mode) {
  if (!P.valid || P.mode != mode || P.sig.size() != 2 * (size_t)n) return false;
  for (int i = 0; i < n; ++i)
    if (P.sig[2 * i] != rows[i] || P.sig[2 * i + 1] != cols[i]) return false;
  return true;
}

// ------------------------------------------------------------------ launches

struct CallMat {
  void* param;        // param (step) / x_in (Newton-Schulz entry)
  const void* grad;
  float* mom;
  void* out;          // o_out (Newton-Schulz entry)
  bool param_bf16, grad_bf16;
  float lrs;          // fl32(lr * sqrt(max(1, rows/cols)))
  float lrwd;         // fl32(lr * weight_decay)
  float* nstate;      // NorMuon second moments (device, min(rows, cols) floats) or null
};

// Per-call options shared by every matrix.
struct CallOpts {
  float mu = 0.f;
  int nesterov = 0;
  int lerp = 0;
  int cautious = 0;
  const float* coeffs = nullptr;
  int ns_steps = 5;
  float eps = 0.f;
  muon_mode mode = MUON_MODE_BF16;
  int normuon = 0;
  float nb2 = 0.f, neps = 0.f;
};

enum EwPass { kPassMomentum = 0, kPassOut = 1, kPassNormuon = 2 };

void* work_ptr(muon_handle* h, const MatPlan& m, int buf) {
  const Plan& P = h->plan;
  const GroupPlan& g = P.groups[m.group];
  const size_t esz = (P.mode == MUON_MODE_BF16) ? 2 : 4;
  return h->ws + g.off_x[buf] + (size_t)m.idx * g.s * g.ld_x * esz;
}

// Tensor maps of the TMA momentum pass for caller matrix i (tall, bf16 gradient, row
// length a multiple of 8): gradient and momentum in the caller's layout, workspace X =
// U^T (s x L with leading dimension ld).  Written into the handle's cache at slot i.
CUresult encode_ew_maps(muon_handle* h, int i, const EwMat& m) {
  CUtensorMap* out = h->ewmap.data() + (size_t)i * kEwMapsPerMat;
  const cuuint32_t estr[2] = {1, 1};
  auto enc = [&](CUtensorMap* map, CUtensorMapDataType dt, const void* base, uint64_t inner, uint64_t outer,
                 uint64_t stride_bytes, uint32_t box_inner) {
    const cuuint64_t dims[2] = {inner, outer};
    const cuuint64_t strides[1] = {stride_bytes};
    const cuuint32_t box[2] = {box_inner, (cuuint32_t)kEwTile};
    return h->encode(map, dt, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                     CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  };
  const uint64_t rows = (uint64_t)m.rows, cols = (uint64_t)m.cols;
  CUresult r = enc(&out[0], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, m.grad, cols, rows, cols * 2, 64);
  if (r == CUDA_SUCCESS) r = enc(&out[1], CU_TENSOR_MAP_DATA_TYPE_FLOAT32, m.mom, cols, rows, cols * 4, 32);
  if (r == CUDA_SUCCESS) r = enc(&out[2], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, m.work, rows, cols, (uint64_t)m.ld * 2, 64);
  return r;
}

// Momentum pass of one batch in bf16 mode (batch = caller matrices b .. b + n_mats - 1).
// Wide matrices whose workspace copy has the caller's layout go to the bulk-copy kernel
// in units of kFlatUnit contiguous elements; tall ones to the TMA tile kernel, whose
// tensor maps travel by value with the launch (re-encoded only for matrices whose
// pointers changed); matrices that fit neither (fp32 gradients, row lengths not a
// multiple of 8, unaligned buffers) to the register tile kernel.  The norm finalize
// sees every matrix with the unit count of its kernel.
cudaError_t launch_momentum_bf16(muon_handle* h, const EwParams& ep, int b, int* launches, cudaStream_t st) {
  const size_t n_all = h->plan.mats.size();
  if (h->ewmap.size() != n_all * kEwMapsPerMat) {
    h->ewmap.assign(n_all * kEwMapsPerMat, CUtensorMap{});
    h->ewmap_key.assign(n_all * kEwMapsPerMat, nullptr);
  }
  EwParams* flat = new EwParams(ep);
  EwParams* rest = new EwParams(ep);
  EwParams* all = new EwParams(ep);
  const int max_tiled = (ep.n_mats + kMaxTiledPerLaunch - 1) / kMaxTiledPerLaunch;
  EwTiledParams* tiled = new EwTiledParams[max_tiled > 0 ? max_tiled : 1]();
  int n_tiled = 0;
  flat->n_mats = rest->n_mats = 0;
  int uf = 0, ur = 0;
  cudaError_t err = cudaSuccess;
  for (int j = 0; j < ep.n_mats; ++j) {
    const EwMat& m = ep.mats[j];
    const int i = b + j;  // caller index: cache slot of this matrix's maps
    const bool aligned = (reinterpret_cast<uintptr_t>(m.grad) % 16 == 0) &&
                         (reinterpret_cast<uintptr_t>(m.mom) % 16 == 0) &&
                         (reinterpret_cast<uintptr_t>(m.work) % 16 == 0);
    const bool eligible = m.grad_bf16 && m.cols % 8 == 0 && aligned;
    EwMat e = m;
    if (eligible && !m.transposed && m.ld == m.cols) {
      const int64_t numel = (int64_t)m.rows * m.cols;
      e.n_units = (int32_t)((numel + kFlatUnit - 1) / kFlatUnit);
      e.unit_begin = uf;
      uf += e.n_units;
      flat->mats[flat->n_mats++] = e;
    } else if (eligible && m.transposed) {
      const void** key = h->ewmap_key.data() + (size_t)i * kEwMapsPerMat;
      if (key[0] != m.grad || key[1] != m.mom || key[2] != m.work) {
        if (encode_ew_maps(h, i, m) != CUDA_SUCCESS) {
          err = cudaErrorInvalidValue;
          break;
        }
        key[0] = m.grad;
        key[1] = m.mom;
        key[2] = m.work;
      }
      if (n_tiled == 0 || tiled[n_tiled - 1].n_mats == kMaxTiledPerLaunch) {
        EwTiledParams& tp = tiled[n_tiled++];
        tp.mu = ep.mu;
        tp.nesterov = ep.nesterov;
        tp.lerp = ep.lerp;
        tp.omu = ep.omu;
        tp.partials = ep.partials;
        tp.status = ep.status;
      }
      EwTiledParams& tp = tiled[n_tiled - 1];
      std::memcpy(&tp.maps[tp.n_mats * kEwMapsPerMat], &h->ewmap[(size_t)i * kEwMapsPerMat],
                  kEwMapsPerMat * sizeof(CUtensorMap));
      e.unit_begin = tp.total_units;
      tp.total_units += e.n_units;
      tp.mats[tp.n_mats++] = e;
    } else {
      e.unit_begin = ur;
      ur += e.n_units;
      rest->mats[rest->n_mats++] = e;
    }
    all->mats[j].n_units = e.n_units;
  }
  flat->total_units = uf;
  rest->total_units = ur;
  if (err == cudaSuccess) err = launch_momentum_split(*flat, tiled, n_tiled, *rest, *all, h->sm_count, launches, st);
  delete flat;
  delete rest;
  delete all;
  delete[] tiled;
  return err;
}

// Weight-update pass of one batch in bf16 mode (bf16 weights): wide matrices whose
// workspace copy has the caller's layout through the bulk-copy kernel, tall ones through
// the TMA tile kernel (weight and workspace maps by value, re-encoded only when
// pointers change), the others through the register tile kernel.
cudaError_t launch_apply_bf16(muon_handle* h, const EwParams& ep, int b, int* launches, cudaStream_t st) {
  const size_t n_all = h->plan.mats.size();
  if (h->ewmap_apply.size() != n_all * 2) {
    h->ewmap_apply.assign(n_all * 2, CUtensorMap{});
    h->ewmap_apply_key.assign(n_all * 2, nullptr);
  }
  EwParams* flat = new EwParams(ep);
  EwParams* rest = new EwParams(ep);
  const int max_tiled = (ep.n_mats + kMaxTiledPerLaunch - 1) / kMaxTiledPerLaunch;
  EwTiledParams* tiled = new EwTiledParams[max_tiled > 0 ? max_tiled : 1]();
  int n_tiled = 0;
  flat->n_mats = rest->n_mats = 0;
  int uf = 0, ur = 0;
  cudaError_t err = cudaSuccess;
  for (int j = 0; j < ep.n_mats; ++j) {
    const EwMat& m = ep.mats[j];
    const int i = b + j;
    const bool aligned = (reinterpret_cast<uintptr_t>(m.param) % 16 == 0) &&
                         (reinterpret_cast<uintptr_t>(m.work) % 16 == 0);
    const bool eligible = m.param_bf16 && m.cols % 8 == 0 && aligned;
    EwMat e = m;
    if (eligible && !m.transposed && m.ld == m.cols) {
      const int64_t numel = (int64_t)m.rows * m.cols;
      e.n_units = (int32_t)((numel + kApplyUnit - 1) / kApplyUnit);
      e.unit_begin = uf;
      uf += e.n_units;
      flat->mats[flat->n_mats++] = e;
    } else if (eligible && m.transposed) {
      const void** key = h->ewmap_apply_key.data() + (size_t)i * 2;
      CUtensorMap* maps = h->ewmap_apply.data() + (size_t)i * 2;
      if (key[0] != m.param || key[1] != m.work) {
        const cuuint32_t estr[2] = {1, 1};
        const cuuint32_t box[2] = {(cuuint32_t)kEwTile, (cuuint32_t)kEwTile};
        const cuuint64_t wdims[2] = {(cuuint64_t)m.cols, (cuuint64_t)m.rows};
        const cuuint64_t wstr[1] = {(cuuint64_t)m.cols * 2};
        const cuuint64_t xdims[2] = {(cuuint64_t)m.rows, (cuuint64_t)m.cols};
        const cuuint64_t xstr[1] = {(cuuint64_t)m.ld * 2};
        CUresult r = h->encode(&maps[0], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, m.param, wdims, wstr, box, estr,
                               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
        if (r == CUDA_SUCCESS)
          r = h->encode(&maps[1], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, m.work, xdims, xstr, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
        if (r != CUDA_SUCCESS) {
          err = cudaErrorInvalidValue;
          break;
        }
        key[0] = m.param;
        key[1] = m.work;
      }
      if (n_tiled == 0 || tiled[n_tiled - 1].n_mats == kMaxTiledPerLaunch) {
        EwTiledParams& tp = tiled[n_tiled++];
        tp.status = ep.status;
        tp.cautious = ep.cautious;
        tp.normuon = ep.normuon;
        tp.rowsq = ep.rowsq;
      }
      EwTiledParams& tp = tiled[n_tiled - 1];
      std::memcpy(&tp.maps[tp.n_mats * kEwMapsPerMat], maps, 2 * sizeof(CUtensorMap));
      e.unit_begin = tp.total_units;
      tp.total_units += e.n_units;
      tp.mats[tp.n_mats++] = e;
    } else {
      e.unit_begin = ur;
      ur += e.n_units;
      rest->mats[rest->n_mats++] = e;
    }
  }
  flat->total_units = uf;
  rest->total_units = ur;
  if (err == cudaSuccess) err = launch_apply_split(*flat, tiled, n_tiled, *rest, h->sm_count, launches, st);
  delete flat;
  delete rest;
  delete[] tiled;
  return err;
}

muon_status launch_elementwise(muon_handle* h, const std::vector<CallMat>& cm, int pass, int out_kind,
                               int work_buf, const CallOpts& o, cudaStream_t st) {
  const bool momentum_pass = pass == kPassMomentum;
  const float mu = o.mu, eps = o.eps;
  const int nesterov = o.nesterov;
  const Plan& P = h->plan;
  const int n = (int)cm.size();
  const bool f32 = (P.mode != MUON_MODE_BF16);
  for (int b = 0; b < n; b += kMaxMatsPerLaunch) {
    EwParams* ep = new EwParams();
    std::memset(ep, 0, sizeof(EwParams));
    ep->n_mats = std::min(kMaxMatsPerLaunch, n - b);
    ep->mu = mu;
    ep->nesterov = nesterov;
    ep->use_momentum = (momentum_pass && cm[b].mom != nullptr) ? 1 : 0;
    ep->lerp = o.lerp;
    ep->omu = 1.0f - mu;
    ep->cautious = o.cautious;
    ep->normuon = (pass == kPassOut && o.normuon) ? 1 : 0;
    ep->nb2 = o.nb2;
    ep->neps = o.neps;
    ep->rowsq = reinterpret_cast<float*>(h->ws + P.off_rowsq);
    ep->rowf = reinterpret_cast<float*>(h->ws + P.off_rowf);
    ep->eps = eps;
    ep->partials = reinterpret_cast<float*>(h->ws + P.off_partials);
    ep->scale = reinterpret_cast<float*>(h->ws + P.off_scale);
    ep->status = h->dev_status;
    int units = 0;
    for (int j = 0; j < ep->n_mats; ++j) {
      const int i = b + j;
      const MatPlan& m = P.mats[i];
      const GroupPlan& g = P.groups[m.group];
      EwMat& e = ep->mats[j];
      const bool export_pass = !momentum_pass && out_kind == kEwExport;
      e.param = export_pass ? cm[i].out : cm[i].param;
      e.grad = cm[i].grad;
      e.mom = cm[i].mom;
      e.work = work_ptr(h, m, work_buf);
      e.rows = (int32_t)m.rows;
      e.cols = (int32_t)m.cols;
      e.ld = g.ld_x;
      e.tiles_c = m.tiles_c;
      e.unit_begin = units;
      e.gid = g.gid_base + m.idx;
      e.part_base = m.part_base;
      e.n_units = m.n_units;
      e.transposed = m.transposed ? 1 : 0;
      e.vec_ok = (m.cols % 8 == 0) ? 1 : 0;
      e.param_bf16 = cm[i].param_bf16 ? 1 : 0;
      e.grad_bf16 = cm[i].grad_bf16 ? 1 : 0;
      e.lrs = cm[i].lrs;
      e.lrwd = cm[i].lrwd;
      e.nstate = cm[i].nstate;
      e.row_base = m.row_base;
      units += m.n_units;
    }
    ep->total_units = units;
    const int grid = std::max(1, std::min(units, h->sm_count * 8));
    int launches = pass == kPassOut ? 1 : 2;
    prof_begin(h, st, pass == kPassMomentum ? MUON_KIND_MOMENTUM_NORM : MUON_KIND_APPLY);
    cudaError_t err;
    if (pass == kPassMomentum && ep->use_momentum && !f32) {
      err = launch_momentum_bf16(h, *ep, b, &launches, st);
    } else if (pass == kPassOut && out_kind == kEwApply && !f32) {
      err = launch_apply_bf16(h, *ep, b, &launches, st);
    } else {
      err = pass == kPassMomentum ? launch_momentum_norm(*ep, f32, grid, st)
            : pass == kPassNormuon ? launch_normuon(*ep, f32, h->sm_count * 8, st)
                                   : launch_apply(*ep, f32, out_kind, grid, st);
    }
    prof_end(h, pass == kPassMomentum ? MUON_KIND_MOMENTUM_NORM : MUON_KIND_APPLY, st);
    delete ep;
    if (err != cudaSuccess)
      return cuda_fail(h, err, pass == kPassMomentum ? "momentum/norm launch"
                               : pass == kPassNormuon ? "NorMuon launch" : "apply launch");
    h->last_launches += launches;
  }
  return MUON_OK;
}

// True when every chunk's matrices fit one fused weight-update table.
bool can_fuse_apply(const Plan& P) {
  if (P.mode != MUON_MODE_BF16) return false;
  for (const ChunkPlan& ch : P.chunks) {
    const GroupPlan& last = P.groups[ch.g_end - 1];
    if (last.gid_base + last.n - P.groups[ch.g_begin].gid_base > kMaxFusedApply) return false;
  }
  return true;
}

// Fills the handle's fused weight-update table for the matrices of chunk `ch`.
void fill_apply_table(muon_handle* h, const ChunkPlan& ch, const std::vector<CallMat>& fuse_cm, int cautious) {
  const Plan& P = h->plan;
  TcApplyTable& at = *h->apply_table;
  at.base = P.groups[ch.g_begin].gid_base;
  const GroupPlan& last = P.groups[ch.g_end - 1];
  at.n = last.gid_base + last.n - at.base;
  for (int j = 0; j < at.n; ++j) {
    const int i = P.mat_of_gid[at.base + j];
    const CallMat& c = fuse_cm[i];
    const MatPlan& m = P.mats[i];
    TcApply& a = at.m[j];
    a.w = c.param;
    a.lrs = c.lrs;
    a.lrwd = c.lrwd;
    a.flags = (uint16_t)((c.param_bf16 ? kApplyBf16 : 0) | (m.transposed ? kApplyTransposed : 0) |
                         (m.cols % 8 == 0 ? kApplyVec : 0) | (cautious ? kApplyCautious : 0));
    a.pad = 0;
    a.pad2 = 0;
  }
}

// True when the whole Newton-Schulz loop of this plan can run as one persistent launch.
bool can_persist(const Plan& P) {
  return P.mode == MUON_MODE_BF16 && P.chunks.size() == 1 && P.groups.size() <= (size_t)kMaxGroupsPersist;
}

// Launch form for this call: the persistent launch removes the per-phase launches and
// the idle time between phases, which dominates small sets; large sets keep one launch
// per phase (six operand stages instead of five).
bool use_persistent(const muon_handle* h, const Plan& P) {
  if (!can_persist(P)) return false;
  if (h->launch_mode == MUON_LAUNCH_PERSISTENT) return true;
  if (h->launch_mode == MUON_LAUNCH_PER_PHASE) return false;
  double flops = 0.0;  // algorithmic work of one Newton-Schulz step
  for (const GroupPlan& g : P.groups)
    flops += (double)g.n * ((double)g.L * g.s * (g.s + 1) + (double)g.s * g.s * (g.s + 1) + 2.0 * g.L * g.s * g.s);
  return flops < kPersistentMaxFlops;
}

// The whole Newton-Schulz loop as one persistent launch (see TcPersistParams).
muon_status launch_ns_persistent(muon_handle* h, const float* coeffs, int ns_steps,
                                 const std::vector<CallMat>* fuse_cm, int cautious, cudaStream_t st) {
  const Plan& P = h->plan;
  const ChunkPlan& ch = P.chunks[0];
  if (!h->persist) {
    h->persist = new (std::nothrow) TcPersistParams();
    if (!h->persist) return fail(h, MUON_ERR_OOM, "host allocation of the persistent-launch parameters failed");
  }
  TcPersistParams& pp = *h->persist;
  std::memset(&pp, 0, sizeof(pp));
  for (int gg = ch.g_begin; gg < ch.g_end; ++gg) {
    const int li = gg - ch.g_begin;
    const GroupPlan& g = P.groups[gg];
    TcGroup& t = pp.g[li];
    t.s = g.s; t.L = g.L; t.ld_x = g.ld_x; t.ld_s = g.ld_s; t.gid_base = g.gid_base;
    t.x_cur = reinterpret_cast<__nv_bfloat16*>(h->ws + g.off_x[0]);
    t.x_next = reinterpret_cast<__nv_bfloat16*>(h->ws + g.off_x[1]);
    t.gram = reinterpret_cast<__nv_bfloat16*>(h->ws + g.off_gram);
    t.poly = reinterpret_cast<__nv_bfloat16*>(h->ws + g.off_poly);
    for (int b = 0; b < 2; ++b) {
      pp.xk[li][b] = P.map_xk[b][gg];
      pp.xmn[li][b] = P.map_xmn[b][gg];
      pp.xout[li][b] = P.map_xout[b][gg];
    }
    pp.gram[li] = P.map_gram[gg];
    pp.gram_out[li] = P.map_gram_out[gg];
    pp.poly[li] = P.map_poly[gg];
    pp.poly_out[li] = P.map_poly_out[gg];
  }
  const TcTile* dev_tiles = reinterpret_cast<const TcTile*>(h->ws + P.off_tiles);
  pp.tiles_syrk = dev_tiles + ch.off_ptiles[0];
  pp.tiles_upd = dev_tiles + ch.off_ptiles[1];
  pp.n_syrk = ch.n_tiles[kPhaseGram];
  pp.n_upd = ch.n_tiles[kPhaseUpdate];
  pp.ns_steps = ns_steps;
  for (int k = 0; k < ns_steps; ++k) {
    const float* c = coeffs ? coeffs + 3 * k : kDefaultCoeffs;
    pp.ca[k] = c[0];
    pp.cb[k] = c[1];
    pp.cc[k] = c[2];
  }
  pp.scale = reinterpret_cast<const float*>(h->ws + P.off_scale);
  pp.status = h->dev_status;
  pp.queue = reinterpret_cast<unsigned*>(h->ws + P.off_sched);
  pp.done = pp.queue + 1;
  pp.stall_ns = h->stall_ns;
  h->stall_ns = 0;
  if (fuse_cm) fill_apply_table(h, ch, *fuse_cm, cautious);
  const int n_items = ns_steps * (2 * pp.n_syrk + pp.n_upd);
  const int clusters = std::max(1, std::min(tc_persistent_clusters(), n_items));
  prof_begin(h, st, MUON_KIND_NS_PERSISTENT);
  cudaError_t e = cudaMemsetAsync(pp.queue, 0, (size_t)(1 + P.mats.size()) * 4, st);
  if (e == cudaSuccess) e = launch_tc_persistent(pp, fuse_cm ? h->apply_table : nullptr, clusters, st);
  prof_end(h, MUON_KIND_NS_PERSISTENT, st);
  if (e != cudaSuccess) return cuda_fail(h, e, "persistent Newton-Schulz launch");
  h->last_launches += 1;
  return MUON_OK;
}

// fp32 validation mode on the tensor cores (3xTF32): split X0 into its hi and lo parts,
// then one grouped launch per phase and step; the last Update stores X_K unsplit for the
// weight-update / export pass.
muon_status launch_ns_tf32x3(muon_handle* h, const float* coeffs, int ns_steps, cudaStream_t st) {
  const Plan& P = h->plan;
  for (const GroupPlan& g : P.groups) {
    prof_begin(h, st, MUON_KIND_MOMENTUM_NORM);
    cudaError_t e = launch_tf32_split(reinterpret_cast<float*>(h->ws + g.off_x[0]),
                                      reinterpret_cast<float*>(h->ws + g.off_xlo[0]), (size_t)g.n * g.s * g.ld_x, st);
    prof_end(h, MUON_KIND_MOMENTUM_NORM, st);
    if (e != cudaSuccess) return cuda_fail(h, e, "3xTF32 split launch");
    h->last_launches++;
  }
  Tc32Params* tp = new (std::nothrow) Tc32Params();
  if (!tp) return fail(h, MUON_ERR_OOM, "host allocation of the 3xTF32 launch parameters failed");
  auto f = [&](size_t off) { return reinterpret_cast<float*>(h->ws + off); };
  for (int k = 0; k < ns_steps; ++k) {
    const int cur = k & 1;
    const float* c = coeffs ? coeffs + 3 * k : kDefaultCoeffs;
    for (int ph = 0; ph < 3; ++ph) {
      for (const ChunkPlan& ch : P.chunks) {
        std::memset(tp, 0, sizeof(Tc32Params));
        for (int gg = ch.g_begin; gg < ch.g_end; ++gg) {
          const int li = gg - ch.g_begin;
          const GroupPlan& g = P.groups[gg];
          Tc32Group& t = tp->g[li];
          t.s = g.s; t.L = g.L; t.gid_base = g.gid_base;
          const size_t xs = (size_t)g.s * g.ld_x, ss = (size_t)g.s * g.ld_s;
          if (ph == kPhaseGram) {
            tp->a_hi[li] = P.t_xk[0][cur][gg];
            tp->a_lo[li] = P.t_xk[1][cur][gg];
            t.out_hi = f(g.off_gram); t.out_lo = f(g.off_gram_lo); t.ld_out = g.ld_s; t.out_stride = ss;
          } else if (ph == kPhasePoly) {
            tp->a_hi[li] = P.t_gram[0][gg];
            tp->a_lo[li] = P.t_gram[1][gg];
            t.in_hi = f(g.off_gram); t.in_lo = f(g.off_gram_lo); t.ld_in = g.ld_s; t.in_stride = ss;
            t.out_hi = f(g.off_poly); t.out_lo = f(g.off_poly_lo); t.ld_out = g.ld_s; t.out_stride = ss;
          } else {
            tp->a_hi[li] = P.t_poly[0][gg];
            tp->a_lo[li] = P.t_poly[1][gg];
            tp->b_hi[li] = P.t_xmn[0][cur][gg];
            tp->b_lo[li] = P.t_xmn[1][cur][gg];
            t.in_hi = f(g.off_x[cur]); t.in_lo = f(g.off_xlo[cur]); t.ld_in = g.ld_x; t.in_stride = xs;
            t.out_hi = f(g.off_x[cur ^ 1]); t.out_lo = f(g.off_xlo[cur ^ 1]); t.ld_out = g.ld_x; t.out_stride = xs;
          }
        }
        tp->tiles = reinterpret_cast<const TcTile*>(h->ws + P.off_tiles) + ch.off_tiles[ph];
        tp->n_tiles = ch.n_tiles[ph];
        tp->first_iter = (k == 0) ? 1 : 0;
        tp->plain_out = (ph == kPhaseUpdate && k == ns_steps - 1) ? 1 : 0;
        tp->ca = c[0];
        tp->cb = c[1];
        tp->cc = c[2];
        tp->scale = f(P.off_scale);
        tp->status = h->dev_status;
        prof_begin(h, st, MUON_KIND_GRAM + ph);
        const cudaError_t e = launch_tc32(ph, *tp, st);
        prof_end(h, MUON_KIND_GRAM + ph, st);
        if (e != cudaSuccess) {
          delete tp;
          return cuda_fail(h, e, "3xTF32 Newton-Schulz launch");
        }
        h->last_launches++;
      }
    }
  }
  delete tp;
  return MUON_OK;
}

// fuse_cm: caller matrices whose weight update is fused into the last Update pass
// (nullptr: the last pass stores X_K for a separate apply / export pass).
muon_status launch_ns(muon_handle* h, const float* coeffs, int ns_steps, const std::vector<CallMat>* fuse_cm,
                      int cautious, cudaStream_t st) {
  const Plan& P = h->plan;
  if (use_persistent(h, P)) return launch_ns_persistent(h, coeffs, ns_steps, fuse_cm, cautious, st);
  float* scale = reinterpret_cast<float*>(h->ws + P.off_scale);
  if (P.mode == MUON_MODE_FP32_VALIDATE) return launch_ns_tf32x3(h, coeffs, ns_steps, st);
  if (P.mode == MUON_MODE_FP32_SIMT) {
    for (int k = 0; k < ns_steps; ++k) {
      const int cur = k & 1;
      const float* c = coeffs ? coeffs + 3 * k : kDefaultCoeffs;
      for (size_t i = 0; i < P.mats.size(); ++i) {
        const MatPlan& m = P.mats[i];
        const GroupPlan& g = P.groups[m.group];
        F32Mat f;
        f.x_cur = reinterpret_cast<float*>(work_ptr(h, m, cur));
        f.x_next = reinterpret_cast<float*>(work_ptr(h, m, cur ^ 1));
        f.gram = reinterpret_cast<float*>(h->ws + g.off_gram + (size_t)m.idx * g.s * g.ld_s * 4);
        f.poly = reinterpret_cast<float*>(h->ws + g.off_poly + (size_t)m.idx * g.s * g.ld_s * 4);
        f.s = g.s; f.L = g.L; f.ld_x = g.ld_x; f.ld_s = g.ld_s; f.gid = g.gid_base + m.idx;
        prof_begin(h, st, MUON_KIND_GRAM);
        cudaError_t e = launch_f32_gram(f, k == 0, scale, st);
        prof_end(h, MUON_KIND_GRAM, st);
        prof_begin(h, st, MUON_KIND_POLY);
        if (e == cudaSuccess) e = launch_f32_poly(f, c[1], c[2], st);
        prof_end(h, MUON_KIND_POLY, st);
        prof_begin(h, st, MUON_KIND_UPDATE);
        if (e == cudaSuccess) e = launch_f32_update(f, k == 0, scale, c[0], st);
        prof_end(h, MUON_KIND_UPDATE, st);
        if (e != cudaSuccess) return cuda_fail(h, e, "fp32 Newton-Schulz launch");
        h->last_launches += 3;
      }
    }
    return MUON_OK;
  }
  TcParams* tp = new TcParams();
  for (int k = 0; k < ns_steps; ++k) {
    const int cur = k & 1;
    const float* c = coeffs ? coeffs + 3 * k : kDefaultCoeffs;
    for (int ph = 0; ph < 3; ++ph) {
      for (const ChunkPlan& ch : P.chunks) {
        std::memset(tp, 0, sizeof(TcParams));
        for (int gg = ch.g_begin; gg < ch.g_end; ++gg) {
          const int li = gg - ch.g_begin;
          const GroupPlan& g = P.groups[gg];
          TcGroup& t = tp->g[li];
          t.s = g.s; t.L = g.L; t.ld_x = g.ld_x; t.ld_s = g.ld_s; t.gid_base = g.gid_base;
          t.x_cur = reinterpret_cast<__nv_bfloat16*>(h->ws + g.off_x[cur]);
          t.x_next = reinterpret_cast<__nv_bfloat16*>(h->ws + g.off_x[cur ^ 1]);
          t.gram = reinterpret_cast<__nv_bfloat16*>(h->ws + g.off_gram);
          t.poly = reinterpret_cast<__nv_bfloat16*>(h->ws + g.off_poly);
          if (ph == kPhaseGram) {
            tp->map_a[li] = P.map_xk[cur][gg];
            tp->map_out[li] = P.map_gram_out[gg];
          } else if (ph == kPhasePoly) {
            tp->map_a[li] = P.map_gram[gg];
            tp->map_out[li] = P.map_poly_out[gg];
            tp->map_in[li] = P.map_gram_out[gg];
          } else {
            tp->map_a[li] = P.map_poly[gg];
            tp->map_b[li] = P.map_xmn[cur][gg];
            tp->map_out[li] = P.map_xout[cur ^ 1][gg];
            tp->map_in[li] = P.map_xout[cur][gg];
          }
        }
        tp->tiles = reinterpret_cast<const TcTile*>(h->ws + P.off_tiles) + ch.off_tiles[ph];
        tp->n_tiles = ch.n_tiles[ph];
        tp->first_iter = (k == 0) ? 1 : 0;
        tp->ca = c[0];
        tp->cb = c[1];
        tp->cc = c[2];
        tp->scale = scale;
        tp->status = h->dev_status;
        const int clusters = tc_grid_clusters(tp->n_tiles);
        cudaError_t e = cudaSuccess;
        if (fuse_cm && ph == kPhaseUpdate && k == ns_steps - 1) {
          fill_apply_table(h, ch, *fuse_cm, cautious);
          prof_begin(h, st, MUON_KIND_UPDATE_APPLY);
          e = launch_tc_update_apply(*tp, *h->apply_table, clusters, st);
          prof_end(h, MUON_KIND_UPDATE_APPLY, st);
        } else {
          prof_begin(h, st, MUON_KIND_GRAM + ph);
          e = launch_tc(ph, *tp, clusters, st);
          prof_end(h, MUON_KIND_GRAM + ph, st);
        }
        if (e != cudaSuccess) {
          delete tp;
          return cuda_fail(h, e, "tensor-core Newton-Schulz launch");
        }
        h->last_launches++;
      }
    }
  }
  delete tp;
  return MUON_OK;
}

muon_status ensure_status(muon_handle* h) {
  if (h->dev_status) return MUON_OK;
  cudaError_t e = cudaMalloc(&h->dev_status, sizeof(int));
  if (e != cudaSuccess) return fail(h, MUON_ERR_OOM, "status word allocation failed");
  e = cudaMemset(h->dev_status, 0, sizeof(int));
  if (e == cudaSuccess) e = cudaHostAlloc(&h->host_status, sizeof(int), cudaHostAllocDefault);
  if (e == cudaSuccess) e = cudaEventCreateWithFlags(&h->status_event, cudaEventDisableTiming);
  if (e != cudaSuccess) return cuda_fail(h, e, "status set-up");
  *h->host_status = 0;
  return MUON_OK;
}

// Reports a device-side time-out of earlier work, if its status copy has landed.
muon_status poll_status(muon_handle* h, bool wait) {
  if (!h->status_pending) return MUON_OK;
  cudaError_t e = wait ? cudaEventSynchronize(h->status_event) : cudaEventQuery(h->status_event);
  if (e == cudaErrorNotReady) {
    cudaGetLastError();
    return MUON_OK;
  }
  if (e != cudaSuccess) return cuda_fail(h, e, "status event");
  h->status_pending = false;
  if (*h->host_status != kDevOk) {
    *h->host_status = kDevOk;
    cudaMemset(h->dev_status, 0, sizeof(int));
    return fail(h, MUON_ERR_TIMEOUT, "a device-side wait of an earlier call timed out");
  }
  return MUON_OK;
}

muon_status finish_call(muon_handle* h, cudaStream_t st) {
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  cudaStreamIsCapturing(st, &cs);
  if (cs != cudaStreamCaptureStatusNone) return MUON_OK;
  if (h->debug) {
    const muon_status g = check_guards(h, st);
    if (g != MUON_OK) return g;
  }
  cudaError_t e = cudaMemcpyAsync(h->host_status, h->dev_status, sizeof(int), cudaMemcpyDeviceToHost, st);
  if (e == cudaSuccess) e = cudaEventRecord(h->status_event, st);
  if (e != cudaSuccess) return cuda_fail(h, e, "status copy");
  h->status_pending = true;
  return MUON_OK;
}

muon_status run_impl(muon_handle* h, const std::vector<CallMat>& cm, const int64_t* rows, const int64_t* cols,
                     bool step, const CallOpts& o, cudaStream_t st);

muon_status run(muon_handle* h, const std::vector<CallMat>& cm, const int64_t* rows, const int64_t* cols,
                bool step, const CallOpts& o, cudaStream_t st) {
  if (h->nvtx) nvtxRangePushA(step ? "muon_step" : "muon_newton_schulz");
  const muon_status s = run_impl(h, cm, rows, cols, step, o, st);
  if (h->nvtx) nvtxRangePop();
  return s;
}

muon_status run_impl(muon_handle* h, const std::vector<CallMat>& cm, const int64_t* rows, const int64_t* cols,
                     bool step, const CallOpts& o, cudaStream_t st) {
  const float* coeffs = o.coeffs;
  const int ns_steps = o.ns_steps;
  const muon_mode mode = o.mode;
  const int n = (int)cm.size();
  DeviceGuard dg(h->device);
  if (!dg.ok) return fail(h, MUON_ERR_CUDA, "cannot select device %d", h->device);
  muon_status s = ensure_status(h);
  if (s) return s;
  s = poll_status(h, false);
  if (s) return s;
  h->last_launches = 0;
  if (!plan_matches(h->plan, rows, cols, n, mode)) {
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    cudaStreamIsCapturing(st, &cs);
    if (cs != cudaStreamCaptureStatusNone)
      return fail(h, MUON_ERR_INVALID_ARG,
                  "a new list of shapes needs workspace set-up, which cannot run under stream capture");
    if ((s = build_plan(h, rows, cols, n, mode, st))) return s;
  }
  const int final_buf = ns_steps & 1;
  const bool fuse = step && !o.normuon && can_fuse_apply(h->plan);
  if (fuse && !h->apply_table) {
    h->apply_table = new (std::nothrow) TcApplyTable();
    if (!h->apply_table) return fail(h, MUON_ERR_OOM, "host allocation of the weight-update table failed");
  }
  if ((s = launch_elementwise(h, cm, kPassMomentum, 0, 0, o, st))) return s;
  if ((s = launch_ns(h, coeffs, ns_steps, fuse ? &cm : nullptr, o.cautious, st))) return s;
  if (step && o.normuon && (s = launch_elementwise(h, cm, kPassNormuon, 0, final_buf, o, st))) return s;
  if (!fuse && (s = launch_elementwise(h, cm, kPassOut, step ? kEwApply : kEwExport, final_buf, o, st))) return s;
  return finish_call(h, st);
}

}  // namespace

extern "C" {

muon_status muon_init(muon_handle_t* out, int device) {
  if (!out) return MUON_ERR_INVALID_ARG;
  *out = nullptr;
  int count = 0;
  if (cudaGetDeviceCount(&count) != cudaSuccess) {
    cudaGetLastError();
    return MUON_ERR_CUDA;
  }
  if (device < 0 || device >= count) return MUON_ERR_INVALID_ARG;
  cudaDeviceProp prop;
  if (cudaGetDeviceProperties(&prop, device) != cudaSuccess) return MUON_ERR_CUDA;
  if (prop.major != 10 || prop.minor != 0) return MUON_ERR_UNSUPPORTED;
  void* fn = nullptr;
  cudaDriverEntryPointQueryResult q;
  if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
      q != cudaDriverEntryPointSuccess || fn == nullptr)
    return MUON_ERR_CUDA;
  muon_handle* h = new (std::nothrow) muon_handle();
  if (!h) return MUON_ERR_OOM;
  h->device = device;
  h->sm_count = prop.multiProcessorCount;
  h->encode = reinterpret_cast<EncodeTiledFn>(fn);
  const char* lg = getenv("MUON_LOG");
  h->log = lg != nullptr && lg[0] != '\0' && strcmp(lg, "0") != 0;
  const char* dbg = getenv("MUON_DEBUG");
  h->debug = dbg != nullptr && dbg[0] != '\0' && strcmp(dbg, "0") != 0;
  const char* nv = getenv("MUON_NVTX");
  h->nvtx = nv != nullptr && nv[0] != '\0' && strcmp(nv, "0") != 0;
  if (h->log) fprintf(stderr, "muon: handle on device %d (%s, %d SMs)\n", device, prop.name, h->sm_count);
  *out = h;
  return MUON_OK;
}

}  // extern "C"

namespace {

muon_status step_impl(muon_handle_t h, const muon_matrix* mats, int n, float lr, float momentum, int nesterov,
                      int lerp, const float* coeffs, int ns_steps, float eps, muon_mode mode, float weight_decay,
                      int cautious, int normuon, float nb2, float neps, float* const* nstate, void* cuda_stream) {
  if (!h) return MUON_ERR_INVALID_ARG;
  h->err.clear();
  if (!finite(weight_decay) || weight_decay < 0.f)
    return fail(h, MUON_ERR_INVALID_ARG, "weight_decay must be finite and >= 0");
  if (normuon) {
    if (!finite(nb2) || nb2 < 0.f || nb2 >= 1.f)
      return fail(h, MUON_ERR_INVALID_ARG, "normuon_beta2 must lie in [0, 1)");
    if (!finite(neps) || neps <= 0.f) return fail(h, MUON_ERR_INVALID_ARG, "normuon_eps must be finite and > 0");
    if (n > 0 && !nstate) return fail(h, MUON_ERR_INVALID_ARG, "normuon_state is NULL");
  }
  if (n < 0 || n > kMaxMatrices) return fail(h, MUON_ERR_INVALID_ARG, "n = %d outside 0..%d", n, kMaxMatrices);
  if (n == 0) return MUON_OK;
  if (!mats) return fail(h, MUON_ERR_INVALID_ARG, "mats is NULL");
  if (!finite(lr) || lr < 0.f) return fail(h, MUON_ERR_INVALID_ARG, "lr must be finite and >= 0");
  if (!finite(momentum) || momentum < 0.f || momentum >= 1.f)
    return fail(h, MUON_ERR_INVALID_ARG, "momentum must lie in [0, 1)");
  if (!finite(eps) || eps < 0.f) return fail(h, MUON_ERR_INVALID_ARG, "eps must be finite and >= 0");
  if (mode != MUON_MODE_BF16 && mode != MUON_MODE_FP32_VALIDATE && mode != MUON_MODE_FP32_SIMT)
    return fail(h, MUON_ERR_INVALID_ARG, "unknown mode %d", (int)mode);
  muon_status s = check_coeffs(h, coeffs, ns_steps);
  if (s) return s;
  std::vector<Range> ranges;
  std::vector<int64_t> rows(n), cols(n);
  std::vector<CallMat> cm(n);
  for (int i = 0; i < n; ++i) {
    const muon_matrix& m = mats[i];
    if (!m.param || !m.grad || !m.momentum) return fail(h, MUON_ERR_INVALID_ARG, "matrix %d has a NULL pointer", i);
    if (m.rows < 1 || m.cols < 1 || m.rows > kMaxDim || m.cols > kMaxDim)
      return fail(h, MUON_ERR_INVALID_ARG, "matrix %d has shape %lld x %lld", i, (long long)m.rows,
                  (long long)m.cols);
    if ((m.param_dtype != MUON_F32 && m.param_dtype != MUON_BF16) ||
        (m.grad_dtype != MUON_F32 && m.grad_dtype != MUON_BF16))
      return fail(h, MUON_ERR_INVALID_ARG, "matrix %d has an unknown dtype", i);
    if ((reinterpret_cast<uintptr_t>(m.param) | reinterpret_cast<uintptr_t>(m.grad) |
         reinterpret_cast<uintptr_t>(m.momentum)) & 15u)
      return fail(h, MUON_ERR_INVALID_ARG, "matrix %d has a pointer that is not 16-byte aligned", i);
    const uint64_t numel = (uint64_t)m.rows * (uint64_t)m.cols;
    const size_t pb = numel * (m.param_dtype == MUON_BF16 ? 2 : 4);
    const size_t gb = numel * (m.grad_dtype == MUON_BF16 ? 2 : 4);
    ranges.push_back({(uintptr_t)m.param, (uintptr_t)m.param + pb, i});
    ranges.push_back({(uintptr_t)m.grad, (uintptr_t)m.grad + gb, i});
    ranges.push_back({(uintptr_t)m.momentum, (uintptr_t)m.momentum + numel * 4, i});
    rows[i] = m.rows;
    cols[i] = m.cols;
    const double scale = std::sqrt(std::max(1.0, (double)m.rows / (double)m.cols));
    float* ns_ptr = nullptr;
    if (normuon) {
      ns_ptr = nstate[i];
      if (!ns_ptr || (reinterpret_cast<uintptr_t>(ns_ptr) & 15u))
        return fail(h, MUON_ERR_INVALID_ARG, "normuon_state[%d] is NULL or not 16-byte aligned", i);
      const size_t sb = (size_t)std::min(m.rows, m.cols) * 4;
      ranges.push_back({(uintptr_t)ns_ptr, (uintptr_t)ns_ptr + sb, i});
    }
    cm[i] = CallMat{m.param, m.grad, m.momentum, nullptr, m.param_dtype == MUON_BF16, m.grad_dtype == MUON_BF16,
                    (float)((double)lr * scale), (float)((double)lr * (double)weight_decay), ns_ptr};
  }
  if ((s = check_overlaps(h, ranges))) return s;
  {
    std::vector<const void*> ptrs;
    ptrs.reserve((size_t)n * (normuon ? 4 : 3));
    for (int i = 0; i < n; ++i) {
      ptrs.push_back(mats[i].param);
      ptrs.push_back(mats[i].grad);
      ptrs.push_back(mats[i].momentum);
      if (normuon) ptrs.push_back(nstate[i]);
    }
    DeviceGuard dg(h->device);
    if (!dg.ok) return fail(h, MUON_ERR_CUDA, "cannot select device %d", h->device);
    if ((s = check_device_pointers(h, ptrs))) return s;
  }
  mode = fp32_form(mode, rows.data(), cols.data(), n);
  CallOpts o;
  o.mu = momentum;
  o.nesterov = nesterov ? 1 : 0;
  o.lerp = lerp ? 1 : 0;
  o.cautious = cautious ? 1 : 0;
  o.coeffs = coeffs;
  o.ns_steps = ns_steps;
  o.eps = eps;
  o.mode = mode;
  o.normuon = normuon ? 1 : 0;
  o.nb2 = nb2;
  o.neps = neps;
  return run(h, cm, rows.data(), cols.data(), true, o, static_cast<cudaStream_t>(cuda_stream));
}

}  // namespace

extern "C" {

muon_status muon_step(muon_handle_t h, const muon_matrix* mats, int n, float lr, float momentum, int nesterov,
                      const float* coeffs, int ns_steps, float eps, muon_mode mode, void* cuda_stream) {
  return step_impl(h, mats, n, lr, momentum, nesterov, 0, coeffs, ns_steps, eps, mode, 0.f, 0, 0, 0.f, 0.f, nullptr,
                   cuda_stream);
}

muon_status muon_step_ex(muon_handle_t h, const muon_matrix* mats, int n, const muon_options* opt,
                         void* cuda_stream) {
  if (!h) return MUON_ERR_INVALID_ARG;
  if (!opt) return fail(h, MUON_ERR_INVALID_ARG, "options pointer is NULL");
  if (opt->momentum_form != MUON_MOMENTUM_SGD && opt->momentum_form != MUON_MOMENTUM_LERP)
    return fail(h, MUON_ERR_INVALID_ARG, "unknown momentum form %d", (int)opt->momentum_form);
  return step_impl(h, mats, n, opt->lr, opt->momentum, opt->nesterov, opt->momentum_form == MUON_MOMENTUM_LERP,
                   opt->coeffs, opt->ns_steps, opt->eps, opt->mode, opt->weight_decay, opt->cautious, opt->normuon,
                   opt->normuon_beta2, opt->normuon_eps, opt->normuon_state, cuda_stream);
}

muon_status muon_newton_schulz(muon_handle_t h, const void* const* x_in, void* const* o_out, const int64_t* rows,
                               const int64_t* cols, int n, muon_dtype dtype, const float* coeffs, int ns_steps,
                               float eps, muon_mode mode, void* cuda_stream) {
  if (!h) return MUON_ERR_INVALID_ARG;
  h->err.clear();
  if (n < 0 || n > kMaxMatrices) return fail(h, MUON_ERR_INVALID_ARG, "n = %d outside 0..%d", n, kMaxMatrices);
  if (n == 0) return MUON_OK;
  if (!x_in || !o_out || !rows || !cols) return fail(h, MUON_ERR_INVALID_ARG, "NULL array argument");
  if (dtype != MUON_F32 && dtype != MUON_BF16) return fail(h, MUON_ERR_INVALID_ARG, "unknown dtype");
  if (!finite(eps) || eps < 0.f) return fail(h, MUON_ERR_INVALID_ARG, "eps must be finite and >= 0");
  if (mode != MUON_MODE_BF16 && mode != MUON_MODE_FP32_VALIDATE && mode != MUON_MODE_FP32_SIMT)
    return fail(h, MUON_ERR_INVALID_ARG, "unknown mode %d", (int)mode);
  muon_status s = check_coeffs(h, coeffs, ns_steps);
  if (s) return s;
  std::vector<Range> ranges;
  std::vector<CallMat> cm(n);
  const size_t esz = dtype == MUON_BF16 ? 2 : 4;
  for (int i = 0; i < n; ++i) {
    if (!x_in[i] || !o_out[i]) return fail(h, MUON_ERR_INVALID_ARG, "matrix %d has a NULL pointer", i);
    if (rows[i] < 1 || cols[i] < 1 || rows[i] > kMaxDim || cols[i] > kMaxDim)
      return fail(h, MUON_ERR_INVALID_ARG, "matrix %d has shape %lld x %lld", i, (long long)rows[i],
                  (long long)cols[i]);
    if ((reinterpret_cast<uintptr_t>(x_in[i]) | reinterpret_cast<uintptr_t>(o_out[i])) & 15u)
      return fail(h, MUON_ERR_INVALID_ARG, "matrix %d has a pointer that is not 16-byte aligned", i);
    const size_t bytes = (size_t)rows[i] * (size_t)cols[i] * esz;
    ranges.push_back({(uintptr_t)o_out[i], (uintptr_t)o_out[i] + bytes, i});
    cm[i] = CallMat{const_cast<void*>(x_in[i]), nullptr, nullptr, o_out[i], dtype == MUON_BF16, false, 0.f, 0.f,
                    nullptr};
  }
  if ((s = check_overlaps(h, ranges))) return s;
  // outputs must not overlap any input either
  for (int i = 0; i < n; ++i) {
    const uintptr_t lo = (uintptr_t)x_in[i], hi = lo + (size_t)rows[i] * (size_t)cols[i] * esz;
    for (const Range& r : ranges)
      if (lo < r.hi && r.lo < hi)
        return fail(h, MUON_ERR_INVALID_ARG, "output of matrix %d overlaps input of matrix %d", r.mat, i);
  }
  {
    std::vector<const void*> ptrs;
    ptrs.reserve(2 * (size_t)n);
    for (int i = 0; i < n; ++i) {
      ptrs.push_back(x_in[i]);
      ptrs.push_back(o_out[i]);
    }
    DeviceGuard dg(h->device);
    if (!dg.ok) return fail(h, MUON_ERR_CUDA, "cannot select device %d", h->device);
    if ((s = check_device_pointers(h, ptrs))) return s;
  }
  CallOpts o;
  o.coeffs = coeffs;
  o.ns_steps = ns_steps;
  o.eps = eps;
  o.mode = fp32_form(mode, rows, cols, n);
  return run(h, cm, rows, cols, false, o, static_cast<cudaStream_t>(cuda_stream));
}

muon_status muon_selftest_wait_timeout(muon_handle_t h, int64_t limit_ns, void* cuda_stream) {
  if (!h) return MUON_ERR_INVALID_ARG;
  h->err.clear();
  if (limit_ns < 0 || limit_ns > 10000000000ll) return fail(h, MUON_ERR_INVALID_ARG, "limit_ns out of range");
  DeviceGuard dg(h->device);
  if (!dg.ok) return fail(h, MUON_ERR_CUDA, "cannot select device %d", h->device);
  muon_status s = ensure_status(h);
  if (s) return s;
  if ((s = poll_status(h, false))) return s;
  cudaStream_t st = static_cast<cudaStream_t>(cuda_stream);
  cudaError_t e = launch_wait_selftest(h->dev_status, (unsigned long long)limit_ns, st);
  if (e != cudaSuccess) return cuda_fail(h, e, "self-test launch");
  h->last_launches = 1;
  return finish_call(h, st);
}

muon_status muon_set_launch_mode(muon_handle_t h, muon_launch_mode mode) {
  if (!h) return MUON_ERR_INVALID_ARG;
  if (mode != MUON_LAUNCH_AUTO && mode != MUON_LAUNCH_PER_PHASE && mode != MUON_LAUNCH_PERSISTENT)
    return fail(h, MUON_ERR_INVALID_ARG, "unknown launch mode %d", (int)mode);
  h->launch_mode = mode;
  return MUON_OK;
}

muon_status muon_selftest_stall_persistent(muon_handle_t h, int64_t limit_ns) {
  if (!h) return MUON_ERR_INVALID_ARG;
  h->err.clear();
  if (limit_ns <= 0 || limit_ns > 10000000000ll) return fail(h, MUON_ERR_INVALID_ARG, "limit_ns out of range");
  h->stall_ns = (unsigned long long)limit_ns;
  return MUON_OK;
}

muon_status muon_selftest_corrupt_guard(muon_handle_t h) {
  if (!h) return MUON_ERR_INVALID_ARG;
  h->err.clear();
  if (!h->debug || !h->plan.valid || h->plan.guards.empty())
    return fail(h, MUON_ERR_INVALID_ARG, "no guard bands: the handle is not in debug mode or has no workspace yet");
  DeviceGuard dg(h->device);
  if (!dg.ok) return fail(h, MUON_ERR_CUDA, "cannot select device %d", h->device);
  const size_t last = h->plan.guards.size() - 1;
  const cudaError_t e = cudaMemset(h->ws + h->plan.guards[last].first + 3, 0, 1);
  if (e != cudaSuccess) return cuda_fail(h, e, "guard band write");
  return MUON_OK;
}

muon_status muon_selftest_fail_next_alloc(muon_handle_t h) {
  if (!h) return MUON_ERR_INVALID_ARG;
  h->fail_next_alloc = true;
  return MUON_OK;
}

muon_status muon_sync(muon_handle_t h) {
  if (!h) return MUON_ERR_INVALID_ARG;
  DeviceGuard dg(h->device);
  return poll_status(h, true);
}

muon_status muon_profile_enable(muon_handle_t h, int enable) {
  if (!h) return MUON_ERR_INVALID_ARG;
  h->profiling = enable != 0;
  return MUON_OK;
}

muon_status muon_profile_read(muon_handle_t h, double* ms, int64_t* launches) {
  if (!h || !ms || !launches) return MUON_ERR_INVALID_ARG;
  DeviceGuard dg(h->device);
  muon_status st = MUON_OK;
  for (auto& p : h->ev_pending) {
    float t = 0.f;
    cudaError_t e = cudaEventSynchronize(p.b);
    if (e == cudaSuccess) e = cudaEventElapsedTime(&t, p.a, p.b);
    if (e != cudaSuccess) {
      st = cuda_fail(h, e, "profile event");
    } else {
      h->prof_ms[p.kind] += t;
      h->prof_launches[p.kind] += 1;
    }
    h->ev_free.push_back(p.a);
    h->ev_free.push_back(p.b);
  }
  h->ev_pending.clear();
  for (int k = 0; k < MUON_KIND_COUNT; ++k) {
    ms[k] = h->prof_ms[k];
    launches[k] = h->prof_launches[k];
    h->prof_ms[k] = 0.0;
    h->prof_launches[k] = 0;
  }
  return st;
}

int64_t muon_workspace_bytes(muon_handle_t h) { return h ? (int64_t)h->ws_bytes : 0; }

int muon_last_launch_count(muon_handle_t h) { return h ? h->last_launches : 0; }

muon_status muon_destroy(muon_handle_t h) {
  if (!h) return MUON_OK;
  muon_status s = MUON_OK;
  {
    DeviceGuard dg(h->device);
    s = poll_status(h, true);
    if (h->ws) cudaFree(h->ws);
    if (h->dev_status) cudaFree(h->dev_status);
    if (h->host_status) cudaFreeHost(h->host_status);
    if (h->status_event) cudaEventDestroy(h->status_event);

    for (auto& p : h->ev_pending) {
      cudaEventDestroy(p.a);
      cudaEventDestroy(p.b);
    }
    for (cudaEvent_t e : h->ev_free) cudaEventDestroy(e);
  }
  delete h->apply_table;
  delete h->persist;
  delete h;
  return s;
}

const char* muon_status_string(muon_status s) {
  switch (s) {
    case MUON_OK: return "MUON_OK";
    case MUON_ERR_INVALID_ARG: return "MUON_ERR_INVALID_ARG: invalid argument";
    case MUON_ERR_UNSUPPORTED: return "MUON_ERR_UNSUPPORTED: unsupported device or combination";
    case MUON_ERR_OOM: return "MUON_ERR_OOM: device allocation failed";
    case MUON_ERR_CUDA: return "MUON_ERR_CUDA: CUDA call failed";
    case MUON_ERR_TIMEOUT: return "MUON_ERR_TIMEOUT: a device-side wait timed out";
    case MUON_ERR_TOO_LARGE: return "MUON_ERR_TOO_LARGE: matrix exceeds the fixed scratch of the allocation-free entry point";
    case MUON_ERR_CORRUPT: return "MUON_ERR_CORRUPT: a workspace guard band was overwritten (debug mode)";
    default: return "unknown muon_status";
  }
}

const char* muon_last_error(muon_handle_t h) { return h ? h->err.c_str() : ""; }

}  // extern "C"
