// muon_api.cu -- the C ABI: argument validation, the wave / workspace planner,
// tensor-map construction, the launch sequence of one Muon step, AdamW
// dispatch, the device status word and the optional per-kernel profiler.
//
// Launch sequence of muon_step, per wave of matrices (all on the caller's
// stream, no host synchronisation):
//   momentum_norm (per <=256 matrices) -> norm_finalize
//   ns_steps x [ gram -> poly -> axpy ]    (grouped over every shape of the wave)
//   the last axpy applies the cautious update itself (or a separate update
//   kernel with MUON_UNFUSED_UPDATE / ns_steps == 0)
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <vector>

#include "../../include/muon_b200.h"
#include "common.cuh"
#include "elt_params.cuh"

namespace muon {
// kernels (k_elementwise.cu, k_gemm_tc.cu, k_gemm_simt.cu)
int elt_chunk();
int adam_chunk();
cudaError_t launch_momentum_norm(const EltParams& p, int sms, cudaStream_t s);
cudaError_t launch_momentum_bulk(const EltParams& p, int sms, cudaStream_t s);
int bulk_chunks();
cudaError_t launch_momentum_rowq(const EltParams& p, int cls, int sms, cudaStream_t s);
int rowq_class(int cols, bool vec);
cudaError_t launch_norm_finalize(const EltParams& p, cudaStream_t s);
cudaError_t launch_normuon_update(const EltParams& p, int sms, cudaStream_t s);
cudaError_t launch_update(const EltParams& p, bool emit, int sms, cudaStream_t s);
cudaError_t launch_adamw(const AdamParams& p, int sms, cudaStream_t s);
cudaError_t launch_adamw_bulk(const AdamParams& p, int sms, cudaStream_t s);
cudaError_t adamw_status_address(unsigned int** addr);
cudaError_t launch_replicate(const ReplParams& p, int sms, cudaStream_t s);
cudaError_t launch_reduce_mean(const MeanParams& p, int sms, cudaStream_t s);
int repl_chunk();
cudaError_t launch_schedule_advance(DevSched* s, long long total, double wu, double wd, double fin,
                                    cudaStream_t st);
cudaError_t launch_schedule_cosine(DevSched* s, long long total, long long warm, double fin, cudaStream_t st);
int tc_tile_m(bool pair);
int tc_tile_n(bool wide);
int tc_b_box_rows(bool pair);
int tc_bk(bool pair, bool wide);
cudaError_t launch_tc_gemm(const TcGemmParams& p, int epi, bool pair, bool wide, int num_sms, cudaStream_t s);
cudaError_t launch_selftest_wait(unsigned int* status, unsigned long long limit_ns, cudaStream_t s);
int simt_tile();
cudaError_t launch_simt_gemm(const SimtGemmParams& p, int epi, int num_sms, cudaStream_t s);
}  // namespace muon

using namespace muon;

// =========================================================== error state
static thread_local char g_err[512] = "";

static muon_status fail(muon_status st, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err, sizeof(g_err), fmt, ap);
  va_end(ap);
  return st;
}
static muon_status cuda_fail(cudaError_t e, const char* what) {
  return fail(MUON_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

// Lets other translation units of this library set the muon_last_error() text.
void muon_set_last_error(const char* msg) { snprintf(g_err, sizeof(g_err), "%s", msg); }

// ============================================================== profiler
namespace {
enum Kind {
  K_MOMENTUM = 0, K_NORM, K_GRAM, K_POLY, K_AXPY, K_AXPY_UPDATE, K_UPDATE, K_EMIT, K_ADAMW,
  K_GRAM_F32, K_POLY_F32, K_AXPY_F32, K_AXPY_UPDATE_F32, K_NORMUON_UPDATE, K_MOMENTUM_ROWEQ, K_COUNT
};
const char* const kKindNames[K_COUNT] = {
    "momentum_norm", "norm_finalize", "ns_gram", "ns_poly", "ns_axpy", "ns_axpy_update",
    "update", "emit", "adamw", "ns_gram_f32", "ns_poly_f32", "ns_axpy_f32", "ns_axpy_update_f32",
    "normuon_update", "momentum_rowq"};

struct ProfRec {
  int kind;
  cudaEvent_t a, b;
};
std::mutex g_prof_mu;
bool g_prof_on = false;
std::vector<ProfRec> g_recs;
std::vector<cudaEvent_t> g_pool;
double g_ms[K_COUNT];
int64_t g_cnt[K_COUNT];

cudaEvent_t pool_get() {
  if (!g_pool.empty()) {
    cudaEvent_t e = g_pool.back();
    g_pool.pop_back();
    return e;
  }
  cudaEvent_t e = nullptr;
  cudaEventCreate(&e);
  return e;
}

// Wraps one kernel launch: events on its stream when profiling is on.
template <typename F>
cudaError_t timed_launch(int kind, cudaStream_t s, F&& f) {
  bool on;
  {
    std::lock_guard<std::mutex> lk(g_prof_mu);
    on = g_prof_on;
  }
  if (!on) return f();
  cudaEvent_t a, b;
  {
    std::lock_guard<std::mutex> lk(g_prof_mu);
    a = pool_get();
    b = pool_get();
  }
  cudaEventRecord(a, s);
  cudaError_t e = f();
  cudaEventRecord(b, s);
  std::lock_guard<std::mutex> lk(g_prof_mu);
  g_recs.push_back({kind, a, b});
  g_cnt[kind] += 1;
  return e;
}
}  // namespace

// =================================================== driver entry points
namespace {
typedef CUresult (*PFN_encodeTiled_t)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                      const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                      const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                      CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
PFN_encodeTiled_t g_encode = nullptr;
std::once_flag g_encode_once;

PFN_encodeTiled_t get_encode() {
  std::call_once(g_encode_once, [] {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_encode = reinterpret_cast<PFN_encodeTiled_t>(fn);
  });
  return g_encode;
}

struct DevInfo {
  int sms = 0, major = 0, minor = 0;
  bool valid = false;
};
std::mutex g_dev_mu;
DevInfo g_dev[64];

muon_status device_info(DevInfo* out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= 64) return fail(MUON_ERR_UNSUPPORTED, "device index %d out of range", dev);
  std::lock_guard<std::mutex> lk(g_dev_mu);
  if (!g_dev[dev].valid) {
    DevInfo d;
    if ((e = cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess ||
        (e = cudaDeviceGetAttribute(&d.major, cudaDevAttrComputeCapabilityMajor, dev)) != cudaSuccess ||
        (e = cudaDeviceGetAttribute(&d.minor, cudaDevAttrComputeCapabilityMinor, dev)) != cudaSuccess)
      return cuda_fail(e, "cudaDeviceGetAttribute");
    d.valid = true;
    g_dev[dev] = d;
  }
  *out = g_dev[dev];
  if (out->major != 10 || out->minor != 0)
    return fail(MUON_ERR_UNSUPPORTED,
                "compute capability %d.%d: this library is built for sm_100a (compute capability 10.0)",
                out->major, out->minor);
  return MUON_OK;
}
}  // namespace

// ================================================================ planner
namespace {
inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }
inline int round_up_int(int x, int a) { return (x + a - 1) / a * a; }

struct GroupGeom {
  int r, c, m, n, tall, ldc, ldm, esz;
  size_t xstride, bstride;  // bytes per matrix
  long long nblk;           // momentum-kernel blocks per matrix
  long long npart;          // Frobenius partial sums per matrix: one per block, or per row (MuonEq)
};

GroupGeom geom_of(const muon_group& g, bool f32, bool row_eq) {
  GroupGeom q;
  q.r = g.rows;
  q.c = g.cols;
  q.tall = g.rows > g.cols;
  q.m = std::min(g.rows, g.cols);
  q.n = std::max(g.rows, g.cols);
  q.esz = f32 ? 4 : 2;
  q.ldc = round_up_int(g.cols, 8);
  q.ldm = round_up_int(q.m, 8);
  q.xstride = static_cast<size_t>(q.r) * q.ldc * q.esz;
  q.bstride = static_cast<size_t>(q.m) * q.ldm * q.esz;
  const long long numel = static_cast<long long>(g.rows) * g.cols;
  q.nblk = (numel + elt_chunk() - 1) / elt_chunk();
  q.npart = row_eq ? q.r : q.nblk;
  return q;
}

struct WaveItem {
  int g, first, count;  // matrices [first, first+count) of group g (group-relative)
  size_t x0, x1, b;     // byte offsets in the workspace
  int sbase;            // index of the item's first matrix in the wave's scale array
  long long pbase;      // first partial sum of the item's first matrix (wave-relative)
  size_t dsc = 0;       // byte offset of the item's diagonal scales of B' (ldm floats per matrix)
};

struct Wave {
  std::vector<WaveItem> items;
  size_t scales_off = 0, partials_off = 0, total = 0;
  int nmats = 0;
  long long nblocks = 0;  // partial sums of the wave
};

// Lay out a wave and return its byte size.
size_t layout_wave(Wave& w, const std::vector<GroupGeom>& geo) {
  w.nmats = 0;
  w.nblocks = 0;
  for (auto& it : w.items) {
    it.sbase = w.nmats;
    it.pbase = w.nblocks;
    w.nmats += it.count;
    w.nblocks += geo[it.g].npart * it.count;
  }
  size_t off = kWsHeaderBytes;
  w.scales_off = off;
  off = align_up(off + 4ull * w.nmats, 256);
  w.partials_off = off;
  off = align_up(off + 4ull * w.nblocks, 1024);
  for (auto& it : w.items) {
    const GroupGeom& q = geo[it.g];
    it.x0 = off;
    off = align_up(off + q.xstride * it.count, 1024);
    it.x1 = off;
    off = align_up(off + q.xstride * it.count, 1024);
    it.b = off;
    off = align_up(off + q.bstride * it.count, 1024);
    it.dsc = off;
    off = align_up(off + 4ull * q.ldm * it.count, 1024);
  }
  w.total = off;
  return off;
}

muon_status validate_groups(const muon_group* groups, int n_groups) {
  if (n_groups < 0) return fail(MUON_ERR_INVALID_ARG, "n_groups < 0");
  if (n_groups > 0 && !groups) return fail(MUON_ERR_INVALID_ARG, "groups is NULL");
  for (int i = 0; i < n_groups; ++i) {
    const muon_group& g = groups[i];
    if (g.rows <= 0 || g.cols <= 0 || g.count < 0 || g.first < 0)
      return fail(MUON_ERR_INVALID_ARG, "group %d: rows, cols must be > 0, count and first >= 0", i);
    if (g.rows > 65536 || g.cols > 65536 || static_cast<long long>(g.rows) * g.cols >= (1ll << 31))
      return fail(MUON_ERR_INVALID_ARG, "group %d: %d x %d exceeds the supported matrix size", i,
                  g.rows, g.cols);
    if (g.grad_dtype != MUON_F32 && g.grad_dtype != MUON_BF16)
      return fail(MUON_ERR_INVALID_ARG, "group %d: grad_dtype %d unknown", i, g.grad_dtype);
    if (!std::isfinite(g.lr_scale)) return fail(MUON_ERR_INVALID_ARG, "group %d: lr_scale not finite", i);
    if (static_cast<long long>(g.first) + g.count > (1ll << 30))
      return fail(MUON_ERR_INVALID_ARG, "group %d: first + count too large", i);
  }
  // the groups' pointer ranges [first, first + count) must not overlap: one
  // matrix in two groups would be updated twice by concurrent kernels
  std::vector<std::pair<int, int>> ranges;
  for (int i = 0; i < n_groups; ++i)
    if (groups[i].count > 0) ranges.emplace_back(groups[i].first, i);
  std::sort(ranges.begin(), ranges.end());
  for (size_t k = 1; k < ranges.size(); ++k) {
    const muon_group& prev = groups[ranges[k - 1].second];
    if (prev.first + prev.count > ranges[k].first)
      return fail(MUON_ERR_INVALID_ARG, "groups %d and %d index overlapping pointer ranges", ranges[k - 1].second,
                  ranges[k].second);
  }
  return MUON_OK;
}

// Greedy waves: whole groups in order, split only where the workspace runs out.
muon_status plan_waves(const muon_group* groups, int n_groups, bool f32, bool row_eq, size_t ws_bytes,
                       std::vector<GroupGeom>& geo, std::vector<Wave>& waves) {
  geo.clear();
  for (int i = 0; i < n_groups; ++i) geo.push_back(geom_of(groups[i], f32, row_eq));
  waves.clear();
  Wave cur;
  for (int gi = 0; gi < n_groups; ++gi) {
    for (int j = 0; j < groups[gi].count; ++j) {
      Wave trial = cur;
      if (!trial.items.empty() && trial.items.back().g == gi &&
          trial.items.back().count < kMaxUpdMats)
        trial.items.back().count += 1;
      else
        trial.items.push_back({gi, j, 1, 0, 0, 0, 0, 0});
      if (layout_wave(trial, geo) <= ws_bytes) {
        cur = trial;
        continue;
      }
      if (cur.items.empty())
        return fail(MUON_ERR_WORKSPACE, "workspace of %zu bytes cannot hold one %d x %d matrix", ws_bytes,
                    groups[gi].rows, groups[gi].cols);
      layout_wave(cur, geo);
      waves.push_back(cur);
      cur = Wave();
      cur.items.push_back({gi, j, 1, 0, 0, 0, 0, 0});
      if (layout_wave(cur, geo) > ws_bytes)
        return fail(MUON_ERR_WORKSPACE, "workspace of %zu bytes cannot hold one %d x %d matrix", ws_bytes,
                    groups[gi].rows, groups[gi].cols);
    }
  }
  if (!cur.items.empty()) {
    layout_wave(cur, geo);
    waves.push_back(cur);
  }
  return MUON_OK;
}

size_t full_wave_size(const muon_group* groups, int n_groups, bool f32, bool row_eq) {
  std::vector<GroupGeom> geo;
  for (int i = 0; i < n_groups; ++i) geo.push_back(geom_of(groups[i], f32, row_eq));
  Wave w;
  for (int gi = 0; gi < n_groups; ++gi) {
    int left = groups[gi].count, first = 0;
    while (left > 0) {
      const int c = std::min(left, kMaxUpdMats);
      w.items.push_back({gi, first, c, 0, 0, 0, 0, 0});
      first += c;
      left -= c;
    }
  }
  return layout_wave(w, geo);
}

size_t min_wave_size(const muon_group* groups, int n_groups, bool f32, bool row_eq) {
  size_t mx = kWsHeaderBytes;
  std::vector<GroupGeom> geo;
  for (int i = 0; i < n_groups; ++i) geo.push_back(geom_of(groups[i], f32, row_eq));
  for (int gi = 0; gi < n_groups; ++gi) {
    if (groups[gi].count == 0) continue;
    Wave w;
    w.items.push_back({gi, 0, 1, 0, 0, 0, 0, 0});
    mx = std::max(mx, layout_wave(w, geo));
  }
  return mx;
}

inline bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// ------------------------------------------------------------ tensor maps
muon_status make_map(CUtensorMap* map, void* base, int inner, int rows, int batch, size_t row_bytes,
                     size_t batch_bytes, int box_inner, int box_rows,
                     CUtensorMapSwizzle swizzle = CU_TENSOR_MAP_SWIZZLE_128B) {
  PFN_encodeTiled_t enc = get_encode();
  if (!enc) return fail(MUON_ERR_CUDA, "cuTensorMapEncodeTiled entry point unavailable");
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(inner), static_cast<cuuint64_t>(rows),
                        static_cast<cuuint64_t>(batch)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(row_bytes), static_cast<cuuint64_t>(batch_bytes)};
  cuuint32_t box[3] = {static_cast<cuuint32_t>(box_inner), static_cast<cuuint32_t>(box_rows), 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, base, dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS)
    return fail(MUON_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d) for %d x %d x %d", static_cast<int>(r),
                inner, rows, batch);
  return MUON_OK;
}

// A chunked 4-D view (64, rows, inner / 64, batch) of the same buffer: the
// 64-element chunks of a row become a dimension of stride 128 bytes, so one
// box of box_chunks chunks brings several 64-wide column blocks at once.
// Used only where inner is a multiple of 64 and the row pitch equals inner
// (no chunk reaches past a row); chunks beyond the view read as zeros.
muon_status make_map_chunked(CUtensorMap* map, void* base, int inner, int rows, int batch, size_t row_bytes,
                             size_t batch_bytes, int box_rows, int box_chunks) {
  PFN_encodeTiled_t enc = get_encode();
  if (!enc) return fail(MUON_ERR_CUDA, "cuTensorMapEncodeTiled entry point unavailable");
  if (inner % 64 != 0 || row_bytes != static_cast<size_t>(inner) * 2)
    return fail(MUON_ERR_UNSUPPORTED, "chunked tensor map over a ragged or padded row (%d, %zu)", inner, row_bytes);
  cuuint64_t dims[4] = {64, static_cast<cuuint64_t>(rows), static_cast<cuuint64_t>(inner / 64),
                        static_cast<cuuint64_t>(batch)};
  cuuint64_t strides[3] = {static_cast<cuuint64_t>(row_bytes), 128, static_cast<cuuint64_t>(batch_bytes)};
  cuuint32_t box[4] = {64, static_cast<cuuint32_t>(box_rows), static_cast<cuuint32_t>(box_chunks), 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, base, dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS)
    return fail(MUON_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d) for the chunked view of %d x %d x %d",
                static_cast<int>(r), inner, rows, batch);
  return MUON_OK;
}

// ============================================================ step driver
struct StepArgs {
  // muon_step: params/grads/momentum; muon_orthogonalize: grads = inputs, outs
  float* const* params;
  const void* const* grads;
  float* const* momentum;
  float* const* outs;
  const muon_group* groups;
  int n_groups;
  float lr, beta, wd;
  int ns_steps;
  const float* coeffs;
  uint32_t flags;
  char* ws;
  cudaStream_t stream;
  bool orth;  // orthogonaliser mode
  const DevSched* sched;  // device schedule (lr multiplier), or nullptr
  float* const* const* replicas = nullptr;  // [nrep][pointer index]: copies of each param
  int nrep = 0;
};

// MuonEq row equilibration applies to muon_step only (the orthogonaliser has
// no momentum stage).
inline bool row_equilibrate(const StepArgs& a) { return !a.orth && (a.flags & MUON_ROW_EQUILIBRATE) != 0; }

struct Ctx {
  const StepArgs& a;
  const std::vector<GroupGeom>& geo;
  const DevInfo& dev;
};

// MuonEq momentum: one launch per row class (rowq_class: by row width and
// alignment) and grad dtype, at most kMaxMatsPerLaunch matrices each.  Rows
// are numbered per launch; each matrix's partials start at its wave-relative
// first row (pbase), the order norm_finalize reads them in.
muon_status run_momentum_rowq(const Ctx& C, const Wave& w) {
  const StepArgs& a = C.a;
  float* partials = reinterpret_cast<float*>(a.ws + w.partials_off);
  EltParams P;
  std::memset(&P, 0, sizeof(P));
  int pending_dtype = -1;
  auto flush = [&](int cls) -> muon_status {
    if (P.nmats == 0) return MUON_OK;
    P.beta = a.beta;
    P.nesterov = (a.flags & MUON_NESTEROV) ? 1 : 0;
    P.x_f32 = (a.flags & MUON_FP32_DEBUG) ? 1 : 0;
    P.row_eq = 1;
    P.partials = partials;
    P.grad_bf16 = pending_dtype == MUON_BF16;
    cudaError_t e = timed_launch(K_MOMENTUM_ROWEQ, a.stream,
                                 [&] { return launch_momentum_rowq(P, cls, C.dev.sms, a.stream); });
    if (e != cudaSuccess) return cuda_fail(e, "MuonEq momentum launch");
    std::memset(&P, 0, sizeof(P));
    pending_dtype = -1;
    return MUON_OK;
  };
  for (int cls = 0; cls < 4; ++cls) {
    long long pbase = 0;
    for (const auto& it : w.items) {
      const GroupGeom& q = C.geo[it.g];
      const muon_group& g = a.groups[it.g];
      for (int j = 0; j < it.count; ++j, pbase += q.npart) {
        const int pi = g.first + it.first + j;
        const size_t ga = (g.grad_dtype == MUON_BF16) ? 8 : 16;
        const bool vec = (q.c % 4) == 0 && aligned(a.grads[pi], ga) && aligned(a.momentum[pi], 16);
        if (rowq_class(q.c, vec) != cls) continue;
        if (P.nmats == kMaxMatsPerLaunch || (pending_dtype != -1 && pending_dtype != g.grad_dtype)) {
          muon_status st = flush(cls);
          if (st != MUON_OK) return st;
        }
        pending_dtype = g.grad_dtype;
        MatRef& r = P.mats[P.nmats];
        r.rows = q.r;
        r.cols = q.c;
        r.ldx = q.ldc;
        r.sidx = it.sbase + j;
        r.x = a.ws + it.x0 + q.xstride * j;
        r.g = a.grads[pi];
        r.m = a.momentum[pi];
        r.vec = vec ? 1 : 0;
        r.blk_begin = P.total_blocks;  // rows, numbered across the launch
        r.pbase = static_cast<int>(pbase);
        P.total_blocks += q.r;
        P.nmats += 1;
      }
    }
    muon_status st = flush(cls);
    if (st != MUON_OK) return st;
  }
  return MUON_OK;
}

muon_status run_elementwise(const Ctx& C, const Wave& w, int kind) {
  // kind: 0 momentum_norm (row-wise with MuonEq), 1 finalize, 2 update, 3 emit,
  // 4 NorMuon update (row-wise)
  const StepArgs& a = C.a;
  const bool f32 = (a.flags & MUON_FP32_DEBUG) != 0;
  const bool row_eq = row_equilibrate(a);
  if (kind == 0 && row_eq) return run_momentum_rowq(C, w);
  float* scales = reinterpret_cast<float*>(a.ws + w.scales_off);
  float* partials = reinterpret_cast<float*>(a.ws + w.partials_off);
  // matrices of the wave in order, batched <= kMaxMatsPerLaunch per launch and,
  // for the momentum kernel, one grad dtype per launch
  EltParams P;
  std::memset(&P, 0, sizeof(P));
  long long launch_blk0 = 0;  // wave-relative first block of the pending launch
  int pending_dtype = -1;
  // momentum: the bulk-copy kernel when every matrix of the launch allows it
  // (momentum present, bf16 X0 of pitch cols, 16-byte aligned G, m and X0,
  // numel a multiple of 8); it gives the same bits as momentum_norm_kernel
  bool bulk_ok = true;
  auto flush = [&]() -> muon_status {
    if (P.nmats == 0) return MUON_OK;
    P.beta = a.beta;
    P.wd = a.wd;
    P.nesterov = (a.flags & MUON_NESTEROV) ? 1 : 0;
    P.cautious = (a.flags & MUON_CAUTIOUS_WD) ? 1 : 0;
    P.x_f32 = f32 ? 1 : 0;
    P.use_scale = (a.ns_steps == 0) ? 1 : 0;
    P.scales = scales;
    P.sched = a.sched;
    P.row_eq = row_eq ? 1 : 0;
    cudaError_t e = cudaSuccess;
    if (kind == 0) {
      P.partials = partials + launch_blk0;
      P.grad_bf16 = pending_dtype == MUON_BF16;
      P.status = reinterpret_cast<unsigned int*>(a.ws);
      e = timed_launch(K_MOMENTUM, a.stream, [&] {
        return bulk_ok ? launch_momentum_bulk(P, C.dev.sms, a.stream) : launch_momentum_norm(P, C.dev.sms, a.stream);
      });
    } else if (kind == 1) {
      P.partials = partials;
      e = timed_launch(K_NORM, a.stream, [&] { return launch_norm_finalize(P, a.stream); });
    } else if (kind == 4) {
      e = timed_launch(K_NORMUON_UPDATE, a.stream,
                       [&] { return launch_normuon_update(P, C.dev.sms, a.stream); });
    } else {
      e = timed_launch(kind == 2 ? K_UPDATE : K_EMIT, a.stream,
                       [&] { return launch_update(P, kind == 3, C.dev.sms, a.stream); });
    }
    if (e != cudaSuccess) return cuda_fail(e, "elementwise launch");
    launch_blk0 += P.total_blocks;
    std::memset(&P, 0, sizeof(P));
    bulk_ok = true;
    return MUON_OK;
  };
  long long wave_blk = 0;
  for (const auto& it : w.items) {
    const GroupGeom& q = C.geo[it.g];
    const muon_group& g = a.groups[it.g];
    for (int j = 0; j < it.count; ++j) {
      const int pi = g.first + it.first + j;  // pointer-array index
      if (P.nmats == kMaxMatsPerLaunch || (kind == 0 && pending_dtype != -1 && pending_dtype != g.grad_dtype)) {
        muon_status st = flush();
        if (st != MUON_OK) return st;
      }
      if (kind == 0) pending_dtype = g.grad_dtype;
      if (kind == 1 && P.nmats == 0) launch_blk0 = 0;
      MatRef& r = P.mats[P.nmats];
      r.rows = q.r;
      r.cols = q.c;
      r.ldx = q.ldc;
      r.sidx = it.sbase + j;
      r.lr = a.lr * g.lr_scale;
      // X buffer holding this matrix's current iterate
      const int cur = (a.ns_steps % 2 == 0) ? 0 : 1;
      const size_t xoff = (kind <= 1 || cur == 0) ? it.x0 : it.x1;
      r.x = a.ws + xoff + q.xstride * j;
      r.g = a.grads ? a.grads[pi] : nullptr;
      r.m = (!a.orth && a.momentum) ? a.momentum[pi] : nullptr;
      r.w = a.params ? a.params[pi] : nullptr;
      r.out = a.outs ? a.outs[pi] : nullptr;
      const bool c4 = (q.c % 4) == 0;
      if (kind == 0) {
        const size_t ga = (g.grad_dtype == MUON_BF16) ? 8 : 16;
        r.vec = c4 && aligned(r.g, ga) && (!r.m || aligned(r.m, 16));
        r.blk_begin = P.total_blocks;
        P.total_blocks += static_cast<int>(q.nblk);
        const long long numel = static_cast<long long>(q.r) * q.c;
        bulk_ok = bulk_ok && r.m && !f32 && q.ldc == q.c && numel % 8 == 0 && aligned(r.g, 16) &&
                  aligned(r.m, 16) && aligned(r.x, 16);
        r.item_begin = P.total_items;
        P.total_items += static_cast<int>((q.nblk + bulk_chunks() - 1) / bulk_chunks());
      } else if (kind == 1) {
        r.blk_begin = static_cast<int>(wave_blk);
      } else if (kind == 2) {
        r.vec = c4 && aligned(r.w, 16);
        r.blk_begin = P.total_blocks;
        P.total_blocks += static_cast<int>(q.nblk);
      } else if (kind == 4) {
        r.vec = (q.c % 8) == 0 && aligned(r.w, 16);
        r.blk_begin = P.total_blocks;  // rows, numbered across the launch
        P.total_blocks += q.r;
      } else {
        r.vec = c4 && aligned(r.out, 16);
        r.blk_begin = P.total_blocks;
        P.total_blocks += static_cast<int>(q.nblk);
      }
      wave_blk += q.npart;
      P.nmats += 1;
    }
  }
  return flush();
}

// Build and launch one NS product (epi) for every item of the wave.
// Products that may run on 512-column CTA-pair tiles (bit per EpiKind).  The
// wide tile reads 25% fewer operand bytes from L2 per FLOP, so at the same SM
// cycles it draws less power and runs at a higher clock under the 1 kW cap;
// its single 512-column accumulator is drained without overlap.  Measured on
// 8 layers of the 8B shapes: the Gram and B'X (whose epilogue only scales and
// stores) take the same cycles on either tile and less time on the wide one;
// A*A (epilogue reads A) and the fused-update B'X (reads and writes W) take
// 4-40% more time on it.  A problem of those products takes the wide tile
// where its output width is a multiple of 512 (no partly empty tiles) and its
// K at least kWideMinK (the undrained accumulator's epilogue is then a small
// part of each tile); on the d=768 and d=1664 transformer sets, with K of 768
// and 1664 and widths of 768 and 1664, the narrow tile was 13% and 5% faster
// per step.  MUON_TC_NARROW_TILES / MUON_TC_WIDE_TILES force one tile for
// every problem (same bits either way).
#ifndef MUON_TC_WIDE_EPIS
#define MUON_TC_WIDE_EPIS 0x5
#endif
constexpr int kWideMinK = 2048;

muon_status run_gemm(const Ctx& C, const Wave& w, int epi, int k, bool x_in_0) {
  const StepArgs& a = C.a;
  const bool f32 = (a.flags & MUON_FP32_DEBUG) != 0;
  const float ca = a.coeffs[3 * k], cb = a.coeffs[3 * k + 1], cc = a.coeffs[3 * k + 2];
  const float* scales = reinterpret_cast<const float*>(a.ws + w.scales_off);
  const bool pair = (a.flags & MUON_TC_SINGLE_CTA) == 0;
  const bool wide_ok = pair && !f32 && (a.flags & MUON_TC_NARROW_TILES) == 0 && ((MUON_TC_WIDE_EPIS >> epi) & 1);
  const bool wide_all = wide_ok && (a.flags & MUON_TC_WIDE_TILES) != 0;
  // the tile width of one item's problem (see above)
  auto item_wide = [&](const GroupGeom& q) {
    if (!wide_ok) return false;
    if (wide_all) return true;
    const int width = (epi == EPI_GRAM || epi == EPI_POLY) ? q.m : q.c;   // output columns
    const int K = (epi == EPI_GRAM) ? q.n : q.m;
    return width % 512 == 0 && K >= kWideMinK;
  };
  const int BM = f32 ? simt_tile() : tc_tile_m(pair);
  const int b_rows = tc_b_box_rows(pair);
  bool wide = false;   // tile width of the launch being built
  int BN = 0;

  static thread_local TcGemmParams TP;
  static thread_local SimtGemmParams SP;
  int nprob = 0, nw = 0, tiles = 0;
  auto reset = [&] {
    nprob = nw = tiles = 0;
  };
  auto flush = [&]() -> muon_status {
    if (nprob == 0) return MUON_OK;
    cudaError_t e;
    if (f32) {
      SP.nprob = nprob;
      SP.total_tiles = tiles;
      SP.scales = scales;
      SP.wd = a.wd;
      SP.cautious = (a.flags & MUON_CAUTIOUS_WD) ? 1 : 0;
      SP.sched = a.sched;
      const int kind = epi == EPI_GRAM ? K_GRAM_F32 : epi == EPI_POLY ? K_POLY_F32
                     : epi == EPI_AXPY ? K_AXPY_F32 : K_AXPY_UPDATE_F32;
      e = timed_launch(kind, a.stream, [&] { return launch_simt_gemm(SP, epi, C.dev.sms, a.stream); });
    } else {
      TP.nprob = nprob;
      TP.total_tiles = tiles;
      TP.scales = scales;
      TP.status = reinterpret_cast<unsigned int*>(a.ws);
      TP.wd = a.wd;
      TP.cautious = (a.flags & MUON_CAUTIOUS_WD) ? 1 : 0;
      TP.sched = a.sched;
      TP.nrep = (epi == EPI_AXPY_UPDATE) ? a.nrep : 0;
      const int kind = epi == EPI_GRAM ? K_GRAM : epi == EPI_POLY ? K_POLY
                     : epi == EPI_AXPY ? K_AXPY : K_AXPY_UPDATE;
      e = timed_launch(kind, a.stream, [&] { return launch_tc_gemm(TP, epi, pair, wide, C.dev.sms, a.stream); });
    }
    if (e != cudaSuccess) return cuda_fail(e, "NS GEMM launch");
    reset();
    return MUON_OK;
  };

  // two passes: the problems on wide tiles, then those on narrow ones
  for (int pass = 0; pass < 2; ++pass) {
    wide = (pass == 0);
    if (wide && !wide_ok) continue;
    BN = f32 ? simt_tile() : tc_tile_n(wide);
    for (const auto& it : w.items) {
      if (item_wide(C.geo[it.g]) != wide) continue;
      if (nprob == kMaxProblems || nw + it.count > kMaxUpdMats) {
        muon_status st = flush();
        if (st != MUON_OK) return st;
      }
      const GroupGeom& q = C.geo[it.g];
      const muon_group& g = a.groups[it.g];
      char* xcur = a.ws + (x_in_0 ? it.x0 : it.x1);
      char* xoth = a.ws + (x_in_0 ? it.x1 : it.x0);
      char* bbuf = a.ws + it.b;
      const long long xs_el = static_cast<long long>(q.xstride / q.esz);
      const long long bs_el = static_cast<long long>(q.bstride / q.esz);
      GemmProblem P;
      std::memset(&P, 0, sizeof(P));
      P.batch = it.count;
      P.scale_base = it.sbase;
      P.ca = ca;
      P.cb = cb;
      P.cc = cc;
      P.lr = a.lr * g.lr_scale;
      P.w_first = nw;
      // operand / output roles
      if (epi == EPI_GRAM) {
        P.M = P.N = q.m;
        P.K = q.n;
        P.a_mn = P.b_mn = q.tall;
        P.a = P.b = xcur;
        P.a_bs = P.b_bs = xs_el;
        P.a_ld = P.b_ld = q.ldc;
        P.sym = 1;
        P.out = xoth; P.out_bs = xs_el; P.out_ld = q.ldm;   // A lives in the other X buffer
        P.scale_mode = (k == 0) ? 1 : 0;
      } else if (epi == EPI_POLY) {
        P.M = P.N = P.K = q.m;
        P.a = P.b = xoth;
        P.a_bs = P.b_bs = xs_el;
        P.a_ld = P.b_ld = q.ldm;
        P.sym = 1;
        P.out = bbuf; P.out_bs = bs_el; P.out_ld = q.ldm;   // B' = a I + b A + c A A
        P.ein = xoth; P.ein_bs = xs_el; P.ein_ld = q.ldm;
        if (!f32) { P.dsc = reinterpret_cast<float*>(a.ws + it.dsc); P.dsc_bs = q.ldm; }
      } else {
        P.M = q.r;
        P.N = q.c;
        P.K = q.m;
        // a X + B X = B' X with B' = a I + B from the A*A epilogue
        if (!q.tall) {  // X' = B' X : Aop = B' (K-major), Bop = X (MN-major)
          P.a = bbuf; P.a_bs = bs_el; P.a_ld = q.ldm; P.a_mn = 0;
          P.b = xcur; P.b_bs = xs_el; P.b_ld = q.ldc; P.b_mn = 1;
        } else {        // X' = X B' : Aop = X (K-major), Bop = B' (K-major, symmetric)
          P.a = xcur; P.a_bs = xs_el; P.a_ld = q.ldc; P.a_mn = 0;
          P.b = bbuf; P.b_bs = bs_el; P.b_ld = q.ldm; P.b_mn = 0;
        }
        P.out = xoth; P.out_bs = xs_el; P.out_ld = q.ldc;
        P.scale_mode = (k == 0) ? 2 : 0;
        if (!f32) {
          // row (wide) or column (tall) i of the product scaled by
          // B'_ii / bf16(B'_ii): its diagonal term is then exact
          P.dsc = reinterpret_cast<float*>(a.ws + it.dsc); P.dsc_bs = q.ldm; P.dsc_col = q.tall;
        }
      }
      // the tensor-core path stores A and B' in upper form and reads them so;
      // the fp32 scaffold computes and reads full matrices
      if (!f32) {
        if (epi == EPI_POLY) P.a_sym = P.b_sym = 1;
        else if (epi == EPI_AXPY || epi == EPI_AXPY_UPDATE) (q.tall ? P.b_sym : P.a_sym) = 1;
      }
      if (f32) P.sym = 0;
      // B'X of a wide matrix: tile rows fastest, so that B' (m x m, indexed by
      // the tile row) stays in L2 while each X panel streams through once
      P.col_major = (epi == EPI_AXPY || epi == EPI_AXPY_UPDATE) && !q.tall;
      P.tiles_m = (P.M + BM - 1) / BM;
      P.tiles_n = (P.N + BN - 1) / BN;
      if (P.sym) {
        // per tile row, the tiles from its diagonal 256-block to N (the
        // kernel's decode_tile enumerates the same)
        int t = 0;
        for (int I = 0; I < P.tiles_m; ++I) t += (P.N - kSymBlock * ((I * BM) / kSymBlock) + BN - 1) / BN;
        P.tiles_per_mat = t;
      } else {
        P.tiles_per_mat = P.tiles_m * P.tiles_n;
      }
      P.tile_begin = tiles;
      const long long add = static_cast<long long>(P.tiles_per_mat) * it.count;
      if (tiles + add > (1ll << 30)) return fail(MUON_ERR_UNSUPPORTED, "too many tiles in one launch");
      if (!f32) {
        // tensor maps: where every operand row length is a multiple of 64,
        // chunked 4-D views, so that a K-major operand block (op_rows x BK)
        // or an MN-major one (BK k-rows x op_rows) is one box per stage; else
        // the natural 3-D view (inner, rows, batch), one box per 64-wide chunk
        const int bk = tc_bk(pair, wide);
        P.chunked = (q.c % 64 == 0 && q.m % 64 == 0) ? 1 : 0;
        auto map_for = [&](CUtensorMap* m, const void* base, int mn, int inner, int rows, int ld,
                           size_t bstride, int op_rows) {
          if (P.chunked)
            return make_map_chunked(m, const_cast<void*>(base), inner, rows, it.count, static_cast<size_t>(ld) * 2,
                                    bstride, mn ? bk : op_rows, mn ? op_rows / 64 : bk / 64);
          return make_map(m, const_cast<void*>(base), inner, rows, it.count, static_cast<size_t>(ld) * 2,
                          bstride, 64, mn ? bk : op_rows);
        };
        muon_status st;
        // A boxes: 128 rows per CTA; B boxes: the rows of B this CTA stages
        if (epi == EPI_GRAM) {
          st = map_for(&TP.tmA[nprob], xcur, q.tall, q.c, q.r, q.ldc, q.xstride, 128);
          if (st == MUON_OK) st = map_for(&TP.tmB[nprob], xcur, q.tall, q.c, q.r, q.ldc, q.xstride, b_rows);
        } else if (epi == EPI_POLY) {
          // A in upper form: K-major boxes, plus MN-major boxes for its transposed K blocks
          st = map_for(&TP.tmA[nprob], xoth, 0, q.m, q.m, q.ldm, q.xstride, 128);
          if (st == MUON_OK) st = map_for(&TP.tmB[nprob], xoth, 0, q.m, q.m, q.ldm, q.xstride, b_rows);
          if (st == MUON_OK) st = map_for(&TP.tmA2[nprob], xoth, 1, q.m, q.m, q.ldm, q.xstride, 128);
          if (st == MUON_OK) st = map_for(&TP.tmB2[nprob], xoth, 1, q.m, q.m, q.ldm, q.xstride, b_rows);
        } else if (!q.tall) {
          // B' in upper form (A operand here)
          st = map_for(&TP.tmA[nprob], bbuf, 0, q.m, q.m, q.ldm, q.bstride, 128);
          if (st == MUON_OK) st = map_for(&TP.tmB[nprob], xcur, 1, q.c, q.r, q.ldc, q.xstride, b_rows);
          if (st == MUON_OK) st = map_for(&TP.tmA2[nprob], bbuf, 1, q.m, q.m, q.ldm, q.bstride, 128);
        } else {
          // B' in upper form (B operand here)
          st = map_for(&TP.tmA[nprob], xcur, 0, q.c, q.r, q.ldc, q.xstride, 128);
          if (st == MUON_OK) st = map_for(&TP.tmB[nprob], bbuf, 0, q.m, q.m, q.ldm, q.bstride, b_rows);
          if (st == MUON_OK) st = map_for(&TP.tmB2[nprob], bbuf, 1, q.m, q.m, q.ldm, q.bstride, b_rows);
        }
        // Gram and B'X output rows are written by TMA stores of 32 x 32 boxes
        // (64-byte swizzle); A*A and the fused update store directly
        if (st == MUON_OK && (epi == EPI_GRAM || epi == EPI_AXPY)) {
          const bool sq = (epi == EPI_GRAM);
          const int out_inner = sq ? q.m : q.c, out_rows = sq ? q.m : q.r, out_ld = sq ? q.ldm : q.ldc;
          st = make_map(&TP.tmOut[nprob], P.out, out_inner, out_rows, it.count,
                        static_cast<size_t>(out_ld) * 2, q.xstride, 32, 32, CU_TENSOR_MAP_SWIZZLE_64B);
        }
        if (st != MUON_OK) return st;
        TP.prob[nprob] = P;
      } else {
        SP.prob[nprob] = P;
      }
      if (epi == EPI_AXPY_UPDATE) {
        for (int j = 0; j < it.count; ++j) {
          const int pi = g.first + it.first + j;
          if (f32) {
            SP.wptr[nw + j] = a.params[pi];
            SP.wcols[nw + j] = q.c;
          } else {
            TP.wptr[nw + j] = a.params[pi];
            TP.wcols[nw + j] = q.c;
            for (int r = 0; r < a.nrep; ++r) TP.rptr[r][nw + j] = a.replicas[r][pi];
          }
        }
      }
      nw += it.count;
      tiles += static_cast<int>(add);
      nprob += 1;
    }
    muon_status st = flush();
    if (st != MUON_OK) return st;
  }
  return MUON_OK;
}

// dst[r][i] <- params[i] for every matrix of the wave (update paths that do
// not write the copies in their own epilogue).
muon_status run_replicate(const Ctx& C, const Wave& w) {
  const StepArgs& a = C.a;
  ReplParams R;
  std::memset(&R, 0, sizeof(R));
  R.nrep = a.nrep;
  auto flush = [&]() -> muon_status {
    if (R.nmats == 0) return MUON_OK;
    cudaError_t e = launch_replicate(R, C.dev.sms, a.stream);
    if (e != cudaSuccess) return cuda_fail(e, "replicate launch");
    R.nmats = R.total_blocks = 0;
    return MUON_OK;
  };
  for (const auto& it : w.items) {
    const muon_group& g = a.groups[it.g];
    for (int j = 0; j < it.count; ++j) {
      if (R.nmats == kReplMats) {
        muon_status st = flush();
        if (st != MUON_OK) return st;
      }
      const int pi = g.first + it.first + j;
      const long long numel = static_cast<long long>(g.rows) * g.cols;
      R.src[R.nmats] = a.params[pi];
      for (int r = 0; r < a.nrep; ++r) R.dst[r][R.nmats] = a.replicas[r][pi];
      R.numel[R.nmats] = numel;
      R.blk_begin[R.nmats] = R.total_blocks;
      R.total_blocks += static_cast<int>((numel + repl_chunk() - 1) / repl_chunk());
      R.nmats += 1;
    }
  }
  return flush();
}

muon_status run_step(const StepArgs& a, size_t ws_bytes) {
  const bool f32 = (a.flags & MUON_FP32_DEBUG) != 0;
  std::vector<GroupGeom> geo;
  std::vector<Wave> waves;
  const bool normuon = (a.flags & MUON_NORMUON) != 0 && !a.orth;
  muon_status st = plan_waves(a.groups, a.n_groups, f32, row_equilibrate(a), ws_bytes, geo, waves);
  if (st != MUON_OK) return st;
  DevInfo dev;
  if ((st = device_info(&dev)) != MUON_OK) return st;
  cudaError_t e = cudaMemsetAsync(a.ws, 0, 4, a.stream);
  if (e != cudaSuccess) return cuda_fail(e, "status reset");
  Ctx C{a, geo, dev};
  const bool fused = !a.orth && a.ns_steps > 0 && !(a.flags & MUON_UNFUSED_UPDATE) && !normuon;
  for (const Wave& w : waves) {
    if ((st = run_elementwise(C, w, 0)) != MUON_OK) return st;
    if ((st = run_elementwise(C, w, 1)) != MUON_OK) return st;
    bool in0 = true;
    for (int k = 0; k < a.ns_steps; ++k) {
      if ((st = run_gemm(C, w, EPI_GRAM, k, in0)) != MUON_OK) return st;
      if ((st = run_gemm(C, w, EPI_POLY, k, in0)) != MUON_OK) return st;
      const bool last = (k == a.ns_steps - 1);
      if ((st = run_gemm(C, w, (last && fused) ? EPI_AXPY_UPDATE : EPI_AXPY, k, in0)) != MUON_OK) return st;
      in0 = !in0;
    }
    if (a.orth) {
      if ((st = run_elementwise(C, w, 3)) != MUON_OK) return st;
    } else if (!fused) {
      if ((st = run_elementwise(C, w, normuon ? 4 : 2)) != MUON_OK) return st;
    }
    // the tensor-core fused update writes the copies itself
    if (a.nrep > 0 && !(fused && !f32))
      if ((st = run_replicate(C, w)) != MUON_OK) return st;
  }
  return MUON_OK;
}

muon_status validate_common(const muon_group* groups, int n_groups, int ns_steps, const float* coeffs,
                            uint32_t flags, void* workspace, size_t workspace_bytes) {
  muon_status st = validate_groups(groups, n_groups);
  if (st != MUON_OK) return st;
  if (flags & ~(MUON_NESTEROV | MUON_CAUTIOUS_WD | MUON_FP32_DEBUG | MUON_UNFUSED_UPDATE |
                MUON_TC_SINGLE_CTA | MUON_NORMUON | MUON_ROW_EQUILIBRATE | MUON_TC_NARROW_TILES |
                MUON_TC_WIDE_TILES))
    return fail(MUON_ERR_INVALID_ARG, "unknown flag bits 0x%x", flags);
  if (ns_steps < 0 || ns_steps > kMaxNsSteps)
    return fail(MUON_ERR_INVALID_ARG, "ns_steps %d outside [0, %d]", ns_steps, kMaxNsSteps);
  if (ns_steps > 0 && !coeffs) return fail(MUON_ERR_INVALID_ARG, "coeffs is NULL with ns_steps > 0");
  for (int i = 0; i < 3 * ns_steps; ++i)
    if (!std::isfinite(coeffs[i])) return fail(MUON_ERR_INVALID_ARG, "coeffs[%d] not finite", i);
  if (!workspace) return fail(MUON_ERR_WORKSPACE, "workspace is NULL");
  if (!aligned(workspace, 256)) return fail(MUON_ERR_WORKSPACE, "workspace not 256-byte aligned");
  const size_t need = min_wave_size(groups, n_groups, (flags & MUON_FP32_DEBUG) != 0,
                                    (flags & MUON_ROW_EQUILIBRATE) != 0);
  if (workspace_bytes < need)
    return fail(MUON_ERR_WORKSPACE, "workspace of %zu bytes < minimum %zu", workspace_bytes, need);
  return MUON_OK;
}

muon_status validate_ptrs(const char* what, const void* const* arr, const muon_group* groups, int n_groups) {
  if (!arr) return fail(MUON_ERR_INVALID_ARG, "%s array is NULL", what);
  for (int gi = 0; gi < n_groups; ++gi)
    for (int j = 0; j < groups[gi].count; ++j) {
      const void* p = arr[groups[gi].first + j];
      if (!p) return fail(MUON_ERR_INVALID_ARG, "%s[%d] is NULL", what, groups[gi].first + j);
      if (!aligned(p, 16)) return fail(MUON_ERR_INVALID_ARG, "%s[%d] not 16-byte aligned", what, groups[gi].first + j);
    }
  return MUON_OK;
}
}  // namespace

// ============================================================= C entry points
extern "C" {

size_t muon_workspace_size(const muon_group* groups, int n_groups, uint32_t flags) {
  if (validate_groups(groups, n_groups) != MUON_OK) return 0;
  return full_wave_size(groups, n_groups, (flags & MUON_FP32_DEBUG) != 0,
                        (flags & MUON_ROW_EQUILIBRATE) != 0);
}

size_t muon_workspace_min_size(const muon_group* groups, int n_groups, uint32_t flags) {
  if (validate_groups(groups, n_groups) != MUON_OK) return 0;
  return min_wave_size(groups, n_groups, (flags & MUON_FP32_DEBUG) != 0,
                       (flags & MUON_ROW_EQUILIBRATE) != 0);
}

static muon_status muon_step_impl(float* const* params, const void* const* grads,
                                  float* const* momentum, const muon_group* groups, int n_groups,
                                  float lr, float beta, float wd, int ns_steps, const float* coeffs,
                                  uint32_t flags, void* workspace, size_t workspace_bytes,
                                  muon_stream_t stream, const DevSched* sched,
                                  float* const* const* replicas = nullptr, int n_replicas = 0) {
  g_err[0] = '\0';
  muon_status st = validate_common(groups, n_groups, ns_steps, coeffs, flags, workspace, workspace_bytes);
  if (st != MUON_OK) return st;
  if (!std::isfinite(lr) || !std::isfinite(wd)) return fail(MUON_ERR_INVALID_ARG, "lr / wd not finite");
  if (!(beta >= 0.f && beta < 1.f)) return fail(MUON_ERR_INVALID_ARG, "beta %g outside [0, 1)", beta);
  if ((st = validate_ptrs("params", reinterpret_cast<const void* const*>(params), groups, n_groups)) != MUON_OK) return st;
  if ((st = validate_ptrs("grads", grads, groups, n_groups)) != MUON_OK) return st;
  if ((st = validate_ptrs("momentum", reinterpret_cast<const void* const*>(momentum), groups, n_groups)) != MUON_OK) return st;
  if (n_replicas < 0 || n_replicas > kMaxReplicas)
    return fail(MUON_ERR_INVALID_ARG, "n_replicas %d outside [0, %d]", n_replicas, kMaxReplicas);
  if (n_replicas > 0 && !replicas) return fail(MUON_ERR_INVALID_ARG, "replicas is NULL");
  for (int r = 0; r < n_replicas; ++r) {
    char what[32];
    snprintf(what, sizeof(what), "replicas[%d]", r);
    if ((st = validate_ptrs(what, reinterpret_cast<const void* const*>(replicas[r]), groups, n_groups)) != MUON_OK)
      return st;
  }
  StepArgs a{params, grads, momentum, nullptr, groups, n_groups, lr, beta, wd, ns_steps, coeffs,
             flags, static_cast<char*>(workspace), reinterpret_cast<cudaStream_t>(stream), false, sched,
             replicas, n_replicas};
  return run_step(a, workspace_bytes);
}

muon_status muon_step_replicated(float* const* params, const void* const* grads, float* const* momentum,
                                 const muon_group* groups, int n_groups, float lr, float beta, float wd,
                                 int ns_steps, const float* coeffs, uint32_t flags, void* workspace,
                                 size_t workspace_bytes, float* const* const* replicas, int n_replicas,
                                 muon_stream_t stream) {
  return muon_step_impl(params, grads, momentum, groups, n_groups, lr, beta, wd, ns_steps, coeffs,
                        flags, workspace, workspace_bytes, stream, nullptr, replicas, n_replicas);
}

muon_status muon_reduce_mean(void* const* dst, const void* const* const* sources, int n_sources,
                             const int64_t* numel, int count, int32_t dtype, muon_stream_t stream) {
  g_err[0] = '\0';
  if (count < 0) return fail(MUON_ERR_INVALID_ARG, "count < 0");
  if (n_sources < 1 || n_sources > kMaxSources)
    return fail(MUON_ERR_INVALID_ARG, "n_sources %d outside [1, %d]", n_sources, kMaxSources);
  if (dtype != MUON_F32 && dtype != MUON_BF16) return fail(MUON_ERR_INVALID_ARG, "dtype %d unknown", dtype);
  if (count > 0 && (!dst || !sources || !numel)) return fail(MUON_ERR_INVALID_ARG, "dst, sources or numel is NULL");
  for (int r = 0; r < n_sources; ++r)
    if (count > 0 && !sources[r]) return fail(MUON_ERR_INVALID_ARG, "sources[%d] is NULL", r);
  for (int i = 0; i < count; ++i) {
    if (numel[i] < 0 || numel[i] >= (1ll << 40)) return fail(MUON_ERR_INVALID_ARG, "numel[%d] out of range", i);
    if (!dst[i] || !aligned(dst[i], 16)) return fail(MUON_ERR_INVALID_ARG, "dst[%d] NULL or not 16-byte aligned", i);
    for (int r = 0; r < n_sources; ++r)
      if (!sources[r][i] || !aligned(sources[r][i], 16))
        return fail(MUON_ERR_INVALID_ARG, "sources[%d][%d] NULL or not 16-byte aligned", r, i);
  }
  DevInfo dev;
  muon_status st = device_info(&dev);
  if (st != MUON_OK) return st;
  const cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  MeanParams P;
  std::memset(&P, 0, sizeof(P));
  auto flush = [&]() -> muon_status {
    if (P.ntensors == 0) return MUON_OK;
    P.nsrc = n_sources;
    P.bf16 = dtype == MUON_BF16;
    P.inv_n = 1.0f / static_cast<float>(n_sources);
    cudaError_t e = launch_reduce_mean(P, dev.sms, s);
    if (e != cudaSuccess) return cuda_fail(e, "reduce_mean launch");
    std::memset(&P, 0, sizeof(P));
    return MUON_OK;
  };
  for (int i = 0; i < count; ++i) {
    if (numel[i] == 0) continue;
    const long long nblk = (numel[i] + repl_chunk() - 1) / repl_chunk();
    if (P.ntensors == kMeanTensors || P.total_blocks + nblk > (1ll << 30))
      if ((st = flush()) != MUON_OK) return st;
    const int t = P.ntensors;
    for (int r = 0; r < n_sources; ++r) P.src[r][t] = sources[r][i];
    P.dst[t] = dst[i];
    P.numel[t] = numel[i];
    P.blk_begin[t] = P.total_blocks;
    P.total_blocks += static_cast<int>(nblk);
    P.ntensors += 1;
  }
  return flush();
}

muon_status muon_step(float* const* params, const void* const* grads, float* const* momentum,
                      const muon_group* groups, int n_groups, float lr, float beta, float wd,
                      int ns_steps, const float* coeffs, uint32_t flags, void* workspace,
                      size_t workspace_bytes, muon_stream_t stream) {
  return muon_step_impl(params, grads, momentum, groups, n_groups, lr, beta, wd, ns_steps, coeffs,
                        flags, workspace, workspace_bytes, stream, nullptr);
}

muon_status muon_step_scheduled(float* const* params, const void* const* grads,
                                float* const* momentum, const muon_group* groups, int n_groups,
                                float lr, float beta, float wd, int ns_steps, const float* coeffs,
                                uint32_t flags, void* workspace, size_t workspace_bytes,
                                const muon_schedule_state* state, muon_stream_t stream) {
  if (!state || !aligned(state, 8)) {
    g_err[0] = '\0';
    return fail(MUON_ERR_INVALID_ARG, "schedule state is NULL or not 8-byte aligned");
  }
  return muon_step_impl(params, grads, momentum, groups, n_groups, lr, beta, wd, ns_steps, coeffs,
                        flags, workspace, workspace_bytes, stream,
                        reinterpret_cast<const DevSched*>(state));
}

muon_status muon_orthogonalize(const void* const* inputs, float* const* outputs, const muon_group* groups,
                               int n_groups, int ns_steps, const float* coeffs, uint32_t flags,
                               void* workspace, size_t workspace_bytes, muon_stream_t stream) {
  g_err[0] = '\0';
  flags &= (MUON_FP32_DEBUG | MUON_TC_SINGLE_CTA | MUON_TC_NARROW_TILES);
  muon_status st = validate_common(groups, n_groups, ns_steps, coeffs, flags, workspace, workspace_bytes);
  if (st != MUON_OK) return st;
  if ((st = validate_ptrs("inputs", inputs, groups, n_groups)) != MUON_OK) return st;
  if ((st = validate_ptrs("outputs", reinterpret_cast<const void* const*>(outputs), groups, n_groups)) != MUON_OK) return st;
  StepArgs a{nullptr, inputs, nullptr, outputs, groups, n_groups, 0.f, 0.f, 0.f, ns_steps, coeffs,
             flags, static_cast<char*>(workspace), reinterpret_cast<cudaStream_t>(stream), true, nullptr};
  return run_step(a, workspace_bytes);
}

static muon_status adamw_impl(const adamw_group* groups, int n_groups, int64_t step,
                              muon_stream_t stream, const DevSched* sched) {
  g_err[0] = '\0';
  if (n_groups < 0) return fail(MUON_ERR_INVALID_ARG, "n_groups < 0");
  if (n_groups > 0 && !groups) return fail(MUON_ERR_INVALID_ARG, "groups is NULL");
  if (step < 1) return fail(MUON_ERR_INVALID_ARG, "step %lld < 1", static_cast<long long>(step));
  for (int gi = 0; gi < n_groups; ++gi) {
    const adamw_group& g = groups[gi];
    if (g.count < 0) return fail(MUON_ERR_INVALID_ARG, "adamw group %d: count < 0", gi);
    if (g.grad_dtype != MUON_F32 && g.grad_dtype != MUON_BF16)
      return fail(MUON_ERR_INVALID_ARG, "adamw group %d: grad_dtype unknown", gi);
    if (!std::isfinite(g.lr) || !std::isfinite(g.wd) || !std::isfinite(g.eps) || g.eps < 0.f ||
        !(g.beta1 >= 0.f && g.beta1 < 1.f) || !(g.beta2 >= 0.f && g.beta2 < 1.f))
      return fail(MUON_ERR_INVALID_ARG, "adamw group %d: bad hyperparameters", gi);
    if (g.count > 0 && (!g.params || !g.grads || !g.exp_avg || !g.exp_avg_sq || !g.numel))
      return fail(MUON_ERR_INVALID_ARG, "adamw group %d: NULL array", gi);
    for (int i = 0; i < g.count; ++i) {
      if (g.numel[i] < 0) return fail(MUON_ERR_INVALID_ARG, "adamw group %d tensor %d: numel < 0", gi, i);
      if (g.numel[i] == 0) continue;
      const void* ps[4] = {g.params[i], g.grads[i], g.exp_avg[i], g.exp_avg_sq[i]};
      for (const void* p : ps) {
        if (!p) return fail(MUON_ERR_INVALID_ARG, "adamw group %d tensor %d: NULL pointer", gi, i);
        if (!aligned(p, 16)) return fail(MUON_ERR_INVALID_ARG, "adamw group %d tensor %d: not 16-byte aligned", gi, i);
      }
      if (g.numel[i] >= (1ll << 40)) return fail(MUON_ERR_INVALID_ARG, "adamw tensor too large");
    }
  }
  DevInfo dev;
  muon_status st = device_info(&dev);
  if (st != MUON_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  static thread_local AdamParams P;
  const int chunk = adam_chunk();
  for (int dt = 0; dt < 2; ++dt) {
    std::memset(&P, 0, sizeof(P));
    P.grad_bf16 = dt;
    P.sched = sched;
    // the bulk-copy kernel where every tensor of the launch has a multiple of
    // 8 elements (its chunks' byte counts are then multiples of 16); it gives
    // the same bits as adamw_kernel
    bool bulk_ok = true;
    auto flush = [&]() -> muon_status {
      if (P.ntensors == 0) return MUON_OK;
      cudaError_t e = timed_launch(K_ADAMW, s, [&] {
        return bulk_ok ? launch_adamw_bulk(P, dev.sms, s) : launch_adamw(P, dev.sms, s);
      });
      if (e != cudaSuccess) return cuda_fail(e, "adamw launch");
      P.ntensors = 0;
      P.total_blocks = 0;
      P.sched = sched;
      bulk_ok = true;
      return MUON_OK;
    };
    for (int gi = 0; gi < n_groups; ++gi) {
      const adamw_group& g = groups[gi];
      if (g.grad_dtype != dt) continue;
      const double b1 = g.beta1, b2 = g.beta2;
      const double bc1 = 1.0 - std::pow(b1, static_cast<double>(step));
      const double bc2 = 1.0 - std::pow(b2, static_cast<double>(step));
      for (int i = 0; i < g.count; ++i) {
        const long long n = g.numel[i];
        if (n == 0) continue;
        const long long nblk = (n + chunk - 1) / chunk;
        if (P.ntensors == kMaxAdamTensors || P.total_blocks + nblk > (1ll << 30)) {
          if ((st = flush()) != MUON_OK) return st;
        }
        AdamTensor& T = P.t[P.ntensors++];
        T.p = g.params[i];
        T.g = g.grads[i];
        T.m = g.exp_avg[i];
        T.v = g.exp_avg_sq[i];
        T.numel = n;
        T.blk_begin = P.total_blocks;
        T.vec = (n % 4) == 0;
        bulk_ok = bulk_ok && (n % 8) == 0;
        T.decay = static_cast<float>(1.0 - static_cast<double>(g.lr) * g.wd);
        T.b1 = g.beta1;
        T.omb1 = static_cast<float>(1.0 - b1);
        T.b2 = g.beta2;
        T.omb2 = static_cast<float>(1.0 - b2);
        T.step_size = static_cast<float>(g.lr / bc1);
        T.rsqrt_bc2 = static_cast<float>(1.0 / std::sqrt(bc2));
        T.eps = g.eps;
        T.lr = g.lr;
        T.wd = g.wd;
        P.total_blocks += static_cast<int>(nblk);
      }
    }
    if ((st = flush()) != MUON_OK) return st;
  }
  return MUON_OK;
}

muon_status adamw_step(const adamw_group* groups, int n_groups, int64_t step, muon_stream_t stream) {
  return adamw_impl(groups, n_groups, step, stream, nullptr);
}

muon_status adamw_step_scheduled(const adamw_group* groups, int n_groups,
                                 const muon_schedule_state* state, muon_stream_t stream) {
  if (!state || !aligned(state, 8)) {
    g_err[0] = '\0';
    return fail(MUON_ERR_INVALID_ARG, "schedule state is NULL or not 8-byte aligned");
  }
  // the host step only feeds scalars the kernel recomputes from the device state
  return adamw_impl(groups, n_groups, 1, stream, reinterpret_cast<const DevSched*>(state));
}

muon_status muon_schedule_advance(muon_schedule_state* state, int64_t total_steps,
                                  float warmup_frac, float warmdown_frac, float final_frac,
                                  muon_stream_t stream) {
  g_err[0] = '\0';
  if (!state || !aligned(state, 8)) return fail(MUON_ERR_INVALID_ARG, "schedule state is NULL or not 8-byte aligned");
  if (total_steps < 1) return fail(MUON_ERR_INVALID_ARG, "total_steps < 1");
  if (!(warmup_frac >= 0.f && warmdown_frac >= 0.f && warmup_frac + warmdown_frac <= 1.f))
    return fail(MUON_ERR_INVALID_ARG, "warmup/warmdown fractions must be >= 0 and sum to <= 1");
  if (!std::isfinite(final_frac)) return fail(MUON_ERR_INVALID_ARG, "final_frac not finite");
  DevInfo dev;
  muon_status st = device_info(&dev);
  if (st != MUON_OK) return st;
  cudaError_t e = launch_schedule_advance(reinterpret_cast<DevSched*>(state), total_steps, warmup_frac,
                                          warmdown_frac, final_frac, reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "schedule launch");
  return MUON_OK;
}

muon_status muon_schedule_advance_cosine(muon_schedule_state* state, int64_t total_steps,
                                         int64_t warmup_steps, float final_frac, muon_stream_t stream) {
  g_err[0] = '\0';
  if (!state || !aligned(state, 8)) return fail(MUON_ERR_INVALID_ARG, "schedule state is NULL or not 8-byte aligned");
  if (total_steps < 1) return fail(MUON_ERR_INVALID_ARG, "total_steps < 1");
  if (warmup_steps < 0 || warmup_steps > total_steps)
    return fail(MUON_ERR_INVALID_ARG, "warmup_steps must be in [0, total_steps]");
  if (!std::isfinite(final_frac)) return fail(MUON_ERR_INVALID_ARG, "final_frac not finite");
  DevInfo dev;
  muon_status st = device_info(&dev);
  if (st != MUON_OK) return st;
  cudaError_t e = launch_schedule_cosine(reinterpret_cast<DevSched*>(state), total_steps, warmup_steps,
                                         final_frac, reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "schedule launch");
  return MUON_OK;
}

muon_status muon_query_status(const void* workspace, muon_stream_t stream) {
  g_err[0] = '\0';
  if (!workspace) return fail(MUON_ERR_WORKSPACE, "workspace is NULL");
  unsigned int word = 0;
  cudaError_t e = cudaMemcpyAsync(&word, workspace, 4, cudaMemcpyDeviceToHost,
                                  reinterpret_cast<cudaStream_t>(stream));
  if (e == cudaSuccess) e = cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "status read");
  if (word & kDevTimeout) return fail(MUON_ERR_TIMEOUT, "a device-side wait ran out of time");
  return MUON_OK;
}

muon_status adamw_query_status(muon_stream_t stream) {
  g_err[0] = '\0';
  unsigned int* addr = nullptr;
  cudaError_t e = adamw_status_address(&addr);   // looked up per call: the module may be reloaded
  if (e != cudaSuccess) return cuda_fail(e, "adamw status address");
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  unsigned int word = 0;
  e = cudaMemcpyAsync(&word, addr, 4, cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e == cudaSuccess && word != 0) {
    e = cudaMemsetAsync(addr, 0, 4, s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  }
  if (e != cudaSuccess) return cuda_fail(e, "adamw status read");
  if (word & kDevTimeout) return fail(MUON_ERR_TIMEOUT, "a device-side wait in an AdamW step ran out of time");
  return MUON_OK;
}

muon_status muon_selftest_wait_timeout(void* workspace, uint64_t limit_ns, muon_stream_t stream) {
  g_err[0] = '\0';
  if (!workspace) return fail(MUON_ERR_WORKSPACE, "workspace is NULL");
  if (!aligned(workspace, 256)) return fail(MUON_ERR_WORKSPACE, "workspace not 256-byte aligned");
  if (limit_ns < 1000 || limit_ns > 1000000000ull)
    return fail(MUON_ERR_INVALID_ARG, "limit_ns %llu outside [1e3, 1e9]", static_cast<unsigned long long>(limit_ns));
  DevInfo dev;
  muon_status st = device_info(&dev);
  if (st != MUON_OK) return st;
  cudaError_t e = launch_selftest_wait(static_cast<unsigned int*>(workspace), limit_ns,
                                       reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "self-test launch");
  return MUON_OK;
}

const char* muon_status_string(muon_status s) {
  switch (s) {
    case MUON_OK: return "MUON_OK";
    case MUON_ERR_INVALID_ARG: return "MUON_ERR_INVALID_ARG";
    case MUON_ERR_UNSUPPORTED: return "MUON_ERR_UNSUPPORTED";
    case MUON_ERR_WORKSPACE: return "MUON_ERR_WORKSPACE";
    case MUON_ERR_CUDA: return "MUON_ERR_CUDA";
    case MUON_ERR_TIMEOUT: return "MUON_ERR_TIMEOUT";
  }
  return "MUON_ERR_UNKNOWN";
}

const char* muon_last_error(void) { return g_err; }

int muon_profiler_enable(int on) {
  std::lock_guard<std::mutex> lk(g_prof_mu);
  const int prev = g_prof_on ? 1 : 0;
  g_prof_on = on != 0;
  return prev;
}

void muon_profiler_reset(void) {
  std::lock_guard<std::mutex> lk(g_prof_mu);
  for (auto& r : g_recs) {
    cudaEventSynchronize(r.b);
    g_pool.push_back(r.a);
    g_pool.push_back(r.b);
  }
  g_recs.clear();
  for (int k = 0; k < K_COUNT; ++k) g_ms[k] = 0.0, g_cnt[k] = 0;
}

int muon_profiler_read(double* ms_out, int64_t* launches_out, int max_kinds) {
  std::lock_guard<std::mutex> lk(g_prof_mu);
  for (auto& r : g_recs) {
    float ms = 0.f;
    if (cudaEventSynchronize(r.b) == cudaSuccess && cudaEventElapsedTime(&ms, r.a, r.b) == cudaSuccess)
      g_ms[r.kind] += ms;
    g_pool.push_back(r.a);
    g_pool.push_back(r.b);
  }
  g_recs.clear();
  const int n = std::min(max_kinds, static_cast<int>(K_COUNT));
  for (int k = 0; k < n; ++k) {
    if (ms_out) ms_out[k] = g_ms[k];
    if (launches_out) launches_out[k] = g_cnt[k];
  }
  return K_COUNT;
}

int muon_kernel_kind_count(void) { return K_COUNT; }

const char* muon_kernel_kind_name(int kind) {
  return (kind >= 0 && kind < K_COUNT) ? kKindNames[kind] : "";
}

}  // extern "C"
