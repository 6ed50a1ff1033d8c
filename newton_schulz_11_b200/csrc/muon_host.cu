// Host side of the C ABI: argument validation, planning (waves of matrices that fit
// the workspace, shape classes inside a wave, scratch layout, TMA descriptors) and
// the launch sequence of one Muon step.
//
// Launch sequence per wave (all on the caller's stream, no host synchronisation):
//   elementwise (momentum, Nesterov input, hi/lo split, chunk sums of squares)
//   norm finalisation (s = 1 / (||u|| + eps) per matrix)
//   for k in 0 .. ns_steps-1:  Gram -> polynomial -> apply   (the last apply also
//                              updates W and/or writes O)
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstring>
#include <list>
#include <mutex>
#include <vector>

#include "muon_b200.h"
#include "muon_params.h"

namespace muon {
cudaError_t launch_momentum(const EwParams& p, cudaStream_t stream);
cudaError_t launch_norm(const EwParams& p, cudaStream_t stream);
cudaError_t launch_gemm(int mode, const GemmParams* p, int max_pairs, cudaStream_t stream);
int gemm_tile_rows();
int gemm_tile_cols();
}  // namespace muon

namespace {
using namespace muon;

static_assert(sizeof(muon_matrix_t) == 80, "muon_matrix_t layout");
static_assert(sizeof(FinalParams) < 32000, "kernel parameter block too large");
static_assert(sizeof(EwParams) < 32000, "kernel parameter block too large");

constexpr size_t kHeaderBytes = 256;
constexpr size_t kBufAlign = 1024;
constexpr int64_t kChunkElems = 16384;
constexpr int64_t kMaxSide = int64_t(1) << 24;
constexpr int kStagedApplyMaxM = 1024;  // Gram side up to which the staged (64-deep) variants serve

std::atomic<long long> g_timeout_us{2000000};

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }
int64_t round8(int64_t x) { return (x + 7) / 8 * 8; }
int64_t round16(int64_t x) { return (x + 15) / 16 * 16; }
int cdiv(int64_t a, int64_t b) { return static_cast<int>((a + b - 1) / b); }

// ---------------------------------------------------------------- device facts

struct DeviceFacts {
  bool probed = false;
  bool supported = false;
  int sm_count = 0;
};

std::mutex g_dev_mu;
std::vector<DeviceFacts> g_dev;

muon_status_t current_device(int* dev, int* sms) {
  if (cudaGetDevice(dev) != cudaSuccess) return MUON_ERR_NO_DEVICE;
  std::lock_guard<std::mutex> lk(g_dev_mu);
  if (static_cast<int>(g_dev.size()) <= *dev) g_dev.resize(*dev + 1);
  DeviceFacts& f = g_dev[*dev];
  if (!f.probed) {
    int major = 0, minor = 0, count = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, *dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, *dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&count, cudaDevAttrMultiProcessorCount, *dev) != cudaSuccess)
      return MUON_ERR_CUDA;
    f.probed = true;
    f.supported = (major == 10 && minor == 0);
    f.sm_count = count;
  }
  if (!f.supported) return MUON_ERR_NO_DEVICE;
  *sms = f.sm_count;
  return MUON_OK;
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// 3-D bf16 map over `count` matrices of rows x cols (row stride ld elements), boxes of
// 64 columns x box_rows rows, 128-byte swizzle, zero fill outside the matrix.
bool encode_map(CUtensorMap* map, void* base, int64_t count, int64_t rows, int64_t cols, int64_t ld,
                uint32_t box_rows) {
  auto fn = encode_fn();
  if (fn == nullptr) return false;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows),
                        static_cast<cuuint64_t>(count)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(ld * 2), static_cast<cuuint64_t>(ld * rows * 2)};
  cuuint32_t box[3] = {static_cast<cuuint32_t>(kBox), box_rows, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, base, dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// The 8-bit lo buffer: 64 x 128 boxes (64 bytes of a row, 128 rows), 64-byte swizzle.
bool encode_map_lo(CUtensorMap* map, void* base, int64_t count, int64_t rows, int64_t cols, int64_t ldl) {
  auto fn = encode_fn();
  if (fn == nullptr) return false;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows),
                        static_cast<cuuint64_t>(count)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(ldl), static_cast<cuuint64_t>(ldl * rows)};
  cuuint32_t box[3] = {64, 128, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, base, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
            CU_TENSOR_MAP_SWIZZLE_64B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// ---------------------------------------------------------------- per-kernel timing

struct Profiler {
  bool on = false;
  std::vector<std::pair<cudaEvent_t, cudaEvent_t>> pool;  // reused across sessions
  std::vector<int> kinds;                                 // kind of each recorded pair
  size_t used = 0;
};
Profiler g_prof;

// Records the start event of a launch of `kind`; returns the pair index or -1.
int prof_start(int kind, cudaStream_t s) {
  if (!g_prof.on) return -1;
  if (g_prof.used == g_prof.pool.size()) {
    cudaEvent_t a, b;
    if (cudaEventCreate(&a) != cudaSuccess) return -1;
    if (cudaEventCreate(&b) != cudaSuccess) {
      cudaEventDestroy(a);
      return -1;
    }
    g_prof.pool.emplace_back(a, b);
  }
  const int i = static_cast<int>(g_prof.used++);
  if (static_cast<int>(g_prof.kinds.size()) <= i) g_prof.kinds.resize(i + 1);
  g_prof.kinds[i] = kind;
  cudaEventRecord(g_prof.pool[i].first, s);
  return i;
}

void prof_stop(int i, cudaStream_t s) {
  if (i >= 0) cudaEventRecord(g_prof.pool[i].second, s);
}

// ---------------------------------------------------------------- validation

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// A strided 2-D region of memory: `rows` rows of `width` bytes, `pitch` bytes apart.
struct Range {
  uintptr_t lo, hi;  // first byte, one past the last byte
  uintptr_t pitch, width;
  int64_t rows;
  bool written;
};

void add_range(std::vector<Range>& v, const void* base, int64_t rows, int64_t cols, int64_t ld, size_t elt,
               bool written) {
  const uintptr_t lo = reinterpret_cast<uintptr_t>(base);
  const uintptr_t hi = lo + static_cast<uintptr_t>(((rows - 1) * ld + cols) * static_cast<int64_t>(elt));
  v.push_back({lo, hi, static_cast<uintptr_t>(ld) * elt, static_cast<uintptr_t>(cols) * elt, rows, written});
}

// Whether two regions whose byte spans overlap share a byte.  Regions with the same pitch
// (sub-blocks of one matrix, e.g. per-head column blocks) are tested exactly: row by row
// in the frame of the one that starts first.  Other pairs count as sharing.
bool regions_share_bytes(const Range& a, const Range& b) {
  const Range& x = a.lo <= b.lo ? a : b;
  const Range& y = a.lo <= b.lo ? b : a;
  if (x.pitch != y.pitch || x.width > x.pitch || y.width > y.pitch) return true;
  const uintptr_t d = y.lo - x.lo;
  const int64_t q = static_cast<int64_t>(d / x.pitch);  // y's first row, in x's rows
  const uintptr_t off = d % x.pitch;                     // y's column offset in bytes
  auto rows_meet = [&](int64_t first) { return first < x.rows && first + y.rows > 0; };
  // the part of each y row that lies in parent row q + k
  if (off < x.width && rows_meet(q)) return true;
  // the part that spills into parent row q + k + 1 (starting at column 0)
  if (off + y.width > x.pitch && rows_meet(q + 1)) return true;
  return false;
}

muon_status_t validate(const muon_matrix_t* mats, int n, bool ns_only) {
  if (mats == nullptr || n < 1) return MUON_ERR_INVALID_ARG;
  std::vector<Range> ranges;
  ranges.reserve(static_cast<size_t>(n) * 4);
  for (int i = 0; i < n; ++i) {
    const muon_matrix_t& t = mats[i];
    if (t.rows < 1 || t.cols < 1 || t.rows > kMaxSide || t.cols > kMaxSide) return MUON_ERR_UNSUPPORTED_SHAPE;
    if (t.grad == nullptr) return MUON_ERR_INVALID_ARG;
    if (t.ld_grad < t.cols) return MUON_ERR_UNSUPPORTED_SHAPE;
    if (!aligned(t.grad, 4)) return MUON_ERR_ALIGNMENT;
    if (!std::isfinite(t.shape_scale)) return MUON_ERR_INVALID_ARG;
    add_range(ranges, t.grad, t.rows, t.cols, t.ld_grad, 4, false);
    if (t.out_update != nullptr) {
      if (!aligned(t.out_update, 4)) return MUON_ERR_ALIGNMENT;
      add_range(ranges, t.out_update, t.rows, t.cols, t.cols, 4, true);
    } else if (ns_only) {
      return MUON_ERR_INVALID_ARG;
    }
    if (ns_only) continue;
    if (t.param == nullptr || t.momentum == nullptr) return MUON_ERR_INVALID_ARG;
    if (t.param_dtype != MUON_F32 && t.param_dtype != MUON_BF16) return MUON_ERR_UNSUPPORTED_DTYPE;
    const size_t pe = t.param_dtype == MUON_F32 ? 4 : 2;
    if (t.ld_param < t.cols || t.ld_mom < t.cols) return MUON_ERR_UNSUPPORTED_SHAPE;
    if (!aligned(t.param, pe) || !aligned(t.momentum, 4)) return MUON_ERR_ALIGNMENT;
    add_range(ranges, t.param, t.rows, t.cols, t.ld_param, pe, true);
    add_range(ranges, t.momentum, t.rows, t.cols, t.ld_mom, 4, true);
  }
  // No written buffer may share a byte with any other buffer.  Pairs whose byte spans
  // overlap are tested exactly (blocks of one matrix interleave without sharing bytes).
  std::sort(ranges.begin(), ranges.end(), [](const Range& a, const Range& b) { return a.lo < b.lo; });
  for (size_t i = 0; i < ranges.size(); ++i)
    for (size_t j = i + 1; j < ranges.size() && ranges[j].lo < ranges[i].hi; ++j)
      if ((ranges[i].written || ranges[j].written) && regions_share_bytes(ranges[i], ranges[j]))
        return MUON_ERR_INVALID_ARG;
  return MUON_OK;
}

muon_status_t validate_hyper(float lr, float beta, float wd, int nesterov, int ns_steps, const float* coeffs,
                             float eps) {
  if (!(std::isfinite(lr) && lr >= 0.f)) return MUON_ERR_INVALID_ARG;
  if (!(std::isfinite(beta) && beta >= 0.f && beta <= 1.f)) return MUON_ERR_INVALID_ARG;
  if (!(std::isfinite(wd) && wd >= 0.f)) return MUON_ERR_INVALID_ARG;
  if (nesterov != 0 && nesterov != 1) return MUON_ERR_INVALID_ARG;
  if (ns_steps < 1 || ns_steps > MUON_MAX_NS_STEPS || coeffs == nullptr) return MUON_ERR_INVALID_ARG;
  for (int k = 0; k < 3 * ns_steps; ++k)
    if (!std::isfinite(coeffs[k])) return MUON_ERR_INVALID_ARG;
  if (!(std::isfinite(eps) && eps > 0.f)) return MUON_ERR_INVALID_ARG;
  return MUON_OK;
}

// ---------------------------------------------------------------- planning

struct ClassPlan {
  int64_t rows = 0, cols = 0, m = 0, n = 0, ldx = 0, lda = 0;
  int64_t ldl = 0;  // row stride of the 8-bit lo buffer (bytes, multiple of 16)
  int tall = 0;
  std::vector<int> mats;  // global indices
  size_t off_hi[2] = {0, 0}, off_lo = 0, off_a = 0, off_b = 0;
};

struct WavePlan {
  std::vector<int> order;  // global index of each wave-local matrix (class by class)
  std::vector<ClassPlan> classes;
  std::vector<int> rows_per_chunk, nchunks, chunk_begin;
  int total_chunks = 0;
  size_t off_scale = 0, off_norm = 0, off_partials = 0, bytes = 0;
};

int rows_per_chunk_for(int64_t rows, int64_t cols) {
  return static_cast<int>(std::max<int64_t>(1, std::min<int64_t>(rows, kChunkElems / std::max<int64_t>(cols, 1))));
}

// Lays out the scratch of one wave (matrices `idx`, in call order) and returns its size.
WavePlan layout_wave(const muon_matrix_t* mats, const std::vector<int>& idx) {
  WavePlan w;
  for (int i : idx) {
    const muon_matrix_t& t = mats[i];
    ClassPlan* c = nullptr;
    for (auto& cp : w.classes)
      if (cp.rows == t.rows && cp.cols == t.cols) c = &cp;
    if (c == nullptr) {
      w.classes.emplace_back();
      c = &w.classes.back();
      c->rows = t.rows;
      c->cols = t.cols;
      c->m = std::min(t.rows, t.cols);
      c->n = std::max(t.rows, t.cols);
      c->tall = t.rows > t.cols ? 1 : 0;
      c->ldx = round8(t.cols);
      c->ldl = round16(t.cols);
      c->lda = round8(c->m);
    }
    c->mats.push_back(i);
  }
  for (auto& c : w.classes)
    for (int i : c.mats) w.order.push_back(i);
  const int nw = static_cast<int>(w.order.size());
  for (int i : w.order) {
    const int rpc = rows_per_chunk_for(mats[i].rows, mats[i].cols);
    w.rows_per_chunk.push_back(rpc);
    w.chunk_begin.push_back(w.total_chunks);
    w.nchunks.push_back(cdiv(mats[i].rows, rpc));
    w.total_chunks += w.nchunks.back();
  }
  size_t off = kHeaderBytes;
  w.off_scale = off;
  off = align_up(off + 4 * nw, 256);
  w.off_norm = off;
  off = align_up(off + 4 * nw, 256);
  w.off_partials = off;
  off = align_up(off + 4 * static_cast<size_t>(w.total_chunks), kBufAlign);
  for (auto& c : w.classes) {
    const size_t xb = static_cast<size_t>(c.mats.size()) * c.rows * c.ldx * 2;
    const size_t lb = static_cast<size_t>(c.mats.size()) * c.rows * c.ldl;
    const size_t ab = static_cast<size_t>(c.mats.size()) * c.m * c.lda * 2;
    c.off_hi[0] = off;
    off = align_up(off + xb, kBufAlign);
    c.off_hi[1] = off;
    off = align_up(off + xb, kBufAlign);
    c.off_lo = off;
    off = align_up(off + lb, kBufAlign);
    c.off_a = off;
    off = align_up(off + ab, kBufAlign);
    c.off_b = off;
    off = align_up(off + ab, kBufAlign);
  }
  w.bytes = off;
  return w;
}

// Greedy waves in call order: a wave closes when adding the next matrix would exceed
// the matrix or shape-class limit, or the workspace.
muon_status_t form_waves(const muon_matrix_t* mats, int n, size_t ws_limit, std::vector<WavePlan>* out) {
  out->clear();
  std::vector<int> cur;
  WavePlan cur_plan;
  for (int i = 0; i < n; ++i) {
    std::vector<int> trial = cur;
    trial.push_back(i);
    WavePlan tp = layout_wave(mats, trial);
    const bool fits = static_cast<int>(trial.size()) <= kMaxWaveMats &&
                      static_cast<int>(tp.classes.size()) <= kMaxClasses && tp.bytes <= ws_limit;
    if (fits) {
      cur.swap(trial);
      cur_plan = std::move(tp);
      continue;
    }
    if (cur.empty()) return MUON_ERR_WORKSPACE_TOO_SMALL;
    out->push_back(std::move(cur_plan));
    cur.assign(1, i);
    cur_plan = layout_wave(mats, cur);
    if (cur_plan.bytes > ws_limit) return MUON_ERR_WORKSPACE_TOO_SMALL;
  }
  if (!cur.empty()) out->push_back(std::move(cur_plan));
  return MUON_OK;
}

// ---------------------------------------------------------------- launch blocks

struct WaveLaunch {
  EwParams ew;
  GemmParams gram[2];   // indexed by which hi buffer is current
  GemmParams poly;
  GemmParams apply[2];
  FinalParams fin[2];
  std::vector<float> shape_scale;  // per wave-local matrix
  int grid_sym = 0, grid_apply = 0;
};

// Symmetric products: pair tiles (I, J) with J >= I over the m x m output.
void fill_sym_tiles(ClassDesc& d, int64_t m) {
  d.mb = cdiv(m, gemm_tile_rows());
  d.nb = cdiv(m, gemm_tile_cols());
  d.tiles_per_mat = d.nb * (d.nb + 1) / 2;
  d.out_rows = d.out_cols = static_cast<int32_t>(m);
  d.i_fast = 0;
}

muon_status_t build_wave(const muon_matrix_t* mats, const WavePlan& w, uint8_t* ws, int sms, WaveLaunch* L) {
  const int nw = static_cast<int>(w.order.size());
  float* scale = reinterpret_cast<float*>(ws + w.off_scale);
  int32_t* status = reinterpret_cast<int32_t*>(ws);

  // Elementwise stage.
  EwParams& ew = L->ew;
  ew.n = nw;
  ew.total_chunks = w.total_chunks;
  ew.partials = reinterpret_cast<float*>(ws + w.off_partials);
  ew.scale = scale;
  ew.norm = reinterpret_cast<float*>(ws + w.off_norm);
  ew.status = status;
  L->shape_scale.resize(nw);

  int local = 0;
  GemmParams base{};
  base.num_classes = static_cast<int>(w.classes.size());
  base.scale = scale;
  base.status = status;
  int tiles_sym = 0, tiles_apply = 0;
  ClassDesc sym[kMaxClasses], app[kMaxClasses];
  // operand maps: 64 x 128 boxes; epilogue store maps: 64 x 64 boxes
  CUtensorMap op_hi[kMaxClasses][2], op_a[kMaxClasses], op_b[kMaxClasses];
  CUtensorMap st_hi[kMaxClasses][2], st_lo[kMaxClasses], st_a[kMaxClasses], st_b[kMaxClasses];
  for (int ci = 0; ci < static_cast<int>(w.classes.size()); ++ci) {
    const ClassPlan& c = w.classes[ci];
    const int count = static_cast<int>(c.mats.size());
    __nv_bfloat16* hi0 = reinterpret_cast<__nv_bfloat16*>(ws + c.off_hi[0]);
    __nv_bfloat16* hi1 = reinterpret_cast<__nv_bfloat16*>(ws + c.off_hi[1]);
    uint8_t* lo = reinterpret_cast<uint8_t*>(ws + c.off_lo);
    __nv_bfloat16* ab = reinterpret_cast<__nv_bfloat16*>(ws + c.off_a);
    __nv_bfloat16* bb = reinterpret_cast<__nv_bfloat16*>(ws + c.off_b);
    if (!encode_map(&op_hi[ci][0], hi0, count, c.rows, c.cols, c.ldx, 128) ||
        !encode_map(&op_hi[ci][1], hi1, count, c.rows, c.cols, c.ldx, 128) ||
        !encode_map(&op_a[ci], ab, count, c.m, c.m, c.lda, 128) ||
        !encode_map(&op_b[ci], bb, count, c.m, c.m, c.lda, 128) ||
        !encode_map(&st_hi[ci][0], hi0, count, c.rows, c.cols, c.ldx, 64) ||
        !encode_map(&st_hi[ci][1], hi1, count, c.rows, c.cols, c.ldx, 64) ||
        !encode_map_lo(&st_lo[ci], lo, count, c.rows, c.cols, c.ldl) ||
        !encode_map(&st_a[ci], ab, count, c.m, c.m, c.lda, 64) ||
        !encode_map(&st_b[ci], bb, count, c.m, c.m, c.lda, 64))
      return MUON_ERR_CUDA;

    ClassDesc d{};
    d.count = count;
    d.rows = static_cast<int32_t>(c.rows);
    d.cols = static_cast<int32_t>(c.cols);
    d.m = static_cast<int32_t>(c.m);
    d.n = static_cast<int32_t>(c.n);
    d.tall = c.tall;
    d.ldx = static_cast<int32_t>(c.ldx);
    d.lda = static_cast<int32_t>(c.lda);
    d.mat_base = local;
    d.x_stride = c.rows * c.ldx;
    d.lo_stride = c.rows * c.ldl;
    d.ldl = static_cast<int32_t>(c.ldl);
    d.a_stride = c.m * c.lda;
    d.x_lo = lo;
    d.a_buf = ab;
    d.b_buf = bb;

    sym[ci] = d;
    fill_sym_tiles(sym[ci], c.m);
    sym[ci].tile_begin = tiles_sym;
    tiles_sym += count * sym[ci].tiles_per_mat;

    app[ci] = d;
    app[ci].mb = cdiv(c.rows, gemm_tile_rows());
    app[ci].nb = cdiv(c.cols, gemm_tile_cols());
    app[ci].tiles_per_mat = app[ci].mb * app[ci].nb;
    app[ci].out_rows = d.rows;
    app[ci].out_cols = d.cols;
    app[ci].ksize = d.m;
    app[ci].a_mn = 0;
    app[ci].b_mn = c.tall ? 0 : 1;
    app[ci].i_fast = c.tall ? 0 : 1;
    app[ci].tile_begin = tiles_apply;
    tiles_apply += count * app[ci].tiles_per_mat;

    for (int k = 0; k < count; ++k, ++local) {
      const int gi = w.order[local];
      const muon_matrix_t& t = mats[gi];
      EwMat& e = ew.mats[local];
      e.g = t.grad;
      e.m = t.momentum;
      e.hi = hi0 + static_cast<int64_t>(k) * d.x_stride;
      e.lo = lo + static_cast<int64_t>(k) * d.lo_stride;
      e.ld_g = t.ld_grad;
      e.ld_m = t.ld_mom;
      e.rows = d.rows;
      e.cols = d.cols;
      e.ldx = d.ldx;
      e.ldl = d.ldl;
      e.rows_per_chunk = w.rows_per_chunk[local];
      e.chunk_begin = w.chunk_begin[local];
      e.nchunks = w.nchunks[local];
      e.index = gi;
      const bool mom_vec = t.momentum == nullptr || (aligned(t.momentum, 16) && t.ld_mom % 4 == 0);
      const bool mom_v8 = t.momentum == nullptr || (aligned(t.momentum, 32) && t.ld_mom % 8 == 0);
      const bool vec16 = t.ld_grad % 4 == 0 && aligned(t.grad, 16) && mom_vec;
      const bool vec32 = t.ld_grad % 8 == 0 && aligned(t.grad, 32) && mom_v8;
      // eight elements per thread when the rows allow it: 2 (32-byte rows), 3 (16-byte rows);
      // else 1 (four elements, 16-byte rows) or 0 (one by one)
      e.vec = (t.cols % 8 == 0 && vec32) ? 2 : (t.cols % 8 == 0 && vec16) ? 3 : (t.cols % 4 == 0 && vec16) ? 1 : 0;

      L->shape_scale[local] =
          t.shape_scale > 0.f ? t.shape_scale
                              : static_cast<float>(std::sqrt(std::max(1.0, double(t.rows) / double(t.cols))));
      for (int cur = 0; cur < 2; ++cur) {
        UpdMat& u = L->fin[cur].upd[local];
        u.param = t.param;
        u.out = t.out_update;
        u.ld_param = t.ld_param;
        u.param_bf16 = t.param_dtype == MUON_BF16 ? 1 : 0;
        const int pv = u.param_bf16 ? 8 : 4;
        // 1: rows 16-byte aligned (128-bit accesses); 2: 32-byte aligned (256-bit accesses)
        u.vec_param = (t.param != nullptr && aligned(t.param, 16) && t.ld_param % pv == 0)
                          ? ((aligned(t.param, 32) && t.ld_param % (2 * pv) == 0) ? 2 : 1)
                          : 0;
        u.vec_out = (t.out_update != nullptr && aligned(t.out_update, 16) && t.cols % 4 == 0)
                        ? ((aligned(t.out_update, 32) && t.cols % 8 == 0) ? 2 : 1)
                        : 0;
      }
    }
  }

  // Classes with the longest reductions (the most expensive tiles) go first, so the
  // round-robin tile assignment balances the pairs' work.
  const int nc = base.num_classes;
  std::vector<int> ord_sym(nc), ord_app(nc);
  for (int i = 0; i < nc; ++i) ord_sym[i] = ord_app[i] = i;
  std::stable_sort(ord_sym.begin(), ord_sym.end(),
                   [&](int x, int y) { return w.classes[x].n > w.classes[y].n; });
  std::stable_sort(ord_app.begin(), ord_app.end(),
                   [&](int x, int y) { return w.classes[x].m > w.classes[y].m; });
  tiles_sym = tiles_apply = 0;
  for (int k = 0; k < nc; ++k) {
    sym[ord_sym[k]].tile_begin = tiles_sym;
    tiles_sym += sym[ord_sym[k]].count * sym[ord_sym[k]].tiles_per_mat;
    app[ord_app[k]].tile_begin = tiles_apply;
    tiles_apply += app[ord_app[k]].count * app[ord_app[k]].tiles_per_mat;
  }
  // The polynomial and the applies run the staged variant while every Gram side is
  // short: tiles then have short reductions, and moving the epilogue's data by TMA matters
  // more than the main loop's k-block depth.  There K-major operands load 64 x 128 boxes
  // (one per 64-deep k-block) and MN-major ones 64 x 64 boxes.  The Gram, whose epilogue
  // has no inputs, always streams (deeper operand ring).
  int max_m = 0;
  for (const ClassPlan& c : w.classes) max_m = std::max(max_m, static_cast<int>(c.m));
  const bool staged = max_m <= kStagedApplyMaxM;
  for (int cur = 0; cur < 2; ++cur) {
    GemmParams g = base;
    GemmParams a = base;
    g.staged = kStreamed;  // (five 64-deep stages measured no faster than three 128-deep ones)
    a.staged = staged ? kStaged : kStreamed;
    for (int k = 0; k < nc; ++k) {
      const int ci = ord_sym[k];
      g.cls[k] = sym[ci];
      g.cls[k].ksize = static_cast<int32_t>(w.classes[ci].n);
      g.cls[k].a_mn = g.cls[k].b_mn = w.classes[ci].tall;
      // 64-deep k-blocks of MN-major (tall) operands load 64 x 64 boxes
      g.map_a[k] = g.map_b[k] = (g.staged == kStaged && w.classes[ci].tall) ? st_hi[ci][cur] : op_hi[ci][cur];
      g.map_out[k] = st_a[ci];

      const int cj = ord_app[k];
      a.cls[k] = app[cj];
      a.cls[k].x_hi_cur = reinterpret_cast<__nv_bfloat16*>(ws + w.classes[cj].off_hi[cur]);
      a.cls[k].x_hi_next = reinterpret_cast<__nv_bfloat16*>(ws + w.classes[cj].off_hi[cur ^ 1]);
      // staged: K-major operands load 128-row boxes, MN-major ones 64 x 64 boxes
      const bool x_mn = !w.classes[cj].tall;  // wide: X is the MN-major B operand
      const CUtensorMap& x_op = (staged && x_mn) ? st_hi[cj][cur] : op_hi[cj][cur];
      const CUtensorMap& b_op = op_b[cj];
      if (w.classes[cj].tall) {
        a.map_a[k] = x_op;
        a.map_b[k] = b_op;
      } else {
        a.map_a[k] = b_op;
        a.map_b[k] = x_op;
      }
      a.map_in[k] = st_hi[cj][cur];
      a.map_out[k] = st_hi[cj][cur ^ 1];
      a.map_out2[k] = st_lo[cj];
    }
    g.total_tiles = tiles_sym;
    a.total_tiles = tiles_apply;
    L->gram[cur] = g;
    L->apply[cur] = a;
    static_cast<GemmParams&>(L->fin[cur]) = a;
  }
  GemmParams pp = base;
  pp.staged = staged ? kStaged : kStreamed;
  for (int k = 0; k < nc; ++k) {
    const int ci = ord_app[k];  // the polynomial's reduction is m, like the apply's
    pp.cls[k] = sym[ci];
    pp.cls[k].ksize = static_cast<int32_t>(w.classes[ci].m);
    pp.cls[k].a_mn = pp.cls[k].b_mn = 0;
    pp.map_a[k] = pp.map_b[k] = op_a[ci];
    pp.map_in[k] = st_a[ci];
    pp.map_out[k] = st_b[ci];
  }
  {
    int tb = 0;
    for (int k = 0; k < nc; ++k) {
      pp.cls[k].tile_begin = tb;
      tb += pp.cls[k].count * pp.cls[k].tiles_per_mat;
    }
  }
  pp.total_tiles = tiles_sym;
  L->poly = pp;
  L->grid_sym = std::max(1, sms / 2);   // CTA pairs available
  L->grid_apply = std::max(1, sms / 2);
  return MUON_OK;
}

// ---------------------------------------------------------------- plan cache

struct Plan {
  std::vector<uint8_t> key;
  std::vector<WavePlan> waves;
  std::vector<WaveLaunch> launches;
};

std::mutex g_plan_mu;
std::list<Plan> g_plans;  // most recent first
constexpr size_t kMaxPlans = 16;

std::vector<uint8_t> plan_key(const muon_matrix_t* mats, int n, const void* ws, size_t ws_bytes, int dev,
                              bool ns_only) {
  std::vector<uint8_t> k(sizeof(muon_matrix_t) * n + 32);
  std::memcpy(k.data(), mats, sizeof(muon_matrix_t) * n);
  uint8_t* tail = k.data() + sizeof(muon_matrix_t) * n;
  const uint64_t f[4] = {reinterpret_cast<uint64_t>(ws), static_cast<uint64_t>(ws_bytes),
                         static_cast<uint64_t>(dev), ns_only ? 1ull : 0ull};
  std::memcpy(tail, f, sizeof(f));
  return k;
}

// Returns the cached or newly built plan (the list node stays valid under the lock's owner
// until the next insertion evicts it, so the caller copies what it launches).
muon_status_t get_plan(const muon_matrix_t* mats, int n, void* ws, size_t ws_bytes, int dev, int sms,
                       bool ns_only, std::vector<WaveLaunch>* out) {
  std::vector<uint8_t> key = plan_key(mats, n, ws, ws_bytes, dev, ns_only);
  std::lock_guard<std::mutex> lk(g_plan_mu);
  for (auto it = g_plans.begin(); it != g_plans.end(); ++it) {
    if (it->key == key) {
      g_plans.splice(g_plans.begin(), g_plans, it);
      *out = g_plans.front().launches;
      return MUON_OK;
    }
  }
  Plan p;
  p.key = std::move(key);
  muon_status_t st = form_waves(mats, n, ws_bytes, &p.waves);
  if (st != MUON_OK) return st;
  p.launches.resize(p.waves.size());
  for (size_t i = 0; i < p.waves.size(); ++i) {
    st = build_wave(mats, p.waves[i], static_cast<uint8_t*>(ws), sms, &p.launches[i]);
    if (st != MUON_OK) return st;
  }
  *out = p.launches;
  g_plans.push_front(std::move(p));
  if (g_plans.size() > kMaxPlans) g_plans.pop_back();
  return MUON_OK;
}

// ---------------------------------------------------------------- the step

muon_status_t run(const muon_matrix_t* mats, int n, float lr, float beta, float wd, int nesterov, int ns_steps,
                  const float* coeffs, float eps, void* ws, size_t ws_bytes, void* stream_v, bool ns_only) {
  muon_status_t st = validate(mats, n, ns_only);
  if (st != MUON_OK) return st;
  st = validate_hyper(lr, beta, wd, nesterov, ns_steps, coeffs, eps);
  if (st != MUON_OK) return st;
  if (ws == nullptr || !aligned(ws, 256) || ws_bytes < kHeaderBytes) return MUON_ERR_INVALID_ARG;
  int dev = 0, sms = 0;
  st = current_device(&dev, &sms);
  if (st != MUON_OK) return st;
  std::vector<WaveLaunch> launches;
  st = get_plan(mats, n, ws, ws_bytes, dev, sms, ns_only, &launches);
  if (st != MUON_OK) return st;

  cudaStream_t stream = static_cast<cudaStream_t>(stream_v);
  const unsigned long long budget = static_cast<unsigned long long>(g_timeout_us.load()) * 1000ull;
  for (WaveLaunch& L : launches) {
    L.ew.beta = beta;
    L.ew.nesterov = nesterov;
    L.ew.ns_only = ns_only ? 1 : 0;
    L.ew.eps = eps;
    int ev = prof_start(MUON_KIND_MOMENTUM, stream);
    if (launch_momentum(L.ew, stream) != cudaSuccess) return MUON_ERR_CUDA;
    prof_stop(ev, stream);
    ev = prof_start(MUON_KIND_NORM, stream);
    if (launch_norm(L.ew, stream) != cudaSuccess) return MUON_ERR_CUDA;
    prof_stop(ev, stream);
    for (int k = 0; k < ns_steps; ++k) {
      const int cur = k & 1;
      const float a = coeffs[3 * k], b = coeffs[3 * k + 1], c = coeffs[3 * k + 2];
      GemmParams& g = L.gram[cur];
      g.first_iter = k == 0;
      g.timeout_ns = budget;
      ev = prof_start(MUON_KIND_GRAM, stream);
      if (launch_gemm(kGram, &g, L.grid_sym, stream) != cudaSuccess) return MUON_ERR_CUDA;
      prof_stop(ev, stream);
      GemmParams& pp = L.poly;
      pp.b = b;
      pp.c = c;
      pp.timeout_ns = budget;
      ev = prof_start(MUON_KIND_POLY, stream);
      if (launch_gemm(kPoly, &pp, L.grid_sym, stream) != cudaSuccess) return MUON_ERR_CUDA;
      prof_stop(ev, stream);
      if (k + 1 < ns_steps) {
        GemmParams& ap = L.apply[cur];
        ap.a = a;
        ap.first_iter = k == 0;
        ap.timeout_ns = budget;
        ev = prof_start(MUON_KIND_APPLY, stream);
        if (launch_gemm(kApply, &ap, L.grid_apply, stream) != cudaSuccess) return MUON_ERR_CUDA;
        prof_stop(ev, stream);
      } else {
        FinalParams& fp = L.fin[cur];
        fp.a = a;
        fp.first_iter = k == 0;
        fp.timeout_ns = budget;
        fp.decay = 1.0f - lr * wd;
        for (int i = 0; i < static_cast<int>(L.shape_scale.size()); ++i) {
          fp.upd[i].lr_scale = lr * L.shape_scale[i];
          if (ns_only) fp.upd[i].param = nullptr;
        }
        ev = prof_start(MUON_KIND_APPLY_LAST, stream);
        if (launch_gemm(kApplyLast, &fp, L.grid_apply, stream) != cudaSuccess) return MUON_ERR_CUDA;
        prof_stop(ev, stream);
      }
    }
  }
  return MUON_OK;
}

}  // namespace

// ---------------------------------------------------------------- C ABI

extern "C" {

int muon_abi_version(void) { return MUON_ABI_VERSION; }

const char* muon_status_str(int status) {
  switch (status) {
    case MUON_OK: return "ok";
    case MUON_ERR_INVALID_ARG: return "invalid argument";
    case MUON_ERR_ALIGNMENT: return "misaligned pointer";
    case MUON_ERR_UNSUPPORTED_SHAPE: return "unsupported shape or leading dimension";
    case MUON_ERR_UNSUPPORTED_DTYPE: return "unsupported parameter dtype";
    case MUON_ERR_WORKSPACE_TOO_SMALL: return "workspace too small for the largest matrix";
    case MUON_ERR_CUDA: return "CUDA runtime error";
    case MUON_ERR_TIMEOUT: return "device-side wait timed out";
    case MUON_ERR_NO_DEVICE: return "no sm_100 device is current";
    case MUON_ERR_STATIC_SCRATCH_LIMIT: return "a matrix needs more scratch than the static array holds (64 MiB)";
    case MUON_ERR_NONFINITE: return "a Newton-Schulz input held NaN or infinite values";
    default: return "unknown status";
  }
}

muon_status_t muon_workspace_size(const muon_matrix_t* mats, int n, size_t* bytes) {
  if (bytes == nullptr) return MUON_ERR_INVALID_ARG;
  if (mats == nullptr || n < 1) return MUON_ERR_INVALID_ARG;
  for (int i = 0; i < n; ++i)
    if (mats[i].rows < 1 || mats[i].cols < 1 || mats[i].rows > kMaxSide || mats[i].cols > kMaxSide)
      return MUON_ERR_UNSUPPORTED_SHAPE;
  std::vector<WavePlan> waves;
  muon_status_t st = form_waves(mats, n, ~size_t(0), &waves);
  if (st != MUON_OK) return st;
  size_t mx = kHeaderBytes;
  for (const auto& w : waves) mx = std::max(mx, w.bytes);
  *bytes = mx;
  return MUON_OK;
}

muon_status_t muon_workspace_init(void* workspace, size_t workspace_bytes, void* stream) {
  if (workspace == nullptr || workspace_bytes < kHeaderBytes || !aligned(workspace, 256)) return MUON_ERR_INVALID_ARG;
  if (cudaMemsetAsync(workspace, 0, kHeaderBytes, static_cast<cudaStream_t>(stream)) != cudaSuccess)
    return MUON_ERR_CUDA;
  return MUON_OK;
}

muon_status_t muon_step(const muon_matrix_t* mats, int n, float lr, float beta, float weight_decay, int nesterov,
                        int ns_steps, const float* coeffs, float eps, void* workspace, size_t workspace_bytes,
                        void* stream) {
  return run(mats, n, lr, beta, weight_decay, nesterov, ns_steps, coeffs, eps, workspace, workspace_bytes, stream,
             false);
}

muon_status_t muon_newton_schulz(const muon_matrix_t* mats, int n, int ns_steps, const float* coeffs, float eps,
                                 void* workspace, size_t workspace_bytes, void* stream) {
  return run(mats, n, 0.f, 0.f, 0.f, 0, ns_steps, coeffs, eps, workspace, workspace_bytes, stream, true);
}

muon_status_t muon_scratch_view(const muon_matrix_t* mats, int n, int index, size_t workspace_bytes,
                                muon_scratch_view_t* view) {
  if (view == nullptr || mats == nullptr || n < 1 || index < 0 || index >= n) return MUON_ERR_INVALID_ARG;
  for (int i = 0; i < n; ++i)
    if (mats[i].rows < 1 || mats[i].cols < 1 || mats[i].rows > kMaxSide || mats[i].cols > kMaxSide)
      return MUON_ERR_UNSUPPORTED_SHAPE;
  std::vector<WavePlan> waves;
  muon_status_t st = form_waves(mats, n, workspace_bytes, &waves);
  if (st != MUON_OK) return st;
  for (size_t wi = 0; wi < waves.size(); ++wi) {
    const WavePlan& w = waves[wi];
    int local = 0;
    for (const ClassPlan& c : w.classes) {
      for (size_t k = 0; k < c.mats.size(); ++k, ++local) {
        if (c.mats[k] != index) continue;
        const size_t xoff = k * static_cast<size_t>(c.rows * c.ldx) * 2;
        const size_t aoff = k * static_cast<size_t>(c.m * c.lda) * 2;
        view->x_hi_offset[0] = c.off_hi[0] + xoff;
        view->x_hi_offset[1] = c.off_hi[1] + xoff;
        view->x_lo_offset = c.off_lo + k * static_cast<size_t>(c.rows * c.ldl);
        view->a_offset = c.off_a + aoff;
        view->b_offset = c.off_b + aoff;
        view->scale_offset = w.off_scale + 4 * static_cast<size_t>(local);
        view->norm_offset = w.off_norm + 4 * static_cast<size_t>(local);
        view->x_ld = c.ldx;
        view->x_lo_ld = c.ldl;
        view->a_ld = c.lda;
        view->wave = static_cast<int32_t>(wi);
        view->transposed = c.tall;
        return MUON_OK;
      }
    }
  }
  return MUON_ERR_INVALID_ARG;
}

muon_status_t muon_device_status(const void* workspace, void* stream, int32_t* device_status, int32_t* where) {
  if (workspace == nullptr || device_status == nullptr) return MUON_ERR_INVALID_ARG;
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return MUON_ERR_CUDA;
  int32_t h[2] = {0, 0};
  if (cudaMemcpy(h, workspace, sizeof(h), cudaMemcpyDeviceToHost) != cudaSuccess) return MUON_ERR_CUDA;
  *device_status = h[0];
  if (where != nullptr) *where = h[1];
  return MUON_OK;
}

muon_status_t muon_nonfinite_count(const void* workspace, void* stream, int64_t* count) {
  if (workspace == nullptr || count == nullptr) return MUON_ERR_INVALID_ARG;
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return MUON_ERR_CUDA;
  uint64_t c = 0;
  if (cudaMemcpy(&c, static_cast<const uint8_t*>(workspace) + 8, sizeof(c), cudaMemcpyDeviceToHost) != cudaSuccess)
    return MUON_ERR_CUDA;
  *count = static_cast<int64_t>(c);
  return MUON_OK;
}

muon_status_t muon_set_wait_timeout_us(int64_t us) {
  g_timeout_us.store(us > 0 ? us : 2000000);
  return MUON_OK;
}

muon_status_t muon_profile_begin(void) {
  g_prof.on = true;
  g_prof.used = 0;
  return MUON_OK;
}

muon_status_t muon_profile_end(double* ms_by_kind, int64_t* launches_by_kind, int kinds) {
  if (ms_by_kind == nullptr || launches_by_kind == nullptr || kinds < 1) return MUON_ERR_INVALID_ARG;
  for (int k = 0; k < kinds; ++k) {
    ms_by_kind[k] = 0.0;
    launches_by_kind[k] = 0;
  }
  muon_status_t st = MUON_OK;
  for (size_t i = 0; i < g_prof.used; ++i) {
    float ms = 0.f;
    if (cudaEventSynchronize(g_prof.pool[i].second) != cudaSuccess ||
        cudaEventElapsedTime(&ms, g_prof.pool[i].first, g_prof.pool[i].second) != cudaSuccess) {
      st = MUON_ERR_CUDA;
      continue;
    }
    const int k = g_prof.kinds[i];
    if (k < kinds) {
      ms_by_kind[k] += ms;
      launches_by_kind[k] += 1;
    }
  }
  g_prof.on = false;
  g_prof.used = 0;
  return st;
}

}  // extern "C"

// ---------------------------------------------------------------- static scratch

namespace {

constexpr size_t kStaticScratchBytes = MUON_STATIC_SCRATCH_BYTES;
constexpr int kMaxDevices = 64;

// Scratch of muon_newton_schulz_static.  In host code `g_static_scratch` only names the
// symbol; its device address comes from cudaGetSymbolAddress, per device.
static __device__ __align__(256) uint8_t g_static_scratch[kStaticScratchBytes];

// The array's address on each device, with the id of the context it was looked up in.  A
// context id is never reused within a process, so after the device's primary context has
// been torn down and re-created (cudaDeviceReset), the first call looks the address up
// again instead of using one from an unloaded module.
struct StaticAddr {
  unsigned long long ctx_id = 0;
  void* addr = nullptr;
};
std::mutex g_static_mu;
StaticAddr g_static_addr[kMaxDevices];

using CtxGetCurrentFn = CUresult (*)(CUcontext*);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long*);

// Unique id of the current context (0 if it cannot be read).
unsigned long long current_context_id() {
  static CtxGetCurrentFn get_cur = nullptr;
  static CtxGetIdFn get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_cur = reinterpret_cast<CtxGetCurrentFn>(p);
    p = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<CtxGetIdFn>(p);
  });
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (get_cur == nullptr || get_id == nullptr || get_cur(&ctx) != CUDA_SUCCESS || ctx == nullptr ||
      get_id(ctx, &id) != CUDA_SUCCESS)
    return 0;
  return id;
}

// Device address of the array on device `dev`, which is current: looked up once per
// device and context (cudaGetSymbolAddress), then reused.
muon_status_t static_scratch(int dev, void** addr) {
  if (dev < 0 || dev >= kMaxDevices) return MUON_ERR_NO_DEVICE;
  std::lock_guard<std::mutex> lk(g_static_mu);
  const unsigned long long ctx = current_context_id();
  StaticAddr& e = g_static_addr[dev];
  if (e.addr == nullptr || ctx == 0 || e.ctx_id != ctx) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_static_scratch) != cudaSuccess || p == nullptr) return MUON_ERR_CUDA;
    e.addr = p;
    e.ctx_id = ctx;
  }
  *addr = e.addr;
  return MUON_OK;
}

}  // namespace

extern "C" muon_status_t muon_newton_schulz_static(const muon_matrix_t* mats, int n, int ns_steps,
                                                   const float* coeffs, float eps, int32_t* device_status,
                                                   void* stream) {
  muon_status_t st = validate(mats, n, true);
  if (st != MUON_OK) return st;
  st = validate_hyper(0.f, 0.f, 0.f, 0, ns_steps, coeffs, eps);
  if (st != MUON_OK) return st;
  {
    std::vector<WavePlan> waves;
    st = form_waves(mats, n, kStaticScratchBytes, &waves);
    if (st == MUON_ERR_WORKSPACE_TOO_SMALL) return MUON_ERR_STATIC_SCRATCH_LIMIT;
    if (st != MUON_OK) return st;
  }
  int dev = 0, sms = 0;
  st = current_device(&dev, &sms);
  if (st != MUON_OK) return st;
  void* ws = nullptr;
  st = static_scratch(dev, &ws);
  if (st != MUON_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(ws, 0, kHeaderBytes, s) != cudaSuccess) return MUON_ERR_CUDA;
  st = run(mats, n, 0.f, 0.f, 0.f, 0, ns_steps, coeffs, eps, ws, kStaticScratchBytes, stream, true);
  if (st != MUON_OK) return st;
  if (device_status != nullptr &&
      cudaMemcpyAsync(device_status, ws, 2 * sizeof(int32_t), cudaMemcpyDefault, s) != cudaSuccess)
    return MUON_ERR_CUDA;
  return MUON_OK;
}
