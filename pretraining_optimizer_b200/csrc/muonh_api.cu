// C ABI of the MuonH step and its host-side scheduler.
//
// muonh_init groups the matrices by their padded Newton-Schulz shape
// (r_pad x c_pad, r = min(rows, cols) on the wide orientation, both padded
// to multiples of 256), allocates one zero-filled workspace per shape class
// ([count][r_pad][c_pad] iterate ping-pong buffers and [count][r_pad][r_pad]
// buffers for A = Y Y^T and B' = a I + b A + c A A, plus C = b I + c A in
// FP32 mode), encodes one TMA descriptor per buffer and box shape, and
// builds the tile lists of the grouped GEMM launches.  Zero padding is exact
// for the iteration: padded rows and columns of Y, A and B' stay zero, so no
// GEMM tile is ragged.
//
// muonh_step enqueues, per matrix group:
//   momentum       (M update, ||X||^2 partials, 16-bit X)       -> finalize_input
//   write_x        (rewrites X where the momentum pass's scale was unsafe)
//   ns_steps x { GRAM, SQUARE, APPLY }   (tcgen05 GEMMs; the last APPLY also
//                                         forms ||O||^2 and <W, O>)
//   update_dots    (only matrices the last APPLY does not cover) -> finalize_update
//   project        (W <- R (W - lr R O/||O||) / ||.||, Eq. (1))  -> finalize_step
// One group runs everything on the caller's stream.  With two groups the
// GEMMs move to an internal highest-priority stream, and each group's
// elementwise launches overlap the other group's GEMMs (see muonh_step).
#include <algorithm>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <map>
#include <string>
#include <vector>

#include "muonh_common.cuh"

using namespace muonh;

namespace {

thread_local std::string g_last_error;

muonh_status fail(muonh_status st, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return st;
}

#define CUDA_TRY(call)                                                                                \
  do {                                                                                                \
    cudaError_t e_ = (call);                                                                          \
    if (e_ != cudaSuccess) return fail(MUONH_ERR_CUDA, "%s failed: %s", #call, cudaGetErrorString(e_)); \
  } while (0)

constexpr int kRing = 4;
// With at least this many elements the step runs in kGroups matrix groups
// whose elementwise phases overlap the other groups' Newton-Schulz GEMMs;
// below it the overlap cannot pay for the extra launches.
constexpr int64_t kTwoGroupMinElems = int64_t(1) << 24;
constexpr int kGroups = 2;      // the automatic choice
constexpr int kMaxGroups = 3;
// Tiles per block of an elementwise launch that overlaps Newton-Schulz GEMMs:
// short-lived blocks leave the SMs' resources to the GEMMs' blocks, which the
// scheduler places first (they run on the highest-priority stream).
constexpr int64_t kOverlapTilesPerBlock = 4;
constexpr int64_t kMaxDim = 1 << 20;
constexpr int64_t kMaxRPad = 16384;
constexpr int32_t kMaxNsSteps = 64;
constexpr uint32_t kStateMagic = 0x484E554Du;   // "MUNH"

struct TileList {
  TileDesc* dev = nullptr;
  int32_t count = 0;
  int64_t sum_nk = 0, sum_nk_sq = 0;   // k-blocks over the tiles, as GRAM/APPLY and as SQUARE
};

// Run lengths of the Gram-space form for `steps` iterations: as few runs of
// at most three as possible, longer runs first (5 -> 3, 2).
std::vector<int> gram_runs(int steps) {
  std::vector<int> runs;
  if (steps <= 0) return runs;
  const int nruns = (steps + 2) / 3;
  for (int j = 0; j < nruns; ++j) runs.push_back(steps / nruns + (j < steps % nruns ? 1 : 0));
  return runs;
}

struct ClassHost {
  int32_t r_pad, c_pad, count = 0;
  bool gram = false;         // holds a matrix in the Gram-space form (P1, T buffers)
  ClassDev dev{};
};

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  }
  return fn;
}

// Largest power-of-two exponent e with bound * 2^e <= 60000 (fp16 max 65504).
int safe_exponent(double bound) {
  if (!(bound > 0.0) || !std::isfinite(bound)) return 0;
  int e = static_cast<int>(std::floor(std::log2(60000.0 / bound)));
  return std::max(-24, std::min(15, e));
}

// Bounds on the entries of the stored operands over all iterations: Y,
// A = Y Y^T, C = b I + c A and B' = a I + b A + c A^2.  Entries are bounded
// by spectral norms, which follow from the scalar map
// s -> a s + b s^3 + c s^5 on the singular values, starting from
// sigma_max(Y_0) <= 1 after the Frobenius normalisation.
void scale_exponents(float a, float b, float c, int steps, int prec, int32_t* ex, int32_t* ea, int32_t* ec,
                     int32_t* eb) {
  if (prec == P_BF16) {
    *ex = *ea = *ec = *eb = 0;
    return;
  }
  double smax = 1.0, s_all = 1.0;
  for (int k = 0; k < steps; ++k) {
    double m = 0.0;
    const int n = 8192;
    for (int i = 0; i <= n; ++i) {
      const double s = smax * i / n;
      m = std::max(m, std::fabs(a * s + b * s * s * s + c * s * s * s * s * s));
    }
    smax = std::max(m * 1.001, 1e-30);
    s_all = std::max(s_all, smax);
    if (!std::isfinite(s_all) || s_all > 1e6) break;
  }
  const double xmax = s_all * 1.02;
  const double amax = xmax * xmax;
  double cmax = 0.0, bmax = 0.0;
  for (int i = 0; i <= 8192; ++i) {
    const double l = amax * i / 8192;
    cmax = std::max(cmax, std::fabs(b + c * l));
    bmax = std::max(bmax, std::fabs(a + b * l + c * l * l));
  }
  *ex = safe_exponent(xmax);
  *ea = safe_exponent(amax);
  *ec = safe_exponent(std::max(cmax, 1e-30));
  *eb = safe_exponent(std::max(bmax, 1e-30));
}

// Scale of a stored product Q of `run` consecutive factors p(A_k) = a I +
// b A_k + c A_k^2 (Gram-space form).  On a singular direction of the run's
// first Y with value s, Q acts as prod_k q(s_k), q(s) = a + b s^2 + c s^4 and
// s_{k+1} = s_k q(s_k); |Q| is bounded by the largest such product over s in
// [0, smax], smax the bound on every iterate's singular values (at s = 0 it
// is a^run).  The products A_k p(A_k) are bounded like A (they act as
// s_k s_{k+1}) and share A's scale.
int q_exponent(float a, float b, float c, int run, double smax) {
  double qmax = 0.0;
  const int n = 8192;
  for (int i = 0; i <= n; ++i) {
    double s = smax * i / n, q = 1.0;
    for (int k = 0; k < run; ++k) {
      const double f = a + b * s * s + c * s * s * s * s;
      q *= f;
      s *= f;
    }
    qmax = std::max(qmax, std::fabs(q));
  }
  return safe_exponent(std::max(qmax * 1.02, 1e-30));
}

// Bound on the singular values of every iterate (the s_all of scale_exponents).
double iterate_bound(float a, float b, float c, int steps) {
  double smax = 1.0, s_all = 1.0;
  for (int k = 0; k < steps; ++k) {
    double m = 0.0;
    const int n = 8192;
    for (int i = 0; i <= n; ++i) {
      const double s = smax * i / n;
      m = std::max(m, std::fabs(a * s + b * s * s * s + c * s * s * s * s * s));
    }
    smax = std::max(m * 1.001, 1e-30);
    s_all = std::max(s_all, smax);
    if (!std::isfinite(s_all) || s_all > 1e6) break;
  }
  return s_all * 1.02;
}

int64_t round_up(int64_t v, int64_t m) { return (v + m - 1) / m * m; }

}  // namespace

void muonh::set_error_message(const char* msg) { g_last_error = msg; }

struct muonh_ctx {
  int32_t n = 0;
  int32_t prec = 0;
  float eps = 0.f;
  int device = 0;
  int sm_count = 148;
  int32_t max_steps = 0;
  bool pairs = false;        // 16-bit operands: CTA-pair GEMMs on 256 x 256 tiles
  std::vector<int> runs;     // Gram-space form: iterations per run
  double step_flops[MUONH_NUM_PHASES] = {};   // tensor-core FLOPs of the last step's launches
  int64_t n_et = 0;
  int64_t step_count = 0;
  int32_t last_launches = 0;
  cudaStream_t last_stream = nullptr;

  std::vector<MatDev> mats;
  std::vector<ClassHost> classes;
  // The step runs in one or kGroups matrix groups (contiguous index ranges
  // of about equal Newton-Schulz work): the elementwise phases of one group
  // overlap the Newton-Schulz GEMMs of its neighbours.
  // The matrices of a group in one Newton-Schulz form (0: Y-space, 1:
  // Gram-space): their elementwise tiles [e_first, e_end) (a group stores
  // the Y-space matrices' tiles first) and their indices in d_mlist.
  struct Subset {
    int64_t e_first = 0, e_end = 0;
    int32_t m_off = 0, m_count = 0;
    bool any_unfused = false, any_general = false, any_wt[2] = {false, false};
  };
  struct Group {
    int32_t m_first = 0, m_count = 0;
    int64_t e_first = 0, e_end = 0;
    bool any_unfused = false, any_general = false, any_wt[2] = {false, false};
    Subset sub[2];
    std::vector<TileList> gram_lists, apply_lists;   // per Newton-Schulz iteration (Y-space form)
    bool any_gram = false;                           // Gram-space form: its upper and APPLY tiles
    TileList gram_upper, gram_apply;
  };
  std::vector<Group> groups;
  cudaStream_t ns_stream = nullptr;   // highest-priority stream for the GEMMs of a grouped step
  std::vector<cudaEvent_t> gev;       // grouped step: per group, front done (2g) and GEMMs done (2g+1)
  cudaEvent_t split_ev[2] = {};       // grouped step: first group's Y-space front done; last group's
                                      // Gram-space GEMMs done
  std::vector<void*> allocs;

  MatDev* d_mats = nullptr;
  ClassDev* d_classes = nullptr;
  MatScal* d_scal = nullptr;
  MatStep* d_step = nullptr;
  const MatStep* step_src = nullptr;   // per-step arguments the next launches read (d_step or the caller's)
  int32_t* d_et_mat = nullptr;
  int32_t* d_mlist = nullptr;      // per group: Y-space matrix indices, then Gram-space ones
  std::vector<int32_t> h_mlist;
  float* d_part = nullptr;
  double* d_part64 = nullptr;
  float* d_part_ns = nullptr;      // fused last-APPLY partials
  CUtensorMap* d_wmaps = nullptr;  // per matrix fp32 W tiles (fused matrices)
  int64_t n_ns_slots = 0;
  int ew_warp_grid[4] = {148, 148, 148, 148};   // blocks of the warp-tiled kernels (one wave each)
  float* d_part8 = nullptr;
  CUtensorMap* d_tmaps = nullptr;
  int* d_err = nullptr;

  MatStep* h_step[kRing] = {};
  cudaEvent_t ev[kRing] = {};
  int ring = 0;

  // optional per-kernel timing: (phase, begin event, end event)
  bool timing = false;
  struct Timed {
    int phase;
    cudaEvent_t begin, end;
  };
  std::vector<Timed> timed;
  std::vector<cudaEvent_t> event_pool;

  cudaEvent_t take_event() {
    if (!event_pool.empty()) {
      cudaEvent_t e = event_pool.back();
      event_pool.pop_back();
      return e;
    }
    cudaEvent_t e = nullptr;
    cudaEventCreate(&e);
    return e;
  }

  // whole-context launch (init) or one group's launch (g >= 0)
  // Elementwise launch parameters: the whole set (g < 0), group g, or the
  // matrices of group g in one form (sub 0: Y-space, 1: Gram-space)
  EwParams ew(muonh_stats* stats_out, int g = -1, int sub = -1) const {
    EwParams p{};
    p.e_first = g < 0 ? 0 : groups[g].e_first;
    p.e_end = g < 0 ? n_et : groups[g].e_end;
    p.m_first = g < 0 ? 0 : groups[g].m_first;
    p.m_count = g < 0 ? n : groups[g].m_count;
    if (g >= 0 && sub >= 0) {
      const Subset& su = groups[g].sub[sub];
      p.e_first = su.e_first;
      p.e_end = su.e_end;
      p.m_first = su.m_off;
      p.m_count = su.m_count;
      p.mlist = d_mlist;
    }
    p.mats = d_mats;
    p.step = step_src ? step_src : d_step;
    p.scal = d_scal;
    p.classes = d_classes;
    p.et_mat = d_et_mat;
    p.n_et = n_et;
    p.part = d_part;
    p.part64 = d_part64;
    p.part8 = d_part8;
    p.part_ns = d_part_ns;
    p.n = n;
    p.eps = eps;
    p.prec = prec;
    p.stats_out = stats_out;
    p.err = d_err;
    p.any_rewrite = d_err + 1 + (g < 0 ? 0 : g);
    return p;
  }
};

namespace {

muonh_status enqueue_step(muonh_ctx* ctx, const MatStep* step_args, muonh_stats* stats, cudaStream_t s);

cudaError_t dev_alloc(muonh_ctx* ctx, void** p, size_t bytes) {
  cudaError_t e = cudaMalloc(p, bytes);
  if (e == cudaSuccess) ctx->allocs.push_back(*p);
  return e;
}

void release(muonh_ctx* ctx) {
  if (!ctx) return;
  for (void* p : ctx->allocs) cudaFree(p);
  ctx->allocs.clear();
  if (ctx->ns_stream) cudaStreamDestroy(ctx->ns_stream);
  for (cudaEvent_t e : ctx->gev)
    if (e) cudaEventDestroy(e);
  ctx->gev.clear();
  for (cudaEvent_t& e : ctx->split_ev)
    if (e) {
      cudaEventDestroy(e);
      e = nullptr;
    }
  for (int i = 0; i < kRing; ++i) {
    if (ctx->h_step[i]) cudaFreeHost(ctx->h_step[i]);
    if (ctx->ev[i]) cudaEventDestroy(ctx->ev[i]);
  }
  for (auto& t : ctx->timed) {
    cudaEventDestroy(t.begin);
    cudaEventDestroy(t.end);
  }
  for (cudaEvent_t e : ctx->event_pool) cudaEventDestroy(e);
  delete ctx;
}

// 4-D 16-bit map over a row-major buffer (rows x inner, count matrices):
// dimensions (64 columns, rows, 64-column chunks, matrix), the chunk stride
// 128 bytes, so that a 64 x box_rows x 2 box lands in shared memory as two
// box_rows x 64 chunks one after the other (128-byte swizzle).  Read as a
// K-major operand the chunks are two k-blocks; read as an MN-major one,
// the two 64-wide column chunks of a 128-column half.
muonh_status encode_map_chunks(CUtensorMap* out, void* base, int prec16_is_bf16, int64_t inner, int64_t rows,
                               int64_t count, int box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return fail(MUONH_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
  const cuuint64_t dims[4] = {64u, static_cast<cuuint64_t>(rows), static_cast<cuuint64_t>(inner / 64),
                              static_cast<cuuint64_t>(count)};
  const cuuint64_t strides[3] = {static_cast<cuuint64_t>(inner * 2), 128u, static_cast<cuuint64_t>(inner * rows * 2)};
  const cuuint32_t box[4] = {64u, static_cast<cuuint32_t>(box_rows), 2u, 1u};
  const cuuint32_t estr[4] = {1u, 1u, 1u, 1u};
  CUresult r = fn(out, prec16_is_bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 4,
                  base, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(MUONH_ERR_CUDA, "cuTensorMapEncodeTiled (MN pair box) failed (%d)", static_cast<int>(r));
  return MUONH_OK;
}

muonh_status encode_map(CUtensorMap* out, void* base, int prec16_is_bf16, int64_t inner, int64_t rows,
                        int64_t count, int box_rows, int box_inner = 64,
                        CUtensorMapSwizzle swizzle = CU_TENSOR_MAP_SWIZZLE_128B) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return fail(MUONH_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(inner), static_cast<cuuint64_t>(rows),
                              static_cast<cuuint64_t>(count)};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(inner * 2), static_cast<cuuint64_t>(inner * rows * 2)};
  const cuuint32_t box[3] = {static_cast<cuuint32_t>(box_inner), static_cast<cuuint32_t>(box_rows), 1u};
  const cuuint32_t estr[3] = {1u, 1u, 1u};
  CUresult r = fn(out, prec16_is_bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 3,
                  base, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(MUONH_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", static_cast<int>(r));
  return MUONH_OK;
}

// 2-D fp32 map over a caller's W (rows x cols, row stride ld elements):
// wide W: 32 x 128 boxes (128-byte swizzle); tall W: 128 x 32 boxes.
muonh_status encode_w_map(CUtensorMap* out, const MatDev& md) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return fail(MUONH_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(md.cols), static_cast<cuuint64_t>(md.rows)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(md.ld * 4)};
  const cuuint32_t box[2] = {md.transposed ? 128u : 32u, md.transposed ? 32u : 128u};
  const cuuint32_t estr[2] = {1u, 1u};
  CUresult r = fn(out, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, md.w, dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE,
                  md.transposed ? CU_TENSOR_MAP_SWIZZLE_NONE : CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(MUONH_ERR_CUDA, "cuTensorMapEncodeTiled (W) failed (%d)", static_cast<int>(r));
  return MUONH_OK;
}

muonh_status check_launch(cudaError_t e, const char* what) {
  if (e != cudaSuccess) return fail(MUONH_ERR_CUDA, "launch of %s failed: %s", what, cudaGetErrorString(e));
  return MUONH_OK;
}

#define LAUNCH_TRY(expr, name)                              \
  do {                                                      \
    muonh_status st_ = check_launch((expr), name);          \
    if (st_ != MUONH_OK) return st_;                        \
    ++launches;                                             \
  } while (0)

// A launch of the step on stream `strm`, bracketed by events when timing is on.
#define STEP_LAUNCH_ON(phase, expr, name, strm)                          \
  do {                                                                   \
    cudaEvent_t ev_b = nullptr, ev_e = nullptr;                          \
    if (ctx->timing) {                                                   \
      ev_b = ctx->take_event();                                          \
      ev_e = ctx->take_event();                                          \
      CUDA_TRY(cudaEventRecord(ev_b, strm));                             \
    }                                                                    \
    LAUNCH_TRY(expr, name);                                              \
    if (ctx->timing) {                                                   \
      CUDA_TRY(cudaEventRecord(ev_e, strm));                             \
      ctx->timed.push_back(muonh_ctx::Timed{phase, ev_b, ev_e});         \
    }                                                                    \
  } while (0)

}  // namespace

extern "C" {

const char* muonh_status_string(muonh_status s) {
  switch (s) {
    case MUONH_OK: return "ok";
    case MUONH_ERR_INVALID_ARG: return "invalid argument";
    case MUONH_ERR_ALIGNMENT: return "misaligned pointer or stride";
    case MUONH_ERR_CUDA: return "CUDA error";
    case MUONH_ERR_OOM: return "out of device memory";
    case MUONH_ERR_TIMEOUT: return "device wait timed out";
    case MUONH_ERR_UNSUPPORTED: return "unsupported device or size";
  }
  return "unknown status";
}

const char* muonh_last_error(void) { return g_last_error.c_str(); }

muonh_status muonh_init(muonh_ctx** out, const muonh_matrix_desc* mats, int32_t n, const muonh_config* cfg,
                        void* stream) {
  g_last_error.clear();
  if (!out) return fail(MUONH_ERR_INVALID_ARG, "out is NULL");
  *out = nullptr;
  if (!mats || n <= 0 || !cfg) return fail(MUONH_ERR_INVALID_ARG, "mats/cfg NULL or n <= 0");
  if (cfg->ns_precision < 0 || cfg->ns_precision > 2)
    return fail(MUONH_ERR_INVALID_ARG, "ns_precision %d is not FP16, BF16 or FP32", cfg->ns_precision);
  if (!(cfg->eps >= 0.f) || !std::isfinite(cfg->eps)) return fail(MUONH_ERR_INVALID_ARG, "eps must be finite and >= 0");
  if (cfg->groups < 0 || cfg->groups > kMaxGroups)
    return fail(MUONH_ERR_INVALID_ARG, "groups %d is not 0 (automatic), 1, 2 or 3", cfg->groups);
  if (cfg->ns_form < MUONH_NS_FORM_AUTO || cfg->ns_form > MUONH_NS_FORM_GRAM)
    return fail(MUONH_ERR_INVALID_ARG, "ns_form %d is not MUONH_NS_FORM_AUTO, _Y or _GRAM", cfg->ns_form);
  for (int32_t i = 0; i < n; ++i) {
    const muonh_matrix_desc& d = mats[i];
    if (!d.w || !d.m) return fail(MUONH_ERR_INVALID_ARG, "matrix %d: w or m is NULL", i);
    if (d.rows <= 0 || d.cols <= 0 || d.rows > kMaxDim || d.cols > kMaxDim)
      return fail(MUONH_ERR_INVALID_ARG, "matrix %d: rows/cols out of range (1..%lld)", i, (long long)kMaxDim);
    if (d.ld < d.cols) return fail(MUONH_ERR_INVALID_ARG, "matrix %d: ld < cols", i);
    if ((reinterpret_cast<uintptr_t>(d.w) & 15) || (reinterpret_cast<uintptr_t>(d.m) & 15))
      return fail(MUONH_ERR_ALIGNMENT, "matrix %d: w and m must be 16-byte aligned", i);
    if (d.ns_steps < 0 || d.ns_steps > kMaxNsSteps)
      return fail(MUONH_ERR_INVALID_ARG, "matrix %d: ns_steps %d outside [0, %d]", i, d.ns_steps, kMaxNsSteps);
    if (!std::isfinite(d.beta) || !std::isfinite(d.ns_a) || !std::isfinite(d.ns_b) || !std::isfinite(d.ns_c) ||
        !std::isfinite(d.radius))
      return fail(MUONH_ERR_INVALID_ARG, "matrix %d: beta, coefficients and radius must be finite", i);
    if (d.update_rule < 0 || d.update_rule > 2 || !std::isfinite(d.weight_decay) || !std::isfinite(d.update_scale) ||
        (d.update_rule != 0 && !(d.update_scale > 0.f)))
      return fail(MUONH_ERR_INVALID_ARG, "matrix %d: update_rule in 0..2, finite weight_decay, update_scale > 0", i);
    if (round_up(std::min(d.rows, d.cols), kPad) > kMaxRPad)
      return fail(MUONH_ERR_UNSUPPORTED, "matrix %d: min(rows, cols) above %lld", i, (long long)kMaxRPad);
  }

  int dev = 0;
  CUDA_TRY(cudaGetDevice(&dev));
  cudaDeviceProp prop;
  CUDA_TRY(cudaGetDeviceProperties(&prop, dev));
  if (prop.major != 10)
    return fail(MUONH_ERR_UNSUPPORTED, "device %d is sm_%d%d; this library is built for sm_100a", dev, prop.major,
                prop.minor);
  CUDA_TRY(ns_gemm_set_attributes());

  muonh_ctx* ctx = new muonh_ctx();
  ctx->n = n;
  ctx->prec = cfg->ns_precision;
  ctx->eps = cfg->eps;
  ctx->device = dev;
  ctx->sm_count = prop.multiProcessorCount;
  for (int k = 0; k < 4; ++k) ctx->ew_warp_grid[k] = ctx->sm_count * ew_warp_blocks_per_sm(k);
  ctx->pairs = cfg->ns_precision != P_FP32;
  // matrix groups: 1, the automatic 2 for a large enough set, or as asked
  const int want_groups = cfg->groups == 0 ? kGroups : cfg->groups;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  ctx->last_stream = s;

  struct Guard {
    muonh_ctx*& c;
    bool ok = false;
    ~Guard() {
      if (!ok) release(c);
    }
  } guard{ctx};

  // ---- per-matrix layout and shape classes
  std::map<std::pair<int64_t, int64_t>, int> class_of;
  ctx->mats.resize(n);
  int64_t n_et = 0;
  for (int32_t i = 0; i < n; ++i) {
    const muonh_matrix_desc& d = mats[i];
    MatDev& md = ctx->mats[i];
    md = MatDev{};
    md.w = d.w;
    md.m = d.m;
    md.rows = d.rows;
    md.cols = d.cols;
    md.ld = d.ld;
    md.r = static_cast<int32_t>(std::min(d.rows, d.cols));
    md.c = static_cast<int32_t>(std::max(d.rows, d.cols));
    md.transposed = d.rows > d.cols ? 1 : 0;
    md.vec = (d.cols % 4 == 0 && d.ld % 4 == 0) ? 1 : 0;
    md.warp_tiled = (md.vec && ctx->prec != P_FP32) ? 1 : 0;
    md.beta = d.beta;
    md.nesterov = d.nesterov ? 1 : 0;
    md.ns_steps = d.ns_steps;
    md.a = d.ns_a;
    md.b = d.ns_b;
    md.c_coef = d.ns_c;
    md.rule = d.update_rule;
    md.wd = d.weight_decay;
    md.uscale = d.update_rule == 0 ? 1.f : d.update_scale;
    scale_exponents(d.ns_a, d.ns_b, d.ns_c, d.ns_steps, ctx->prec, &md.ex, &md.ea, &md.ec, &md.eb);
    if (md.transposed) {
      md.et_th = md.et_tw = kEwTile;
    } else {
      int tw = kEwTile;
      while (tw < 512 && tw < d.cols) tw *= 2;
      md.et_tw = tw;
      md.et_th = kEwTile * kEwTile / tw;
    }
    md.et_rows = static_cast<int32_t>((d.rows + md.et_th - 1) / md.et_th);
    md.et_cols = static_cast<int32_t>((d.cols + md.et_tw - 1) / md.et_tw);
    md.et_begin = n_et;
    n_et += static_cast<int64_t>(md.et_rows) * md.et_cols;
    const std::pair<int64_t, int64_t> key(round_up(md.r, kPad), round_up(md.c, kPad));
    auto it = class_of.find(key);
    if (it == class_of.end()) {
      ClassHost ch;
      ch.r_pad = static_cast<int32_t>(key.first);
      ch.c_pad = static_cast<int32_t>(key.second);
      it = class_of.emplace(key, static_cast<int>(ctx->classes.size())).first;
      ctx->classes.push_back(ch);
    }
    md.cls = it->second;
    md.z = ctx->classes[md.cls].count++;
    ctx->max_steps = std::max(ctx->max_steps, d.ns_steps);
  }
  ctx->n_et = n_et;

  // ---- Newton-Schulz form per matrix: the Gram-space form (fp16 CTA pairs,
  // the context's full step count) where it saves FLOPs, c >= 2r (5
  // iterations: 6 r^2 c + 14 r^3 against 15 r^2 c + 5 r^3, 26% fewer at
  // c = 2r) with r >= 1024, or wherever it can run when asked for
  ctx->runs = gram_runs(ctx->max_steps);
  for (int32_t i = 0; i < n; ++i) {
    MatDev& md = ctx->mats[i];
    ClassHost& ch = ctx->classes[md.cls];
    const bool can = ctx->pairs && ctx->prec == P_FP16 && md.ns_steps == ctx->max_steps && md.ns_steps > 1;
    const bool pays = ch.r_pad >= 1024 && ch.c_pad >= 2 * ch.r_pad;
    md.gram = (can && (cfg->ns_form == MUONH_NS_FORM_GRAM || (cfg->ns_form == MUONH_NS_FORM_AUTO && pays))) ? 1 : 0;
    md.eq = 0;
    if (md.gram) {
      const int longest = *std::max_element(ctx->runs.begin(), ctx->runs.end());
      md.eq = q_exponent(md.a, md.b, md.c_coef, longest, iterate_bound(md.a, md.b, md.c_coef, md.ns_steps));
      ch.gram = true;
    }
    md.o_buf = md.gram ? static_cast<int32_t>(ctx->runs.size() & 1) : (md.ns_steps & 1);
  }

  // ---- fused ||O||^2, <W, O> in the last APPLY (CTA pairs, vector path,
  // matrices whose last iteration is the last launch): 2 slots per pair tile
  for (int32_t i = 0; i < n; ++i) {
    MatDev& md = ctx->mats[i];
    const ClassHost& ch = ctx->classes[md.cls];
    md.fused_dots = (ctx->pairs && md.vec && md.ns_steps > 0 && md.ns_steps == ctx->max_steps) ? 1 : 0;
    md.ns_tiles_bj = ch.c_pad / kBN;
    if (md.fused_dots) {
      md.ns_slots = 8 * (ch.r_pad / (2 * kBM)) * md.ns_tiles_bj;   // per pair tile: 2 CTAs x 4 epilogue warps
      md.ns_slot_base = ctx->n_ns_slots;
      ctx->n_ns_slots += md.ns_slots;
    }
  }
  // ---- matrix groups: with the CTA-pair path and enough elements (or when
  // asked), split the matrices into index ranges of Newton-Schulz work
  {
    std::vector<double> work(n);
    double total = 0.0;
    int64_t elems = 0;
    for (int32_t i = 0; i < n; ++i) {
      const MatDev& md = ctx->mats[i];
      const double r = md.r, c = md.c;
      work[i] = md.ns_steps * (4.0 * r * r * c + 2.0 * r * r * r);
      if (md.gram) {   // per run: Y Y^T and Q Y, plus 4 g - 3 products of r x r factors
        work[i] = 0.0;
        for (int g : ctx->runs) work[i] += 6.0 * r * r * c + (4.0 * g - 3.0) * 2.0 * r * r * r;
      }
      total += work[i];
      elems += md.rows * md.cols;
    }
    // group g ends after the first matrix at which the running work reaches
    // the group's share of the total: halves for two groups; for three, a
    // quarter, a half and a quarter, so that the two exposed phases (the
    // first group's momentum pass, the last group's projection) are short
    // while the middle group's elementwise work hides under the GEMMs of
    // its neighbours.  Every group keeps at least one matrix.
    std::vector<int32_t> bounds{0};
    const int G = want_groups;
    const bool big = cfg->groups > 1 || elems >= kTwoGroupMinElems;
    if (ctx->pairs && G > 1 && n >= G && big && total > 0.0) {
      const double ends2[2] = {0.5, 1.0}, ends3[3] = {0.25, 0.75, 1.0};
      const double* ends = G == 2 ? ends2 : ends3;
      double acc = 0.0;
      for (int32_t i = 0; i < n && static_cast<int>(bounds.size()) < G; ++i) {
        acc += work[i];
        const int g = static_cast<int>(bounds.size()) - 1;
        if (acc >= total * ends[g] && i + 1 > bounds.back() && n - (i + 1) >= G - g - 1) bounds.push_back(i + 1);
      }
    }
    bounds.push_back(n);
    // elementwise tiles, group by group: a group's Y-space matrices first,
    // then its Gram-space ones, so that the tiles of each form are one range
    int64_t e = 0;
    for (size_t g = 0; g + 1 < bounds.size(); ++g) {
      muonh_ctx::Group gr;
      gr.m_first = bounds[g];
      gr.m_count = bounds[g + 1] - bounds[g];
      gr.e_first = e;
      for (int f = 0; f < 2; ++f) {
        muonh_ctx::Subset& su = gr.sub[f];
        su.e_first = e;
        su.m_off = static_cast<int32_t>(ctx->h_mlist.size());
        for (int32_t i = bounds[g]; i < bounds[g + 1]; ++i) {
          MatDev& md = ctx->mats[i];
          if ((md.gram != 0) != (f == 1)) continue;
          md.et_begin = e;
          e += static_cast<int64_t>(md.et_rows) * md.et_cols;
          ctx->h_mlist.push_back(i);
          su.any_unfused |= !md.fused_dots;
          su.any_general |= md.warp_tiled == 0;
          if (md.warp_tiled) su.any_wt[md.transposed ? 1 : 0] = true;
        }
        su.e_end = e;
        su.m_count = static_cast<int32_t>(ctx->h_mlist.size()) - su.m_off;
        gr.any_unfused |= su.any_unfused;
        gr.any_general |= su.any_general;
        for (int k = 0; k < 2; ++k) gr.any_wt[k] |= su.any_wt[k];
      }
      gr.e_end = e;
      gr.any_gram = gr.sub[1].m_count > 0;
      ctx->groups.push_back(gr);
    }
    if (ctx->groups.size() > 1) {
      int least = 0, greatest = 0;
      CUDA_TRY(cudaDeviceGetStreamPriorityRange(&least, &greatest));
      CUDA_TRY(cudaStreamCreateWithPriority(&ctx->ns_stream, cudaStreamNonBlocking, greatest));
      ctx->gev.assign(2 * ctx->groups.size(), nullptr);
      for (cudaEvent_t& ev : ctx->gev) CUDA_TRY(cudaEventCreateWithFlags(&ev, cudaEventDisableTiming));
      for (cudaEvent_t& ev : ctx->split_ev) CUDA_TRY(cudaEventCreateWithFlags(&ev, cudaEventDisableTiming));
    }
  }

  // ---- workspace
  const int parts = ctx->prec == P_FP32 ? 2 : 1;
  for (ClassHost& ch : ctx->classes) {
    ClassDev& cd = ch.dev;
    cd.r_pad = ch.r_pad;
    cd.c_pad = ch.c_pad;
    cd.count = ch.count;
    cd.x_stride = static_cast<int64_t>(ch.r_pad) * ch.c_pad;
    cd.a_stride = static_cast<int64_t>(ch.r_pad) * ch.r_pad;
    const size_t xb = static_cast<size_t>(cd.x_stride) * ch.count * 2;
    const size_t ab = static_cast<size_t>(cd.a_stride) * ch.count * 2;
    for (int part = 0; part < parts; ++part) {
      for (int buf = 0; buf < 2; ++buf) {
        if (dev_alloc(ctx, &cd.x[buf][part], xb) != cudaSuccess)
          return fail(MUONH_ERR_OOM, "workspace allocation of %zu bytes failed", xb);
        CUDA_TRY(cudaMemsetAsync(cd.x[buf][part], 0, xb, s));
      }
      // C = b I + c A is a separate operand of the FP32-mode kernel only
      if (dev_alloc(ctx, &cd.a[part], ab) != cudaSuccess || dev_alloc(ctx, &cd.b[part], ab) != cudaSuccess ||
          (!ctx->pairs && dev_alloc(ctx, &cd.c[part], ab) != cudaSuccess))
        return fail(MUONH_ERR_OOM, "workspace allocation of %zu bytes failed", ab);
      CUDA_TRY(cudaMemsetAsync(cd.a[part], 0, ab, s));
      CUDA_TRY(cudaMemsetAsync(cd.b[part], 0, ab, s));
      if (!ctx->pairs) CUDA_TRY(cudaMemsetAsync(cd.c[part], 0, ab, s));
    }
    if (ctx->prec == P_BF16) {   // residual of B's stored diagonal, per matrix and row
      const size_t db = static_cast<size_t>(ch.r_pad) * ch.count * sizeof(float);
      if (dev_alloc(ctx, reinterpret_cast<void**>(&cd.bdiag), db) != cudaSuccess)
        return fail(MUONH_ERR_OOM, "workspace allocation of %zu bytes failed", db);
      CUDA_TRY(cudaMemsetAsync(cd.bdiag, 0, db, s));
    }
    if (ch.gram) {   // Gram-space form: the second p(A) buffer and the product buffer
      if (dev_alloc(ctx, &cd.p1, ab) != cudaSuccess || dev_alloc(ctx, &cd.t, ab) != cudaSuccess)
        return fail(MUONH_ERR_OOM, "workspace allocation of %zu bytes failed", ab);
      CUDA_TRY(cudaMemsetAsync(cd.p1, 0, ab, s));
      CUDA_TRY(cudaMemsetAsync(cd.t, 0, ab, s));
    }
  }

  // ---- tensor maps: TM_PER_CLASS per class
  std::vector<CUtensorMap> maps(ctx->classes.size() * TM_PER_CLASS);
  std::memset(maps.data(), 0, maps.size() * sizeof(CUtensorMap));
  for (size_t ci = 0; ci < ctx->classes.size(); ++ci) {
    ClassDev& cd = ctx->classes[ci].dev;
    cd.tm_base = static_cast<int32_t>(ci * TM_PER_CLASS);
    CUtensorMap* m = &maps[cd.tm_base];
    for (int part = 0; part < parts; ++part) {
      const int bf = (ctx->prec == P_BF16 && part == 0) ? 1 : 0;
      for (int buf = 0; buf < 2; ++buf) {
        muonh_status st;
        if ((st = encode_map(&m[tm_x(TM_X_K128, buf, part)], cd.x[buf][part], bf, cd.c_pad, cd.r_pad, cd.count, kBM)))
          return st;
        if ((st = encode_map(&m[tm_x(TM_X_K256, buf, part)], cd.x[buf][part], bf, cd.c_pad, cd.r_pad, cd.count, kBN)))
          return st;
        if ((st = encode_map(&m[tm_x(TM_X_MN, buf, part)], cd.x[buf][part], bf, cd.c_pad, cd.r_pad, cd.count, kBK)))
          return st;
        if (part == 0 && ctx->pairs &&
            ((st = encode_map_chunks(&m[TM_X_C64 + buf], cd.x[buf][0], bf, cd.c_pad, cd.r_pad, cd.count, kBK)) ||
             (st = encode_map_chunks(&m[TM_X_C128 + buf], cd.x[buf][0], bf, cd.c_pad, cd.r_pad, cd.count, 2 * kBK))))
          return st;
        if (part == 0 && (st = encode_map(&m[TM_X_ST + buf], cd.x[buf][0], bf, cd.c_pad, cd.r_pad, cd.count, 32, 32,
                                          CU_TENSOR_MAP_SWIZZLE_64B)))
          return st;
      }
      muonh_status st;
      if ((st = encode_map(&m[TM_A_K128 + part], cd.a[part], bf, cd.r_pad, cd.r_pad, cd.count, kBM))) return st;
      if ((st = encode_map(&m[TM_B_K128 + part], cd.b[part], bf, cd.r_pad, cd.r_pad, cd.count, kBM))) return st;
      if (!ctx->pairs &&
          (st = encode_map(&m[TM_C_K256 + part], cd.c[part], bf, cd.r_pad, cd.r_pad, cd.count, kBN)))
        return st;
      if (part == 0 && ctx->pairs) {
        // two k-blocks of A or B' per TMA box
        if ((st = encode_map_chunks(&m[TM_A_C128], cd.a[0], bf, cd.r_pad, cd.r_pad, cd.count, kBM)) ||
            (st = encode_map_chunks(&m[TM_B_C128], cd.b[0], bf, cd.r_pad, cd.r_pad, cd.count, kBM)))
          return st;
        // GRAM and SYMPROD store boxes: 32 x 64 direct, 64 x 32 mirrored
        if ((st = encode_map(&m[TM_A_ST2], cd.a[0], bf, cd.r_pad, cd.r_pad, cd.count, 32, 64, CU_TENSOR_MAP_SWIZZLE_128B)) ||
            (st = encode_map(&m[TM_A_STM], cd.a[0], bf, cd.r_pad, cd.r_pad, cd.count, 64, 32, CU_TENSOR_MAP_SWIZZLE_64B)) ||
            (st = encode_map(&m[TM_B_ST2], cd.b[0], bf, cd.r_pad, cd.r_pad, cd.count, 32, 64, CU_TENSOR_MAP_SWIZZLE_128B)) ||
            (st = encode_map(&m[TM_B_STM], cd.b[0], bf, cd.r_pad, cd.r_pad, cd.count, 64, 32, CU_TENSOR_MAP_SWIZZLE_64B)))
          return st;
        // epilogue store boxes: 32 rows x 32 columns, one per epilogue warp
        if ((st = encode_map(&m[TM_A_ST], cd.a[0], bf, cd.r_pad, cd.r_pad, cd.count, 32, 32, CU_TENSOR_MAP_SWIZZLE_64B)))
          return st;
        if ((st = encode_map(&m[TM_B_ST], cd.b[0], bf, cd.r_pad, cd.r_pad, cd.count, 32, 32, CU_TENSOR_MAP_SWIZZLE_64B)))
          return st;
        if (ctx->classes[ci].gram) {
          if ((st = encode_map(&m[TM_P1_K128], cd.p1, bf, cd.r_pad, cd.r_pad, cd.count, kBM))) return st;
          if ((st = encode_map(&m[TM_T_K128], cd.t, bf, cd.r_pad, cd.r_pad, cd.count, kBM))) return st;
          if ((st = encode_map_chunks(&m[TM_P1_C128], cd.p1, bf, cd.r_pad, cd.r_pad, cd.count, kBM)) ||
              (st = encode_map_chunks(&m[TM_T_C128], cd.t, bf, cd.r_pad, cd.r_pad, cd.count, kBM)))
            return st;
          if ((st = encode_map(&m[TM_P1_ST2], cd.p1, bf, cd.r_pad, cd.r_pad, cd.count, 32, 64, CU_TENSOR_MAP_SWIZZLE_128B)) ||
              (st = encode_map(&m[TM_P1_STM], cd.p1, bf, cd.r_pad, cd.r_pad, cd.count, 64, 32, CU_TENSOR_MAP_SWIZZLE_64B)) ||
              (st = encode_map(&m[TM_T_ST2], cd.t, bf, cd.r_pad, cd.r_pad, cd.count, 32, 64, CU_TENSOR_MAP_SWIZZLE_128B)) ||
              (st = encode_map(&m[TM_T_STM], cd.t, bf, cd.r_pad, cd.r_pad, cd.count, 64, 32, CU_TENSOR_MAP_SWIZZLE_64B)))
            return st;
          if ((st = encode_map(&m[TM_P1_ST], cd.p1, bf, cd.r_pad, cd.r_pad, cd.count, 32, 32,
                               CU_TENSOR_MAP_SWIZZLE_64B)))
            return st;
          if ((st = encode_map(&m[TM_T_ST], cd.t, bf, cd.r_pad, cd.r_pad, cd.count, 32, 32, CU_TENSOR_MAP_SWIZZLE_64B)))
            return st;
        }
      }
    }
  }

  // ---- device tables
  if (dev_alloc(ctx, reinterpret_cast<void**>(&ctx->d_tmaps), maps.size() * sizeof(CUtensorMap)) != cudaSuccess ||
      dev_alloc(ctx, reinterpret_cast<void**>(&ctx->d_mats), n * sizeof(MatDev)) != cudaSuccess ||
      dev_alloc(ctx, reinterpret_cast<void**>(&ctx->d_classes), ctx->classes.size() * sizeof(ClassDev)) !=
          cudaSuccess ||
      dev_alloc(ctx, reinterpret_cast<void**>(&ctx->d_scal), n * sizeof(MatScal)) != cudaSuccess ||
      dev_alloc(ctx, reinterpret_cast<void**>(&ctx->d_step), n * sizeof(MatStep)) != cudaSuccess ||
      dev_alloc(ctx, reinterpret_cast<void**>(&ctx->d_et_mat), n_et * sizeof(int32_t)) != cudaSuccess ||
      dev_alloc(ctx, reinterpret_cast<void**>(&ctx->d_mlist), n * sizeof(int32_t)) != cudaSuccess ||
      dev_alloc(ctx, reinterpret_cast<void**>(&ctx->d_part), 2 * n_et * sizeof(float)) != cudaSuccess ||
      dev_alloc(ctx, reinterpret_cast<void**>(&ctx->d_part64), n_et * sizeof(double)) != cudaSuccess ||
      dev_alloc(ctx, reinterpret_cast<void**>(&ctx->d_part8), kStreamSlots * n_et * sizeof(float)) != cudaSuccess ||
      dev_alloc(ctx, reinterpret_cast<void**>(&ctx->d_part_ns),
                std::max<int64_t>(1, 2 * ctx->n_ns_slots) * sizeof(float)) != cudaSuccess ||
      dev_alloc(ctx, reinterpret_cast<void**>(&ctx->d_wmaps), n * sizeof(CUtensorMap)) != cudaSuccess ||
      dev_alloc(ctx, reinterpret_cast<void**>(&ctx->d_err), (1 + kMaxGroups) * sizeof(int)) != cudaSuccess)   // err, any_rewrite[]
    return fail(MUONH_ERR_OOM, "allocation of the device tables failed");

  std::vector<ClassDev> cdev;
  for (const ClassHost& ch : ctx->classes) cdev.push_back(ch.dev);
  std::vector<int32_t> et_mat(n_et);
  for (int32_t i = 0; i < n; ++i) {
    const MatDev& md = ctx->mats[i];
    std::fill(et_mat.begin() + md.et_begin, et_mat.begin() + md.et_begin + int64_t(md.et_rows) * md.et_cols, i);
  }
  std::vector<MatScal> scal(n);
  for (int32_t i = 0; i < n; ++i) {
    scal[i] = MatScal{};
    scal[i].R = mats[i].radius > 0.f ? mats[i].radius : 0.f;
  }
  std::vector<CUtensorMap> wmaps(n);
  std::memset(wmaps.data(), 0, n * sizeof(CUtensorMap));
  for (int32_t i = 0; i < n; ++i)
    if (ctx->mats[i].fused_dots) {
      muonh_status st = encode_w_map(&wmaps[i], ctx->mats[i]);
      if (st != MUONH_OK) return st;
    }
  CUDA_TRY(cudaMemcpyAsync(ctx->d_wmaps, wmaps.data(), n * sizeof(CUtensorMap), cudaMemcpyHostToDevice, s));
  CUDA_TRY(cudaMemcpyAsync(ctx->d_tmaps, maps.data(), maps.size() * sizeof(CUtensorMap), cudaMemcpyHostToDevice, s));
  CUDA_TRY(cudaMemcpyAsync(ctx->d_mats, ctx->mats.data(), n * sizeof(MatDev), cudaMemcpyHostToDevice, s));
  CUDA_TRY(cudaMemcpyAsync(ctx->d_classes, cdev.data(), cdev.size() * sizeof(ClassDev), cudaMemcpyHostToDevice, s));
  CUDA_TRY(cudaMemcpyAsync(ctx->d_et_mat, et_mat.data(), n_et * sizeof(int32_t), cudaMemcpyHostToDevice, s));
  CUDA_TRY(cudaMemcpyAsync(ctx->d_mlist, ctx->h_mlist.data(), n * sizeof(int32_t), cudaMemcpyHostToDevice, s));
  CUDA_TRY(cudaMemcpyAsync(ctx->d_scal, scal.data(), n * sizeof(MatScal), cudaMemcpyHostToDevice, s));
  CUDA_TRY(cudaMemsetAsync(ctx->d_err, 0, (1 + kMaxGroups) * sizeof(int), s));

  // ---- Newton-Schulz tile lists: per group, one pair (upper-triangle tiles,
  // APPLY tiles) per iteration of the Y-space form (shared when equal), and
  // one pair for the matrices in the Gram-space form
  const int tm = ctx->pairs ? 2 * kBM : kBM;   // tile rows: 128 (single CTA, FP32 mode) or 256 (CTA pairs)
  auto make_lists = [&](const std::vector<int32_t>& active, TileList& gl, TileList& al) -> muonh_status {
    // longest tiles first (the K extent), then matrix by matrix for L2 reuse
    std::vector<int32_t> order = active;
    std::stable_sort(order.begin(), order.end(), [&](int32_t x, int32_t y) {
      const ClassHost& cx = ctx->classes[ctx->mats[x].cls];
      const ClassHost& cy = ctx->classes[ctx->mats[y].cls];
      if (cx.c_pad != cy.c_pad) return cx.c_pad > cy.c_pad;
      return cx.r_pad > cy.r_pad;
    });
    std::vector<TileDesc> gram, apply;
    for (int32_t i : order) {
      const ClassHost& ch = ctx->classes[ctx->mats[i].cls];
      for (int bi = 0; bi < ch.r_pad / tm; ++bi)
        for (int bj = 0; bj < ch.r_pad / kBN; ++bj)
          if (bj * kBN + kBN - 1 >= bi * tm) gram.push_back(TileDesc{i, int16_t(bi), int16_t(bj), ch.c_pad / kBK, ch.r_pad / kBK});
    }
    std::stable_sort(order.begin(), order.end(), [&](int32_t x, int32_t y) {
      return ctx->classes[ctx->mats[x].cls].r_pad > ctx->classes[ctx->mats[y].cls].r_pad;
    });
    for (int32_t i : order) {
      const ClassHost& ch = ctx->classes[ctx->mats[i].cls];
      for (int bi = 0; bi < ch.r_pad / tm; ++bi)
        for (int bj = 0; bj < ch.c_pad / kBN; ++bj)
          apply.push_back(TileDesc{i, int16_t(bi), int16_t(bj), ch.r_pad / kBK, ch.r_pad / kBK});
    }
    gl.count = static_cast<int32_t>(gram.size());
    al.count = static_cast<int32_t>(apply.size());
    for (const TileDesc& td : gram) {
      gl.sum_nk += td.nk;
      gl.sum_nk_sq += td.nk_sq;
    }
    for (const TileDesc& td : apply) al.sum_nk += td.nk;
    if (dev_alloc(ctx, reinterpret_cast<void**>(&gl.dev), std::max<size_t>(1, gram.size()) * sizeof(TileDesc)) !=
            cudaSuccess ||
        dev_alloc(ctx, reinterpret_cast<void**>(&al.dev), std::max<size_t>(1, apply.size()) * sizeof(TileDesc)) !=
            cudaSuccess)
      return fail(MUONH_ERR_OOM, "tile list allocation failed");
    if (!gram.empty())
      CUDA_TRY(cudaMemcpyAsync(gl.dev, gram.data(), gram.size() * sizeof(TileDesc), cudaMemcpyHostToDevice, s));
    if (!apply.empty())
      CUDA_TRY(cudaMemcpyAsync(al.dev, apply.data(), apply.size() * sizeof(TileDesc), cudaMemcpyHostToDevice, s));
    return MUONH_OK;
  };
  for (muonh_ctx::Group& gr : ctx->groups) {
    std::vector<int32_t> prev_active;
    for (int32_t k = 0; k < ctx->max_steps; ++k) {
      std::vector<int32_t> active;
      for (int32_t i = gr.m_first; i < gr.m_first + gr.m_count; ++i)
        if (ctx->mats[i].ns_steps > k && !ctx->mats[i].gram) active.push_back(i);
      if (k > 0 && active == prev_active) {
        gr.gram_lists.push_back(gr.gram_lists.back());
        gr.apply_lists.push_back(gr.apply_lists.back());
        continue;
      }
      prev_active = active;
      TileList gl, al;
      muonh_status st;
      if ((st = make_lists(active, gl, al))) return st;
      gr.gram_lists.push_back(gl);
      gr.apply_lists.push_back(al);
    }
    if (gr.any_gram) {
      std::vector<int32_t> active;
      for (int32_t i = gr.m_first; i < gr.m_first + gr.m_count; ++i)
        if (ctx->mats[i].gram) active.push_back(i);
      muonh_status st;
      if ((st = make_lists(active, gr.gram_upper, gr.gram_apply))) return st;
    }
  }

  // ---- pinned staging ring for the per-step table
  for (int i = 0; i < kRing; ++i) {
    CUDA_TRY(cudaMallocHost(reinterpret_cast<void**>(&ctx->h_step[i]), n * sizeof(MatStep)));
    CUDA_TRY(cudaEventCreateWithFlags(&ctx->ev[i], cudaEventDisableTiming));
  }

  // ---- R = ||W_0||_F where asked, and ||W_0||^2 for every matrix
  const EwParams p = ctx->ew(nullptr);
  int launches = 0;
  const int grid = ctx->sm_count * 8;
  LAUNCH_TRY(launch_init_norm(p, grid, s), "init_norm");
  LAUNCH_TRY(launch_finalize_init(p, s), "finalize_init");
  CUDA_TRY(cudaStreamSynchronize(s));
  guard.ok = true;
  *out = ctx;
  return MUONH_OK;
}

muonh_status muonh_step(muonh_ctx* ctx, const float* lr, const float* const* grads, muonh_stats* stats,
                        void* stream) {
  g_last_error.clear();
  if (!ctx || !lr || !grads) return fail(MUONH_ERR_INVALID_ARG, "ctx, lr or grads is NULL");
  for (int32_t i = 0; i < ctx->n; ++i) {
    if (!grads[i]) return fail(MUONH_ERR_INVALID_ARG, "grads[%d] is NULL", i);
    if (reinterpret_cast<uintptr_t>(grads[i]) & 15) return fail(MUONH_ERR_ALIGNMENT, "grads[%d] not 16-byte aligned", i);
    if (!std::isfinite(lr[i])) return fail(MUONH_ERR_INVALID_ARG, "lr[%d] is not finite", i);
  }
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  // stage (grad pointer, lr) in a pinned slot; reuse waits only if the GPU is kRing steps behind
  const int slot = ctx->ring;
  ctx->ring = (ctx->ring + 1) % kRing;
  CUDA_TRY(cudaEventSynchronize(ctx->ev[slot]));
  for (int32_t i = 0; i < ctx->n; ++i) ctx->h_step[slot][i] = MatStep{grads[i], lr[i], 0.f};
  CUDA_TRY(cudaMemcpyAsync(ctx->d_step, ctx->h_step[slot], ctx->n * sizeof(MatStep), cudaMemcpyHostToDevice, s));
  CUDA_TRY(cudaEventRecord(ctx->ev[slot], s));
  return enqueue_step(ctx, ctx->d_step, stats, s);
}

muonh_status muonh_step_device(muonh_ctx* ctx, const muonh_step_args* args, muonh_stats* stats, void* stream) {
  g_last_error.clear();
  if (!ctx || !args) return fail(MUONH_ERR_INVALID_ARG, "ctx or args is NULL");
  if (reinterpret_cast<uintptr_t>(args) & 15) return fail(MUONH_ERR_ALIGNMENT, "args not 16-byte aligned");
  return enqueue_step(ctx, reinterpret_cast<const MatStep*>(args), stats, static_cast<cudaStream_t>(stream));
}

}  // extern "C"

namespace {

// Every launch of one step, reading the per-matrix (gradient, lr) table from
// device memory `step_args`: kernels and event record/waits only.
muonh_status enqueue_step(muonh_ctx* ctx, const MatStep* step_args, muonh_stats* stats, cudaStream_t s) {
  ctx->step_src = step_args;
  int launches = 0;
  const int grid = ctx->sm_count * 8;
  // elementwise grids: one resident wave, or short blocks when the launch
  // overlaps the other group's GEMMs
  auto ew_grid = [&](int kind, const EwParams& p, bool overlap) {
    if (!overlap) return ctx->ew_warp_grid[kind];
    const int64_t tiles = p.e_end - p.e_first;
    return static_cast<int>(std::max<int64_t>(1, (tiles + kOverlapTilesPerBlock - 1) / kOverlapTilesPerBlock));
  };
  // the elementwise work of group g, or of its matrices in one form (sub 0:
  // Y-space, 1: Gram-space)
  auto front = [&](int g, cudaStream_t st, bool overlap, int sub) -> muonh_status {   // momentum, ||X||, X
    const muonh_ctx::Group& gr = ctx->groups[g];
    const EwParams p = ctx->ew(stats, g, sub);
    const bool* any_wt = sub < 0 ? gr.any_wt : gr.sub[sub].any_wt;
    const bool any_general = sub < 0 ? gr.any_general : gr.sub[sub].any_general;
    for (int tall = 0; tall < 2; ++tall)
      if (any_wt[tall])
        STEP_LAUNCH_ON(MUONH_PHASE_MOMENTUM_NORM, launch_momentum_warp(p, tall != 0, ew_grid(tall, p, overlap), st),
                       "momentum_warp", st);
    if (any_general) STEP_LAUNCH_ON(MUONH_PHASE_MOMENTUM_NORM, launch_momentum_norm(p, grid, st), "momentum_norm", st);
    STEP_LAUNCH_ON(MUONH_PHASE_FINALIZE_INPUT, launch_finalize_input(p, st), "finalize_input", st);
    STEP_LAUNCH_ON(MUONH_PHASE_WRITE_X, launch_write_x(p, grid, st), "write_x", st);
    return MUONH_OK;
  };
  for (double& f : ctx->step_flops) f = 0.0;
  // tensor-core FLOPs of a launch over `sum_k` k-blocks of tiles (tile rows x 256 x 64 each)
  const double tile_flops = 2.0 * (ctx->pairs ? 2 * kBM : kBM) * kBN * kBK * (ctx->pairs ? 1 : 3);
  // the GEMMs of group g: its Y-space iterations (parts & 1) and its
  // Gram-space runs (parts & 2)
  auto newton_schulz = [&](int g, cudaStream_t st, int parts) -> muonh_status {
    const muonh_ctx::Group& gr = ctx->groups[g];
    NsParams base{};
    base.mats = ctx->d_mats;
    base.classes = ctx->d_classes;
    base.tmaps = ctx->d_tmaps;
    base.err = ctx->d_err;
    base.scal = ctx->d_scal;
    base.wmaps = ctx->d_wmaps;
    base.part_ns = ctx->d_part_ns;
    const int pairs_max = std::max(1, ctx->sm_count / 2);
    auto pair_grid = [&](int ntiles) { return std::min(pairs_max, std::max(1, ntiles)); };
    // ---- Y-space form: A = Y Y^T, B' = a I + b A + c A A, Y <- B' Y per iteration
    for (int32_t k = 0; k < ((parts & 1) ? ctx->max_steps : 0); ++k) {
      NsParams np = base;
      np.src = k & 1;
      np.iter = k;
      np.lhs = RR_A;
      np.rhs = RR_A;
      np.out = RR_B;
      np.tiles = gr.gram_lists[k].dev;
      np.ntiles = gr.gram_lists[k].count;
      if (np.ntiles == 0) continue;   // no matrix of this group iterates k times in this form
      ctx->step_flops[MUONH_PHASE_NS_GRAM] += tile_flops * gr.gram_lists[k].sum_nk;
      ctx->step_flops[MUONH_PHASE_NS_SQUARE] += tile_flops * gr.gram_lists[k].sum_nk_sq;
      ctx->step_flops[MUONH_PHASE_NS_APPLY] += tile_flops * gr.apply_lists[k].sum_nk;
      if (ctx->pairs) {
        STEP_LAUNCH_ON(MUONH_PHASE_NS_GRAM, launch_ns_gemm_pair(M_GRAM, ctx->prec, np, pair_grid(np.ntiles), st),
                       "ns_gram", st);
        STEP_LAUNCH_ON(MUONH_PHASE_NS_SQUARE, launch_ns_gemm_pair(M_SQUARE, ctx->prec, np, pair_grid(np.ntiles), st),
                       "ns_square", st);
        np.tiles = gr.apply_lists[k].dev;
        np.ntiles = gr.apply_lists[k].count;
        np.lhs = RR_B;
        np.lhs_kind = RK_P;
        np.apply_kappa = k == 0;
        const int amode = (k == ctx->max_steps - 1) ? M_APPLY_LAST : M_APPLY;
        STEP_LAUNCH_ON(MUONH_PHASE_NS_APPLY, launch_ns_gemm_pair(amode, ctx->prec, np, pair_grid(np.ntiles), st),
                       "ns_apply", st);
      } else {
        const int ggrid = std::min(ctx->sm_count, std::max(1, np.ntiles));
        STEP_LAUNCH_ON(MUONH_PHASE_NS_GRAM, launch_ns_gemm(M_GRAM, ctx->prec, np, ggrid, st), "ns_gram", st);
        STEP_LAUNCH_ON(MUONH_PHASE_NS_SQUARE, launch_ns_gemm(M_SQUARE, ctx->prec, np, ggrid, st), "ns_square", st);
        np.tiles = gr.apply_lists[k].dev;
        np.ntiles = gr.apply_lists[k].count;
        STEP_LAUNCH_ON(MUONH_PHASE_NS_APPLY,
                       launch_ns_gemm(M_APPLY, ctx->prec, np, std::min(ctx->sm_count, std::max(1, np.ntiles)), st),
                       "ns_apply", st);
      }
    }
    // ---- Gram-space form, run by run (see muonh_ns_gemm.cu): A_0 = Y Y^T; per
    // iteration P = p(A) into B' or P1 (alternating); between iterations
    // T = A P, A = T P; the run's product Q = P1 P0 (into T) and P2 Q (into
    // P1); one Y <- Q Y (or P0 Y for a run of one) ends the run
    if (gr.any_gram && (parts & 2)) {
      const TileList& up = gr.gram_upper;
      const TileList& ap = gr.gram_apply;
      int k0 = 0;
      for (size_t j = 0; j < ctx->runs.size(); ++j) {
        const int run = ctx->runs[j];
        NsParams np = base;
        np.src = static_cast<int>(j & 1);
        np.iter = k0;
        np.tiles = up.dev;
        np.ntiles = up.count;
        ctx->step_flops[MUONH_PHASE_NS_GRAM] += tile_flops * up.sum_nk;
        STEP_LAUNCH_ON(MUONH_PHASE_NS_GRAM, launch_ns_gemm_pair(M_GRAM, ctx->prec, np, pair_grid(up.count), st),
                       "ns_gram", st);
        auto product = [&](int lhs, int lk, int rhs, int rk, int out, int ok) -> muonh_status {
          NsParams pp = np;
          pp.lhs = lhs;
          pp.lhs_kind = lk;
          pp.rhs = rhs;
          pp.rhs_kind = rk;
          pp.out = out;
          pp.out_kind = ok;
          ctx->step_flops[MUONH_PHASE_NS_PRODUCT] += tile_flops * up.sum_nk_sq;
          STEP_LAUNCH_ON(MUONH_PHASE_NS_PRODUCT, launch_ns_gemm_pair(M_SYMPROD, ctx->prec, pp, pair_grid(up.count), st),
                         "ns_product", st);
          return MUONH_OK;
        };
        int qbuf = RR_B, qkind = RK_P;
        for (int i = 0; i < run; ++i) {
          const int pbuf = (i & 1) ? RR_P1 : RR_B;
          np.iter = k0 + i;
          np.lhs = RR_A;
          np.rhs = RR_A;
          np.out = pbuf;
          ctx->step_flops[MUONH_PHASE_NS_SQUARE] += tile_flops * up.sum_nk_sq;
          STEP_LAUNCH_ON(MUONH_PHASE_NS_SQUARE, launch_ns_gemm_pair(M_SQUARE, ctx->prec, np, pair_grid(up.count), st),
                         "ns_square", st);
          muonh_status ps;
          if (i + 1 < run) {   // A_{k+1} = (A_k P_k) P_k
            if ((ps = product(RR_A, RK_A, pbuf, RK_P, RR_T, RK_A)) || (ps = product(RR_T, RK_A, pbuf, RK_P, RR_A, RK_A)))
              return ps;
          }
          if (i == 1) {        // Q = P1 P0
            if ((ps = product(RR_P1, RK_P, RR_B, RK_P, RR_T, RK_Q))) return ps;
            qbuf = RR_T;
            qkind = RK_Q;
          } else if (i == 2) { // Q = P2 Q (P2 is in B')
            if ((ps = product(RR_B, RK_P, RR_T, RK_Q, RR_P1, RK_Q))) return ps;
            qbuf = RR_P1;
          }
        }
        np.iter = k0 + run - 1;
        np.tiles = ap.dev;
        np.ntiles = ap.count;
        np.lhs = qbuf;
        np.lhs_kind = qkind;
        np.apply_kappa = j == 0;
        ctx->step_flops[MUONH_PHASE_NS_APPLY] += tile_flops * ap.sum_nk;
        const int amode = (j + 1 == ctx->runs.size()) ? M_APPLY_LAST : M_APPLY;
        STEP_LAUNCH_ON(MUONH_PHASE_NS_APPLY, launch_ns_gemm_pair(amode, ctx->prec, np, pair_grid(ap.count), st),
                       "ns_apply", st);
        k0 += run;
      }
    }
    return MUONH_OK;
  };
  auto back = [&](int g, cudaStream_t st, bool overlap, int sub) -> muonh_status {   // dots, projection, stats
    const muonh_ctx::Group& gr = ctx->groups[g];
    const EwParams p = ctx->ew(stats, g, sub);
    const bool* any_wt = sub < 0 ? gr.any_wt : gr.sub[sub].any_wt;
    const bool any_general = sub < 0 ? gr.any_general : gr.sub[sub].any_general;
    const bool any_unfused = sub < 0 ? gr.any_unfused : gr.sub[sub].any_unfused;
    if (any_unfused) STEP_LAUNCH_ON(MUONH_PHASE_UPDATE_DOTS, launch_update_dots(p, grid, st), "update_dots", st);
    STEP_LAUNCH_ON(MUONH_PHASE_FINALIZE_UPDATE, launch_finalize_update(p, st), "finalize_update", st);
    for (int tall = 0; tall < 2; ++tall)
      if (any_wt[tall])
        STEP_LAUNCH_ON(MUONH_PHASE_PROJECT, launch_project_warp(p, tall != 0, ew_grid(2 + tall, p, overlap), st),
                       "project_warp", st);
    if (any_general) STEP_LAUNCH_ON(MUONH_PHASE_PROJECT, launch_project(p, grid, st), "project", st);
    STEP_LAUNCH_ON(MUONH_PHASE_FINALIZE_STEP, launch_finalize_step(p, st), "finalize_step", st);
    return MUONH_OK;
  };
  muonh_status st;
  if (ctx->groups.size() == 1) {
    if ((st = front(0, s, false, -1)) || (st = newton_schulz(0, s, 3)) || (st = back(0, s, false, -1))) return st;
  } else {
    // caller's stream: front(0) | front(1) | back(0), front(2) | ... | back(G-1)
    // GEMM stream:              | NS(0) ...| NS(1) ............| ... |
    // group g's front work overlaps NS(g-1), its back work NS(g+1).  The two
    // ends, where nothing else runs, are split by Newton-Schulz form when a
    // group has both: the first group's Y-space GEMMs start after only the
    // Y-space matrices' front work, and its Gram-space front work overlaps
    // them; the last group runs its Gram-space GEMMs first, and their back
    // work overlaps its Y-space GEMMs.
    cudaStream_t hs = ctx->ns_stream;
    const int G = static_cast<int>(ctx->groups.size());
    auto both = [&](int g) { return ctx->groups[g].sub[0].m_count > 0 && ctx->groups[g].sub[1].m_count > 0; };
    const bool split_first = both(0), split_last = both(G - 1);
    if (split_first) {
      if ((st = front(0, s, false, 0))) return st;
      CUDA_TRY(cudaEventRecord(ctx->split_ev[0], s));
      if ((st = front(0, s, true, 1))) return st;
    } else if ((st = front(0, s, false, -1))) {
      return st;
    }
    CUDA_TRY(cudaEventRecord(ctx->gev[0], s));
    for (int g = 0; g < G; ++g) {
      if (g == 0 && split_first) {
        CUDA_TRY(cudaStreamWaitEvent(hs, ctx->split_ev[0], 0));
        if ((st = newton_schulz(g, hs, 1))) return st;
        CUDA_TRY(cudaStreamWaitEvent(hs, ctx->gev[0], 0));
        if ((st = newton_schulz(g, hs, 2))) return st;
      } else if (g == G - 1 && split_last) {
        CUDA_TRY(cudaStreamWaitEvent(hs, ctx->gev[2 * g], 0));
        if ((st = newton_schulz(g, hs, 2))) return st;
        CUDA_TRY(cudaEventRecord(ctx->split_ev[1], hs));
        if ((st = newton_schulz(g, hs, 1))) return st;
      } else {
        CUDA_TRY(cudaStreamWaitEvent(hs, ctx->gev[2 * g], 0));
        if ((st = newton_schulz(g, hs, 3))) return st;
      }
      CUDA_TRY(cudaEventRecord(ctx->gev[2 * g + 1], hs));
      if (g + 1 < G) {
        if ((st = front(g + 1, s, true, -1))) return st;
        CUDA_TRY(cudaEventRecord(ctx->gev[2 * (g + 1)], s));   // before back(g - 1): NS(g + 1) need not wait for it
      }
      if (g >= 1) {
        CUDA_TRY(cudaStreamWaitEvent(s, ctx->gev[2 * (g - 1) + 1], 0));
        if ((st = back(g - 1, s, true, -1))) return st;
      }
    }
    if (split_last) {
      CUDA_TRY(cudaStreamWaitEvent(s, ctx->split_ev[1], 0));
      if ((st = back(G - 1, s, true, 1))) return st;
      CUDA_TRY(cudaStreamWaitEvent(s, ctx->gev[2 * (G - 1) + 1], 0));
      if ((st = back(G - 1, s, false, 0))) return st;
    } else {
      CUDA_TRY(cudaStreamWaitEvent(s, ctx->gev[2 * (G - 1) + 1], 0));
      if ((st = back(G - 1, s, false, -1))) return st;
    }
  }
  ctx->last_launches = launches;
  ctx->last_stream = s;
  ++ctx->step_count;
  return MUONH_OK;
}

}  // namespace

extern "C" {

muonh_status muonh_get_stats(muonh_ctx* ctx, muonh_stats* host_out) {
  g_last_error.clear();
  if (!ctx || !host_out) return fail(MUONH_ERR_INVALID_ARG, "ctx or host_out is NULL");
  CUDA_TRY(cudaStreamSynchronize(ctx->last_stream));
  std::vector<MatScal> scal(ctx->n);
  CUDA_TRY(cudaMemcpy(scal.data(), ctx->d_scal, ctx->n * sizeof(MatScal), cudaMemcpyDeviceToHost));
  for (int32_t i = 0; i < ctx->n; ++i) host_out[i] = scal[i].stats;
  return MUONH_OK;
}

muonh_status muonh_get_update(muonh_ctx* ctx, int32_t i, float* dst, int64_t ld, void* stream) {
  g_last_error.clear();
  if (!ctx || !dst) return fail(MUONH_ERR_INVALID_ARG, "ctx or dst is NULL");
  if (i < 0 || i >= ctx->n) return fail(MUONH_ERR_INVALID_ARG, "matrix index %d out of range", i);
  if (ld < ctx->mats[i].cols) return fail(MUONH_ERR_INVALID_ARG, "ld < cols");
  int launches = 0;
  LAUNCH_TRY(launch_export_update(ctx->ew(nullptr), i, dst, ld, static_cast<cudaStream_t>(stream)), "export_update");
  return MUONH_OK;
}

muonh_status muonh_get_radius(const muonh_ctx* ctx, float* host_R) {
  g_last_error.clear();
  if (!ctx || !host_R) return fail(MUONH_ERR_INVALID_ARG, "ctx or host_R is NULL");
  CUDA_TRY(cudaStreamSynchronize(ctx->last_stream));
  std::vector<MatScal> scal(ctx->n);
  CUDA_TRY(cudaMemcpy(scal.data(), ctx->d_scal, ctx->n * sizeof(MatScal), cudaMemcpyDeviceToHost));
  for (int32_t i = 0; i < ctx->n; ++i) host_R[i] = scal[i].R;
  return MUONH_OK;
}

muonh_status muonh_export_state(muonh_ctx* ctx, void* buf, size_t* len) {
  g_last_error.clear();
  if (!ctx || !len) return fail(MUONH_ERR_INVALID_ARG, "ctx or len is NULL");
  const size_t need = 16 + static_cast<size_t>(ctx->n) * (2 * sizeof(float) + sizeof(double));
  if (!buf) {
    *len = need;
    return MUONH_OK;
  }
  if (*len < need) return fail(MUONH_ERR_INVALID_ARG, "buffer of %zu bytes, %zu needed", *len, need);
  CUDA_TRY(cudaStreamSynchronize(ctx->last_stream));
  std::vector<MatScal> scal(ctx->n);
  CUDA_TRY(cudaMemcpy(scal.data(), ctx->d_scal, ctx->n * sizeof(MatScal), cudaMemcpyDeviceToHost));
  uint8_t* o = static_cast<uint8_t*>(buf);
  const uint32_t hdr[2] = {kStateMagic, static_cast<uint32_t>(ctx->n)};
  std::memcpy(o, hdr, 8);
  std::memcpy(o + 8, &ctx->step_count, 8);
  o += 16;
  for (int32_t i = 0; i < ctx->n; ++i) {
    std::memcpy(o, &scal[i].R, sizeof(float));
    std::memcpy(o + sizeof(float), &scal[i].wnorm2, sizeof(double));
    std::memcpy(o + sizeof(float) + sizeof(double), &scal[i].sigma, sizeof(float));
    o += 2 * sizeof(float) + sizeof(double);
  }
  *len = need;
  return MUONH_OK;
}

muonh_status muonh_import_state(muonh_ctx* ctx, const void* buf, size_t len) {
  g_last_error.clear();
  if (!ctx || !buf) return fail(MUONH_ERR_INVALID_ARG, "ctx or buf is NULL");
  const size_t need = 16 + static_cast<size_t>(ctx->n) * (2 * sizeof(float) + sizeof(double));
  if (len != need) return fail(MUONH_ERR_INVALID_ARG, "state of %zu bytes, %zu expected", len, need);
  const uint8_t* in = static_cast<const uint8_t*>(buf);
  uint32_t hdr[2];
  std::memcpy(hdr, in, 8);
  if (hdr[0] != kStateMagic || hdr[1] != static_cast<uint32_t>(ctx->n))
    return fail(MUONH_ERR_INVALID_ARG, "state was not exported from a context with %d matrices", ctx->n);
  CUDA_TRY(cudaStreamSynchronize(ctx->last_stream));
  std::vector<MatScal> scal(ctx->n);
  CUDA_TRY(cudaMemcpy(scal.data(), ctx->d_scal, ctx->n * sizeof(MatScal), cudaMemcpyDeviceToHost));
  int64_t steps;
  std::memcpy(&steps, in + 8, 8);
  in += 16;
  for (int32_t i = 0; i < ctx->n; ++i) {
    std::memcpy(&scal[i].R, in, sizeof(float));
    std::memcpy(&scal[i].wnorm2, in + sizeof(float), sizeof(double));
    std::memcpy(&scal[i].sigma, in + sizeof(float) + sizeof(double), sizeof(float));
    in += 2 * sizeof(float) + sizeof(double);
  }
  CUDA_TRY(cudaMemcpy(ctx->d_scal, scal.data(), ctx->n * sizeof(MatScal), cudaMemcpyHostToDevice));
  ctx->step_count = steps;
  return MUONH_OK;
}

muonh_status muonh_device_status(muonh_ctx* ctx) {
  g_last_error.clear();
  if (!ctx) return fail(MUONH_ERR_INVALID_ARG, "ctx is NULL");
  CUDA_TRY(cudaStreamSynchronize(ctx->last_stream));
  int err = 0;
  CUDA_TRY(cudaMemcpy(&err, ctx->d_err, sizeof(int), cudaMemcpyDeviceToHost));
  if (err) {
    CUDA_TRY(cudaMemset(ctx->d_err, 0, sizeof(int)));
    return fail(MUONH_ERR_TIMEOUT, "a device-side wait gave up (Newton-Schulz GEMM pipeline)");
  }
  return MUONH_OK;
}

int32_t muonh_last_launch_count(const muonh_ctx* ctx) { return ctx ? ctx->last_launches : 0; }

muonh_status muonh_check_wait_timeout(double seconds, void* stream) {
  g_last_error.clear();
  if (!(seconds > 0.0 && seconds <= 10.0)) return fail(MUONH_ERR_INVALID_ARG, "seconds must be in (0, 10]");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int* d_flag = nullptr;
  CUDA_TRY(cudaMalloc(&d_flag, sizeof(int)));
  int flag = 0;
  cudaError_t e = cudaMemsetAsync(d_flag, 0, sizeof(int), s);
  if (e == cudaSuccess) e = launch_wait_probe(d_flag, static_cast<uint64_t>(seconds * 1e9), s);
  if (e == cudaSuccess) e = cudaMemcpyAsync(&flag, d_flag, sizeof(int), cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  cudaFree(d_flag);
  if (e != cudaSuccess) return fail(MUONH_ERR_CUDA, "wait probe: %s", cudaGetErrorString(e));
  if (!flag) return fail(MUONH_ERR_CUDA, "wait probe: the bounded wait did not give up");
  return fail(MUONH_ERR_TIMEOUT, "wait probe: the bounded wait gave up as designed");
}

muonh_status muonh_enable_timing(muonh_ctx* ctx, int32_t enable) {
  g_last_error.clear();
  if (!ctx) return fail(MUONH_ERR_INVALID_ARG, "ctx is NULL");
  ctx->timing = enable != 0;
  return MUONH_OK;
}

muonh_status muonh_phase_times(muonh_ctx* ctx, float* ms_out, int64_t* launches_out) {
  g_last_error.clear();
  if (!ctx || !ms_out) return fail(MUONH_ERR_INVALID_ARG, "ctx or ms_out is NULL");
  CUDA_TRY(cudaStreamSynchronize(ctx->last_stream));
  double acc[MUONH_NUM_PHASES] = {};
  int64_t cnt[MUONH_NUM_PHASES] = {};
  for (auto& t : ctx->timed) {
    float ms = 0.f;
    CUDA_TRY(cudaEventElapsedTime(&ms, t.begin, t.end));
    acc[t.phase] += ms;
    cnt[t.phase] += 1;
    ctx->event_pool.push_back(t.begin);
    ctx->event_pool.push_back(t.end);
  }
  ctx->timed.clear();
  for (int i = 0; i < MUONH_NUM_PHASES; ++i) {
    ms_out[i] = static_cast<float>(acc[i]);
    if (launches_out) launches_out[i] = cnt[i];
  }
  return MUONH_OK;
}

muonh_status muonh_phase_flops(const muonh_ctx* ctx, double* flops_out) {
  g_last_error.clear();
  if (!ctx || !flops_out) return fail(MUONH_ERR_INVALID_ARG, "ctx or flops_out is NULL");
  for (int i = 0; i < MUONH_NUM_PHASES; ++i) flops_out[i] = ctx->step_flops[i];
  return MUONH_OK;
}

void muonh_destroy(muonh_ctx* ctx) {
  if (!ctx) return;
  cudaDeviceSynchronize();
  release(ctx);
}

}  // extern "C"
