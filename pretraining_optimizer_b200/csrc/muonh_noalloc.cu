// Allocation-free variant of the first kernel stage of the MuonH step for a
// single matrix: M <- beta M + G and ||X||_F of the Newton-Schulz input
// X = G + beta M (Nesterov) or M.
//
// Some callers cannot call cudaMalloc: code that runs while a stream is being
// captured into a CUDA graph in the global capture mode, programs whose
// device memory is wholly owned by a framework's caching allocator or a
// fixed arena, and real-time loops that must not take the driver's
// allocation locks.  This entry point allocates nothing.  Its scratch (one
// fp32 partial sum per 4096-element tile) is the file-scope array below,
// which every GPU that loads the library holds until the process exits.
//
// The arithmetic and the tile decomposition are those of the context-based
// step (muonh_step), so for the same inputs the momentum is bitwise equal and
// the norm agrees to rounding of the final square root.
#include <mutex>

#include "muonh_common.cuh"

namespace muonh {
namespace {

constexpr int64_t kNoAllocMaxTiles = 65536;   // 256 KB of scratch: up to 268,435,456 elements
static __device__ __align__(256) float g_noalloc_partials[kNoAllocMaxTiles];

constexpr int kMaxDevices = 64;
std::mutex g_setup_mutex;
// Per device ordinal, looked up once in the primary context: the scratch
// array's device address and the SM count that sizes the grid.
float* g_partials_ptr[kMaxDevices] = {};
int g_sm_count[kMaxDevices] = {};

struct OneMatrix {
  float* m;
  const float* g;
  int64_t rows, cols, ld;
  int32_t vec, nesterov;
  float beta;
  int32_t th, tw, tiles_c;
  int64_t tiles;
};

__device__ __forceinline__ float4 ld4(const float* base, const OneMatrix& a, int64_t row, int64_t col) {
  float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
  if (row >= a.rows) return v;
  const float* src = base + row * a.ld + col;
  if (a.vec) {
    if (col < a.cols) v = *reinterpret_cast<const float4*>(src);
  } else {
    if (col + 0 < a.cols) v.x = src[0];
    if (col + 1 < a.cols) v.y = src[1];
    if (col + 2 < a.cols) v.z = src[2];
    if (col + 3 < a.cols) v.w = src[3];
  }
  return v;
}

__device__ __forceinline__ void st4(float* base, const OneMatrix& a, int64_t row, int64_t col, float4 v) {
  if (row >= a.rows) return;
  float* dst = base + row * a.ld + col;
  if (a.vec) {
    if (col < a.cols) *reinterpret_cast<float4*>(dst) = v;
  } else {
    if (col + 0 < a.cols) dst[0] = v.x;
    if (col + 1 < a.cols) dst[1] = v.y;
    if (col + 2 < a.cols) dst[2] = v.z;
    if (col + 3 < a.cols) dst[3] = v.w;
  }
}

template <typename T>
__device__ __forceinline__ T block_sum_na(T v, T* red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  __syncthreads();
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
  __syncthreads();
  T s = 0;
  if (threadIdx.x == 0)
    for (int i = 0; i < kEwThreads / 32; ++i) s += red[i];
  return s;
}

__global__ void __launch_bounds__(kEwThreads) momentum_norm_noalloc_kernel(const OneMatrix a, float* partials) {
  __shared__ float red[kEwThreads / 32];
  const int tpr = a.tw / 4;
  const int rin = threadIdx.x / tpr, cin = (threadIdx.x % tpr) * 4, rstep = kEwThreads / tpr;
  for (int64_t e = blockIdx.x; e < a.tiles; e += gridDim.x) {
    const int64_t r0 = (e / a.tiles_c) * a.th, c0 = (e % a.tiles_c) * a.tw;
    float4 gv[4], mv[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      gv[j] = ld4(a.g, a, r0 + rin + rstep * j, c0 + cin);
      mv[j] = ld4(a.m, a, r0 + rin + rstep * j, c0 + cin);
    }
    float acc = 0.f;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      float4 m = mv[j];
      m.x = fmaf(a.beta, m.x, gv[j].x);
      m.y = fmaf(a.beta, m.y, gv[j].y);
      m.z = fmaf(a.beta, m.z, gv[j].z);
      m.w = fmaf(a.beta, m.w, gv[j].w);
      st4(a.m, a, r0 + rin + rstep * j, c0 + cin, m);
      float4 x = m;
      if (a.nesterov) {
        x.x = fmaf(a.beta, m.x, gv[j].x);
        x.y = fmaf(a.beta, m.y, gv[j].y);
        x.z = fmaf(a.beta, m.z, gv[j].z);
        x.w = fmaf(a.beta, m.w, gv[j].w);
      }
      acc = fmaf(x.x, x.x, acc);
      acc = fmaf(x.y, x.y, acc);
      acc = fmaf(x.z, x.z, acc);
      acc = fmaf(x.w, x.w, acc);
    }
    const float s = block_sum_na(acc, red);
    if (threadIdx.x == 0) partials[e] = s;
  }
}

__global__ void __launch_bounds__(kEwThreads) norm_noalloc_kernel(const float* partials, int64_t tiles,
                                                                 double* out) {
  __shared__ double red[kEwThreads / 32];
  double s = 0.0;
  for (int64_t i = threadIdx.x; i < tiles; i += kEwThreads) s += static_cast<double>(partials[i]);
  s = block_sum_na(s, red);
  if (threadIdx.x == 0) *out = sqrt(s);
}

muonh_status na_fail(muonh_status st, const char* msg) {
  set_error_message(msg);
  return st;
}

}  // namespace
}  // namespace muonh

using namespace muonh;

extern "C" muonh_status muonh_momentum_norm_noalloc(float* m, const float* g, int64_t rows, int64_t cols,
                                                    int64_t ld, float beta, int32_t nesterov, double* x_norm,
                                                    void* stream) {
  set_error_message("");
  if (!m || !g || !x_norm) return na_fail(MUONH_ERR_INVALID_ARG, "m, g or x_norm is NULL");
  if (rows <= 0 || cols <= 0 || ld < cols) return na_fail(MUONH_ERR_INVALID_ARG, "need rows, cols > 0 and ld >= cols");
  if ((reinterpret_cast<uintptr_t>(m) & 15) || (reinterpret_cast<uintptr_t>(g) & 15))
    return na_fail(MUONH_ERR_ALIGNMENT, "m and g must be 16-byte aligned");
  if (!std::isfinite(beta)) return na_fail(MUONH_ERR_INVALID_ARG, "beta must be finite");

  OneMatrix a;
  a.m = m;
  a.g = g;
  a.rows = rows;
  a.cols = cols;
  a.ld = ld;
  a.vec = (cols % 4 == 0 && ld % 4 == 0) ? 1 : 0;
  a.nesterov = nesterov ? 1 : 0;
  a.beta = beta;
  // tile shapes of the context-based step (tall matrices: 64 x 64)
  if (rows > cols) {
    a.th = a.tw = kEwTile;
  } else {
    int tw = kEwTile;
    while (tw < 512 && tw < cols) tw *= 2;
    a.tw = tw;
    a.th = kEwTile * kEwTile / tw;
  }
  const int64_t tiles_r = (rows + a.th - 1) / a.th;
  a.tiles_c = static_cast<int32_t>((cols + a.tw - 1) / a.tw);
  a.tiles = tiles_r * a.tiles_c;
  if (a.tiles > kNoAllocMaxTiles)
    return na_fail(MUONH_ERR_UNSUPPORTED,
                   "matrix too large for the allocation-free path (more than 65536 tiles of 4096 elements)");

  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices)
    return na_fail(MUONH_ERR_CUDA, "cudaGetDevice failed");
  float* partials = nullptr;
  int sms = 0;
  {
    std::lock_guard<std::mutex> lock(g_setup_mutex);
    if (!g_partials_ptr[dev]) {
      void* ptr = nullptr;
      if (cudaGetSymbolAddress(&ptr, g_noalloc_partials) != cudaSuccess || !ptr)
        return na_fail(MUONH_ERR_CUDA, "cudaGetSymbolAddress of the scratch array failed");
      int count = 0;
      if (cudaDeviceGetAttribute(&count, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || count <= 0)
        return na_fail(MUONH_ERR_CUDA, "cudaDeviceGetAttribute(multiProcessorCount) failed");
      g_sm_count[dev] = count;
      g_partials_ptr[dev] = static_cast<float*>(ptr);
    }
    partials = g_partials_ptr[dev];
    sms = g_sm_count[dev];
  }
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int64_t grid = std::min<int64_t>(a.tiles, static_cast<int64_t>(sms) * 8);
  momentum_norm_noalloc_kernel<<<static_cast<int>(grid), kEwThreads, 0, s>>>(a, partials);
  if (cudaGetLastError() != cudaSuccess) return na_fail(MUONH_ERR_CUDA, "launch of momentum_norm_noalloc failed");
  norm_noalloc_kernel<<<1, kEwThreads, 0, s>>>(partials, a.tiles, x_norm);
  if (cudaGetLastError() != cudaSuccess) return na_fail(MUONH_ERR_CUDA, "launch of norm_noalloc failed");
  return MUONH_OK;
}
