// Auxiliary HBM-bound kernels of the optimizer (sm_100a):
//  * checkpoint parameter averaging: the Puro-2B release is the equal
//    average of six checkpoints of its constant-LR continuation (Sec. 3.4);
//  * AdamW for the parameter group outside MuonH (Table 8: embeddings,
//    normalisation layers, LM head; decoupled weight decay, bias-corrected
//    moments).
// Both stream their operands once with 16-byte vector accesses in a grid
// sized to the SM count.
#include <algorithm>
#include <cmath>

#include "muonh_common.cuh"

namespace muonh {
namespace {

constexpr int kAvgMax = 16;
constexpr int kAdamMax = 32;
constexpr int kAuxThreads = 256;
constexpr int64_t kAdamChunk = 4096;

struct AvgParams {
  const void* in[kAvgMax];
  void* out;
  int32_t k, in_bf16, out_bf16;
  int64_t count;
};

// Elements of one 16-byte input vector and their conversion to fp32.
template <bool BF16>
struct InVec;
template <>
struct InVec<false> {
  static constexpr int kElems = 4;
  __device__ static void add(float* acc, const uint4& r) {
    acc[0] += __uint_as_float(r.x);
    acc[1] += __uint_as_float(r.y);
    acc[2] += __uint_as_float(r.z);
    acc[3] += __uint_as_float(r.w);
  }
  __device__ static float load1(const void* base, int64_t j) { return static_cast<const float*>(base)[j]; }
};
template <>
struct InVec<true> {
  static constexpr int kElems = 8;
  __device__ static void add2(float* acc, uint32_t u) {
    // bf16 -> fp32 is exact: the 16 bits become the high half of the fp32 word
    acc[0] += __uint_as_float(u << 16);
    acc[1] += __uint_as_float(u & 0xffff0000u);
  }
  __device__ static void add(float* acc, const uint4& r) {
    add2(acc + 0, r.x);
    add2(acc + 2, r.y);
    add2(acc + 4, r.z);
    add2(acc + 6, r.w);
  }
  __device__ static float load1(const void* base, int64_t j) {
    return __bfloat162float(static_cast<const __nv_bfloat16*>(base)[j]);
  }
};

template <bool BF16, int N>
__device__ __forceinline__ void store_vec(void* base, int64_t j, const float* v) {
  if constexpr (!BF16) {
    float* d = static_cast<float*>(base) + j;
#pragma unroll
    for (int q = 0; q < N; q += 4) *reinterpret_cast<float4*>(d + q) = make_float4(v[q], v[q + 1], v[q + 2], v[q + 3]);
  } else {
    uint32_t w[N / 2];
#pragma unroll
    for (int q = 0; q < N / 2; ++q) {
      __nv_bfloat162 h = __floats2bfloat162_rn(v[2 * q], v[2 * q + 1]);
      w[q] = *reinterpret_cast<uint32_t*>(&h);
    }
    __nv_bfloat16* d = static_cast<__nv_bfloat16*>(base) + j;
    if constexpr (N == 8)
      *reinterpret_cast<uint4*>(d) = make_uint4(w[0], w[1], w[2], w[3]);
    else
      *reinterpret_cast<uint2*>(d) = make_uint2(w[0], w[1]);
  }
}

template <bool BF16>
__device__ __forceinline__ void store1(void* base, int64_t j, float v) {
  if constexpr (!BF16)
    static_cast<float*>(base)[j] = v;
  else
    static_cast<__nv_bfloat16*>(base)[j] = __float2bfloat16_rn(v);
}

// out = (in[0] + in[1] + ... + in[k-1]) / k, added in that order in fp32.
// Each thread owns one 16-byte vector of every input per iteration; the
// inputs are read in groups of 8 whose loads are all issued before the first
// add, so a thread keeps up to 128 bytes in flight.
template <bool IN_BF16, bool OUT_BF16>
__global__ void __launch_bounds__(kAuxThreads) average_kernel(const __grid_constant__ AvgParams p) {
  constexpr int E = InVec<IN_BF16>::kElems;
  constexpr int kGroup = 8;
  const int64_t nvec = p.count / E;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  const float kk = static_cast<float>(p.k);
  for (int64_t v = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; v < nvec; v += stride) {
    const int64_t j = E * v;
    float acc[E];
#pragma unroll
    for (int e = 0; e < E; ++e) acc[e] = 0.f;
    for (int g0 = 0; g0 < p.k; g0 += kGroup) {
      uint4 r[kGroup];
#pragma unroll
      for (int q = 0; q < kGroup; ++q)
        if (g0 + q < p.k)
          r[q] = *reinterpret_cast<const uint4*>(static_cast<const char*>(p.in[g0 + q]) +
                                                 j * (IN_BF16 ? 2 : 4));
#pragma unroll
      for (int q = 0; q < kGroup; ++q)
        if (g0 + q < p.k) InVec<IN_BF16>::add(acc, r[q]);
    }
#pragma unroll
    for (int e = 0; e < E; ++e) acc[e] /= kk;
    store_vec<OUT_BF16, E>(p.out, j, acc);
  }
  // ragged tail (count % E elements)
  for (int64_t j = E * nvec + blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; j < p.count; j += stride) {
    float acc = 0.f;
    for (int i = 0; i < p.k; ++i) acc += InVec<IN_BF16>::load1(p.in[i], j);
    store1<OUT_BF16>(p.out, j, acc / kk);
  }
}

struct AdamBatch {
  int32_t n;
  int32_t vec[kAdamMax];
  int64_t chunk_begin[kAdamMax + 1];
  muonh_adamw_tensor t[kAdamMax];
  float lr, beta1, beta2, eps, decay, bc1, bc2;
};

__device__ __forceinline__ void adamw_one(float& p, float& m, float& v, float g, const AdamBatch& b) {
  p *= b.decay;                                        // decoupled weight decay on the current p
  m = fmaf(b.beta1, m, (1.f - b.beta1) * g);
  v = fmaf(b.beta2, v, (1.f - b.beta2) * g * g);
  const float m_hat = m / b.bc1;
  const float v_hat = v / b.bc2;
  p -= b.lr * m_hat / (sqrtf(v_hat) + b.eps);
}

__global__ void __launch_bounds__(kAuxThreads) adamw_kernel(const __grid_constant__ AdamBatch b) {
  const int64_t nchunks = b.chunk_begin[b.n];
  for (int64_t c = blockIdx.x; c < nchunks; c += gridDim.x) {
    int i = 0;
    while (c >= b.chunk_begin[i + 1]) ++i;
    const muonh_adamw_tensor& t = b.t[i];
    const int64_t base = (c - b.chunk_begin[i]) * kAdamChunk;
    const int64_t end = base + kAdamChunk < t.count ? base + kAdamChunk : t.count;
    if (b.vec[i]) {
      for (int64_t j = base + 4 * threadIdx.x; j < end; j += 4 * kAuxThreads) {
        if (j + 3 < end) {
          float4 p = *reinterpret_cast<const float4*>(t.p + j);
          float4 m = *reinterpret_cast<const float4*>(t.m + j);
          float4 v = *reinterpret_cast<const float4*>(t.v + j);
          const float4 g = *reinterpret_cast<const float4*>(t.g + j);
          adamw_one(p.x, m.x, v.x, g.x, b);
          adamw_one(p.y, m.y, v.y, g.y, b);
          adamw_one(p.z, m.z, v.z, g.z, b);
          adamw_one(p.w, m.w, v.w, g.w, b);
          *reinterpret_cast<float4*>(t.p + j) = p;
          *reinterpret_cast<float4*>(t.m + j) = m;
          *reinterpret_cast<float4*>(t.v + j) = v;
        } else {
          for (int64_t q = j; q < end; ++q) adamw_one(t.p[q], t.m[q], t.v[q], t.g[q], b);
        }
      }
    } else {
      for (int64_t q = base + threadIdx.x; q < end; q += kAuxThreads) adamw_one(t.p[q], t.m[q], t.v[q], t.g[q], b);
    }
  }
}

int aux_grid(int64_t work_units) {
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  return static_cast<int>(std::max<int64_t>(1, std::min<int64_t>(work_units, static_cast<int64_t>(sms) * 8)));
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

muonh_status aux_fail(muonh_status st, const char* msg) {
  set_error_message(msg);
  return st;
}

}  // namespace
}  // namespace muonh

using namespace muonh;

extern "C" muonh_status muonh_average(void* out, int32_t out_dtype, const void* const* in, int32_t in_dtype,
                                      int32_t k, int64_t count, void* stream) {
  set_error_message("");
  if (!in || k < 1 || k > kAvgMax || count < 0)
    return aux_fail(MUONH_ERR_INVALID_ARG, "need in, 1 <= k <= 16 and count >= 0");
  if ((out_dtype != MUONH_DTYPE_F32 && out_dtype != MUONH_DTYPE_BF16) ||
      (in_dtype != MUONH_DTYPE_F32 && in_dtype != MUONH_DTYPE_BF16))
    return aux_fail(MUONH_ERR_INVALID_ARG, "dtypes must be MUONH_DTYPE_F32 or MUONH_DTYPE_BF16");
  if (count == 0) return MUONH_OK;   // pointers of empty buffers may be NULL
  if (!out) return aux_fail(MUONH_ERR_INVALID_ARG, "out is NULL");
  AvgParams p{};
  for (int i = 0; i < k; ++i) {
    if (!in[i]) return aux_fail(MUONH_ERR_INVALID_ARG, "an input pointer is NULL");
    if (!aligned16(in[i])) return aux_fail(MUONH_ERR_ALIGNMENT, "inputs must be 16-byte aligned");
    p.in[i] = in[i];
  }
  if (!aligned16(out)) return aux_fail(MUONH_ERR_ALIGNMENT, "out must be 16-byte aligned");
  p.out = out;
  p.k = k;
  p.in_bf16 = in_dtype == MUONH_DTYPE_BF16;
  p.out_bf16 = out_dtype == MUONH_DTYPE_BF16;
  p.count = count;
  const int64_t elems_per_vec = p.in_bf16 ? 8 : 4;
  const int grid = aux_grid((count / elems_per_vec + kAuxThreads - 1) / kAuxThreads + 1);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (p.in_bf16 && p.out_bf16)
    average_kernel<true, true><<<grid, kAuxThreads, 0, s>>>(p);
  else if (p.in_bf16)
    average_kernel<true, false><<<grid, kAuxThreads, 0, s>>>(p);
  else if (p.out_bf16)
    average_kernel<false, true><<<grid, kAuxThreads, 0, s>>>(p);
  else
    average_kernel<false, false><<<grid, kAuxThreads, 0, s>>>(p);
  if (cudaGetLastError() != cudaSuccess) return aux_fail(MUONH_ERR_CUDA, "launch of average_kernel failed");
  return MUONH_OK;
}

extern "C" muonh_status muonh_adamw_step(const muonh_adamw_tensor* tensors, int32_t n, const muonh_adamw_config* cfg,
                                         int64_t step, void* stream) {
  set_error_message("");
  if (!tensors || n < 0 || !cfg || step < 1) return aux_fail(MUONH_ERR_INVALID_ARG, "need tensors, cfg and step >= 1");
  if (!std::isfinite(cfg->lr) || !(cfg->beta1 >= 0.f && cfg->beta1 < 1.f) || !(cfg->beta2 >= 0.f && cfg->beta2 < 1.f) ||
      !(cfg->eps >= 0.f) || !std::isfinite(cfg->weight_decay))
    return aux_fail(MUONH_ERR_INVALID_ARG, "lr, weight_decay finite; betas in [0, 1); eps >= 0");
  for (int32_t i = 0; i < n; ++i) {
    const muonh_adamw_tensor& t = tensors[i];
    if (t.count < 0 || (t.count > 0 && (!t.p || !t.m || !t.v || !t.g)))
      return aux_fail(MUONH_ERR_INVALID_ARG, "tensor with NULL pointer or negative count");
    if ((reinterpret_cast<uintptr_t>(t.p) | reinterpret_cast<uintptr_t>(t.m) | reinterpret_cast<uintptr_t>(t.v) |
         reinterpret_cast<uintptr_t>(t.g)) & 3)
      return aux_fail(MUONH_ERR_ALIGNMENT, "tensors must be 4-byte aligned");
  }
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  for (int32_t first = 0; first < n; first += kAdamMax) {
    AdamBatch b{};
    b.n = std::min(kAdamMax, n - first);
    b.chunk_begin[0] = 0;
    for (int32_t i = 0; i < b.n; ++i) {
      b.t[i] = tensors[first + i];
      b.vec[i] = aligned16(b.t[i].p) && aligned16(b.t[i].m) && aligned16(b.t[i].v) && aligned16(b.t[i].g);
      b.chunk_begin[i + 1] = b.chunk_begin[i] + (b.t[i].count + kAdamChunk - 1) / kAdamChunk;
    }
    if (b.chunk_begin[b.n] == 0) continue;
    b.lr = cfg->lr;
    b.beta1 = cfg->beta1;
    b.beta2 = cfg->beta2;
    b.eps = cfg->eps;
    b.decay = static_cast<float>(1.0 - static_cast<double>(cfg->lr) * cfg->weight_decay);
    b.bc1 = static_cast<float>(1.0 - std::pow(static_cast<double>(cfg->beta1), static_cast<double>(step)));
    b.bc2 = static_cast<float>(1.0 - std::pow(static_cast<double>(cfg->beta2), static_cast<double>(step)));
    adamw_kernel<<<aux_grid(b.chunk_begin[b.n]), kAuxThreads, 0, s>>>(b);
    if (cudaGetLastError() != cudaSuccess) return aux_fail(MUONH_ERR_CUDA, "launch of adamw_kernel failed");
  }
  return MUONH_OK;
}
