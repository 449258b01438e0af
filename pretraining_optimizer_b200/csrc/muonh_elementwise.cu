// HBM-bound kernels of the MuonH step (sm_100a): momentum, the Frobenius
// normalisation of the Newton-Schulz input, the hyperball projection of the
// Puro-2B report (Sec. 3.3, Eq. (1)) and the per-matrix reductions.
//
// Every kernel walks 64 x 64 tiles of the weights' own layout (rows x cols,
// row stride ld) in a persistent grid; a tile belongs to one matrix, so all
// branches on matrix properties are block-uniform.  Per-tile partial sums go
// to a fixed slot; the finalize kernels (one block per matrix) add the slots
// of a matrix in a fixed order in fp64, so every result is bitwise
// reproducible run to run.
#include "muonh_common.cuh"

namespace muonh {
namespace {

// Every tile holds 4096 elements: 64 x 64 for tall matrices (whose X/O is
// the transpose), th x tw with tw = min(512, cols rounded up to 64) rows
// otherwise.  A thread covers 4 consecutive columns in each of 4 passes.
constexpr int kPasses = 4;

struct TileCoord {
  int mi;
  int64_t r0, c0;
  int rin, cin;     // this thread's first row / column inside the tile
  int rstep;        // rows between passes
};

__device__ __forceinline__ TileCoord tile_coord(const EwParams& p, int64_t e) {
  TileCoord t;
  t.mi = p.et_mat[e];
  const MatDev& md = p.mats[t.mi];
  const int64_t local = e - md.et_begin;
  t.r0 = (local / md.et_cols) * md.et_th;
  t.c0 = (local % md.et_cols) * md.et_tw;
  const int tpr = md.et_tw / 4;    // threads per tile row
  t.rin = threadIdx.x / tpr;
  t.cin = (threadIdx.x % tpr) * 4;
  t.rstep = kEwThreads / tpr;
  return t;
}

// Load 4 consecutive fp32 (row, col..col+3), zero outside the matrix.
__device__ __forceinline__ float4 load4(const float* base, const MatDev& md, int64_t row, int64_t col) {
  float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
  if (row >= md.rows) return v;
  const float* src = base + row * md.ld + col;
  if (md.vec) {
    if (col < md.cols) v = *reinterpret_cast<const float4*>(src);
  } else {
    if (col + 0 < md.cols) v.x = src[0];
    if (col + 1 < md.cols) v.y = src[1];
    if (col + 2 < md.cols) v.z = src[2];
    if (col + 3 < md.cols) v.w = src[3];
  }
  return v;
}

// Tile-relative variants: base points at the tile's first element, (r, c)
// are tile coordinates, rows_left/cols_left bound the matrix.
__device__ __forceinline__ float4 load4_rel(const float* base, const MatDev& md, int r, int c, int64_t rows_left,
                                            int64_t cols_left) {
  float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
  if (r >= rows_left) return v;
  const float* src = base + r * md.ld + c;
  if (md.vec) {
    if (c < cols_left) v = *reinterpret_cast<const float4*>(src);
  } else {
    if (c + 0 < cols_left) v.x = src[0];
    if (c + 1 < cols_left) v.y = src[1];
    if (c + 2 < cols_left) v.z = src[2];
    if (c + 3 < cols_left) v.w = src[3];
  }
  return v;
}

__device__ __forceinline__ void store4_rel(float* base, const MatDev& md, int r, int c, int64_t rows_left,
                                           int64_t cols_left, float4 v) {
  if (r >= rows_left) return;
  float* dst = base + r * md.ld + c;
  if (md.vec) {
    if (c < cols_left) *reinterpret_cast<float4*>(dst) = v;
  } else {
    if (c + 0 < cols_left) dst[0] = v.x;
    if (c + 1 < cols_left) dst[1] = v.y;
    if (c + 2 < cols_left) dst[2] = v.z;
    if (c + 3 < cols_left) dst[3] = v.w;
  }
}

template <typename T>
__device__ __forceinline__ T block_sum(T v, T* red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  const int w = threadIdx.x >> 5;
  __syncthreads();   // red may still be read by a previous call
  if ((threadIdx.x & 31) == 0) red[w] = v;
  __syncthreads();
  T s = 0;
  if (threadIdx.x == 0)
    for (int i = 0; i < kEwThreads / 32; ++i) s += red[i];
  return s;   // valid in thread 0
}

// ---------------------------------------------------- 16-bit X storage
__device__ __forceinline__ void put16(void* hi, void* lo, int64_t off, float v, int prec) {
  if (prec == P_BF16) {
    reinterpret_cast<__nv_bfloat16*>(hi)[off] = __float2bfloat16_rn(v);
  } else {
    const __half h = __float2half_rn(v);
    reinterpret_cast<__half*>(hi)[off] = h;
    if (prec == P_FP32) reinterpret_cast<__half*>(lo)[off] = __float2half_rn(v - __half2float(h));
  }
}

struct XView {
  void* hi;
  void* lo;
  int64_t ld;   // c_pad
};

__device__ __forceinline__ XView x_view(const EwParams& p, const MatDev& md, int buf) {
  const ClassDev& cd = p.classes[md.cls];
  XView v;
  const int64_t off = md.z * cd.x_stride * 2;
  v.hi = static_cast<uint8_t*>(cd.x[buf][0]) + off;
  v.lo = cd.x[buf][1] ? static_cast<uint8_t*>(cd.x[buf][1]) + off : nullptr;
  v.ld = cd.c_pad;
  return v;
}

// Four consecutive stored values X[row][col..col+3] (8-byte aligned).
__device__ __forceinline__ float4 x4(const XView& xv, int64_t off, int prec) {
  float4 r;
  const uint2 u = *reinterpret_cast<const uint2*>(static_cast<const uint16_t*>(xv.hi) + off);
  if (prec == P_BF16) {
    const __nv_bfloat162 a = *reinterpret_cast<const __nv_bfloat162*>(&u.x);
    const __nv_bfloat162 b = *reinterpret_cast<const __nv_bfloat162*>(&u.y);
    r = make_float4(__low2float(a), __high2float(a), __low2float(b), __high2float(b));
  } else {
    const __half2 a = *reinterpret_cast<const __half2*>(&u.x);
    const __half2 b = *reinterpret_cast<const __half2*>(&u.y);
    r = make_float4(__low2float(a), __high2float(a), __low2float(b), __high2float(b));
    if (prec == P_FP32) {
      const uint2 l = *reinterpret_cast<const uint2*>(static_cast<const uint16_t*>(xv.lo) + off);
      const __half2 c = *reinterpret_cast<const __half2*>(&l.x);
      const __half2 d = *reinterpret_cast<const __half2*>(&l.y);
      r.x += __low2float(c);
      r.y += __high2float(c);
      r.z += __low2float(d);
      r.w += __high2float(d);
    }
  }
  return r;
}

// O(r0 + i, c0 + j) = X[c0 + j][r0 + i] of a tall matrix into tile[i][j]
// (64 x 64), with 16-byte loads along X's rows.
__device__ __forceinline__ void load_o_tile_t(const XView& xv, const TileCoord& tc, int prec,
                                              float (*tile)[kEwTile + 1]) {
#pragma unroll
  for (int pass = 0; pass < 2; ++pass) {
    const int q = threadIdx.x / 8 + 32 * pass;
    const int p0 = (threadIdx.x % 8) * 8;
    const int64_t off = (tc.c0 + q) * xv.ld + tc.r0 + p0;
    const uint4 u = *reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(xv.hi) + off);
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
    float v[8];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      if (prec == P_BF16) {
        const __nv_bfloat162 h = *reinterpret_cast<const __nv_bfloat162*>(&w[k]);
        v[2 * k] = __low2float(h);
        v[2 * k + 1] = __high2float(h);
      } else {
        const __half2 h = *reinterpret_cast<const __half2*>(&w[k]);
        v[2 * k] = __low2float(h);
        v[2 * k + 1] = __high2float(h);
      }
    }
    if (prec == P_FP32) {
      const uint4 l = *reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(xv.lo) + off);
      const uint32_t lw[4] = {l.x, l.y, l.z, l.w};
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const __half2 h = *reinterpret_cast<const __half2*>(&lw[k]);
        v[2 * k] += __low2float(h);
        v[2 * k + 1] += __high2float(h);
      }
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) tile[p0 + i][q] = v[i];
  }
}

// O at W coordinates (row, col..col+3), stored scale: direct for wide
// matrices, from the transposed smem tile for tall ones.
__device__ __forceinline__ float4 o_at(const XView& xv, const MatDev& md, const TileCoord& tc, int r, int c,
                                       int prec, float (*tile)[kEwTile + 1]) {
  if (!md.transposed) {
    // tiles may reach past the padded width when cols is not a multiple of the tile width
    if (tc.c0 + c >= xv.ld) return make_float4(0.f, 0.f, 0.f, 0.f);
    return x4(xv, (tc.r0 + r) * xv.ld + tc.c0 + c, prec);
  }
  return make_float4(tile[r][c], tile[r][c + 1], tile[r][c + 2], tile[r][c + 3]);
}

// X[off .. off+3] = scale * (x, y, z, w) in the 16-bit storage (off multiple of 4).
__device__ __forceinline__ void put4(const XView& xv, int64_t off, float4 x, float scale, int prec) {
  if (prec == P_FP16) {
    __half2 h01 = __floats2half2_rn(x.x * scale, x.y * scale);
    __half2 h23 = __floats2half2_rn(x.z * scale, x.w * scale);
    uint2 u;
    u.x = *reinterpret_cast<uint32_t*>(&h01);
    u.y = *reinterpret_cast<uint32_t*>(&h23);
    *reinterpret_cast<uint2*>(static_cast<__half*>(xv.hi) + off) = u;
  } else {
    put16(xv.hi, xv.lo, off + 0, x.x * scale, prec);
    put16(xv.hi, xv.lo, off + 1, x.y * scale, prec);
    put16(xv.hi, xv.lo, off + 2, x.z * scale, prec);
    put16(xv.hi, xv.lo, off + 3, x.w * scale, prec);
  }
}

// X[c0 + q][r0 + p] = tile[p][q] for a tall matrix's 64 x 64 tile.
__device__ __forceinline__ void store_x_tile_t(const XView& xv, const TileCoord& tc, int prec,
                                               float (*tile)[kEwTile + 1]) {
  const int q = threadIdx.x / 4, p0 = (threadIdx.x % 4) * 16;
  const int64_t off = (tc.c0 + q) * xv.ld + tc.r0 + p0;
  if (prec == P_FP16) {
    uint4 u[2];
    __half* h = reinterpret_cast<__half*>(u);
#pragma unroll
    for (int i = 0; i < 16; ++i) h[i] = __float2half_rn(tile[p0 + i][q]);
    uint4* dst = reinterpret_cast<uint4*>(static_cast<__half*>(xv.hi) + off);
    dst[0] = u[0];
    dst[1] = u[1];
  } else {
#pragma unroll
    for (int i = 0; i < 16; ++i) put16(xv.hi, xv.lo, off + i, tile[p0 + i][q], prec);
  }
}

// Index of this block's last tile of matrix md (the loop increment then
// moves past the matrix): lets the general kernels skip warp-tiled matrices.
__device__ __forceinline__ int64_t skip_matrix(const MatDev& md, int64_t e) {
  const int64_t end = md.et_begin + static_cast<int64_t>(md.et_rows) * md.et_cols;
  return e + ((end - e + gridDim.x - 1) / gridDim.x - 1) * gridDim.x;
}

// ------------------------------------------------------------- kernels
__global__ void __launch_bounds__(kEwThreads) init_norm_kernel(const EwParams p) {
  __shared__ double red[kEwThreads / 32];
  for (int64_t e = p.e_first + blockIdx.x; e < p.e_end; e += gridDim.x) {
    const TileCoord tc = tile_coord(p, e);
    const MatDev& md = p.mats[tc.mi];
    double acc = 0.0;
    for (int j = 0; j < kPasses; ++j) {
      const float4 w = load4(md.w, md, tc.r0 + tc.rin + tc.rstep * j, tc.c0 + tc.cin);
      acc += (double)w.x * w.x + (double)w.y * w.y + (double)w.z * w.z + (double)w.w * w.w;
    }
    const double s = block_sum(acc, red);
    if (threadIdx.x == 0) p.part64[e] = s;
  }
}

// Loads and stores of one thread's 4 consecutive elements at tile coordinates
// (r, c); FULL tiles (whole tile inside the matrix, vector path) skip every
// bounds check and use 32-bit offsets from the tile origin.
template <bool FULL>
__device__ __forceinline__ float4 tile_ld(const float* base, const MatDev& md, int r, int c, int64_t rows_left,
                                          int64_t cols_left) {
  if (FULL) return *reinterpret_cast<const float4*>(base + (r * static_cast<int>(md.ld) + c));
  return load4_rel(base, md, r, c, rows_left, cols_left);
}
template <bool FULL>
__device__ __forceinline__ void tile_st(float* base, const MatDev& md, int r, int c, int64_t rows_left,
                                        int64_t cols_left, float4 v) {
  if (FULL) {
    *reinterpret_cast<float4*>(base + (r * static_cast<int>(md.ld) + c)) = v;
    return;
  }
  store4_rel(base, md, r, c, rows_left, cols_left, v);
}

__device__ __forceinline__ bool tile_is_full(const MatDev& md, const TileCoord& tc) {
  return md.vec && tc.r0 + md.et_th <= md.rows && tc.c0 + md.et_tw <= md.cols;
}

template <bool FULL>
__device__ __forceinline__ float momentum_tile(const EwParams& p, const MatDev& md, const TileCoord& tc,
                                               const float* g, float sigma, const XView& xv,
                                               float (*tile)[kEwTile + 1]) {
  const float beta = md.beta;
  const float* gb = g + tc.r0 * md.ld + tc.c0;
  float* mb = md.m + tc.r0 * md.ld + tc.c0;
  const int64_t rows_left = md.rows - tc.r0, cols_left = md.cols - tc.c0;
  float acc = 0.f;
  // two passes at a time: both loads of each pass issued before its store
#pragma unroll
  for (int j0 = 0; j0 < kPasses; j0 += 2) {
    float4 gv[2], mv[2];
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const int r = tc.rin + tc.rstep * (j0 + u);
      gv[u] = tile_ld<FULL>(gb, md, r, tc.cin, rows_left, cols_left);
      mv[u] = tile_ld<FULL>(mb, md, r, tc.cin, rows_left, cols_left);
    }
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const int r = tc.rin + tc.rstep * (j0 + u);
      float4 m = mv[u];
      m.x = fmaf(beta, m.x, gv[u].x);
      m.y = fmaf(beta, m.y, gv[u].y);
      m.z = fmaf(beta, m.z, gv[u].z);
      m.w = fmaf(beta, m.w, gv[u].w);
      tile_st<FULL>(mb, md, r, tc.cin, rows_left, cols_left, m);
      float4 x = m;
      if (md.nesterov) {
        x.x = fmaf(beta, m.x, gv[u].x);
        x.y = fmaf(beta, m.y, gv[u].y);
        x.z = fmaf(beta, m.z, gv[u].z);
        x.w = fmaf(beta, m.w, gv[u].w);
      }
      acc = fmaf(x.x, x.x, acc);
      acc = fmaf(x.y, x.y, acc);
      acc = fmaf(x.z, x.z, acc);
      acc = fmaf(x.w, x.w, acc);
      if (sigma > 0.f) {
        if (!md.transposed) {
          const int64_t col = tc.c0 + tc.cin;
          if (FULL || col < xv.ld) put4(xv, (tc.r0 + r) * xv.ld + col, x, sigma, p.prec);
        } else {
          tile[r][tc.cin + 0] = x.x * sigma;
          tile[r][tc.cin + 1] = x.y * sigma;
          tile[r][tc.cin + 2] = x.z * sigma;
          tile[r][tc.cin + 3] = x.w * sigma;
        }
      }
    }
  }
  return acc;
}

// M <- beta M + G; X = G + beta M (Nesterov) or M; partial ||X||^2.  When
// sigma > 0 it also writes the 16-bit Newton-Schulz input sigma * X (wide
// orientation; tall matrices through a transposed shared-memory tile).
__global__ void __launch_bounds__(kEwThreads, 5) momentum_norm_kernel(const EwParams p) {
  __shared__ float red[kEwThreads / 32];
  __shared__ float tile[kEwTile][kEwTile + 1];
  for (int64_t e = p.e_first + blockIdx.x; e < p.e_end; e += gridDim.x) {
    const TileCoord tc = tile_coord(p, e);
    const MatDev& md = p.mats[tc.mi];
    if (md.warp_tiled) {
      e = skip_matrix(md, e);
      continue;
    }
    const float* g = p.step[tc.mi].g;
    const float sigma = p.scal[tc.mi].sigma;
    const XView xv = x_view(p, md, 0);
    if (sigma > 0.f && md.transposed) __syncthreads();   // previous tile's readers are done with `tile`
    const float acc = tile_is_full(md, tc) ? momentum_tile<true>(p, md, tc, g, sigma, xv, tile)
                                           : momentum_tile<false>(p, md, tc, g, sigma, xv, tile);
    if (sigma > 0.f && md.transposed) {
      __syncthreads();
      store_x_tile_t(xv, tc, p.prec, tile);
    }
    const float s = block_sum(acc, red);
    if (threadIdx.x == 0) p.part[e] = s;
  }
}

// X_stored = xscale * X into NS buffer 0 (wide orientation, transposed for tall W).
__global__ void __launch_bounds__(kEwThreads, 6) write_x_kernel(const EwParams p) {
  __shared__ float tile[kEwTile][kEwTile + 1];
  if (*reinterpret_cast<const volatile int*>(p.any_rewrite) == 0) return;   // every X already written
  for (int64_t e = p.e_first + blockIdx.x; e < p.e_end; e += gridDim.x) {
    const int mi = p.et_mat[e];
    if (!p.scal[mi].rewrite) {
      // the momentum kernel already wrote this matrix's X: jump past its tiles
      const MatDev& ms = p.mats[mi];
      const int64_t end = ms.et_begin + static_cast<int64_t>(ms.et_rows) * ms.et_cols;
      const int64_t skip = (end - e + gridDim.x - 1) / gridDim.x - 1;
      e += skip * gridDim.x;
      continue;
    }
    const TileCoord tc = tile_coord(p, e);
    const MatDev& md = p.mats[tc.mi];
    const float* g = p.step[tc.mi].g;
    const float beta = md.beta;
    const float xs = p.scal[tc.mi].xscale;
    const XView xv = x_view(p, md, 0);
    if (!md.transposed) {
#pragma unroll
      for (int j = 0; j < kPasses; ++j) {
        const int64_t row = tc.r0 + tc.rin + tc.rstep * j, col = tc.c0 + tc.cin;
        const float4 gv = load4(g, md, row, col);
        const float4 mv = load4(md.m, md, row, col);
        float4 x = mv;
        if (md.nesterov) {
          x.x = fmaf(beta, mv.x, gv.x);
          x.y = fmaf(beta, mv.y, gv.y);
          x.z = fmaf(beta, mv.z, gv.z);
          x.w = fmaf(beta, mv.w, gv.w);
        }
        if (col >= xv.ld) continue;   // past the padded width (see o_at)
        const int64_t off = row * xv.ld + col;
        if (p.prec == P_FP16) {
          __half2 h01 = __floats2half2_rn(x.x * xs, x.y * xs);
          __half2 h23 = __floats2half2_rn(x.z * xs, x.w * xs);
          uint2 u;
          u.x = *reinterpret_cast<uint32_t*>(&h01);
          u.y = *reinterpret_cast<uint32_t*>(&h23);
          *reinterpret_cast<uint2*>(static_cast<__half*>(xv.hi) + off) = u;
        } else {
          put16(xv.hi, xv.lo, off + 0, x.x * xs, p.prec);
          put16(xv.hi, xv.lo, off + 1, x.y * xs, p.prec);
          put16(xv.hi, xv.lo, off + 2, x.z * xs, p.prec);
          put16(xv.hi, xv.lo, off + 3, x.w * xs, p.prec);
        }
      }
    } else {
      __syncthreads();   // previous tile's readers are done with `tile`
      const int tx = tc.cin / 4;
#pragma unroll
      for (int j = 0; j < kPasses; ++j) {
        const int r = tc.rin + tc.rstep * j;
        const int64_t row = tc.r0 + r, col = tc.c0 + tx * 4;
        const float4 gv = load4(g, md, row, col);
        const float4 mv = load4(md.m, md, row, col);
        float4 x = mv;
        if (md.nesterov) {
          x.x = fmaf(beta, mv.x, gv.x);
          x.y = fmaf(beta, mv.y, gv.y);
          x.z = fmaf(beta, mv.z, gv.z);
          x.w = fmaf(beta, mv.w, gv.w);
        }
        tile[r][tx * 4 + 0] = x.x * xs;
        tile[r][tx * 4 + 1] = x.y * xs;
        tile[r][tx * 4 + 2] = x.z * xs;
        tile[r][tx * 4 + 3] = x.w * xs;
      }
      __syncthreads();
      // X[q][p] = tile[p][q]: thread writes 16 consecutive p of one q
      const int q = threadIdx.x / 4, p0 = (threadIdx.x % 4) * 16;
      const int64_t off = (tc.c0 + q) * xv.ld + tc.r0 + p0;
      if (p.prec == P_FP16) {
        uint4 u[2];
        __half* h = reinterpret_cast<__half*>(u);
#pragma unroll
        for (int i = 0; i < 16; ++i) h[i] = __float2half_rn(tile[p0 + i][q]);
        uint4* dst = reinterpret_cast<uint4*>(static_cast<__half*>(xv.hi) + off);
        dst[0] = u[0];
        dst[1] = u[1];
      } else {
#pragma unroll
        for (int i = 0; i < 16; ++i) put16(xv.hi, xv.lo, off + i, tile[p0 + i][q], p.prec);
      }
    }
  }
}

// Partial ||O||^2 and <W, O> (O at its stored scale).
__global__ void __launch_bounds__(kEwThreads, 8) update_dots_kernel(const EwParams p) {
  __shared__ float tile[kEwTile][kEwTile + 1];
  __shared__ float red[kEwThreads / 32];
  for (int64_t e = p.e_first + blockIdx.x; e < p.e_end; e += gridDim.x) {
    const TileCoord tc = tile_coord(p, e);
    const MatDev& md = p.mats[tc.mi];
    if (md.fused_dots) continue;   // the last APPLY produced this matrix's partials
    const XView xv = x_view(p, md, md.o_buf);
    if (md.transposed) {
      __syncthreads();
      load_o_tile_t(xv, tc, p.prec, tile);
      __syncthreads();
    }
    float oo = 0.f, wo = 0.f;
#pragma unroll
    for (int j = 0; j < kPasses; ++j) {
      const int r = tc.rin + tc.rstep * j;
      const float4 w = load4(md.w, md, tc.r0 + r, tc.c0 + tc.cin);
      const float4 o = o_at(xv, md, tc, r, tc.cin, p.prec, tile);
      oo = fmaf(o.x, o.x, fmaf(o.y, o.y, fmaf(o.z, o.z, fmaf(o.w, o.w, oo))));
      wo = fmaf(w.x, o.x, fmaf(w.y, o.y, fmaf(w.z, o.z, fmaf(w.w, o.w, wo))));
    }
    const float s_oo = block_sum(oo, red);
    const float s_wo = block_sum(wo, red);
    if (threadIdx.x == 0) {
      p.part[2 * e] = s_oo;
      p.part[2 * e + 1] = s_wo;
    }
  }
}

template <bool FULL>
__device__ __forceinline__ float project_tile(const EwParams& p, const MatDev& md, const TileCoord& tc, int mode,
                                              float kw, float ko, const XView& xv, float (*tile)[kEwTile + 1]) {
  float* wb = md.w + tc.r0 * md.ld + tc.c0;
  const int64_t rows_left = md.rows - tc.r0, cols_left = md.cols - tc.c0;
  float acc = 0.f;
#pragma unroll
  for (int j0 = 0; j0 < kPasses; j0 += 2) {
    float4 wv[2], ov[2];
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const int r = tc.rin + tc.rstep * (j0 + u);
      wv[u] = tile_ld<FULL>(wb, md, r, tc.cin, rows_left, cols_left);
      if (mode != 0)
        ov[u] = make_float4(0.f, 0.f, 0.f, 0.f);
      else if (FULL && !md.transposed)
        ov[u] = x4(xv, (tc.r0 + r) * xv.ld + tc.c0 + tc.cin, p.prec);
      else
        ov[u] = o_at(xv, md, tc, r, tc.cin, p.prec, tile);
    }
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const int r = tc.rin + tc.rstep * (j0 + u);
      float4 w = wv[u];
      const float4 o = ov[u];
      w.x = fmaf(ko, o.x, kw * w.x);
      w.y = fmaf(ko, o.y, kw * w.y);
      w.z = fmaf(ko, o.z, kw * w.z);
      w.w = fmaf(ko, o.w, kw * w.w);
      tile_st<FULL>(wb, md, r, tc.cin, rows_left, cols_left, w);
      acc = fmaf(w.x, w.x, fmaf(w.y, w.y, fmaf(w.z, w.z, fmaf(w.w, w.w, acc))));
    }
  }
  return acc;
}

// W <- kw W + ko O (Eq. (1) with both normalisations folded into kw, ko).
__global__ void __launch_bounds__(kEwThreads, 6) project_kernel(const EwParams p) {
  __shared__ float tile[kEwTile][kEwTile + 1];
  __shared__ float red[kEwThreads / 32];
  for (int64_t e = p.e_first + blockIdx.x; e < p.e_end; e += gridDim.x) {
    const TileCoord tc = tile_coord(p, e);
    const MatDev& md = p.mats[tc.mi];
    if (md.warp_tiled) {
      e = skip_matrix(md, e);
      continue;
    }
    const MatScal& sc = p.scal[tc.mi];
    const int mode = sc.mode;
    if (mode == 2) {
      if (threadIdx.x == 0) p.part[e] = 0.f;
      continue;
    }
    const float kw = sc.kw, ko = sc.ko;
    const XView xv = x_view(p, md, md.o_buf);
    if (mode == 0 && md.transposed) {
      __syncthreads();
      load_o_tile_t(xv, tc, p.prec, tile);
      __syncthreads();
    }
    const float acc = tile_is_full(md, tc) ? project_tile<true>(p, md, tc, mode, kw, ko, xv, tile)
                                           : project_tile<false>(p, md, tc, mode, kw, ko, xv, tile);
    const float s = block_sum(acc, red);
    if (threadIdx.x == 0) p.part[e] = s;
  }
}

// dst (rows x cols, fp32, row stride ld) = O of one matrix, unscaled.
__global__ void __launch_bounds__(kEwThreads) export_update_kernel(const EwParams p, int mi, float* dst,
                                                                   int64_t ld) {
  __shared__ float tile[kEwTile][kEwTile + 1];
  const MatDev& md = p.mats[mi];
  const float unscale = exp2f(static_cast<float>(-md.ex));
  const XView xv = x_view(p, md, md.o_buf);
  const int64_t n_tiles = static_cast<int64_t>(md.et_rows) * md.et_cols;
  for (int64_t local = blockIdx.x; local < n_tiles; local += gridDim.x) {
    const TileCoord tc = tile_coord(p, md.et_begin + local);
    if (md.transposed) {
      __syncthreads();
      load_o_tile_t(xv, tc, p.prec, tile);
      __syncthreads();
    }
    for (int j = 0; j < kPasses; ++j) {
      const int r = tc.rin + tc.rstep * j;
      const float4 o = o_at(xv, md, tc, r, tc.cin, p.prec, tile);
      const int64_t row = tc.r0 + r, col = tc.c0 + tc.cin;
      if (row >= md.rows) continue;
      const float ov[4] = {o.x, o.y, o.z, o.w};
      for (int k = 0; k < 4; ++k)
        if (col + k < md.cols) dst[row * ld + col + k] = ov[k] * unscale;
    }
  }
}

// ------------------------------------------------------ finalize kernels
template <typename T>
__device__ double matrix_sum(const T* part, int64_t begin, int64_t count, int stride, int comp, double* red) {
  double s = 0.0;
  for (int64_t i = threadIdx.x; i < count; i += kEwThreads) s += static_cast<double>(part[(begin + i) * stride + comp]);
  return block_sum(s, red);
}

// Sum of a matrix's per-tile partials of the momentum or project phase: 8
// slots per tile from the warp-tiled kernels, one from the general ones.
__device__ double tile_partials(const EwParams& p, const MatDev& md, double* red) {
  const int64_t cnt = static_cast<int64_t>(md.et_rows) * md.et_cols;
  if (md.warp_tiled) return matrix_sum(p.part8, md.et_begin * kStreamSlots, cnt * kStreamSlots, 1, 0, red);
  return matrix_sum(p.part, md.et_begin, cnt, 1, 0, red);
}

__global__ void __launch_bounds__(kEwThreads) finalize_init_kernel(const EwParams p) {
  __shared__ double red[kEwThreads / 32];
  const int mi = ew_matrix(p, blockIdx.x);
  const MatDev& md = p.mats[mi];
  const int64_t cnt = static_cast<int64_t>(md.et_rows) * md.et_cols;
  const double s = matrix_sum(p.part64, md.et_begin, cnt, 1, 0, red);
  if (threadIdx.x == 0) {
    MatScal& sc = p.scal[mi];
    sc.wnorm2 = s;
    if (!(sc.R > 0.f)) sc.R = static_cast<float>(sqrt(s));
  }
}

__global__ void __launch_bounds__(kEwThreads) finalize_input_kernel(const EwParams p) {
  __shared__ double red[kEwThreads / 32];
  const int mi = ew_matrix(p, blockIdx.x);
  const MatDev& md = p.mats[mi];
  const double s = tile_partials(p, md, red);
  if (threadIdx.x == 0) {
    MatScal& sc = p.scal[mi];
    sc.flags = 0u;
    sc.mode = 0;
    const double xn = sqrt(s);
    sc.stats.input_norm = static_cast<float>(xn);
    // The momentum kernel wrote X at scale sigma (chosen from the previous
    // step's norm).  |X_ij| <= ||X||_F, so its largest stored entry is at
    // most sigma ||X||; keep it when that lies in [2^(ex-6), 60000] and
    // correct the scale exactly in the first GEMM epilogues (kappa);
    // otherwise rewrite X at the ideal scale 2^ex / (||X|| + eps).
    const double sigma = sc.sigma;
    const double peak = sigma * xn;
    sc.kappa = 1.f;
    sc.rewrite = 1;
    if (!isfinite(s)) {
      sc.flags |= MUONH_FLAG_NONFINITE_INPUT;
      sc.xscale = 0.f;
    } else if (s == 0.0) {
      sc.flags |= MUONH_FLAG_ZERO_UPDATE;
      sc.xscale = 0.f;
      if (sigma > 0.0) {   // X was written as zeros already
        sc.rewrite = 0;
        sc.kappa = 0.f;
      }
    } else {
      sc.xscale = static_cast<float>(ldexp(1.0, md.ex) / (xn + static_cast<double>(p.eps)));
      if (sigma > 0.0 && md.ns_steps > 0 && peak <= 60000.0 && peak >= ldexp(1.0, md.ex - 6)) {
        sc.rewrite = 0;
        sc.kappa = static_cast<float>(ldexp(1.0, md.ex) / (sigma * (xn + static_cast<double>(p.eps))));
      }
    }
    if (sc.rewrite) atomicOr(p.any_rewrite, 1);
    // scale for the next step's momentum kernel (not in FP32 mode: hi/lo X)
    sc.sigma = (p.prec != P_FP32 && isfinite(s) && s > 0.0) ? static_cast<float>(ldexp(1.0, md.ex - 2) / xn) : 0.f;
  }
}

__global__ void __launch_bounds__(kEwThreads) finalize_update_kernel(const EwParams p) {
  __shared__ double red[kEwThreads / 32];
  const int mi = ew_matrix(p, blockIdx.x);
  const MatDev& md = p.mats[mi];
  double soo, swo;
  if (md.fused_dots) {
    soo = matrix_sum(p.part_ns, md.ns_slot_base, md.ns_slots, 2, 0, red);
    swo = matrix_sum(p.part_ns, md.ns_slot_base, md.ns_slots, 2, 1, red);
  } else {
    const int64_t cnt = static_cast<int64_t>(md.et_rows) * md.et_cols;
    soo = matrix_sum(p.part, md.et_begin, cnt, 2, 0, red);
    swo = matrix_sum(p.part, md.et_begin, cnt, 2, 1, red);
  }
  if (threadIdx.x == 0) {
    MatScal& sc = p.scal[mi];
    const double unscale = ldexp(1.0, -md.ex);
    const double oo = soo * unscale * unscale;
    const double wo = swo * unscale;
    const double on = sqrt(oo);
    const double wn2 = sc.wnorm2;
    const double wn = sqrt(wn2);
    const double R = sc.R;
    const double lr = p.step[mi].lr;
    sc.kw = 1.f;
    sc.ko = 0.f;
    double elr = 0.0;
    if (sc.flags & MUONH_FLAG_NONFINITE_INPUT) {
      sc.mode = 2;
    } else if (!isfinite(oo) || !isfinite(wo)) {
      sc.flags |= MUONH_FLAG_NONFINITE_UPDATE;
      sc.mode = 2;
    } else if (oo == 0.0) {
      sc.flags |= MUONH_FLAG_ZERO_UPDATE;
      if (md.rule != MUONH_RULE_HYPERBALL) {
        sc.mode = 2;   // ordinary Muon: no update, W kept
      } else if (wn > 0.0) {
        sc.mode = 1;
        sc.kw = static_cast<float>(R / wn);
      } else {
        sc.flags |= MUONH_FLAG_DEGENERATE;
        sc.mode = 2;
      }
    } else if (md.rule != MUONH_RULE_HYPERBALL) {
      // Eq. (3): eta = lr; Eq. (5): eta = lr ||W|| / ||u||; W <- (1 - wd eta) W - eta u, u = s O
      const double un = static_cast<double>(md.uscale) * on;
      const double eta = (md.rule == MUONH_RULE_DECOUPLED_WD) ? lr : lr * wn / un;
      sc.mode = 0;
      sc.kw = static_cast<float>(1.0 - static_cast<double>(md.wd) * eta);
      sc.ko = static_cast<float>(-eta * static_cast<double>(md.uscale) * unscale);
      elr = wn > 0.0 ? eta * un / wn : 0.0;
    } else {
      const double alpha = lr * R / on;
      const double wt2 = wn2 - 2.0 * alpha * wo + alpha * alpha * oo;
      if (!(wt2 > 0.0)) {
        sc.flags |= MUONH_FLAG_DEGENERATE;
        sc.mode = 2;
      } else {
        const double kw = R / sqrt(wt2);
        sc.mode = 0;
        sc.kw = static_cast<float>(kw);
        sc.ko = static_cast<float>(-kw * alpha * unscale);
        elr = alpha * on / wn;
      }
    }
    sc.stats.elr = static_cast<float>(elr);
    sc.stats.pre_norm = static_cast<float>(wn);
    sc.stats.update_norm = (sc.flags & MUONH_FLAG_NONFINITE_INPUT) ? 0.f : static_cast<float>(on);
  }
}

__global__ void __launch_bounds__(kEwThreads) finalize_step_kernel(const EwParams p) {
  __shared__ double red[kEwThreads / 32];
  const int mi = ew_matrix(p, blockIdx.x);
  const MatDev& md = p.mats[mi];
  const double s = tile_partials(p, md, red);
  if (blockIdx.x == 0 && threadIdx.x == 0) *p.any_rewrite = 0;   // write_x of this step has run
  if (threadIdx.x == 0) {
    MatScal& sc = p.scal[mi];
    if (sc.mode != 2) sc.wnorm2 = s;
    sc.stats.post_norm = static_cast<float>(sqrt(sc.wnorm2));
    if (*reinterpret_cast<const volatile int*>(p.err) != 0) sc.flags |= MUONH_FLAG_TIMEOUT;
    sc.stats.flags = sc.flags;
    if (p.stats_out) p.stats_out[mi] = sc.stats;
  }
}

// One thread waits on an mbarrier that nothing arrives on, with the bounded
// wait of the pipelined kernels: it must give up after limit_ns and record
// the failure in *err.
__global__ void wait_probe_kernel(int* err, uint64_t limit_ns) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_mbar_init();
    mbar_wait(&bar, 0u, err, limit_ns);
  }
}

inline int ew_grid(int64_t n_et, int grid) {
  return static_cast<int>(n_et < grid ? (n_et > 0 ? n_et : 1) : grid);
}

}  // namespace

cudaError_t launch_init_norm(const EwParams& p, int grid, cudaStream_t s) {
  init_norm_kernel<<<ew_grid(p.e_end - p.e_first, grid), kEwThreads, 0, s>>>(p);
  return cudaGetLastError();
}
cudaError_t launch_finalize_init(const EwParams& p, cudaStream_t s) {
  finalize_init_kernel<<<p.m_count, kEwThreads, 0, s>>>(p);
  return cudaGetLastError();
}
cudaError_t launch_momentum_norm(const EwParams& p, int grid, cudaStream_t s) {
  momentum_norm_kernel<<<ew_grid(p.e_end - p.e_first, grid), kEwThreads, 0, s>>>(p);
  return cudaGetLastError();
}
cudaError_t launch_finalize_input(const EwParams& p, cudaStream_t s) {
  finalize_input_kernel<<<p.m_count, kEwThreads, 0, s>>>(p);
  return cudaGetLastError();
}
cudaError_t launch_write_x(const EwParams& p, int grid, cudaStream_t s) {
  write_x_kernel<<<ew_grid(p.e_end - p.e_first, grid), kEwThreads, 0, s>>>(p);
  return cudaGetLastError();
}
cudaError_t launch_update_dots(const EwParams& p, int grid, cudaStream_t s) {
  update_dots_kernel<<<ew_grid(p.e_end - p.e_first, grid), kEwThreads, 0, s>>>(p);
  return cudaGetLastError();
}
cudaError_t launch_finalize_update(const EwParams& p, cudaStream_t s) {
  finalize_update_kernel<<<p.m_count, kEwThreads, 0, s>>>(p);
  return cudaGetLastError();
}
cudaError_t launch_project(const EwParams& p, int grid, cudaStream_t s) {
  project_kernel<<<ew_grid(p.e_end - p.e_first, grid), kEwThreads, 0, s>>>(p);
  return cudaGetLastError();
}
cudaError_t launch_wait_probe(int* err, uint64_t limit_ns, cudaStream_t s) {
  wait_probe_kernel<<<1, 32, 0, s>>>(err, limit_ns);
  return cudaGetLastError();
}

cudaError_t launch_finalize_step(const EwParams& p, cudaStream_t s) {
  finalize_step_kernel<<<p.m_count, kEwThreads, 0, s>>>(p);
  return cudaGetLastError();
}
cudaError_t launch_export_update(const EwParams& p, int mat, float* dst, int64_t ld, cudaStream_t s) {
  export_update_kernel<<<256, kEwThreads, 0, s>>>(p, mat, dst, ld);
  return cudaGetLastError();
}

}  // namespace muonh
