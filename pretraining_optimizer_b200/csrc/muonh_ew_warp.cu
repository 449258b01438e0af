// Warp-tiled variants of the two large HBM-bound kernels of the step (sm_100a):
//   momentum:  M <- beta M + G, X = G + beta M (Nesterov) or M, partials of
//              ||X||^2, and the 16-bit Newton-Schulz input sigma X;
//   project:   W <- kw W + ko O (Eq. (1) of the Puro-2B report, Sec. 3.3, with
//              both normalisations folded into kw and ko), partials of ||W||^2.
//
// A block walks elementwise tiles (4096 elements of W) in a grid-stride loop;
// each of its 8 warps owns a fixed eighth of every tile and never waits for
// the others: no shared memory, no block barrier.  A lane issues all of its
// loads for a tile (8 x 16 bytes) before the first use, so a resident warp
// keeps 4 KB in flight, and it fetches the next tile's table entries while
// those loads are in flight (three resident blocks per SM: 80 registers a
// thread).  Tall matrices, whose X is the transpose, are tiled 64 x 64: warp
// w takes a 16 x 32 block and each lane a 4 x 4 sub-block of it (four
// consecutive rows, four columns), so a column of the sub-block is 8
// consecutive bytes of one 16-bit X row and the four lanes sharing a column
// write (or, in project, read) that row's whole 32-byte sector in one
// instruction.
//
// Every warp writes its partial sum of a tile to a fixed slot (8 per tile);
// the finalize kernels add the slots of a matrix in a fixed order in fp64, so
// results are bitwise reproducible.  Matrices whose rows are not 16-byte
// vectors, and the FP32 Newton-Schulz mode (hi/lo operands), take the
// general kernels instead (MatDev::warp_tiled == 0).
#include "muonh_common.cuh"

namespace muonh {
namespace {

constexpr int kWarps = kStreamSlots;          // 8 warps, one partial slot each
constexpr int kWarpThreads = 32 * kWarps;

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__device__ __forceinline__ float4 unpack4(uint2 u, int prec) {
  if (prec == P_BF16) {
    const __nv_bfloat162 a = *reinterpret_cast<const __nv_bfloat162*>(&u.x);
    const __nv_bfloat162 b = *reinterpret_cast<const __nv_bfloat162*>(&u.y);
    return make_float4(__low2float(a), __high2float(a), __low2float(b), __high2float(b));
  }
  const __half2 a = *reinterpret_cast<const __half2*>(&u.x);
  const __half2 b = *reinterpret_cast<const __half2*>(&u.y);
  return make_float4(__low2float(a), __high2float(a), __low2float(b), __high2float(b));
}

// Two fp32 values to a packed pair of 16-bit values (round to nearest even).
__device__ __forceinline__ uint32_t pack2(float a, float b, int prec) {
  if (prec == P_BF16) {
    __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<uint32_t*>(&h);
  }
  __half2 h = __floats2half2_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&h);
}

struct Tile {
  int64_t r0, c0;
  int nr, nc;        // valid rows / columns of the tile inside the matrix
};

__device__ __forceinline__ Tile tile_of(const MatDev& md, int64_t e) {
  Tile t;
  const uint32_t local = static_cast<uint32_t>(e - md.et_begin);
  const uint32_t tr = local / static_cast<uint32_t>(md.et_cols);
  t.r0 = static_cast<int64_t>(tr) * md.et_th;
  t.c0 = static_cast<int64_t>(local - tr * static_cast<uint32_t>(md.et_cols)) * md.et_tw;
  t.nr = static_cast<int>(md.rows - t.r0 < md.et_th ? md.rows - t.r0 : md.et_th);
  t.nc = static_cast<int>(md.cols - t.c0 < md.et_tw ? md.cols - t.c0 : md.et_tw);
  return t;
}

// Next tile of this block that belongs to a warp-tiled matrix of the
// kernel's kind (wide or tall), or e_end.
template <bool TALL>
__device__ __forceinline__ int64_t next_tile(const EwParams& p, int64_t e) {
  while (e < p.e_end) {
    const MatDev& md = p.mats[p.et_mat[e]];
    if (md.warp_tiled && (md.transposed != 0) == TALL) return e;
    const int64_t end = md.et_begin + static_cast<int64_t>(md.et_rows) * md.et_cols;
    e += ((end - e + gridDim.x - 1) / gridDim.x) * gridDim.x;   // first tile of ours past this matrix
  }
  return e;
}

// Everything a warp needs to know about one tile, gathered from the device
// tables; the kernels fetch the next tile's copy while the current tile's
// data loads are in flight, so the dependent table reads (tile -> matrix ->
// pointers, scalars) do not stall the data stream.
struct TileCtx {
  int64_t e;
  const float* a;       // momentum: G tile origin;   project: W tile origin
  float* b;             // momentum: M tile origin;   project: W tile origin (written)
  uint16_t* x;          // X / O at the tile origin (wide: row r0, column c0; tall: row c0, column r0)
  int64_t ld, xld;
  int nr, nc, sh;       // valid rows / columns; log2(tw / 4) for wide tiles
  float s0, s1;         // momentum: beta, sigma;     project: kw, ko
  int flag;             // momentum: nesterov;        project: mode
};

template <bool TALL, bool PROJECT>
__device__ __forceinline__ TileCtx tile_ctx(const EwParams& p, int64_t e) {
  TileCtx c;
  c.e = e;
  if (e >= p.e_end) return c;
  const int mi = p.et_mat[e];
  const MatDev& md = p.mats[mi];
  const Tile t = tile_of(md, e);
  const ClassDev& cd = p.classes[md.cls];
  c.ld = md.ld;
  c.xld = cd.c_pad;
  c.nr = t.nr;
  c.nc = t.nc;
  c.sh = __ffs(md.et_tw) - 3;
  uint16_t* xg = static_cast<uint16_t*>(cd.x[PROJECT ? md.o_buf : 0][0]) + md.z * cd.x_stride;
  c.x = TALL ? xg + t.c0 * c.xld + t.r0 : xg + t.r0 * c.xld + t.c0;
  if (PROJECT) {
    const MatScal& sc = p.scal[mi];
    c.a = md.w + t.r0 * md.ld + t.c0;
    c.b = md.w + t.r0 * md.ld + t.c0;
    c.s0 = sc.kw;
    c.s1 = sc.ko;
    c.flag = sc.mode;
  } else {
    c.a = p.step[mi].g + t.r0 * md.ld + t.c0;
    c.b = md.m + t.r0 * md.ld + t.c0;
    c.s0 = md.beta;
    c.s1 = p.scal[mi].sigma;
    c.flag = md.nesterov;
  }
  return c;
}

// Chunk j (0..3) of lane `lane` in warp w of a wide tile: 4 consecutive
// columns of one row; the warp covers chunks 128w .. 128w + 127.
__device__ __forceinline__ void wide_chunk_sh(int sh, int w, int lane, int j, int& row, int& col) {
  const int q = lane + 32 * j + 128 * w;
  row = q >> sh;
  col = (q & ((1 << sh) - 1)) * 4;
}

// ---------------------------------------------------------------- momentum
template <bool TALL>
__global__ void __launch_bounds__(kWarpThreads, 3) momentum_warp_kernel(const EwParams p) {
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  TileCtx cur = tile_ctx<TALL, false>(p, next_tile<TALL>(p, p.e_first + blockIdx.x));
  while (cur.e < p.e_end) {
    const float beta = cur.s0, sigma = cur.s1;
    float acc = 0.f;
    if (!TALL) {
      int row[4], col[4];
      bool ok[4];
      float4 gv[4], mv[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        wide_chunk_sh(cur.sh, w, lane, j, row[j], col[j]);
        ok[j] = row[j] < cur.nr && col[j] < cur.nc;
        if (ok[j]) {
          gv[j] = *reinterpret_cast<const float4*>(cur.a + row[j] * cur.ld + col[j]);
          mv[j] = *reinterpret_cast<const float4*>(cur.b + row[j] * cur.ld + col[j]);
        }
      }
      const TileCtx nxt = tile_ctx<TALL, false>(p, next_tile<TALL>(p, cur.e + gridDim.x));
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        if (!ok[j]) continue;
        float4 m = mv[j];
        const float4 g = gv[j];
        m.x = fmaf(beta, m.x, g.x);
        m.y = fmaf(beta, m.y, g.y);
        m.z = fmaf(beta, m.z, g.z);
        m.w = fmaf(beta, m.w, g.w);
        *reinterpret_cast<float4*>(cur.b + row[j] * cur.ld + col[j]) = m;
        float4 x = m;
        if (cur.flag) {
          x.x = fmaf(beta, m.x, g.x);
          x.y = fmaf(beta, m.y, g.y);
          x.z = fmaf(beta, m.z, g.z);
          x.w = fmaf(beta, m.w, g.w);
        }
        acc = fmaf(x.x, x.x, acc);
        acc = fmaf(x.y, x.y, acc);
        acc = fmaf(x.z, x.z, acc);
        acc = fmaf(x.w, x.w, acc);
        if (sigma > 0.f) {
          const uint2 u = make_uint2(pack2(x.x * sigma, x.y * sigma, p.prec), pack2(x.z * sigma, x.w * sigma, p.prec));
          *reinterpret_cast<uint2*>(cur.x + row[j] * cur.xld + col[j]) = u;
        }
      }
      acc = warp_sum(acc);
      if (lane == 0) p.part8[cur.e * kWarps + w] = acc;
      cur = nxt;
    } else {
      // tall 64 x 64 tile, X holding its transpose: warp w takes the 16 x 32
      // block of W rows 16 (w >> 1) .. +15 and columns 32 (w & 1) .. +31, and
      // lane l its 4 x 4 sub-block of rows rb .. rb+3 and columns cb .. cb+3.
      // A load instruction then covers four whole 128-byte W rows, and a
      // column of the lane's sub-block is four consecutive entries (8 bytes)
      // of one X row: the four lanes sharing cb write a whole 32-byte sector.
      const int rb = 16 * (w >> 1) + 4 * (lane >> 3);
      const int cb = 32 * (w & 1) + 4 * (lane & 7);
      const bool cok = cb < cur.nc;   // nc is a multiple of 4
      float4 gv[4], mv[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int r = rb + j;
        if (cok && r < cur.nr) {
          gv[j] = *reinterpret_cast<const float4*>(cur.a + r * cur.ld + cb);
          mv[j] = *reinterpret_cast<const float4*>(cur.b + r * cur.ld + cb);
        }
      }
      const TileCtx nxt = tile_ctx<TALL, false>(p, next_tile<TALL>(p, cur.e + gridDim.x));
      float x[4][4];   // [row j][column q], scaled by sigma
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int r = rb + j;
        x[j][0] = x[j][1] = x[j][2] = x[j][3] = 0.f;   // rows past the matrix stay zero in X's padding
        if (!cok || r >= cur.nr) continue;
        float4 m = mv[j];
        const float4 g = gv[j];
        m.x = fmaf(beta, m.x, g.x);
        m.y = fmaf(beta, m.y, g.y);
        m.z = fmaf(beta, m.z, g.z);
        m.w = fmaf(beta, m.w, g.w);
        *reinterpret_cast<float4*>(cur.b + r * cur.ld + cb) = m;
        float4 xv = m;
        if (cur.flag) {
          xv.x = fmaf(beta, m.x, g.x);
          xv.y = fmaf(beta, m.y, g.y);
          xv.z = fmaf(beta, m.z, g.z);
          xv.w = fmaf(beta, m.w, g.w);
        }
        acc = fmaf(xv.x, xv.x, fmaf(xv.y, xv.y, fmaf(xv.z, xv.z, fmaf(xv.w, xv.w, acc))));
        x[j][0] = xv.x * sigma;
        x[j][1] = xv.y * sigma;
        x[j][2] = xv.z * sigma;
        x[j][3] = xv.w * sigma;
      }
      if (sigma > 0.f && cok) {
#pragma unroll
        for (int q = 0; q < 4; ++q) {   // X row cb + q, entries rb .. rb+3
          const uint2 u = make_uint2(pack2(x[0][q], x[1][q], p.prec), pack2(x[2][q], x[3][q], p.prec));
          *reinterpret_cast<uint2*>(cur.x + (cb + q) * cur.xld + rb) = u;
        }
      }
      acc = warp_sum(acc);
      if (lane == 0) p.part8[cur.e * kWarps + w] = acc;
      cur = nxt;
    }
  }
}

// ----------------------------------------------------------------- project
template <bool TALL>
__global__ void __launch_bounds__(kWarpThreads, 3) project_warp_kernel(const EwParams p) {
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  TileCtx cur = tile_ctx<TALL, true>(p, next_tile<TALL>(p, p.e_first + blockIdx.x));
  while (cur.e < p.e_end) {
    const int mode = cur.flag;
    const float kw = cur.s0, ko = cur.s1;
    float acc = 0.f;
    if (mode == 2) {   // W kept
      const TileCtx nxt = tile_ctx<TALL, true>(p, next_tile<TALL>(p, cur.e + gridDim.x));
      if (lane == 0) p.part8[cur.e * kWarps + w] = 0.f;
      cur = nxt;
      continue;
    }
    if (!TALL) {
      int row[4], col[4];
      bool ok[4];
      float4 wv[4];
      uint2 ov[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        wide_chunk_sh(cur.sh, w, lane, j, row[j], col[j]);
        ok[j] = row[j] < cur.nr && col[j] < cur.nc;
        ov[j] = make_uint2(0u, 0u);
        if (ok[j]) {
          wv[j] = *reinterpret_cast<const float4*>(cur.a + row[j] * cur.ld + col[j]);
          if (mode == 0) ov[j] = *reinterpret_cast<const uint2*>(cur.x + row[j] * cur.xld + col[j]);
        }
      }
      const TileCtx nxt = tile_ctx<TALL, true>(p, next_tile<TALL>(p, cur.e + gridDim.x));
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        if (!ok[j]) continue;
        const float4 o = unpack4(ov[j], p.prec);
        float4 v = wv[j];
        v.x = fmaf(ko, o.x, kw * v.x);
        v.y = fmaf(ko, o.y, kw * v.y);
        v.z = fmaf(ko, o.z, kw * v.z);
        v.w = fmaf(ko, o.w, kw * v.w);
        *reinterpret_cast<float4*>(cur.b + row[j] * cur.ld + col[j]) = v;
        acc = fmaf(v.x, v.x, fmaf(v.y, v.y, fmaf(v.z, v.z, fmaf(v.w, v.w, acc))));
      }
      acc = warp_sum(acc);
      if (lane == 0) p.part8[cur.e * kWarps + w] = acc;
      cur = nxt;
    } else {
      // tall 64 x 64 tile: the block of each warp and lane of the momentum
      // kernel; the lane reads O as four 8-byte pieces of X rows cb .. cb+3
      const int rb = 16 * (w >> 1) + 4 * (lane >> 3);
      const int cb = 32 * (w & 1) + 4 * (lane & 7);
      const bool cok = cb < cur.nc;
      float4 wv[4];
      uint2 ov[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        ov[q] = make_uint2(0u, 0u);
        // O(rb + j, cb + q) = X[c0 + cb + q][r0 + rb + j]; X's padding columns are zero
        if (cok && mode == 0) ov[q] = *reinterpret_cast<const uint2*>(cur.x + (cb + q) * cur.xld + rb);
      }
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int r = rb + j;
        if (cok && r < cur.nr) wv[j] = *reinterpret_cast<const float4*>(cur.a + r * cur.ld + cb);
      }
      const TileCtx nxt = tile_ctx<TALL, true>(p, next_tile<TALL>(p, cur.e + gridDim.x));
      const float4 o0 = unpack4(ov[0], p.prec), o1 = unpack4(ov[1], p.prec);
      const float4 o2 = unpack4(ov[2], p.prec), o3 = unpack4(ov[3], p.prec);
      const float oc[4][4] = {{o0.x, o1.x, o2.x, o3.x}, {o0.y, o1.y, o2.y, o3.y},
                              {o0.z, o1.z, o2.z, o3.z}, {o0.w, o1.w, o2.w, o3.w}};   // [row j][column q]
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int r = rb + j;
        if (!cok || r >= cur.nr) continue;
        float4 v = wv[j];
        v.x = fmaf(ko, oc[j][0], kw * v.x);
        v.y = fmaf(ko, oc[j][1], kw * v.y);
        v.z = fmaf(ko, oc[j][2], kw * v.z);
        v.w = fmaf(ko, oc[j][3], kw * v.w);
        *reinterpret_cast<float4*>(cur.b + r * cur.ld + cb) = v;
        acc = fmaf(v.x, v.x, fmaf(v.y, v.y, fmaf(v.z, v.z, fmaf(v.w, v.w, acc))));
      }
      acc = warp_sum(acc);
      if (lane == 0) p.part8[cur.e * kWarps + w] = acc;
      cur = nxt;
    }
  }
}

}  // namespace

// Resident blocks per SM of a warp-tiled kernel: kind 0/1 momentum wide/tall,
// 2/3 project wide/tall.
int ew_warp_blocks_per_sm(int kind) {
  int n = 0;
  cudaError_t e = cudaErrorInvalidValue;
  switch (kind) {
    case 0: e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, momentum_warp_kernel<false>, kWarpThreads, 0); break;
    case 1: e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, momentum_warp_kernel<true>, kWarpThreads, 0); break;
    case 2: e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, project_warp_kernel<false>, kWarpThreads, 0); break;
    case 3: e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, project_warp_kernel<true>, kWarpThreads, 0); break;
  }
  return (e == cudaSuccess && n > 0) ? n : 1;
}

cudaError_t launch_momentum_warp(const EwParams& p, bool tall, int grid, cudaStream_t s) {
  if (tall)
    momentum_warp_kernel<true><<<grid, kWarpThreads, 0, s>>>(p);
  else
    momentum_warp_kernel<false><<<grid, kWarpThreads, 0, s>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_project_warp(const EwParams& p, bool tall, int grid, cudaStream_t s) {
  if (tall)
    project_warp_kernel<true><<<grid, kWarpThreads, 0, s>>>(p);
  else
    project_warp_kernel<false><<<grid, kWarpThreads, 0, s>>>(p);
  return cudaGetLastError();
}

}  // namespace muonh
