// Grouped Newton-Schulz GEMMs on the 5th-generation tensor cores (sm_100a).
//
// One Newton-Schulz iteration on a wide matrix Y (r x c),
//   Y' = a Y + (b A + c A A) Y,   A = Y Y^T
// (quintic iteration of the Muon update; the MuonH wrapper of the Puro-2B
// report, Sec. 3.3, normalises its output), runs as three products with the
// polynomial folded into the products (16-bit operands, CTA pairs):
//   GRAM    A  = Y Y^T  (and, FP32 mode, C = b I + c A)    M = r, N = r, K = c   (symmetric)
//   SQUARE  B' = c A A + b A + a I  (FP32 mode: A C + a I)  M = r, N = r, K = r   (symmetric)
//   APPLY   Y' = B' Y                                      M = r, N = c, K = r
// The Gram-space form (fp16 operands) runs g <= 3 iterations on r x r
// matrices between two passes over Y: with P_k = p(A_k) = a I + b A_k + c A_k^2,
// A_{k+1} = Y_{k+1} Y_{k+1}^T = P_k A_k P_k = (A_k P_k) P_k, since all these
// factors are polynomials in one symmetric matrix and commute; the run ends
// with Y <- Q Y, Q = P_{g-1} ... P_0.  Its r x r products are
//   SYMPROD out = L R   (L, R symmetric and commuting)      M = r, N = r, K = r   (symmetric)
// Every launch covers the tiles of all matrices of the step (grouped), in a
// persistent grid of one CTA per SM (one CTA pair per two SMs for 16-bit
// operands).  Symmetric products compute only the tiles that touch the upper
// triangle and store each off-diagonal block twice, directly and mirrored,
// so that every consumer reads its operands K-major.
//
// Per CTA: producer warps issue TMA loads into a ring of shared-memory
// stages (one warp in the FP32-mode kernel; in the CTA-pair kernel warp 0
// loads the A boxes and warp 6 the B boxes), warp 1 (one thread) issues
// tcgen05.mma into one of two TMEM accumulators (128 lanes x 256 fp32
// columns each), warps 2-5 drain the other accumulator with tcgen05.ld,
// apply the polynomial epilogue and store.  Every wait is bounded
// (muonh::mbar_wait) and records a timeout in *err.
//
// Storage: fp16 operands hold the value times 2^e (e per matrix and per
// operand, chosen on the host so that no entry can overflow); products of
// scaled operands are rescaled exactly in the fp32 epilogue.  In FP32 mode
// each operand is a pair (hi, lo) of fp16 arrays, value = hi + lo, and each
// tile accumulates hi*hi + hi*lo + lo*hi.
#include "muonh_common.cuh"

namespace muonh {
namespace {

template <int PREC>
struct Store16;
template <>
struct Store16<P_FP16> {
  using T = __half;
  static __device__ __forceinline__ T cvt(float v) { return __float2half_rn(v); }
  static __device__ __forceinline__ float back(T v) { return __half2float(v); }
};
template <>
struct Store16<P_BF16> {
  using T = __nv_bfloat16;
  static __device__ __forceinline__ T cvt(float v) { return __float2bfloat16_rn(v); }
  static __device__ __forceinline__ float back(T v) { return __bfloat162float(v); }
};
template <>
struct Store16<P_FP32> : Store16<P_FP16> {};

template <int PREC>
struct Cfg {
  static constexpr int kParts = (PREC == P_FP32) ? 2 : 1;
  static constexpr int kStages = (PREC == P_FP32) ? 2 : 4;
  static constexpr int kABytes = kBM * kBK * 2;                    // 16 KB
  static constexpr int kBBytes = kBN * kBK * 2;                    // 32 KB
  static constexpr int kStageBytes = kParts * (kABytes + kBBytes);
  static constexpr int kBarOffset = kStages * kStageBytes;
  static constexpr int kSmem = kBarOffset + 256 + 1024;            // + barriers + alignment slack
  // FP32 mode: the tensor cores accumulate kChunkBlocks k-blocks (128 of K)
  // into a scratch accumulator; the epilogue adds each chunk to the running
  // sum in IEEE fp32 (the hardware accumulation truncates, with an error
  // that grows with the number of accumulated products).
  static constexpr int kChunkBlocks = 2;
};

// 32 consecutive values of one row, stored as 16-bit (and the fp16 residual in FP32 mode).
template <int PREC>
__device__ __forceinline__ void store_row32(void* hi_base, void* lo_base, int64_t off, const float (&v)[32]) {
  using S = Store16<PREC>;
  using T = typename S::T;
  uint4 hbuf[4], lbuf[4];
  T* h = reinterpret_cast<T*>(hbuf);
  __half* l = reinterpret_cast<__half*>(lbuf);
#pragma unroll
  for (int j = 0; j < 32; ++j) {
    T hv = S::cvt(v[j]);
    h[j] = hv;
    if (PREC == P_FP32) l[j] = __float2half_rn(v[j] - S::back(hv));
  }
  uint4* dh = reinterpret_cast<uint4*>(reinterpret_cast<T*>(hi_base) + off);
#pragma unroll
  for (int q = 0; q < 4; ++q) dh[q] = hbuf[q];
  if (PREC == P_FP32) {
    uint4* dl = reinterpret_cast<uint4*>(reinterpret_cast<__half*>(lo_base) + off);
#pragma unroll
    for (int q = 0; q < 4; ++q) dl[q] = lbuf[q];
  }
}

template <int PREC>
__device__ __forceinline__ void store_one(void* hi_base, void* lo_base, int64_t off, float v) {
  using S = Store16<PREC>;
  using T = typename S::T;
  T hv = S::cvt(v);
  reinterpret_cast<T*>(hi_base)[off] = hv;
  if (PREC == P_FP32) reinterpret_cast<__half*>(lo_base)[off] = __float2half_rn(v - S::back(hv));
}

// Symmetric output: element (row, col) of the upper triangle (col >= row)
// is stored at [row][col]; for col > row also at [col][row].
template <int PREC>
__device__ __forceinline__ void store_symmetric(void* hi, void* lo, int ld, int row, int col0,
                                                const float (&v)[32]) {
  const int64_t roff = static_cast<int64_t>(row) * ld;
  if (col0 >= row) {
    store_row32<PREC>(hi, lo, roff + col0, v);
  } else if (col0 + 31 >= row) {
#pragma unroll
    for (int j = 0; j < 32; ++j)
      if (col0 + j >= row) store_one<PREC>(hi, lo, roff + col0 + j, v[j]);
  }
  if (col0 + 31 > row) {
#pragma unroll
    for (int j = 0; j < 32; ++j)
      if (col0 + j > row) store_one<PREC>(hi, lo, static_cast<int64_t>(col0 + j) * ld + row, v[j]);
  }
}

template <int MODE, int PREC>
__global__ void __launch_bounds__(kGemmThreads, 1) ns_gemm_kernel(const __grid_constant__ NsParams p) {
  using C = Cfg<PREC>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::kBarOffset);
  uint64_t* empty = full + C::kStages;
  uint64_t* tfull = empty + C::kStages;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], 128);
    }
    mbar_init(drain, 1);
    fence_mbar_init();
  }
  if (warp == 1) tmem_alloc(tmem_slot, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      uint32_t issued_parity[C::kStages];
      bool issued[C::kStages];
      for (int s = 0; s < C::kStages; ++s) issued[s] = false;
      bool ok = true;
      for (int t = blockIdx.x; t < p.ntiles && ok; t += gridDim.x) {
        const TileDesc td = p.tiles[t];
        const MatDev& md = p.mats[td.mat];
        const ClassDev& cd = p.classes[md.cls];
        const int z = md.z;
        const int nk = (MODE == M_GRAM ? cd.c_pad : cd.r_pad) / kBK;
        for (int kb = 0; kb < nk; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1u, p.err)) { ok = false; break; }
          mbar_expect_tx(&full[stage], C::kStageBytes);
          uint8_t* sa = smem + stage * C::kStageBytes;
          uint8_t* sb = sa + C::kParts * C::kABytes;
          const int k0 = kb * kBK;
          for (int part = 0; part < C::kParts; ++part) {
            uint8_t* a_dst = sa + part * C::kABytes;
            uint8_t* b_dst = sb + part * C::kBBytes;
            if (MODE == M_GRAM) {
              tma_load_3d(a_dst, p.tmaps + tm_x(cd.tm_base + TM_X_K128, p.src, part), &full[stage], k0,
                          td.bi * kBM, z);
              tma_load_3d(b_dst, p.tmaps + tm_x(cd.tm_base + TM_X_K256, p.src, part), &full[stage], k0,
                          td.bj * kBN, z);
            } else if (MODE == M_SQUARE) {
              tma_load_3d(a_dst, p.tmaps + cd.tm_base + TM_A_K128 + part, &full[stage], k0, td.bi * kBM, z);
              tma_load_3d(b_dst, p.tmaps + cd.tm_base + TM_C_K256 + part, &full[stage], k0, td.bj * kBN, z);
            } else {
              tma_load_3d(a_dst, p.tmaps + cd.tm_base + TM_B_K128 + part, &full[stage], k0, td.bi * kBM, z);
              const CUtensorMap* xm = p.tmaps + tm_x(cd.tm_base + TM_X_MN, p.src, part);
#pragma unroll
              for (int q = 0; q < kBN / 64; ++q)
                tma_load_3d(b_dst + q * (64 * kBK * 2), xm, &full[stage], td.bj * kBN + q * 64, k0, z);
            }
          }
          issued[stage] = true;
          issued_parity[stage] = phase;
          if (++stage == C::kStages) { stage = 0; phase ^= 1u; }
        }
      }
      if (!ok) {
        // let the copies already in flight land before the CTA exits
        for (int s = 0; s < C::kStages; ++s)
          if (issued[s]) {
            const uint64_t t0 = globaltimer();
            while (!mbar_try_wait(&full[s], issued_parity[s]) && globaltimer() - t0 < kWaitLimitNs) {
            }
          }
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0 && PREC == P_FP32) {
      // accumulator S (columns 0..255) holds chunk 0 and the running sum;
      // chunks 1.. go to C (columns 256..511) and are merged by the epilogue.
      constexpr uint32_t kIdesc = idesc_f16(kBM, kBN, 0, MODE == M_APPLY ? 1 : 0);
      uint64_t* cready = &tfull[0];
      uint64_t* sdone = &tfull[1];
      uint64_t* cfree = &tempty[0];
      uint64_t* sfree = &tempty[1];
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      int local = 0, cuse = 0;
      for (int t = blockIdx.x; t < p.ntiles && ok; t += gridDim.x, ++local) {
        const TileDesc td = p.tiles[t];
        const MatDev& md = p.mats[td.mat];
        const ClassDev& cd = p.classes[md.cls];
        const int nk = (MODE == M_GRAM ? cd.c_pad : cd.r_pad) / kBK;
        if (local > 0 && !mbar_wait(sfree, (local - 1) & 1, p.err)) { ok = false; break; }
        tc_fence_after();
        for (int kb = 0; kb < nk && ok; ++kb) {
          const int chunk = kb / C::kChunkBlocks;
          const bool chunk_start = (kb % C::kChunkBlocks) == 0;
          if (chunk >= 1 && chunk_start) {
            if (cuse > 0 && !mbar_wait(cfree, (cuse - 1) & 1, p.err)) { ok = false; break; }
            tc_fence_after();
          }
          const uint32_t d_tmem = tmem_base + (chunk == 0 ? 0 : kBN);
          if (!mbar_wait(&full[stage], phase, p.err)) { ok = false; break; }
          tc_fence_after();
          const uint32_t sa = smem_u32(smem + stage * C::kStageBytes);
          const uint32_t sb = sa + C::kParts * C::kABytes;
#pragma unroll
          for (int k = 0; k < kBK / 16; ++k) {
#pragma unroll
            for (int prod = 0; prod < 3; ++prod) {
              const int pa = (prod == 2) ? 1 : 0;
              const int pb = (prod == 1) ? 1 : 0;
              const uint64_t adesc = sdesc_sw128(sa + pa * C::kABytes + k * 32, 16, 1024);
              uint64_t bdesc;
              if (MODE == M_APPLY)
                bdesc = sdesc_sw128(sb + pb * C::kBBytes + k * 16 * 128, 64 * kBK * 2, 1024);
              else
                bdesc = sdesc_sw128(sb + pb * C::kBBytes + k * 32, 16, 1024);
              umma_f16(d_tmem, adesc, bdesc, kIdesc, (chunk_start && k == 0 && prod == 0) ? 0u : 1u);
            }
          }
          umma_commit(&empty[stage]);
          if (++stage == C::kStages) { stage = 0; phase ^= 1u; }
          const bool chunk_end = ((kb + 1) % C::kChunkBlocks) == 0 || kb + 1 == nk;
          if (chunk >= 1 && chunk_end) {
            umma_commit(cready);
            ++cuse;
          }
        }
        if (!ok) break;
        umma_commit(sdone);
      }
      umma_commit(drain);
      const uint64_t t0 = globaltimer();
      while (!mbar_try_wait(drain, 0) && globaltimer() - t0 < kWaitLimitNs) {
      }
    } else if (lane == 0) {
      constexpr uint32_t kIdesc = idesc_f16(kBM, kBN, PREC == P_BF16 ? 1 : 0, MODE == M_APPLY ? 1 : 0);
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      int local = 0;
      for (int t = blockIdx.x; t < p.ntiles && ok; t += gridDim.x, ++local) {
        const TileDesc td = p.tiles[t];
        const MatDev& md = p.mats[td.mat];
        const ClassDev& cd = p.classes[md.cls];
        const int nk = (MODE == M_GRAM ? cd.c_pad : cd.r_pad) / kBK;
        const int acc = local & 1;
        const uint32_t acc_phase = (local >> 1) & 1;
        if (!mbar_wait(&tempty[acc], acc_phase ^ 1u, p.err)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * kBN;
        for (int kb = 0; kb < nk; ++kb) {
          if (!mbar_wait(&full[stage], phase, p.err)) { ok = false; break; }
          tc_fence_after();
          const uint32_t sa = smem_u32(smem + stage * C::kStageBytes);
          const uint32_t sb = sa + C::kParts * C::kABytes;
#pragma unroll
          for (int k = 0; k < kBK / 16; ++k) {
#pragma unroll
            for (int prod = 0; prod < (C::kParts == 2 ? 3 : 1); ++prod) {
              // products: hi*hi, hi*lo, lo*hi
              const int pa = (prod == 2) ? 1 : 0;
              const int pb = (prod == 1) ? 1 : 0;
              const uint64_t adesc = sdesc_sw128(sa + pa * C::kABytes + k * 32, 16, 1024);
              uint64_t bdesc;
              if (MODE == M_APPLY)
                bdesc = sdesc_sw128(sb + pb * C::kBBytes + k * 16 * 128, 64 * kBK * 2, 1024);
              else
                bdesc = sdesc_sw128(sb + pb * C::kBBytes + k * 32, 16, 1024);
              umma_f16(d_tmem, adesc, bdesc, kIdesc, (kb | k | prod) != 0 ? 1u : 0u);
            }
          }
          umma_commit(&empty[stage]);
          if (++stage == C::kStages) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        umma_commit(&tfull[acc]);
      }
      // make sure no MMA is still writing TMEM when the CTA deallocates it
      umma_commit(drain);
      const uint64_t t0 = globaltimer();
      while (!mbar_try_wait(drain, 0) && globaltimer() - t0 < kWaitLimitNs) {
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue
    const int quarter = warp & 3;            // TMEM lanes 32*quarter .. +31
    const int lrow = quarter * 32 + lane;    // row within the tile
    int local = 0;
    int merges = 0;                          // FP32 mode: chunk merges so far
    for (int t = blockIdx.x; t < p.ntiles; t += gridDim.x, ++local) {
      const TileDesc td = p.tiles[t];
      const MatDev& md = p.mats[td.mat];
      const ClassDev& cd = p.classes[md.cls];
      const int acc = (PREC == P_FP32) ? 0 : (local & 1);
      if (PREC == P_FP32) {
        // merge chunks 1.. of this tile into S, then wait for the tile's end
        const int nk = (MODE == M_GRAM ? cd.c_pad : cd.r_pad) / kBK;
        const int nchunks = (nk + C::kChunkBlocks - 1) / C::kChunkBlocks;
        const uint32_t lane_base = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16);
        bool ok = true;
        for (int c = 1; c < nchunks; ++c) {
          if (!mbar_wait(&tfull[0], merges & 1, p.err)) { ok = false; break; }
          tc_fence_after();
          for (int g = 0; g < kBN / 32; ++g) {
            float sv[32], cv[32];
            tmem_ld32(lane_base + g * 32, sv);
            tmem_ld32(lane_base + kBN + g * 32, cv);
#pragma unroll
            for (int j = 0; j < 32; ++j) sv[j] += cv[j];
            tmem_st32(lane_base + g * 32, sv);
          }
          tc_fence_before();
          mbar_arrive(&tempty[0]);
          ++merges;
        }
        if (!ok || !mbar_wait(&tfull[1], local & 1, p.err)) break;
      } else {
        const uint32_t acc_phase = (local >> 1) & 1;
        if (!mbar_wait(&tfull[acc], acc_phase, p.err)) break;
      }
      tc_fence_after();
      const int row = td.bi * kBM + lrow;
      // tcgen05.ld is warp-collective: chunk skips below depend on the warp's
      // first row only, so a warp never splits around it.
      const int warp_row0 = row - lane;
      const uint32_t taddr = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) + acc * kBN;
      const float kap = (p.iter == 0) ? p.scal[td.mat].kappa : 1.f;
      if (MODE == M_GRAM) {
        // acc = 2^(2ex) A;  A_s = 2^ea A;  C_s = 2^ec (b I + c A)
        const float sa = kap * kap * exp2f(static_cast<float>(md.ea - 2 * md.ex));
        const float sc = kap * kap * md.c_coef * exp2f(static_cast<float>(md.ec - 2 * md.ex));
        const float diag = md.b * exp2f(static_cast<float>(md.ec));
        const int64_t mo = md.z * cd.a_stride * 2;
        void* ahi = static_cast<uint8_t*>(cd.a[0]) + mo;
        void* alo = cd.a[1] ? static_cast<uint8_t*>(cd.a[1]) + mo : nullptr;
        void* chi = static_cast<uint8_t*>(cd.c[0]) + mo;
        void* clo = cd.c[1] ? static_cast<uint8_t*>(cd.c[1]) + mo : nullptr;
        for (int ch = 0; ch < kBN / 32; ++ch) {
          const int col0 = td.bj * kBN + ch * 32;
          if (col0 + 31 < warp_row0) continue;   // whole chunk below the diagonal for this warp
          float v[32], w[32];
          tmem_ld32(taddr + ch * 32, v);
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            w[j] = sc * v[j];
            v[j] *= sa;
          }
          const int dj = row - col0;   // diagonal element of this row, if in the chunk
#pragma unroll
          for (int j = 0; j < 32; ++j)
            if (j == dj) w[j] += diag;
          store_symmetric<PREC>(ahi, alo, cd.r_pad, row, col0, v);
          store_symmetric<PREC>(chi, clo, cd.r_pad, row, col0, w);
        }
      } else if (MODE == M_SQUARE) {
        // acc = 2^(ea+ec) A C;  B'_s = 2^eb (A C + a I)
        const float sb = exp2f(static_cast<float>(md.eb - md.ea - md.ec));
        const float diag = md.a * exp2f(static_cast<float>(md.eb));
        const int64_t mo = md.z * cd.a_stride * 2;
        void* bhi = static_cast<uint8_t*>(cd.b[0]) + mo;
        void* blo = cd.b[1] ? static_cast<uint8_t*>(cd.b[1]) + mo : nullptr;
        for (int ch = 0; ch < kBN / 32; ++ch) {
          const int col0 = td.bj * kBN + ch * 32;
          if (col0 + 31 < warp_row0) continue;   // whole chunk below the diagonal for this warp
          float v[32];
          tmem_ld32(taddr + ch * 32, v);
#pragma unroll
          for (int j = 0; j < 32; ++j) v[j] *= sb;
          const int dj = row - col0;   // diagonal element of this row, if in the chunk
#pragma unroll
          for (int j = 0; j < 32; ++j)
            if (j == dj) v[j] += diag;
          store_symmetric<PREC>(bhi, blo, cd.r_pad, row, col0, v);
        }
      } else {
        // acc = 2^(eb+ex) B' Y;  Y'_s = 2^ex B' Y
        const float ks = kap * exp2f(static_cast<float>(-md.eb));
        const int64_t xo = md.z * cd.x_stride * 2;
        void* yhi = static_cast<uint8_t*>(cd.x[p.src ^ 1][0]) + xo;
        void* ylo = cd.x[p.src ^ 1][1] ? static_cast<uint8_t*>(cd.x[p.src ^ 1][1]) + xo : nullptr;
        for (int ch = 0; ch < kBN / 32; ++ch) {
          const int col0 = td.bj * kBN + ch * 32;
          float v[32];
          tmem_ld32(taddr + ch * 32, v);
#pragma unroll
          for (int j = 0; j < 32; ++j) v[j] *= ks;
          store_row32<PREC>(yhi, ylo, static_cast<int64_t>(row) * cd.c_pad + col0, v);
        }
      }
      tc_fence_before();
      mbar_arrive(&tempty[PREC == P_FP32 ? 1 : acc]);
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem_base, 512);
}


// ---------------------------------------------------------------------------
// CTA-pair variant (fp16 / bf16 operands): a cluster of two CTAs on two SMs
// computes a 256 x 256 tile with tcgen05.mma.cta_group::2.  Each CTA loads
// its own 128 rows of the A operand and its own 128-column half of the B
// operand (no multicast), so a pair moves a third less operand data per
// FLOP than two single-CTA 128 x 256 tiles.  Each operand of a stage is one
// 4-D TMA box covering two k-blocks, issued by one of two producer warps:
// a TMA instruction holds its issuing thread for a few hundred cycles, and
// one box per operand and k-block from a single thread starved the MMAs.
// The leader CTA (rank 0) issues the MMAs; both CTAs' TMA loads complete on
// the leader's stage barrier, and the leader's commits arrive on the
// matching barriers of both CTAs.  Each CTA drains its own TMEM (its 128
// rows) in the epilogue.
//
// Symmetric results (A, B', the Gram-space factors) are computed on the
// 256 x 256 tiles of the upper block triangle; the epilogue of an
// off-diagonal tile also writes its transpose (stmatrix.trans from the
// accumulator fragments into a second store box), so SQUARE, SYMPROD and
// APPLY read them as K-major operands.  (Reading a lower block through its
// stored transpose as an MN-major operand instead ran SQUARE about 30%
// slower on B200.)
template <int PREC, int MODE>
struct PairCfg {
  // the last APPLY gives staging space to the fp32 W boxes of its <W, O> partials
  static constexpr bool kLast = MODE == M_APPLY_LAST;
  static constexpr bool kSquare = MODE == M_SQUARE;
  // Operand ring: stages of kKB k-blocks, each operand of a stage one TMA
  // box (two 64-column chunks of a 4-D map): 3 stages of 64 KB, or, in the
  // last APPLY, which also stages W, 5 stages of one k-block (32 KB)
  static constexpr int kKB = kLast ? 1 : 2;
  static constexpr int kStages = kLast ? 5 : 3;
  static constexpr int kWBufs = 2;
  static constexpr int kABlock = 128 * kBK * 2;                 // 16 KB: one k-block of this CTA's 128 rows
  static constexpr int kABytes = kKB * kABlock;
  static constexpr int kBBytes = kKB * kABlock;                 // this CTA's half of N
  static constexpr int kStageBytes = kABytes + kBBytes;
  static constexpr int kBarOffset = kStages * kStageBytes;
  // Epilogue warps: one per TMEM lane quarter
  static constexpr int kEpiWarps = 4;
  static constexpr int kProducerB = 2 + kEpiWarps;   // the B-operand producer warp, after the epilogue warps
  static constexpr int kThreads = 96 + 32 * kEpiWarps;
  // Epilogue output staging: each epilogue warp owns kWarpBufs boxes of
  // 32 rows x 32 columns (16-bit, 64-byte swizzle) that it writes to global
  // memory with its own TMA stores
  // GRAM and SYMPROD store two chunks per box (a 32 x 64 direct box, a 64 x
  // 32 mirror box): half the TMA stores
  static constexpr bool kPairStore = MODE == M_GRAM || MODE == M_SYMPROD;
  static constexpr int kWarpBox = kPairStore ? 32 * 64 * 2 : 32 * 32 * 2;
  static constexpr int kWarpBufs = (kLast || kSquare || kPairStore) ? 2 : 4;
  static constexpr int kStoreOffset = (kBarOffset + 256 + 1023) / 1024 * 1024;
  // SQUARE: each epilogue warp stages A's 32 x 32 box of its next chunk (for
  // the b A term) by TMA, two buffers, and reads it back with ldmatrix
  static constexpr int kABoxOffset = kStoreOffset + kEpiWarps * kWarpBufs * kWarpBox;
  static constexpr int kABoxBytes = kSquare ? kEpiWarps * 2 * kWarpBox : 0;
  // Last APPLY: kWBufs fp32 W boxes (128 rows x 32 columns, or 32 x 128 for
  // a tall W) filled kWBufs chunks ahead, for the <W, O> partials
  static constexpr int kWBox = 128 * 32 * 4;
  static constexpr int kWOffset = kABoxOffset + kABoxBytes;
  static constexpr int kSmem = kWOffset + (kLast ? kWBufs * kWBox : 0) + 1024;
  static_assert(kSmem <= 227 * 1024, "shared memory of the pair kernel exceeds 227 KB");
  static_assert(!kPairStore || kEpiWarps == 4, "a box of two consecutive chunks needs one warp per lane quarter");
  static_assert(2 * kStages + 2 + 2 + 1 + 4 + 4 + 8 <= 31, "mbarriers exceed their 256-byte region");
};

// Row `r` of a 16-bit box with 64-byte rows (32 columns; 32 or 64 rows),
// 16-byte piece q, in the 64-byte swizzle pattern of the TMA box.
__device__ __forceinline__ uint32_t store_box_offset(int r, int q) {
  return static_cast<uint32_t>(r * 64 + ((q ^ ((r >> 1) & 3)) << 4));
}

// Row `r` (0..31) of a 32 x 64 16-bit box, 16-byte piece q (0..7), in the
// 128-byte swizzle pattern of the TMA store box.
__device__ __forceinline__ uint32_t store_box_offset128(int r, int q) {
  return static_cast<uint32_t>(r * 128 + ((q ^ (r & 7)) << 4));
}

// TMA-store staging private to one epilogue warp: the warp writes a box of
// kBox bytes into an acquired buffer and lane 0 issues its store.  Acquire
// and commit alternate; a buffer is reused only after the store issued from
// it kBufs boxes earlier has read it, so the warps never wait on one
// another.
template <int kBufs, int kBox>
struct WarpStager {
  uint8_t* base;
  int count;   // boxes handed out so far
  // The next buffer, once the store issued from it kBufs puts ago has read it.
  __device__ __forceinline__ uint8_t* acquire(int lane) {
    uint8_t* buf = base + (count % kBufs) * kBox;
    if (count >= kBufs) {
      if (lane == 0) bulk_wait_read<kBufs - 1>();
      __syncwarp();
    }
    return buf;
  }
  // Store the box the warp wrote into the acquired buffer.
  __device__ __forceinline__ void commit(uint8_t* buf, const CUtensorMap* map, int lane, int x, int y, int z) {
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) {
      tma_store_3d(map, buf, x, y, z);
      bulk_commit();
    }
    ++count;
  }
  __device__ __forceinline__ void put(const CUtensorMap* map, int lane, const uint4 (&row)[4], int x, int y,
                                      int z) {
    uint8_t* buf = acquire(lane);
#pragma unroll
    for (int q = 0; q < 4; ++q) *reinterpret_cast<uint4*>(buf + store_box_offset(lane, q)) = row[q];
    commit(buf, map, lane, x, y, z);
  }
};

// Two fp32 values to a packed pair of 16-bit values, the first in the low half.
template <int PREC>
__device__ __forceinline__ uint32_t pack_pair(float lo, float hi) {
  if (PREC == P_BF16) {
    __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&h);
  }
  __half2 h = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}
template <int PREC>
__device__ __forceinline__ float unpack_lo(uint32_t u) {
  using T = typename Store16<PREC>::T;
  return Store16<PREC>::back(*reinterpret_cast<const T*>(&u));
}
template <int PREC>
__device__ __forceinline__ float unpack_hi(uint32_t u) {
  using T = typename Store16<PREC>::T;
  return Store16<PREC>::back(reinterpret_cast<const T*>(&u)[1]);
}

template <int PREC>
__device__ __forceinline__ void pack32(const float (&v)[32], uint4 (&packed)[4]) {
  using T = typename Store16<PREC>::T;
  T* h = reinterpret_cast<T*>(packed);
#pragma unroll
  for (int j = 0; j < 32; ++j) h[j] = Store16<PREC>::cvt(v[j]);
}
constexpr int kPairM = 256;

template <int MODE, int PREC>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(PairCfg<PREC, MODE>::kThreads, 1)
    ns_gemm_pair_kernel(const __grid_constant__ NsParams p) {
  using C = PairCfg<PREC, MODE>;
  constexpr bool kApply = MODE == M_APPLY || MODE == M_APPLY_LAST;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::kBarOffset);
  uint64_t* empty = full + C::kStages;
  uint64_t* tfull = empty + C::kStages;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint64_t* wfull = drain + 1;                       // last APPLY / SQUARE: staged boxes landed
  uint64_t* wempty = wfull + 4;                      // ... and consumed by the 4 epilogue warps
  uint64_t* abar = wempty + 4;                       // SQUARE: A boxes landed, per epilogue warp and buffer
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(abar + 8);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();          // 0 = leader
  const int pair = blockIdx.x >> 1;
  const int npairs = gridDim.x >> 1;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(&full[s], 1);                        // leader: one expect_tx arrival per phase
      mbar_init(&empty[s], 1);                       // one multicast commit per phase
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], 2 * 32 * C::kEpiWarps);  // both CTAs' epilogue threads
    }
    mbar_init(drain, 1);
    for (int b = 0; b < C::kWBufs; ++b) {
      mbar_init(&wfull[b], 1);
      mbar_init(&wempty[b], C::kEpiWarps);
    }
    for (int b = 0; b < 8; ++b) mbar_init(&abar[b], 1);
    fence_mbar_init();
  }
  if (warp == 1) tmem_alloc_pair(tmem_slot, 512);
  tc_fence_before();
  __syncthreads();
  cluster_sync();                                    // barriers initialised in both CTAs
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0 || warp == C::kProducerB) {
    // ------------------------------------------------------------ TMA producers (both CTAs)
    // warp 0 loads the A operand of every stage (and, in the leader, sets
    // the stage's expected bytes); warp kProducerB loads the B operand, so
    // that the two boxes of a stage are issued from two warps at once
    const bool role_a = warp == 0;
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      uint32_t issued_parity[C::kStages];
      bool issued[C::kStages];
      for (int s = 0; s < C::kStages; ++s) issued[s] = false;
      bool ok = true;
      for (int t = pair; t < p.ntiles && ok; t += npairs) {
        const TileDesc td = p.tiles[t];
        const MatDev& md = p.mats[td.mat];
        const ClassDev& cd = p.classes[md.cls];
        const int z = md.z;
        const int nk = (MODE == M_SQUARE || MODE == M_SYMPROD) ? td.nk_sq : td.nk;
        const int abase = td.bi * kPairM, bbase = td.bj * kBN;                // tile origin
        const int arow = abase + static_cast<int>(rank) * 128;              // this CTA's A rows
        const int bcol = bbase + static_cast<int>(rank) * 128;              // this CTA's B half
        for (int kb = 0; kb < nk; kb += C::kKB) {
          if (!mbar_wait(&empty[stage], phase ^ 1u, p.err)) { ok = false; break; }
          if (rank == 0 && role_a) mbar_expect_tx(&full[stage], 2 * C::kStageBytes);
          const uint32_t bar = map_shared_rank(&full[stage], 0);
          uint8_t* sa = smem + stage * C::kStageBytes;
          uint8_t* sb = sa + C::kABytes;
          const int k0 = kb * kBK;
          if (C::kKB == 2) {
            // one 4-D box per operand and stage: K-major operands as the two
            // 64-column chunks (k-blocks) kb, kb + 1 of this CTA's 128 rows;
            // in APPLY, Y's rows k0 .. k0+127 in this CTA's two 64-column
            // chunks (read MN-major).  Half the TMA instructions of one box
            // per k-block.
            if (MODE == M_GRAM) {
              const CUtensorMap* xm = p.tmaps + cd.tm_base + TM_X_C128 + p.src;
              if (role_a) tma_load_4d_pair(sa, xm, bar, 0, arow, kb, z);
              if (!role_a) tma_load_4d_pair(sb, xm, bar, 0, bcol, kb, z);
            } else if (MODE == M_SQUARE || MODE == M_SYMPROD) {
              if (role_a) tma_load_4d_pair(sa, p.tmaps + cd.tm_base + tm_rr_c128(p.lhs), bar, 0, arow, kb, z);
              if (!role_a) tma_load_4d_pair(sb, p.tmaps + cd.tm_base + tm_rr_c128(p.rhs), bar, 0, bcol, kb, z);
            } else {
              if (role_a) tma_load_4d_pair(sa, p.tmaps + cd.tm_base + tm_rr_c128(p.lhs), bar, 0, arow, kb, z);
              if (!role_a) tma_load_4d_pair(sb, p.tmaps + cd.tm_base + TM_X_C128 + p.src, bar, 0, k0, bcol / 64, z);
            }
          } else if (MODE == M_GRAM) {
            if (role_a) tma_load_3d_pair(sa, p.tmaps + tm_x(cd.tm_base + TM_X_K128, p.src, 0), bar, k0, arow, z);
            if (!role_a) tma_load_3d_pair(sb, p.tmaps + tm_x(cd.tm_base + TM_X_K128, p.src, 0), bar, k0, bcol, z);
          } else if (MODE == M_SQUARE || MODE == M_SYMPROD) {
            // A A (SQUARE) or L R (SYMPROD) with both operands stored whole
            // (every block and its mirror): both K-major; the right operand is
            // symmetric, so its rows serve as the N x K operand
            if (role_a) tma_load_3d_pair(sa, p.tmaps + cd.tm_base + tm_rr_k128(p.lhs), bar, k0, arow, z);
            if (!role_a) tma_load_3d_pair(sb, p.tmaps + cd.tm_base + tm_rr_k128(p.rhs), bar, k0, bcol, z);
          } else {
            // APPLY: rows of B' or Q (stored with its mirror, K-major) times Y,
            // read as an MN-major operand: both 64-column chunks of this CTA's
            // half in one box (one TMA instruction fewer per stage: APPLY ran
            // 4-5% faster than with a box per chunk)
            if (role_a) tma_load_3d_pair(sa, p.tmaps + cd.tm_base + tm_rr_k128(p.lhs), bar, k0, arow, z);
            if (!role_a) tma_load_4d_pair(sb, p.tmaps + cd.tm_base + TM_X_C64 + p.src, bar, 0, k0, bcol / 64, z);
          }
          issued[stage] = true;
          issued_parity[stage] = phase;
          if (++stage == C::kStages) { stage = 0; phase ^= 1u; }
        }
      }
      if (!ok && rank == 0 && role_a) {
        for (int s = 0; s < C::kStages; ++s)
          if (issued[s]) {
            const uint64_t t0 = globaltimer();
            while (!mbar_try_wait(&full[s], issued_parity[s]) && globaltimer() - t0 < kWaitLimitNs) {
            }
          }
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer (leader only)
    if (lane == 0 && rank == 0) {
      // A operand always K-major; B operand MN-major in APPLY (Y read as stored)
      constexpr uint32_t kIdesc = idesc_f16(kPairM, kBN, PREC == P_BF16 ? 1 : 0, kApply ? 1 : 0);
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      int local = 0;
      TileDesc td = pair < p.ntiles ? p.tiles[pair] : TileDesc{};
      for (int t = pair; t < p.ntiles && ok; t += npairs, ++local) {
        const TileDesc next = (t + npairs < p.ntiles) ? p.tiles[t + npairs] : td;   // prefetch
        const int nk = (MODE == M_SQUARE || MODE == M_SYMPROD) ? td.nk_sq : td.nk;
        const int acc = local & 1;
        const uint32_t acc_phase = (local >> 1) & 1;
        if (!mbar_wait(&tempty[acc], acc_phase ^ 1u, p.err)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * kBN;
        for (int kb = 0; kb < nk; kb += C::kKB) {
          if (!mbar_wait(&full[stage], phase, p.err)) { ok = false; break; }
          tc_fence_after();
          const uint32_t s0 = smem_u32(smem + stage * C::kStageBytes);
#pragma unroll
          for (int j = 0; j < C::kKB; ++j) {
            // k-block kb + j: A chunk j; B chunk j (K-major), or rows 64 j ..
            // of both 64-column chunks (MN-major APPLY: chunk stride kKB x 8 KB)
            const uint32_t sa = s0 + j * C::kABlock;
            const uint32_t sb = s0 + C::kABytes + j * (kApply ? 64 * 128 : C::kABlock);
#pragma unroll
            for (int k = 0; k < kBK / 16; ++k) {
              const uint64_t adesc = sdesc_sw128(sa + k * 32, 16, 1024);
              const uint64_t bdesc = kApply ? sdesc_sw128(sb + k * 16 * 128, C::kKB * 64 * 128, 1024)
                                            : sdesc_sw128(sb + k * 32, 16, 1024);
              umma_f16_pair(d_tmem, adesc, bdesc, kIdesc, ((kb + j) | k) != 0 ? 1u : 0u);
            }
          }
          umma_commit_pair(&empty[stage]);
          if (++stage == C::kStages) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        umma_commit_pair(&tfull[acc]);
        td = next;
      }
      umma_commit(drain);
      const uint64_t t0 = globaltimer();
      while (!mbar_try_wait(drain, 0) && globaltimer() - t0 < kWaitLimitNs) {
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue (both CTAs)
    const int quarter = warp & 3;             // TMEM lanes 32 quarter .. +31 (a warp reaches lanes of warp id mod 4)
    const int epi = warp - 2;                 // 0 .. kEpiWarps-1
    constexpr int kChStep = C::kEpiWarps / 4; // warps sharing a lane quarter split its chunks
    const int ch0 = epi / 4;
    const int lrow = quarter * 32 + lane;
    const uint32_t tempty_leader[2] = {map_shared_rank(&tempty[0], 0), map_shared_rank(&tempty[1], 0)};
    WarpStager<C::kWarpBufs, C::kWarpBox> stager{smem + C::kStoreOffset + epi * C::kWarpBufs * C::kWarpBox, 0};
    const int wrow0_off = quarter * 32;   // this warp's rows inside the CTA's 128
    // SQUARE: A boxes of this warp (two buffers), their landing barriers and
    // phases, and whether a box is still in flight (for the give-up path)
    uint8_t* const abox = smem + C::kABoxOffset + epi * 2 * C::kWarpBox;
    uint64_t* const abar_w = abar + 2 * epi;
    uint32_t aphase[2] = {0u, 0u};
    bool a_inflight[2] = {false, false};
    int a_count = 0;   // A boxes issued so far; box i lands in buffer i % 2
    auto a_issue = [&](const CUtensorMap* amap, int x, int y, int z) {
      const int b = a_count & 1;
      if (lane == 0) {
        fence_proxy_async_smem();   // the buffer's previous box was read with ldmatrix
        mbar_expect_tx(&abar_w[b], C::kWarpBox);
        tma_load_3d(abox + b * C::kWarpBox, amap, &abar_w[b], x, y, z);
      }
      a_inflight[b] = true;
      ++a_count;
    };
    uint32_t wphase[C::kWBufs] = {};   // phases of the staging buffers
    int w_pending[C::kWBufs] = {};     // thread 64: staged loads issued and not yet consumed
    int w_issued[C::kWBufs] = {};      // thread 64: loads issued into each buffer so far
    bool werr = false;
    // thread 64 loads the last APPLY's W box of chunk `chk` into buffer b
    auto w_issue = [&](const TileDesc& td, const MatDev& md, const ClassDev& cd, int row0, int b, int chk) {
      const int c0 = td.bj * kBN + chk * 32;
      // the buffer's previous contents must have been read by all epilogue warps
      if (w_issued[b] > 0 && !mbar_wait(&wempty[b], static_cast<uint32_t>(w_issued[b] - 1) & 1u, p.err)) {
        werr = true;
        return;
      }
      ++w_issued[b];
      mbar_expect_tx(&wfull[b], C::kWBox);
      uint8_t* dst = smem + C::kWOffset + b * C::kWBox;
      (void)cd;
      if (!md.transposed)
        tma_load_2d(dst, p.wmaps + td.mat, &wfull[b], c0, row0);
      else
        tma_load_2d(dst, p.wmaps + td.mat, &wfull[b], row0, c0);
      ++w_pending[b];
    };
    int local = 0;
    for (int t = pair; t < p.ntiles; t += npairs, ++local) {
      const TileDesc td = p.tiles[t];
      const MatDev& md = p.mats[td.mat];
      const ClassDev& cd = p.classes[md.cls];
      const int acc = local & 1;
      const uint32_t acc_phase = (local >> 1) & 1;
      if (threadIdx.x == 64 && C::kLast && md.fused_dots && p.iter == md.ns_steps - 1) {
        const int r0 = td.bi * kPairM + static_cast<int>(rank) * 128;
        for (int b = 0; b < C::kWBufs; ++b) w_issue(td, md, cd, r0, b, b);   // first chunks while the MMAs run
      }
      // SQUARE reads A (written by GRAM, read-only here) for its b A term:
      // the 32 x 32 box of this warp's rows and the chunk's columns, staged
      // by TMA one chunk ahead and read with ldmatrix straight into the
      // accumulator fragment layout (rows lane/4 + 8p + 16h of the warp's
      // 32, columns 8k + 2 (lane % 4) (+1) of the chunk)
      const CUtensorMap* amap = p.tmaps + cd.tm_base + TM_A_ST;
      const int arow_w = td.bi * kPairM + static_cast<int>(rank) * 128 + quarter * 32;
      if (C::kSquare) a_issue(amap, td.bj * kBN + ch0 * 32, arow_w, md.z);
      if (!mbar_wait(&tfull[acc], acc_phase, p.err)) break;
      tc_fence_after();
      const int row0 = td.bi * kPairM + static_cast<int>(rank) * 128;   // this CTA's first row
      const int row = row0 + lrow;
      const uint32_t taddr = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) + acc * kBN;
      // iteration 0 reads X at the momentum kernel's scale: kappa corrects it
      const float kap = (MODE == M_GRAM && p.iter == 0) ? p.scal[td.mat].kappa : 1.f;
      const bool mirror = td.bj > td.bi;   // off-diagonal block: also store its transpose
      if (MODE == M_GRAM || MODE == M_SYMPROD || MODE == M_SQUARE) {
        // Symmetric outputs, drained in the accumulator fragment layout
        // (tcgen05.ld.16x256b): the warp writes its 32 x 32 box with
        // stmatrix and, for an off-diagonal tile, the mirrored box with
        // stmatrix.trans, so the transpose costs no extra shared-memory pass.
        //   GRAM:    stored A   = 2^ea Y Y^T from the stored Y (2^ex Y)
        //   SYMPROD: stored out = 2^e_out L R from the stored L and R
        //   SQUARE:  stored B'  = 2^eb (c A A + b A + a I) from the stored A
        float sa = 1.f, s2 = 0.f, s1 = 0.f, diag = 0.f;
        if (MODE == M_GRAM) sa = kap * kap * exp2f(static_cast<float>(md.ea - 2 * md.ex));
        if (MODE == M_SYMPROD)
          sa = exp2f(static_cast<float>(rr_exp(md, p.out_kind) - rr_exp(md, p.lhs_kind) - rr_exp(md, p.rhs_kind)));
        if (MODE == M_SQUARE) {
          s2 = md.c_coef * exp2f(static_cast<float>(md.eb - 2 * md.ea));
          s1 = md.b * exp2f(static_cast<float>(md.eb - md.ea));
          diag = md.a * exp2f(static_cast<float>(md.eb));
        }
        const CUtensorMap* omap = p.tmaps + cd.tm_base + (MODE == M_GRAM ? TM_A_ST : tm_rr_st(p.out));
        // GRAM, SYMPROD: 32 x 64 direct and 64 x 32 mirror boxes of two chunks
        const CUtensorMap* omap2 = p.tmaps + cd.tm_base + (MODE == M_GRAM ? TM_A_ST2 : tm_rr_st2(p.out));
        const CUtensorMap* omapm = p.tmaps + cd.tm_base + (MODE == M_GRAM ? TM_A_STM : tm_rr_stm(p.out));
        uint32_t wprev[2][2][4];   // the first chunk of a pair, held for its box
        const int grow = row0 + wrow0_off;            // this warp's first row
        const int frow = lane >> 2, fcol = 2 * (lane & 3);
        for (int ch = ch0; ch < kBN / 32; ch += kChStep) {
          const int col0 = td.bj * kBN + ch * 32;
          uint32_t u[2][16];
          tmem_ld16x32_nowait(taddr + ch * 32, u[0]);                       // rows 0..15 of the warp's 32
          tmem_ld16x32_nowait(taddr + (16u << 16) + ch * 32, u[1]);         // rows 16..31
          tmem_wait_ld();
          if (ch + kChStep >= kBN / 32) {   // this warp's last chunk of the tile
            tc_fence_before();
            mbar_arrive_cluster(tempty_leader[acc]);   // accumulator drained
          }
          uint32_t a_cur[16];
          if (MODE == M_SQUARE) {
            const int b = (a_count - 1) & 1;   // this chunk's box (the latest issued)
            if (ch + kChStep < kBN / 32) a_issue(amap, col0 + kChStep * 32, arow_w, md.z);
            if (!mbar_wait(&abar_w[b], aphase[b], p.err)) {
              werr = true;
              break;
            }
            aphase[b] ^= 1u;
            a_inflight[b] = false;
            const uint32_t ab = smem_u32(abox + b * C::kWarpBox);
#pragma unroll
            for (int hp = 0; hp < 4; ++hp)
              ldmatrix_x4(ab + store_box_offset(8 * hp + (lane & 7), lane >> 3), a_cur[4 * hp], a_cur[4 * hp + 1],
                          a_cur[4 * hp + 2], a_cur[4 * hp + 3]);
          }
          uint32_t w[2][2][4];   // [h][p][k]: rows 16h + 8p + lane/4, columns 8k + 2 (lane % 4) (+1)
#pragma unroll
          for (int h = 0; h < 2; ++h)
#pragma unroll
            for (int pp = 0; pp < 2; ++pp)
#pragma unroll
              for (int k = 0; k < 4; ++k) {
                float v0 = __uint_as_float(u[h][4 * k + 2 * pp]), v1 = __uint_as_float(u[h][4 * k + 2 * pp + 1]);
                if (MODE == M_SQUARE) {
                  const uint32_t av = a_cur[4 * (2 * h + pp) + k];
                  v0 = fmaf(s2, v0, s1 * unpack_lo<PREC>(av));
                  v1 = fmaf(s2, v1, s1 * unpack_hi<PREC>(av));
                  const int rg = grow + 16 * h + 8 * pp + frow, cg = col0 + 8 * k + fcol;
                  if (rg == cg || rg == cg + 1) {
                    float& vd = rg == cg ? v0 : v1;
                    vd += diag;
                    // bf16 keeps 8 significant bits of the diagonal (near a = 3.44
                    // in early iterations): APPLY adds back the rounding residual
                    if (PREC == P_BF16)
                      cd.bdiag[static_cast<int64_t>(md.z) * cd.r_pad + rg] =
                          vd - Store16<PREC>::back(Store16<PREC>::cvt(vd));
                  }
                } else {
                  v0 *= sa;
                  v1 *= sa;
                }
                w[h][pp][k] = pack_pair<PREC>(v0, v1);
              }
          if (C::kPairStore) {
            const int c = ch & 1;   // chunk of the pair (every warp walks every chunk)
            if (c == 0) {
#pragma unroll
              for (int h = 0; h < 2; ++h)
#pragma unroll
                for (int pp = 0; pp < 2; ++pp)
#pragma unroll
                  for (int k = 0; k < 4; ++k) wprev[h][pp][k] = w[h][pp][k];
              continue;
            }
            // direct box: chunk cc's matrix (h, p, k) is rows 16h + 8p .. +7, 16-byte piece 4 cc + k
            uint8_t* buf = stager.acquire(lane);
            const uint32_t sb = smem_u32(buf);
#pragma unroll
            for (int h = 0; h < 2; ++h)
#pragma unroll
              for (int pp = 0; pp < 2; ++pp) {
                stmatrix_x4(sb + store_box_offset128(16 * h + 8 * pp + (lane & 7), lane >> 3), wprev[h][pp][0],
                            wprev[h][pp][1], wprev[h][pp][2], wprev[h][pp][3]);
                stmatrix_x4(sb + store_box_offset128(16 * h + 8 * pp + (lane & 7), 4 + (lane >> 3)), w[h][pp][0],
                            w[h][pp][1], w[h][pp][2], w[h][pp][3]);
              }
            stager.commit(buf, omap2, lane, col0 - 32, grow, md.z);
            if (mirror) {
              // chunk cc transposed: mirror-box rows 32 cc + 8k .. +7, piece 2h + p
              uint8_t* mb = stager.acquire(lane);
              const uint32_t smb = smem_u32(mb);
#pragma unroll
              for (int h = 0; h < 2; ++h)
#pragma unroll
                for (int pp = 0; pp < 2; ++pp) {
                  stmatrix_x4_trans(smb + store_box_offset(lane, 2 * h + pp), wprev[h][pp][0], wprev[h][pp][1],
                                    wprev[h][pp][2], wprev[h][pp][3]);
                  stmatrix_x4_trans(smb + store_box_offset(32 + lane, 2 * h + pp), w[h][pp][0], w[h][pp][1],
                                    w[h][pp][2], w[h][pp][3]);
                }
              stager.commit(mb, omapm, lane, grow, col0 - 32, md.z);
            }
            continue;
          }
          // direct box: matrix (h, p, k) is box rows 16h + 8p .. +7, 16-byte piece k
          uint8_t* buf = stager.acquire(lane);
          const uint32_t sb = smem_u32(buf);
#pragma unroll
          for (int h = 0; h < 2; ++h)
#pragma unroll
            for (int pp = 0; pp < 2; ++pp)
              stmatrix_x4(sb + store_box_offset(16 * h + 8 * pp + (lane & 7), lane >> 3), w[h][pp][0], w[h][pp][1],
                          w[h][pp][2], w[h][pp][3]);
          stager.commit(buf, omap, lane, col0, grow, md.z);
          if (mirror) {
            // out[col][row] = out[row][col]: matrix (h, p, k) transposed is
            // mirror-box rows 8k .. 8k+7, piece 2h + p; lane l addresses row l
            uint8_t* mb = stager.acquire(lane);
            const uint32_t smb = smem_u32(mb);
#pragma unroll
            for (int h = 0; h < 2; ++h)
#pragma unroll
              for (int pp = 0; pp < 2; ++pp)
                stmatrix_x4_trans(smb + store_box_offset(lane, 2 * h + pp), w[h][pp][0], w[h][pp][1], w[h][pp][2],
                                  w[h][pp][3]);
            stager.commit(mb, omap, lane, grow, col0, md.z);
          }
        }
        if (werr) break;
      } else {
        // Y' = 2^ex (B' or Q) Y from the stored operand and Y; kappa where Y
        // is the momentum kernel's X
        const float ks = (p.apply_kappa ? p.scal[td.mat].kappa : 1.f) *
                         exp2f(static_cast<float>(-rr_exp(md, p.lhs_kind)));
        const CUtensorMap* ymap = p.tmaps + cd.tm_base + TM_X_ST + (p.src ^ 1);
        // Last APPLY: Y' is the update O; accumulate ||O||^2 and <W, O> over
        // the stored values, W staged per 32-column chunk by TMA (wide W: box
        // of W[row0.., col0..]; tall W: box of W[col0.., row0..]).
        const bool dots = C::kLast && md.fused_dots && p.iter == md.ns_steps - 1;
        float oo = 0.f, wo = 0.f;
        // bf16 operands: Y' = (B'_stored + diag(residual)) Y, the residual of
        // this row times its own Y row, read from L2 one chunk ahead
        float dres = 0.f;
        const uint16_t* yrow = nullptr;
        uint4 y_next[4];
        if (PREC == P_BF16) {
          dres = cd.bdiag[static_cast<int64_t>(md.z) * cd.r_pad + row];
          yrow = static_cast<const uint16_t*>(cd.x[p.src][0]) + md.z * cd.x_stride +
                 static_cast<int64_t>(row) * cd.c_pad + td.bj * kBN;
#pragma unroll
          for (int q = 0; q < 4; ++q) y_next[q] = __ldg(reinterpret_cast<const uint4*>(yrow + ch0 * 32) + q);
        }
        for (int ch = ch0; ch < kBN / 32; ch += kChStep) {
          const int col0 = td.bj * kBN + ch * 32;
          float v[32];
          tmem_ld32(taddr + ch * 32, v);
          if (ch + kChStep >= kBN / 32) {   // this warp's last chunk of the tile
            tc_fence_before();
            mbar_arrive_cluster(tempty_leader[acc]);
          }
          if (PREC == P_BF16) {
            uint4 y_cur[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) y_cur[q] = y_next[q];
            if (ch + kChStep < kBN / 32) {
#pragma unroll
              for (int q = 0; q < 4; ++q) y_next[q] = __ldg(reinterpret_cast<const uint4*>(yrow + (ch + kChStep) * 32) + q);
            }
            using T16 = typename Store16<PREC>::T;
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const T16* h = reinterpret_cast<const T16*>(&y_cur[q]);
#pragma unroll
              for (int e = 0; e < 8; ++e) v[8 * q + e] = fmaf(dres, Store16<PREC>::back(h[e]), v[8 * q + e]);
            }
          }
#pragma unroll
          for (int j = 0; j < 32; ++j) v[j] *= ks;
          uint4 packed[4];
          pack32<PREC>(v, packed);
          stager.put(ymap, lane, packed, col0, row0 + wrow0_off, md.z);
          if (C::kLast && dots) {
            const int b = ch % C::kWBufs;
            if (!mbar_wait(&wfull[b], wphase[b], p.err)) { werr = true; break; }
            wphase[b] ^= 1u;
            if (threadIdx.x == 64) --w_pending[b];
            const uint8_t* wb = smem + C::kWOffset + b * C::kWBox;
            using T16 = typename Store16<PREC>::T;
            const T16* h = reinterpret_cast<const T16*>(packed);
            if (!md.transposed) {
#pragma unroll
              for (int q = 0; q < 8; ++q) {
                const float4 w4 = *reinterpret_cast<const float4*>(wb + lrow * 128 + ((q ^ (lrow & 7)) << 4));
                const float o0 = Store16<PREC>::back(h[4 * q]), o1 = Store16<PREC>::back(h[4 * q + 1]);
                const float o2 = Store16<PREC>::back(h[4 * q + 2]), o3 = Store16<PREC>::back(h[4 * q + 3]);
                oo = fmaf(o0, o0, fmaf(o1, o1, fmaf(o2, o2, fmaf(o3, o3, oo))));
                wo = fmaf(w4.x, o0, fmaf(w4.y, o1, fmaf(w4.z, o2, fmaf(w4.w, o3, wo))));
              }
            } else {
#pragma unroll
              for (int j = 0; j < 32; ++j) {
                const float w = *reinterpret_cast<const float*>(wb + j * 512 + lrow * 4);
                const float o = Store16<PREC>::back(h[j]);
                oo = fmaf(o, o, oo);
                wo = fmaf(w, o, wo);
              }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&wempty[b]);   // this warp is done with W buffer b
            if (threadIdx.x == 64 && ch + C::kWBufs < kBN / 32) w_issue(td, md, cd, row0, b, ch + C::kWBufs);
          }
        }
        if (werr) break;
        if (C::kLast && dots) {
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) {
            oo += __shfl_xor_sync(0xffffffffu, oo, o);
            wo += __shfl_xor_sync(0xffffffffu, wo, o);
          }
          if (lane == 0) {   // one slot per (pair tile, CTA, epilogue warp)
            const int64_t slot =
                md.ns_slot_base + ((static_cast<int64_t>(td.bi) * md.ns_tiles_bj + td.bj) * 2 + rank) * 4 + quarter;
            p.part_ns[2 * slot] = oo;
            p.part_ns[2 * slot + 1] = wo;
          }
        }
      }
    }
    if (lane == 0) bulk_wait_all();   // every TMA store of this warp has completed
    // on a give-up path, let this warp's A boxes in flight land before the CTA exits
    for (int b = 0; b < 2; ++b)
      if (C::kSquare && a_inflight[b]) {
        const uint64_t t0 = globaltimer();
        while (!mbar_try_wait(&abar_w[b], aphase[b]) && globaltimer() - t0 < kWaitLimitNs) {
        }
      }
    if (threadIdx.x == 64) {
      // on a give-up path, let issued W loads land before the CTA exits
      for (int b = 0; b < C::kWBufs; ++b)
        for (; w_pending[b] > 0; --w_pending[b]) {
          const uint64_t t0 = globaltimer();
          while (!mbar_try_wait(&wfull[b], wphase[b]) && globaltimer() - t0 < kWaitLimitNs) {
          }
          wphase[b] ^= 1u;
        }
    }
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync();              // the leader's MMAs into both CTAs' TMEM have drained
  tc_fence_after();
  if (warp == 1) tmem_dealloc_pair(tmem_base, 512);
}

}  // namespace

template <int MODE, int PREC>
static cudaError_t set_attr() {
  return cudaFuncSetAttribute(ns_gemm_kernel<MODE, PREC>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              Cfg<PREC>::kSmem);
}

template <int MODE, int PREC>
static cudaError_t set_pair_attr() {
  return cudaFuncSetAttribute(ns_gemm_pair_kernel<MODE, PREC>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              PairCfg<PREC, MODE>::kSmem);
}

cudaError_t ns_gemm_set_attributes() {
  cudaError_t e;
#define MUONH_SET_PAIR(MD, PR) \
  if ((e = set_pair_attr<MD, PR>()) != cudaSuccess) return e;
  MUONH_SET_PAIR(M_GRAM, P_FP16) MUONH_SET_PAIR(M_SQUARE, P_FP16) MUONH_SET_PAIR(M_APPLY, P_FP16)
  MUONH_SET_PAIR(M_APPLY_LAST, P_FP16) MUONH_SET_PAIR(M_SYMPROD, P_FP16)
  MUONH_SET_PAIR(M_GRAM, P_BF16) MUONH_SET_PAIR(M_SQUARE, P_BF16) MUONH_SET_PAIR(M_APPLY, P_BF16)
  MUONH_SET_PAIR(M_APPLY_LAST, P_BF16)
#undef MUONH_SET_PAIR
#define MUONH_SET(MD, PR) \
  if ((e = set_attr<MD, PR>()) != cudaSuccess) return e;
  MUONH_SET(M_GRAM, P_FP16) MUONH_SET(M_SQUARE, P_FP16) MUONH_SET(M_APPLY, P_FP16)
  MUONH_SET(M_GRAM, P_BF16) MUONH_SET(M_SQUARE, P_BF16) MUONH_SET(M_APPLY, P_BF16)
  MUONH_SET(M_GRAM, P_FP32) MUONH_SET(M_SQUARE, P_FP32) MUONH_SET(M_APPLY, P_FP32)
#undef MUONH_SET
  return cudaSuccess;
}

size_t ns_gemm_smem_bytes(int prec) {
  return prec == P_FP32 ? Cfg<P_FP32>::kSmem : Cfg<P_FP16>::kSmem;
}

cudaError_t launch_ns_gemm_pair(int mode, int prec, const NsParams& p, int pairs, cudaStream_t s) {
  if (p.ntiles <= 0) return cudaSuccess;
#define MUONH_LAUNCH_PAIR(MD, PR)                                                              \
  if (mode == MD && prec == PR) {                                                              \
    ns_gemm_pair_kernel<MD, PR><<<2 * pairs, PairCfg<PR, MD>::kThreads, PairCfg<PR, MD>::kSmem, s>>>(p);   \
    return cudaGetLastError();                                                                 \
  }
  MUONH_LAUNCH_PAIR(M_GRAM, P_FP16) MUONH_LAUNCH_PAIR(M_SQUARE, P_FP16) MUONH_LAUNCH_PAIR(M_APPLY, P_FP16)
  MUONH_LAUNCH_PAIR(M_APPLY_LAST, P_FP16) MUONH_LAUNCH_PAIR(M_SYMPROD, P_FP16)
  MUONH_LAUNCH_PAIR(M_GRAM, P_BF16) MUONH_LAUNCH_PAIR(M_SQUARE, P_BF16) MUONH_LAUNCH_PAIR(M_APPLY, P_BF16)
  MUONH_LAUNCH_PAIR(M_APPLY_LAST, P_BF16)
#undef MUONH_LAUNCH_PAIR
  return cudaErrorInvalidValue;
}

cudaError_t launch_ns_gemm(int mode, int prec, const NsParams& p, int grid, cudaStream_t s) {
  if (p.ntiles <= 0) return cudaSuccess;
  const size_t smem = ns_gemm_smem_bytes(prec);
#define MUONH_LAUNCH(MD, PR)                                                   \
  if (mode == MD && prec == PR) {                                              \
    ns_gemm_kernel<MD, PR><<<grid, kGemmThreads, smem, s>>>(p);                \
    return cudaGetLastError();                                                 \
  }
  MUONH_LAUNCH(M_GRAM, P_FP16) MUONH_LAUNCH(M_SQUARE, P_FP16) MUONH_LAUNCH(M_APPLY, P_FP16)
  MUONH_LAUNCH(M_GRAM, P_BF16) MUONH_LAUNCH(M_SQUARE, P_BF16) MUONH_LAUNCH(M_APPLY, P_BF16)
  MUONH_LAUNCH(M_GRAM, P_FP32) MUONH_LAUNCH(M_SQUARE, P_FP32) MUONH_LAUNCH(M_APPLY, P_FP32)
#undef MUONH_LAUNCH
  return cudaErrorInvalidValue;
}

}  // namespace muonh
