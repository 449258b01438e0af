// Internal definitions shared by the CUDA translation units of libmuonh:
// device-side tables, launch parameters and inline-PTX wrappers for
// mbarrier, TMA and tcgen05 (sm_100a).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <cuda_fp16.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "../../include/muonh.h"

namespace muonh {

// ------------------------------------------------------------------ sizes
constexpr int kEwTile = 64;          // elementwise tiles: 64 x 64 elements of W
constexpr int kEwThreads = 256;
constexpr int kBM = 128;             // Newton-Schulz GEMM tile: 128 x 256 x 64
constexpr int kBN = 256;
constexpr int kBK = 64;
constexpr int kPad = 256;            // NS buffers are padded to multiples of 256
constexpr int kGemmThreads = 192;    // warp 0 TMA, warp 1 MMA, warps 2-5 epilogue
constexpr unsigned long long kWaitLimitNs = 2000000000ull;   // 2 s per wait

enum Prec { P_FP16 = 0, P_BF16 = 1, P_FP32 = 2 };
// LAST: also ||O||^2, <W, O>.  SYMPROD: product of two symmetric r x r
// operands that commute (Gram-space form), stored with its mirror.
enum Mode { M_GRAM = 0, M_SQUARE = 1, M_APPLY = 2, M_APPLY_LAST = 3, M_SYMPROD = 4 };

// r x r buffers of a shape class, as operands of SQUARE / SYMPROD / APPLY.
// The Y-space iteration uses A and B'; the Gram-space form also P1 and T.
enum RrBuf { RR_A = 0, RR_B = 1, RR_P1 = 2, RR_T = 3 };
// Power-of-two scale of a stored r x r operand: A-like (A, T = A P), P-like
// (B' = p(A)), Q-like (a product of several p(A)).
enum RrKind { RK_A = 0, RK_P = 1, RK_Q = 2 };

// Tensor-map slots of one shape class.  "hi" buffers hold the 16-bit
// operand (fp16/bf16), "lo" buffers the fp16 residual in FP32 mode.  The
// CTA-pair kernels (16-bit operands) use the store boxes; the
// FP32-mode kernel stores directly and also reads C = b I + c A.
enum TmSlot {
  TM_X_K128 = 0,   // X[buf] as K-major operand, 128-row box   (+buf, +2*part)
  TM_X_K256 = 4,   // X[buf] as K-major operand, 256-row box
  TM_X_MN = 8,     // X[buf] as MN-major operand, 64 x 64 box
  TM_A_K128 = 12,  // A, 128-row box (+part)
  TM_C_K256 = 14,  // C = b I + c A, 256-row box (+part), FP32 mode only
  TM_B_K128 = 16,  // B' = a I + b A + c A A, 128-row box (+part)
  TM_X_ST = 18,    // X[buf] store box 32 x 32 (64-byte swizzle)   (+buf)
  TM_A_ST = 20,    // A store box (direct and mirrored blocks)
  TM_B_ST = 21,    // B' store box (direct and mirrored blocks)
  TM_P1_K128 = 22, // Gram-space form: P1, 128-row box
  TM_T_K128 = 23,  // Gram-space form: T, 128-row box
  TM_P1_ST = 24,   // P1 store box
  TM_T_ST = 25,    // T store box
  // CTA pairs: 4-D maps (64 columns, rows, 64-column chunks, matrix) that
  // load two 64-column chunks with one instruction
  TM_X_C64 = 26,   // X[buf], 64 rows x 2 chunks: an MN-major k-block of a 128-column half (+buf)
  TM_X_C128 = 28,  // X[buf], 128 rows x 2 chunks: two K-major k-blocks, or two MN-major ones (+buf)
  TM_A_C128 = 30,  // A, B', P1, T: 128 rows x 2 chunks, two K-major k-blocks
  TM_B_C128 = 31,
  TM_P1_C128 = 32,
  TM_T_C128 = 33,
  // CTA pairs, GRAM and SYMPROD outputs: 32 x 64 direct boxes (128-byte
  // swizzle) and 64 x 32 mirror boxes (64-byte swizzle) of A, B', P1, T
  TM_A_ST2 = 34,
  TM_B_ST2 = 35,
  TM_P1_ST2 = 36,
  TM_T_ST2 = 37,
  TM_A_STM = 38,
  TM_B_STM = 39,
  TM_P1_STM = 40,
  TM_T_STM = 41,
  TM_PER_CLASS = 42
};
__host__ __device__ inline int tm_rr_k128(int buf) {
  return buf == RR_A ? TM_A_K128 : buf == RR_B ? TM_B_K128 : buf == RR_P1 ? TM_P1_K128 : TM_T_K128;
}
__host__ __device__ inline int tm_rr_c128(int buf) {
  return buf == RR_A ? TM_A_C128 : buf == RR_B ? TM_B_C128 : buf == RR_P1 ? TM_P1_C128 : TM_T_C128;
}
__host__ __device__ inline int tm_rr_st2(int buf) {
  return buf == RR_A ? TM_A_ST2 : buf == RR_B ? TM_B_ST2 : buf == RR_P1 ? TM_P1_ST2 : TM_T_ST2;
}
__host__ __device__ inline int tm_rr_stm(int buf) {
  return buf == RR_A ? TM_A_STM : buf == RR_B ? TM_B_STM : buf == RR_P1 ? TM_P1_STM : TM_T_STM;
}
__host__ __device__ inline int tm_rr_st(int buf) {
  return buf == RR_A ? TM_A_ST : buf == RR_B ? TM_B_ST : buf == RR_P1 ? TM_P1_ST : TM_T_ST;
}
__host__ __device__ inline int tm_x(int base, int buf, int part) { return base + buf + 2 * part; }

struct MatDev {
  float* w;
  float* m;
  int64_t rows, cols, ld;
  int32_t r, c;              // Newton-Schulz orientation, r <= c
  int32_t transposed;        // rows > cols: X holds the transpose
  int32_t cls, z;            // shape class and slot within it
  int32_t vec;               // cols % 4 == 0: float4 path
  float beta;
  int32_t nesterov;
  int32_t ns_steps;
  float a, b, c_coef;
  int32_t ex, ea, ec, eb;    // power-of-two scales of stored X, A, C, B'
  int32_t eq;                // Gram-space form: scale of a stored product of p(A) factors
  int32_t gram;              // 1: Newton-Schulz in the Gram-space form (runs of <= 3 iterations)
  int32_t o_buf;             // Y buffer that holds O after the last iteration
  int32_t rule;              // MUONH_RULE_*
  float wd, uscale;          // ordinary-Muon weight decay and update scale
  int32_t et_rows, et_cols;  // elementwise tile grid
  int32_t et_th, et_tw;      // elementwise tile shape: 64 x 64 for tall W, <= 8 x 512 rows otherwise
  int64_t et_begin;          // first elementwise tile
  int32_t fused_dots;        // ||O||^2, <W, O> come from the last APPLY (else from update_dots)
  int32_t ns_tiles_bj;       // APPLY pair tiles per tile row (c_pad / 256)
  int64_t ns_slot_base;      // first (||O||^2, <W, O>) slot: 8 per pair tile (CTA x epilogue warp)
  int32_t ns_slots;
  int32_t warp_tiled;        // momentum/project run in the warp-tiled kernels (partials in part8)
};

struct ClassDev {
  int32_t r_pad, c_pad, count, tm_base;
  void* x[2][2];             // [buf][part]
  void* a[2];                // [part]: A = Y Y^T
  void* c[2];                // C = b I + c A
  void* b[2];                // B' = a I + A C
  void* p1;                  // Gram-space form only: second p(A) buffer
  void* t;                   // Gram-space form only: A P, or a product of p(A) factors
  float* bdiag;              // bf16 operands only: [count][r_pad] fp32 residual of B's stored diagonal
  int64_t x_stride, a_stride;   // elements per matrix
};

struct MatStep {             // per step, copied from the host
  const float* g;
  float lr;
  float pad_;
};

struct MatScal {             // device-resident per-matrix scalars
  float R;
  float xscale;              // 2^ex / (||X|| + eps): scale of the rewrite pass
  float sigma;               // scale the momentum kernel applies when it writes X (0: it does not)
  float kappa;               // first-iteration correction: stored X times kappa = 2^ex X / (||X|| + eps)
  int32_t rewrite;           // 1: write_x rewrites X at the ideal scale this step
  float kw, ko;              // projection: W <- kw W + ko O_stored
  int32_t mode;              // 0 step, 1 re-project only, 2 keep W
  uint32_t flags;
  double wnorm2;             // ||W_t||^2 (measured on the stored W)
  muonh_stats stats;
};

struct TileDesc {
  int32_t mat;
  int16_t bi, bj;
  int32_t nk;                // k-blocks of 64 along K: GRAM (c_pad/64) or APPLY (r_pad/64)
  int32_t nk_sq;             // SQUARE k-blocks (r_pad/64) for GRAM-list tiles
};

struct NsParams {
  const TileDesc* tiles;
  int32_t ntiles;
  int32_t src;               // X buffer read by this phase
  int32_t iter;              // Newton-Schulz iteration of this launch (0: apply kappa)
  const MatScal* scal;
  const CUtensorMap* wmaps;  // per matrix: fp32 W tiles for the last APPLY's <W, O>
  float* part_ns;            // per (pair tile, CTA): ||O||^2 and <W, O> at the stored scale
  const MatDev* mats;
  const ClassDev* classes;
  const CUtensorMap* tmaps;
  int* err;
  // r x r operands of SQUARE / SYMPROD (lhs, rhs, out) and APPLY (lhs), as
  // RrBuf ids, and the RrKind of each (which power-of-two scale it holds)
  int32_t lhs, rhs, out;
  int32_t lhs_kind, rhs_kind, out_kind;
  int32_t apply_kappa;       // APPLY reads the momentum kernel's X: apply kappa
};

// Scale exponent of a stored r x r operand of the given RrKind.
__host__ __device__ inline int rr_exp(const MatDev& md, int kind) {
  return kind == RK_A ? md.ea : kind == RK_P ? md.eb : md.eq;
}

struct EwParams {
  const MatDev* mats;
  const MatStep* step;
  MatScal* scal;
  const ClassDev* classes;
  const int32_t* et_mat;     // elementwise tile -> matrix
  int64_t n_et;
  // the part of the step one launch covers: elementwise tiles [e_first,
  // e_end) and matrices [m_first, m_first + m_count) (one finalize block
  // each), or, with mlist, the matrices mlist[m_first .. m_first + m_count)
  int64_t e_first, e_end;
  int32_t m_first, m_count;
  const int32_t* mlist;
  float* part;               // per-tile partials
  float* part8;              // warp-tiled kernels: one partial per (tile, warp), 8 per tile
  double* part64;
  const float* part_ns;      // partials of the fused last APPLY (MatDev::fused_dots)
  int32_t n;
  float eps;
  int32_t prec;
  muonh_stats* stats_out;
  const int* err;
  int* any_rewrite;          // this matrix group: set by finalize_input when a matrix needs write_x,
                             // cleared by finalize_step
};

// Matrix of finalize block `b` of a launch.
__device__ __forceinline__ int ew_matrix(const EwParams& p, int b) {
  return p.mlist ? p.mlist[p.m_first + b] : p.m_first + b;
}

// -------------------------------------------------------------- PTX helpers
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t globaltimer() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Wait for the phase with the given parity; gives up after limit_ns (every
// kernel uses kWaitLimitNs) or when another role already recorded an error.
// Returns false on give-up, after recording the error in *err.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, int* err,
                                          uint64_t limit_ns = kWaitLimitNs) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer();
  for (uint32_t spin = 1;; ++spin) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((spin & 255u) == 0u) {
      if (*reinterpret_cast<volatile int*>(err) != 0) return false;
      if (globaltimer() - t0 > limit_ns) {
        atomicOr(err, 1);
        return false;
      }
    }
  }
}

__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* map, uint64_t* bar, int x, int y,
                                            int z) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(x), "r"(y), "r"(z)
      : "memory");
}

// TMA store of a shared-memory box into a tiled tensor (bulk-group completion).
__device__ __forceinline__ void tma_store_3d(const CUtensorMap* map, const void* src, int x, int y, int z) {
  asm volatile("cp.async.bulk.tensor.3d.global.shared::cta.bulk_group [%0, {%2, %3, %4}], [%1];" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(smem_u32(src)), "r"(x), "r"(y), "r"(z)
               : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void bulk_wait_read() {
  asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }
// Make generic-proxy shared-memory writes visible to the async (TMA) proxy.
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, uint64_t* bar, int x, int y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(x), "r"(y)
      : "memory");
}

__device__ __forceinline__ void prefetch_tmap(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

__device__ __forceinline__ void tmem_alloc(uint32_t* slot, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(slot)),
               "r"(ncols)
               : "memory");
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

// D[tmem] (+)= A[smem] * B[smem]^T, kind::f16 (fp16 or bf16 in, fp32 accumulate)
__device__ __forceinline__ void umma_f16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                         uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Arrive on `bar` once all previously issued MMAs of this thread completed.
__device__ __forceinline__ void umma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   smem_u32(bar))
               : "memory");
}

// 32 lanes x 32 consecutive 32-bit columns: thread i gets lane (base+i).
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32]) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]),
        "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]),
        "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]),
        "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

// 16 lanes x 32 consecutive 32-bit columns (.16x256b.x4), the accumulator
// fragment of an m16n8 MMA repeated over four 8-column blocks: thread t
// receives r[4k + 2p + e] = (lane base + t/4 + 8p, column 8k + 2(t%4) + e).
// Completes at the next tmem_wait_ld().
__device__ __forceinline__ void tmem_ld16x32_nowait(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.16x256b.x4.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// Four 8 x 8 16-bit matrices from MMA fragments (thread t: row t/4, columns
// 2(t%4), 2(t%4)+1 of each) to shared memory; thread t gives the address of
// row t%8 of matrix t/8.  The .trans form stores each matrix transposed.
__device__ __forceinline__ void stmatrix_x4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  asm volatile("stmatrix.sync.aligned.m8n8.x4.shared.b16 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b),
               "r"(c), "r"(d)
               : "memory");
}
// Inverse of stmatrix_x4: four 8 x 8 16-bit matrices from shared memory into
// MMA fragments (thread t: row t/4, columns 2(t%4), 2(t%4)+1 of each);
// thread t gives the address of row t%8 of matrix t/8.
__device__ __forceinline__ void ldmatrix_x4(uint32_t addr, uint32_t& a, uint32_t& b, uint32_t& c, uint32_t& d) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(a), "=r"(b), "=r"(c), "=r"(d)
               : "r"(addr)
               : "memory");
}
__device__ __forceinline__ void stmatrix_x4_trans(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  asm volatile("stmatrix.sync.aligned.m8n8.x4.trans.shared.b16 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a),
               "r"(b), "r"(c), "r"(d)
               : "memory");
}

// Inverse of tmem_ld32: thread i writes lane (base+i), 32 consecutive columns.
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const float (&v)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])),
      "r"(__float_as_uint(v[3])), "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])),
      "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7])), "r"(__float_as_uint(v[8])),
      "r"(__float_as_uint(v[9])), "r"(__float_as_uint(v[10])), "r"(__float_as_uint(v[11])),
      "r"(__float_as_uint(v[12])), "r"(__float_as_uint(v[13])), "r"(__float_as_uint(v[14])),
      "r"(__float_as_uint(v[15])), "r"(__float_as_uint(v[16])), "r"(__float_as_uint(v[17])),
      "r"(__float_as_uint(v[18])), "r"(__float_as_uint(v[19])), "r"(__float_as_uint(v[20])),
      "r"(__float_as_uint(v[21])), "r"(__float_as_uint(v[22])), "r"(__float_as_uint(v[23])),
      "r"(__float_as_uint(v[24])), "r"(__float_as_uint(v[25])), "r"(__float_as_uint(v[26])),
      "r"(__float_as_uint(v[27])), "r"(__float_as_uint(v[28])), "r"(__float_as_uint(v[29])),
      "r"(__float_as_uint(v[30])), "r"(__float_as_uint(v[31]))
      : "memory");
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// Shared-memory matrix descriptor, 128-byte swizzle, sm_100 version field.
__device__ __forceinline__ uint64_t sdesc_sw128(uint32_t saddr, uint32_t lbo_bytes, uint32_t sbo_bytes) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((saddr >> 4) & 0x3FFFu);
  d |= static_cast<uint64_t>((lbo_bytes >> 4) & 0x3FFFu) << 16;
  d |= static_cast<uint64_t>((sbo_bytes >> 4) & 0x3FFFu) << 32;
  d |= static_cast<uint64_t>(1) << 46;   // descriptor version (sm_100)
  d |= static_cast<uint64_t>(2) << 61;   // SWIZZLE_128B
  return d;
}

// Instruction descriptor, kind::f16: D fp32, A K-major, B K- or MN-major.
__host__ __device__ constexpr uint32_t idesc_f16(int m, int n, int ab_bf16, int b_mn_major) {
  return (1u << 4) | (static_cast<uint32_t>(ab_bf16) << 7) | (static_cast<uint32_t>(ab_bf16) << 10) |
         (static_cast<uint32_t>(b_mn_major) << 16) | (static_cast<uint32_t>(n >> 3) << 17) |
         (static_cast<uint32_t>(m >> 4) << 24);
}

// Message returned by muonh_last_error() on the calling thread.
void set_error_message(const char* msg);

// ------------------------------------------------- CTA-pair (cluster) helpers
__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
  asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// Address of the same shared-memory location in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t map_shared_rank(const void* p, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(smem_u32(p)), "r"(rank));
  return r;
}

__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}

// TMA load into this CTA's shared memory that signals the pair leader's mbarrier.
// 4-D tiled load for a CTA pair (see tma_load_3d_pair).
__device__ __forceinline__ void tma_load_4d_pair(void* dst, const CUtensorMap* map, uint32_t bar_cluster, int x,
                                                 int y, int z, int w) {
  asm volatile(
      "cp.async.bulk.tensor.4d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5, %6}], [%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar_cluster), "r"(x), "r"(y), "r"(z), "r"(w)
      : "memory");
}

__device__ __forceinline__ void tma_load_3d_pair(void* dst, const CUtensorMap* map, uint32_t bar_cluster, int x,
                                                 int y, int z) {
  asm volatile(
      "cp.async.bulk.tensor.3d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar_cluster), "r"(x), "r"(y), "r"(z)
      : "memory");
}

__device__ __forceinline__ void tmem_alloc_pair(uint32_t* slot, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(slot)),
               "r"(ncols)
               : "memory");
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

// D[tmem of both CTAs] (+)= A * B^T with M = 256 split across the pair.
__device__ __forceinline__ void umma_f16_pair(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                              uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Arrive on `bar` (same offset) in both CTAs of the pair once the leader's MMAs completed.
__device__ __forceinline__ void umma_commit_pair(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(
          smem_u32(bar)),
      "h"(static_cast<uint16_t>(0x3))
      : "memory");
}

// --------------------------------------------------------- launch helpers
cudaError_t launch_ns_gemm(int mode, int prec, const NsParams& p, int grid, cudaStream_t s);
cudaError_t launch_ns_gemm_pair(int mode, int prec, const NsParams& p, int pairs, cudaStream_t s);
size_t ns_gemm_smem_bytes(int prec);
cudaError_t ns_gemm_set_attributes();

cudaError_t launch_init_norm(const EwParams& p, int grid, cudaStream_t s);
cudaError_t launch_finalize_init(const EwParams& p, cudaStream_t s);
cudaError_t launch_momentum_norm(const EwParams& p, int grid, cudaStream_t s);
cudaError_t launch_finalize_input(const EwParams& p, cudaStream_t s);
cudaError_t launch_write_x(const EwParams& p, int grid, cudaStream_t s);
cudaError_t launch_update_dots(const EwParams& p, int grid, cudaStream_t s);
cudaError_t launch_finalize_update(const EwParams& p, cudaStream_t s);
cudaError_t launch_project(const EwParams& p, int grid, cudaStream_t s);
cudaError_t launch_finalize_step(const EwParams& p, cudaStream_t s);
cudaError_t launch_export_update(const EwParams& p, int mat, float* dst, int64_t ld, cudaStream_t s);
cudaError_t launch_wait_probe(int* err, uint64_t limit_ns, cudaStream_t s);
int ew_warp_blocks_per_sm(int kind);
cudaError_t launch_momentum_warp(const EwParams& p, bool tall, int grid, cudaStream_t s);
cudaError_t launch_project_warp(const EwParams& p, bool tall, int grid, cudaStream_t s);
constexpr int kStreamSlots = 8;      // partial slots per tile in EwParams::part8

}  // namespace muonh
