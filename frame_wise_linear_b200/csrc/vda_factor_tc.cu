// Factor step on tcgen05 tensor cores (bf16 path, d = 128): M_t = lambda A_t^{-1}.
//
// "VDN-MiniMax-H3" (aiezz.com), section 03, Video Delta Attention item: each
// frame's state comes from a joint solve of the normal equations; the scan
// uses S_t = M_t (S_{t-1} + B_t / lambda) with M_t = lambda A_t^{-1}.
//
// Method: the sweep operator (vda_sweep.cuh) taken 8 pivots at a time.  For a
// pivot block K with P = A_KK = L L^T and X = A[:, K],
//     X~ = X with X~_K = P - I,   Y = X~ L^{-T},   A <- A - Y Y^T
// (= A - X~ P^{-1} X~^T) leaves the swept block row and column K in place; the
// only missing piece, -2 on the swept diagonal, commutes with later blocks and
// is applied once at the end: after all 16 blocks, -A^{-1} = A - 2I, so
// M = lambda (2I - A).  The Cholesky form keeps the float32 error of the
// blocked update at the level of the one-pivot-at-a-time sweep; an explicit
// P^{-1} would not (P itself can be ill-conditioned).
//
// Layout: one CTA of 4 warps per slot; A lives in TMEM as a 128 x 128 float32
// accumulator (lane i = row i).  Per block: each thread reads its row's 8
// pivot columns from TMEM; the 8 rows of P publish them in shared memory and
// every thread factors P in registers (rsqrt, no divides: a short dependency
// chain instead of a one-warp Cholesky that the other warps would wait for);
// each thread solves for its row of Y; Y goes to shared
// memory as tf32 hi + lo (both rounded to nearest, about 2^-22 together); one
// thread issues the symmetric rank-8 update as three kind::tf32 MMAs (the
// hi/lo products of Y Y^T above float32 rounding, A negated).  Up to 4 CTAs
// share an SM (128 TMEM columns each).  M is written as bf16 hi/lo in the
// scan's MMA operand layout.  A non-positive or non-finite pivot sets the
// NOT_SPD bit; every wait is bounded.
#include "sm100.cuh"
#include "vda_internal.cuh"

namespace vda {
namespace {

using namespace sm100;

constexpr int kThreads = 128;
constexpr uint32_t kTmemCols = 128;
constexpr int kOp = 128 * 8 * 4;              // one operand: 128 rows x 8 tf32 (4 KB)
constexpr uint32_t kIdesc = idesc_tf32_f32(128, 128, /*negate A*/ true);

struct Shared {
  uint64_t mma_done;     // one phase per step: the step's update has completed
  uint64_t final_done;   // every MMA of the CTA has completed
  uint32_t tmem_base;
  int bad;
  int abort;
};

__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
  __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&v);
}

// Row i, K-chunk c (4 tf32 values) of a K-major, non-swizzled operand: 8-row
// core matrices of 128 bytes (SBO = 128), the two K-chunks 2 KB apart (LBO).
__device__ __forceinline__ void store_op(uint8_t* op, int i, const float (&v)[8]) {
  *reinterpret_cast<float4*>(op + i * 16) = make_float4(v[0], v[1], v[2], v[3]);
  *reinterpret_cast<float4*>(op + 2048 + i * 16) = make_float4(v[4], v[5], v[6], v[7]);
}

__global__ void __launch_bounds__(kThreads) factor_tc_kernel(float* __restrict__ Mreg, float lam,
                                                             unsigned* __restrict__ err) {
  __shared__ __align__(1024) uint8_t ops[2 * kOp];   // Y hi | Y lo
  __shared__ __align__(16) float psm[8][8];           // the pivot block P of this step
  __shared__ Shared sh;

  const int i = threadIdx.x;            // row of A = TMEM lane
  const int warp = i / 32, lane = i % 32;
  float* A = Mreg + (size_t)blockIdx.x * 128 * 128;

  if (i == 0) {
    mbar_init(&sh.mma_done, 1);
    mbar_init(&sh.final_done, 1);
    sh.bad = 0;
    sh.abort = 0;
    fence_barrier_init();
  }
  if (warp == 0) {
    tmem_alloc(&sh.tmem_base, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sh.tmem_base;
  const uint32_t trow = tmem + ((uint32_t)(warp * 32) << 16);

  // Row i of A into TMEM lane i.
  {
    const float4* src = reinterpret_cast<const float4*>(A + (size_t)i * 128);
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      uint32_t r[32];
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        const float4 v = src[c * 8 + q];
        r[4 * q] = __float_as_uint(v.x);
        r[4 * q + 1] = __float_as_uint(v.y);
        r[4 * q + 2] = __float_as_uint(v.z);
        r[4 * q + 3] = __float_as_uint(v.w);
      }
      tmem_st_32x32b_x32(trow + c * 32, r);
    }
    tmem_st_wait();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();

  int steps_issued = 0;
#pragma unroll 1
  for (int K = 0; K < 16; ++K) {
    if (K > 0) {
      if (!mbar_wait(&sh.mma_done, (K - 1) & 1)) *reinterpret_cast<volatile int*>(&sh.abort) = 1;
      __syncthreads();
      if (*reinterpret_cast<volatile int*>(&sh.abort)) break;   // the same for every thread
      tc_fence_after();
    }
    float x[8];
    {
      uint32_t r[8];
      tmem_ld_32x32b_x8(trow + 8 * K, r);
      tmem_ld_wait();
#pragma unroll
      for (int j = 0; j < 8; ++j) x[j] = __uint_as_float(r[j]);
    }
    // ---- P = L L^T.  The 8 rows of the pivot block publish their pivot
    // columns; every thread then factors P itself, in registers (rsqrt, no
    // divides; the same operations in the same order, so every copy is
    // identical).  A short dependency chain, and no warp waits for another.
    if ((i >> 3) == K) {
      *reinterpret_cast<float4*>(&psm[i & 7][0]) = make_float4(x[0], x[1], x[2], x[3]);
      *reinterpret_cast<float4*>(&psm[i & 7][4]) = make_float4(x[4], x[5], x[6], x[7]);
    }
    __syncthreads();
    float l[8][8];     // lower triangle: P, then L
    float dinv[8];     // 1 / L_jj
#pragma unroll
    for (int r = 0; r < 8; ++r) {
#pragma unroll
      for (int c = 0; c <= r; ++c) l[r][c] = psm[r][c];
    }
    {
      bool badp = false;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const float piv = l[j][j];
        badp |= !(piv > 0.f) || !isfinite(piv);
        const float rs = rsqrtf(piv);
        dinv[j] = rs;
#pragma unroll
        for (int r = j + 1; r < 8; ++r) l[r][j] *= rs;
#pragma unroll
        for (int r = j + 1; r < 8; ++r) {
#pragma unroll
          for (int c = j + 1; c <= r; ++c) l[r][c] = fmaf(-l[r][j], l[c][j], l[r][c]);
        }
      }
      if (i == 0 && badp) sh.bad = 1;
    }
    // ---- X~ (row i) and Y = X~ L^{-T}: forward substitution L y = x~.
    if ((i >> 3) == K) {
#pragma unroll
      for (int j = 0; j < 8; ++j) x[j] -= (j == (i & 7)) ? 1.f : 0.f;   // static indices only
    }
    float y[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      float acc = x[j];
#pragma unroll
      for (int m = 0; m < j; ++m) acc = fmaf(-l[j][m], y[m], acc);
      y[j] = acc * dinv[j];
    }
    // ---- tf32 hi + lo operand (row i)
    {
      float yh[8], yl[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        yh[j] = to_tf32(y[j]);
        yl[j] = to_tf32(y[j] - yh[j]);
      }
      store_op(ops + 0 * kOp, i, yh);
      store_op(ops + 1 * kOp, i, yl);
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    if (i == 0) {
      tc_fence_after();
      // A -= Y Y^T: Y is the A operand (M x K) and, read K-major from the same
      // rows, the B operand (K x N).  Three tf32 passes: hi hi, hi lo, lo hi;
      // the lo lo product is below float32 rounding of the update.
      const uint32_t opaddr = smem_u32(ops);
      const uint64_t yhi = smem_desc(opaddr + 0 * kOp, 2048, 128, kSwizzleNone);
      const uint64_t ylo = smem_desc(opaddr + 1 * kOp, 2048, 128, kSwizzleNone);
      mma_tf32_ss(tmem, yhi, yhi, kIdesc, 1u);
      mma_tf32_ss(tmem, yhi, ylo, kIdesc, 1u);
      mma_tf32_ss(tmem, ylo, yhi, kIdesc, 1u);
      mma_commit(&sh.mma_done);
    }
    ++steps_issued;
  }

  // One more commit covers every MMA issued; wait for it (bounded), also on
  // the error path, so no MMA still runs when TMEM is read or released.
  if (i == 0) mma_commit(&sh.final_done);
  bool ok = steps_issued > 0 && mbar_wait(&sh.final_done, 0);
  if (!ok) *reinterpret_cast<volatile int*>(&sh.abort) = 1;
  tc_fence_after();
  __syncthreads();
  ok = !*reinterpret_cast<volatile int*>(&sh.abort);
  if (i == 0 && !ok) atomicOr(err, kDevErrTimeout);
  if (i == 0 && sh.bad) atomicOr(err, kDevErrNotSpd);
  // M = lambda (2I - A), row i, as bf16 hi/lo (K-major, swizzled).
  if (ok) {
    uint8_t* hi = reinterpret_cast<uint8_t*>(A);
    uint8_t* lo = hi + 32768;
#pragma unroll 1
    for (int c = 0; c < 4; ++c) {
      uint32_t r[32];
      tmem_ld_32x32b_x32(trow + c * 32, r);
      tmem_ld_wait();
#pragma unroll
      for (int q = 0; q < 4; ++q) {       // 8 columns per 16-byte chunk
        float h[8], l[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const int col = c * 32 + q * 8 + e;
          const float m = lam * ((col == i ? 2.f : 0.f) - __uint_as_float(r[q * 8 + e]));
          h[e] = __bfloat162float(__float2bfloat16_rn(m));
          l[e] = m - h[e];
        }
        const int chunk = c * 4 + q;       // 0..15
        const uint32_t off = (chunk / 8) * 16384u + sw128(i, chunk % 8);
        *reinterpret_cast<uint4*>(hi + off) =
            make_uint4(pack_bf16(h[0], h[1]), pack_bf16(h[2], h[3]), pack_bf16(h[4], h[5]), pack_bf16(h[6], h[7]));
        *reinterpret_cast<uint4*>(lo + off) =
            make_uint4(pack_bf16(l[0], l[1]), pack_bf16(l[2], l[3]), pack_bf16(l[4], l[5]), pack_bf16(l[6], l[7]));
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tmem, kTmemCols);
}

}  // namespace

cudaError_t launch_factor_tc(const vda_problem& p, float* M, unsigned* err, cudaStream_t st) {
  if (p.d_k != 128) return cudaErrorInvalidValue;
  const unsigned slots = (unsigned)(p.B * p.H * (p.T + 1));
  // Unused dynamic shared memory that caps residency at 4 CTAs per SM, the
  // number whose 128-column TMEM allocations fit (a fifth would wait in
  // alloc): with 8.5 KB static and 1 KB reserved per CTA, 4 x 53.5 KB fit in
  // the SM's 228 KB and 5 do not.
  const int pad = 44 * 1024;
  cudaError_t e = cudaFuncSetAttribute(factor_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, pad);
  if (e != cudaSuccess) return e;
  factor_tc_kernel<<<slots, kThreads, pad, st>>>(M, p.lambda, err);
  return cudaGetLastError();
}

}  // namespace vda
