// VDA backward (bf16 inputs, d_k = d_v = 128): the gradients of O with
// respect to Q, K, V, G, K_txt and V_txt for L = sum(dO * O).
//
// The pages give the forward only; this is its exact derivative (the chain
// rule through "VDN-MiniMax-H3" (aiezz.com) section 03's normal-equation
// solve, text injection and gate, and the bidirectional scan of "VDN-H3"
// (comfyui-wiki.com)).  With S_t = S^f_t + S^b_t and P_t = Q_t S_t:
//   dG_t = dO_t * P_t * s (1 - s),  dP_t = dO_t * s  (s = sigmoid(G_t));
//   dQ_t = dP_t S_t^T;  E_t = Q_t^T dP_t.
//   The forward scan's adjoint, run backward in time, and the backward
//   scan's, run forward in time, have the scan's own form:
//     Gf_t = M_t (Gf_{t+1} + E_t / lambda),   Gb_t = M_t (Gb_{t-1} + E_t / lambda),
//   so the scan kernel computes them (E in place of B; its direction 0
//   gives Gb, its direction 1 gives Gf).
//   dB_t = Gf_t + Gb_t,  dA_t = -(Gf_t S^f_t^T + Gb_t S^b_t^T);
//   text: G_0 = M_0 (Gf_1 + Gb_T), S_0 = M_0 B_0 / lambda, dB_0 = G_0,
//   dA_0 = -G_0 S_0^T;
//   dK = K (dA + dA^T) + V dB^T,  dV = K dB  (frames and text alike).
//
// Steps: the forward's Gram+factor and scan kernels (bf16 states), unless a
// vda_forward call has just left them in the workspace; the
// readout's backward in one tensor-core pass over the tokens (dQ, dG, E);
// the scan kernel once more for both adjoints; the 128 x 128 products as
// plain batched GEMMs in cuBLAS (one call per product over all frames: bf16
// adjoints and states for dA, float32 data on TF32 tensor cores for the
// text's) and element-wise kernels here; then the Gram
// products' backward in one tensor-core pass over the tokens (dK, dV).
#include <cublas_v2.h>

#include <mutex>

#include "sm100.cuh"
#include "vda_internal.cuh"

namespace vda {
namespace {

constexpr int kD = 128;
constexpr size_t kMat = (size_t)kD * kD;   // elements of one 128 x 128 matrix

// S = bf16(S^f + S^b) from the bf16 states, eight elements per thread and
// pass (16-byte accesses).
__global__ void sum_states_kernel(const uint4* __restrict__ SF, const uint4* __restrict__ SB, uint4* __restrict__ S,
                                  size_t count8) {
  for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < count8; i += (size_t)gridDim.x * blockDim.x) {
    const uint4 f = SF[i], b = SB[i];
    const __nv_bfloat162* f2 = reinterpret_cast<const __nv_bfloat162*>(&f);
    const __nv_bfloat162* b2 = reinterpret_cast<const __nv_bfloat162*>(&b);
    uint4 o;
    __nv_bfloat162* o2 = reinterpret_cast<__nv_bfloat162*>(&o);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float2 x = __bfloat1622float2(f2[j]), y = __bfloat1622float2(b2[j]);
      o2[j] = __floats2bfloat162_rn(x.x + y.x, x.y + y.y);
    }
    S[i] = o;
  }
}

// The right-hand operands of the Gram backward, per matrix m: W1 = dA + dA^T
// and dB = Gf + Gb (Gb null: dB = Gf), bf16, row-major, written to
// W + m * 2 * 128^2 (W1) and the 128^2 elements after it (dB).  One CTA of
// 32 x 8 threads per 32 x 32 tile: grid (16, matrices); the transposed tile
// goes through shared memory so every global access is coalesced.
__global__ void operands_kernel(const float* __restrict__ dA, const float* __restrict__ Gf,
                                const float* __restrict__ Gb, __nv_bfloat16* __restrict__ W) {
  __shared__ float tt[32][33];
  const size_t m = blockIdx.y;
  const int r0 = (blockIdx.x / 4) * 32, c0 = (blockIdx.x % 4) * 32;
  const float* a = dA + m * kMat;
  const int tx = threadIdx.x, ty = threadIdx.y;
#pragma unroll
  for (int i = 0; i < 4; ++i) tt[ty + 8 * i][tx] = a[(size_t)(c0 + ty + 8 * i) * kD + r0 + tx];
  __syncthreads();
  __nv_bfloat16* w1 = W + m * 2 * kMat;
  __nv_bfloat16* db = w1 + kMat;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int r = r0 + ty + 8 * i, c = c0 + tx;
    const size_t e = (size_t)r * kD + c;
    w1[e] = __float2bfloat16_rn(a[e] + tt[tx][ty + 8 * i]);
    db[e] = __float2bfloat16_rn(Gb ? Gf[m * kMat + e] + Gb[m * kMat + e] : Gf[m * kMat + e]);
  }
}

// M_0 (fp32, row-major) from the bf16 hi/lo operand image of each head's
// text slot, and X_0 = Gf_1 + Gb_T.  One CTA per head.
__global__ void text_inputs_kernel(const uint8_t* __restrict__ Mimg, const float* __restrict__ Gf,
                                   const float* __restrict__ Gb, float* __restrict__ M0, float* __restrict__ X0,
                                   int T) {
  const int bh = blockIdx.x;
  const uint8_t* img = Mimg + (size_t)bh * (T + 1) * 65536;   // the text slot
  const float* gf1 = Gf + ((size_t)bh * T + 0) * kMat;
  const float* gbT = Gb + ((size_t)bh * T + (T - 1)) * kMat;
  for (int e = threadIdx.x; e < kD * kD; e += blockDim.x) {
    const int r = e / kD, c = e % kD;
    const int chunk = c / 8;
    const uint32_t off = (chunk / 8) * 16384u + sm100::sw128(r, chunk % 8) + (c % 8) * 2;
    const float hi = __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(img + off));
    const float lo = __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(img + 32768 + off));
    M0[(size_t)bh * kMat + e] = hi + lo;
    X0[(size_t)bh * kMat + e] = gf1[e] + gbT[e];
  }
}

// Per device, created on first use and kept until exit: the cuBLAS handle,
// and the side stream (non-blocking) with the fork / join events of the
// text's work.
struct Blas {
  std::mutex mu;
  cublasHandle_t h = nullptr;
  cudaStream_t side = nullptr;
  cudaEvent_t fork = nullptr, join = nullptr;
};
constexpr int kMaxDevices = 64;
Blas g_blas[kMaxDevices];

int grid_for(size_t count) {
  size_t b = (count + 255) / 256;
  return (int)(b > 148 * 16 ? 148 * 16 : (b ? b : 1));
}

// Row-major C[m x n] = op(A) op(B) for a batch, through cuBLAS's column-major
// convention (C^T = op(B)^T op(A)^T).  ta / tb: the row-major operand is used
// transposed.  Types: bf16 operands with float32 accumulation (C bf16 or
// float32), or float32 throughout.
cublasStatus_t gemm_rm(cublasHandle_t h, bool ta, bool tb, int m, int n, int k, float alpha, const void* A,
                       cudaDataType at, int lda, long long sa, const void* B, cudaDataType bt, int ldb,
                       long long sb, float beta, void* C, cudaDataType ct, int ldc, long long sc, int batch,
                       cublasComputeType_t ctype = CUBLAS_COMPUTE_32F) {
  return cublasGemmStridedBatchedEx(h, tb ? CUBLAS_OP_T : CUBLAS_OP_N, ta ? CUBLAS_OP_T : CUBLAS_OP_N, n, m, k,
                                    &alpha, B, bt, ldb, sb, A, at, lda, sa, &beta, C, ct, ldc, sc, batch, ctype,
                                    CUBLAS_GEMM_DEFAULT);
}

struct BwdLayout {
  Layout fwd;
  size_t Sb, E, Gf, Gb, GfB, GbB, dA, W, Wt, M0, X0, G0, S0, dA0, total;
};

// After the forward's regions (whose M_t, B_t and bf16 states a preceding
// vda_forward leaves in place): frame-indexed blocks ([frames][128][128]),
// so each product is one batched call; the text's per-head matrices in
// blocks of their own.
BwdLayout make_bwd_layout(const vda_problem& p) {
  BwdLayout L;
  L.fwd = make_layout(p);
  const size_t bh = (size_t)p.B * p.H, frames = bh * p.T;
  size_t off = L.fwd.total;
  auto take = [&](size_t bytes) { const size_t o = off; off = align_up(off + bytes, 256); return o; };
  L.Sb = take(frames * kMat * 2);
  L.E = take(frames * kMat * 4);
  L.Gf = take(frames * kMat * 4);
  L.Gb = take(frames * kMat * 4);
  L.GfB = take(frames * kMat * 2);        // the adjoints as bf16, the dA products' operands
  L.GbB = take(frames * kMat * 2);
  L.dA = take(frames * kMat * 4);
  L.W = take(frames * 2 * kMat * 2);      // per frame: W1 | dB, bf16
  L.Wt = take(bh * 2 * kMat * 2);         // per head, the text's
  L.M0 = take(bh * kMat * 4);
  L.X0 = take(bh * kMat * 4);
  L.G0 = take(bh * kMat * 4);
  L.S0 = take(bh * kMat * 4);
  L.dA0 = take(bh * kMat * 4);
  L.total = off;
  return L;
}

}  // namespace

size_t backward_workspace_bytes(const vda_problem& p) { return make_bwd_layout(p).total; }

cudaError_t run_backward(const vda_problem& p, const __nv_bfloat16* Q, const __nv_bfloat16* K,
                         const __nv_bfloat16* V, const __nv_bfloat16* G, const __nv_bfloat16* Kt,
                         const __nv_bfloat16* Vt, const __nv_bfloat16* dO, __nv_bfloat16* dQ, __nv_bfloat16* dK,
                         __nv_bfloat16* dV, __nv_bfloat16* dG, __nv_bfloat16* dKt, __nv_bfloat16* dVt, char* ws,
                         cudaStream_t st, const char** where, bool from_forward) {
  const BwdLayout L = make_bwd_layout(p);
  const int BH = p.B * p.H, T = p.T, n = p.n, frames = BH * T;
  const size_t slot_stride = (size_t)(T + 1) * kMat;   // elements between a head's slot blocks
  unsigned* err = reinterpret_cast<unsigned*>(ws + L.fwd.err);
  float* M = reinterpret_cast<float*>(ws + L.fwd.M);
  float* Bm = reinterpret_cast<float*>(ws + L.fwd.C);
  __nv_bfloat16* SFb = reinterpret_cast<__nv_bfloat16*>(ws + L.fwd.SF);
  __nv_bfloat16* SBb = reinterpret_cast<__nv_bfloat16*>(ws + L.fwd.SB);
  __nv_bfloat16* Sb = reinterpret_cast<__nv_bfloat16*>(ws + L.Sb);
  float* E = reinterpret_cast<float*>(ws + L.E);
  float* Gf = reinterpret_cast<float*>(ws + L.Gf);
  float* Gb = reinterpret_cast<float*>(ws + L.Gb);
  __nv_bfloat16* GfB = reinterpret_cast<__nv_bfloat16*>(ws + L.GfB);
  __nv_bfloat16* GbB = reinterpret_cast<__nv_bfloat16*>(ws + L.GbB);
  float* dA = reinterpret_cast<float*>(ws + L.dA);
  __nv_bfloat16* W = reinterpret_cast<__nv_bfloat16*>(ws + L.W);
  __nv_bfloat16* Wt = reinterpret_cast<__nv_bfloat16*>(ws + L.Wt);
  float* M0 = reinterpret_cast<float*>(ws + L.M0);
  float* X0 = reinterpret_cast<float*>(ws + L.X0);
  float* G0 = reinterpret_cast<float*>(ws + L.G0);
  float* S0 = reinterpret_cast<float*>(ws + L.S0);
  float* dA0 = reinterpret_cast<float*>(ws + L.dA0);
  const cudaDataType bf = CUDA_R_16BF, f32 = CUDA_R_32F;
  cudaError_t e;
#define VDA_TRY(expr, what)                 \
  if ((e = (expr)) != cudaSuccess) {        \
    *where = what;                          \
    return e;                               \
  }
#define VDA_BLAS(expr, what)                            \
  if ((expr) != CUBLAS_STATUS_SUCCESS) {                \
    *where = what;                                      \
    return cudaErrorUnknown;                            \
  }

  int dev = 0;
  VDA_TRY(cudaGetDevice(&dev), "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  Blas& bl = g_blas[dev];
  std::lock_guard<std::mutex> lock(bl.mu);
  if (!bl.h) VDA_BLAS(cublasCreate(&bl.h), "cublasCreate");
  if (!bl.side) {
    VDA_TRY(cudaStreamCreateWithFlags(&bl.side, cudaStreamNonBlocking), "side stream");
    VDA_TRY(cudaEventCreateWithFlags(&bl.fork, cudaEventDisableTiming), "fork event");
    VDA_TRY(cudaEventCreateWithFlags(&bl.join, cudaEventDisableTiming), "join event");
  }
  cublasHandle_t h = bl.h;
  VDA_BLAS(cublasSetStream(h, st), "cublasSetStream");
  VDA_BLAS(cublasSetMathMode(h, CUBLAS_DEFAULT_MATH), "cublasSetMathMode");

  // 1. The forward's M_t, B_t and bf16 states: recomputed, or left in the
  //    workspace by the vda_forward call that preceded this one (whose
  //    error bits stay set for vda_sync_status).
  if (!from_forward) {
    VDA_TRY(cudaMemsetAsync(err, 0, 256, st), "clearing the error word");
    VDA_TRY(launch_gramfactor_tc(p, K, V, Kt, Vt, M, Bm, err, st), "gram+factor launch");
    VDA_TRY(launch_scan_tc(p, M, Bm, SFb, SBb, nullptr, nullptr, err, st), "scan launch");
  }

  // 2. The readout's gradients in one pass over the tokens: P = Q S, dP,
  //    dG, dQ = dP S^T and E = Q^T dP (vda_readout_bwd_tc.cu).
  const size_t sc = (size_t)frames * kMat;
  sum_states_kernel<<<grid_for(sc / 8), 256, 0, st>>>(reinterpret_cast<const uint4*>(SFb),
                                                      reinterpret_cast<const uint4*>(SBb),
                                                      reinterpret_cast<uint4*>(Sb), sc / 8);
  VDA_TRY(cudaGetLastError(), "sum_states launch");
  VDA_TRY(launch_readout_bwd_tc(p, Q, G, dO, Sb, dQ, dG, E, err, st), "readout backward launch");

  // 3. The scans' adjoints: the scan kernel with E (frame-indexed, nothing
  //    at the text step) for B; direction 0 gives Gb (forward in time),
  //    direction 1 gives Gf.
  VDA_TRY(launch_scan_tc(p, M, E, GbB, GfB, Gb, Gf, err, st, /*b_frames=*/true), "adjoint scan launch");

  // 4. The text's operands on the side stream (five small launches that
  //    overlap the frames' work below): G_0 = M_0 (Gf_1 + Gb_T),
  //    S_0 = M_0 B_0 / lambda, dA_0 = -G_0 S_0^T (TF32 tensor cores).
  const bool text = p.n_txt > 0;
  if (text) {
    VDA_TRY(cudaEventRecord(bl.fork, st), "fork event");
    VDA_TRY(cudaStreamWaitEvent(bl.side, bl.fork, 0), "fork wait");
    VDA_BLAS(cublasSetStream(h, bl.side), "cublasSetStream");
    VDA_BLAS(cublasSetMathMode(h, CUBLAS_TF32_TENSOR_OP_MATH), "cublasSetMathMode");
    text_inputs_kernel<<<BH, 256, 0, bl.side>>>(reinterpret_cast<const uint8_t*>(M), Gf, Gb, M0, X0, T);
    VDA_TRY(cudaGetLastError(), "text_inputs launch");
    VDA_BLAS(gemm_rm(h, false, false, kD, kD, kD, 1.f, M0, f32, kD, kMat, X0, f32, kD, kMat, 0.f, G0, f32, kD, kMat,
                     BH, CUBLAS_COMPUTE_32F_FAST_TF32), "G_0");
    VDA_BLAS(gemm_rm(h, false, false, kD, kD, kD, 1.f / p.lambda, M0, f32, kD, kMat, Bm, f32, kD,
                     (long long)slot_stride, 0.f, S0, f32, kD, kMat, BH, CUBLAS_COMPUTE_32F_FAST_TF32), "S_0");
    VDA_BLAS(gemm_rm(h, false, true, kD, kD, kD, -1.f, G0, f32, kD, kMat, S0, f32, kD, kMat, 0.f, dA0, f32, kD, kMat,
                     BH, CUBLAS_COMPUTE_32F_FAST_TF32), "dA_0");
    operands_kernel<<<dim3(16, BH), dim3(32, 8), 0, bl.side>>>(dA0, G0, nullptr, Wt);
    VDA_TRY(cudaGetLastError(), "operands launch");
    VDA_TRY(cudaEventRecord(bl.join, bl.side), "join event");
    VDA_BLAS(cublasSetMathMode(h, CUBLAS_DEFAULT_MATH), "cublasSetMathMode");
    VDA_BLAS(cublasSetStream(h, st), "cublasSetStream");
  }

  // 5. dA_t = -(Gf_t S^f_t^T + Gb_t S^b_t^T) from the bf16 adjoints and
  //    states (float32 accumulation), then W1 = dA + dA^T and dB (from the
  //    float32 adjoints).
  VDA_BLAS(gemm_rm(h, false, true, kD, kD, kD, -1.f, GfB, bf, kD, kMat, SFb, bf, kD, kMat, 0.f, dA, f32, kD, kMat,
                   frames), "dA (forward part)");
  VDA_BLAS(gemm_rm(h, false, true, kD, kD, kD, -1.f, GbB, bf, kD, kMat, SBb, bf, kD, kMat, 1.f, dA, f32, kD, kMat,
                   frames), "dA (backward part)");
  operands_kernel<<<dim3(16, frames), dim3(32, 8), 0, st>>>(dA, Gf, Gb, W);
  VDA_TRY(cudaGetLastError(), "operands launch");
  if (text) VDA_TRY(cudaStreamWaitEvent(st, bl.join, 0), "join wait");

  // 6. dK = K W1 + V dB^T, dV = K dB, for the frames and the text, in one
  //    pass over the tokens (vda_gram_bwd_tc.cu).
  VDA_TRY(launch_gram_bwd_tc(p, K, V, W, Kt, Vt, Wt, dK, dV, dKt, dVt, err, st), "gram backward launch");
#undef VDA_TRY
#undef VDA_BLAS
  return cudaSuccess;
}

}  // namespace vda
