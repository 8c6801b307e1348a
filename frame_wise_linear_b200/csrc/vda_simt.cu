// Float32 SIMT kernels for every step of VDA forward.
//
// These serve float32 inputs (any d_k, d_v multiple of 16 up to 128), where
// the result must hold float32 accuracy end to end.  Steps, per (b, h), besides
// the factor step (vda_factor.cu, shared with the bf16 path):
//   gram    : A_t = K_t^T K_t + lambda I, B_t = K_t^T V_t (frames and text)
//   scan    : S^f_t = M_t (S^f_{t-1} + B_t / lambda) forward and
//             S^b_t = M_t (S^b_{t+1} + B_t / lambda) backward, with
//             M_t = lambda A_t^{-1} from the factor step (vda_factor.cu); both
//             start from S_0 = M_0 (B_txt / lambda), the text slot
//   readout : O_t = sigmoid(G_t) * (Q_t (S^f_t + S^b_t))
// The equations follow "VDN-MiniMax-H3" (aiezz.com) section 03, items Video
// Delta Attention, text dual-branch injection and gate fusion.
#include "vda_internal.cuh"

namespace vda {
namespace {

__device__ __forceinline__ float ld_in(const float* p) { return __ldg(p); }
__device__ __forceinline__ float ld_in(const __nv_bfloat16* p) { return __bfloat162float(*p); }
__device__ __forceinline__ void st_out(float* p, float v) { *p = v; }
__device__ __forceinline__ void st_out(__nv_bfloat16* p, float v) { *p = __float2bfloat16_rn(v); }

constexpr int kThreads = 256;

// ---------------------------------------------------------------------------
// gram: D = K^T [K | V] for one slot, tiles of 64 x 64 outputs, 32 tokens per
// stage.  Thread (ty, tx) owns rows ty + 16a and columns tx + 16b.
// ---------------------------------------------------------------------------
template <typename TIn>
__global__ void __launch_bounds__(kThreads) gram_simt_kernel(
    const TIn* __restrict__ K, const TIn* __restrict__ V, const TIn* __restrict__ Kt,
    const TIn* __restrict__ Vt, float* __restrict__ A, float* __restrict__ Bm, int T, int n,
    int n_txt, int dk, int dv, float lam) {
  __shared__ float sK[32][65];
  __shared__ float sX[32][65];
  const int slot = blockIdx.y;
  const int bh = slot / (T + 1);
  const int t = slot % (T + 1);
  const int ncol = dk + dv;
  const int tiles_j = (ncol + 63) / 64;
  const int i0 = (blockIdx.x / tiles_j) * 64;
  const int j0 = (blockIdx.x % tiles_j) * 64;
  const TIn* Kp;
  const TIn* Vp;
  int rows;
  if (t == 0) {
    rows = n_txt;
    Kp = Kt + (size_t)bh * n_txt * dk;
    Vp = Vt + (size_t)bh * n_txt * dv;
  } else {
    rows = n;
    Kp = K + ((size_t)bh * T + (t - 1)) * n * dk;
    Vp = V + ((size_t)bh * T + (t - 1)) * n * dv;
  }
  const int tid = threadIdx.x, tx = tid % 16, ty = tid / 16;
  float acc[4][4];
#pragma unroll
  for (int a = 0; a < 4; ++a)
#pragma unroll
    for (int b = 0; b < 4; ++b) acc[a][b] = 0.f;

  for (int r0 = 0; r0 < rows; r0 += 32) {
    for (int e = tid; e < 32 * 64; e += kThreads) {
      const int r = e / 64, f = e % 64;
      const int row = r0 + r;
      const int fi = i0 + f, fj = j0 + f;
      float kv = 0.f, xv = 0.f;
      if (row < rows) {
        if (fi < dk) kv = ld_in(Kp + (size_t)row * dk + fi);
        if (fj < dk) xv = ld_in(Kp + (size_t)row * dk + fj);
        else if (fj < ncol) xv = ld_in(Vp + (size_t)row * dv + (fj - dk));
      }
      sK[r][f] = kv;
      sX[r][f] = xv;
    }
    __syncthreads();
#pragma unroll 8
    for (int k = 0; k < 32; ++k) {
      float a[4], x[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        a[q] = sK[k][ty + 16 * q];
        x[q] = sX[k][tx + 16 * q];
      }
#pragma unroll
      for (int p = 0; p < 4; ++p)
#pragma unroll
        for (int q = 0; q < 4; ++q) acc[p][q] = fmaf(a[p], x[q], acc[p][q]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int p = 0; p < 4; ++p) {
    const int i = i0 + ty + 16 * p;
    if (i >= dk) continue;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int j = j0 + tx + 16 * q;
      if (j < dk) {
        A[(size_t)slot * dk * dk + (size_t)i * dk + j] = acc[p][q] + (i == j ? lam : 0.f);
      } else if (j < ncol) {
        Bm[(size_t)slot * dk * dv + (size_t)i * dv + (j - dk)] = acc[p][q];
      }
    }
  }
}

// ---------------------------------------------------------------------------
// scan: one block per (column slice of 16, direction, b*h).  Every step is
//     X = S_prev + B_t / lambda,   S = M_t X          (M_t = lambda A_t^{-1})
// which equals A_t^{-1} (lambda S_prev + B_t).  The text slot (t = 0) runs it
// from S_prev = 0 to give S_0.  The recurrence is independent per column of
// S, so slices need no communication.
// ---------------------------------------------------------------------------
constexpr int kScanCols = 16;

__global__ void __launch_bounds__(kThreads) scan_simt_kernel(const float* __restrict__ M,
                                                             const float* __restrict__ Bm,
                                                             float* __restrict__ SF,
                                                             float* __restrict__ SB, int T,
                                                             int dk, int dv, float lam) {
  extern __shared__ float smem[];
  const int ldm = dk + 1;
  float* sM = smem;                          // dk x ldm
  float* sX = smem + dk * ldm;               // dk x kScanCols
  const int c0 = blockIdx.x * kScanCols;
  const int dir = blockIdx.y;
  const int bh = blockIdx.z;
  const int tid = threadIdx.x;
  const size_t base = (size_t)bh * (T + 1);
  float* out = dir == 0 ? SF : SB;
  const float inv_lam = 1.f / lam;
  constexpr int kPer = (128 * kScanCols) / kThreads;  // outputs per thread at most
  float res[kPer];
#pragma unroll
  for (int r = 0; r < kPer; ++r) res[r] = 0.f;       // S_prev = 0 before the text

  for (int step = 0; step <= T; ++step) {
    const int t = step == 0 ? 0 : (dir == 0 ? step : T + 1 - step);
    const float* Mp = M + (base + t) * dk * dk;
    const float* Bp = Bm + (base + t) * dk * dv;
    for (int e = tid; e < dk * dk; e += kThreads) sM[(e / dk) * ldm + (e % dk)] = Mp[e];
#pragma unroll
    for (int r = 0; r < kPer; ++r) {
      const int e = tid + r * kThreads;
      if (e < dk * kScanCols) {
        const int i = e / kScanCols, c = e % kScanCols;
        sX[e] = res[r] + Bp[(size_t)i * dv + c0 + c] * inv_lam;
      }
    }
    __syncthreads();
#pragma unroll
    for (int r = 0; r < kPer; ++r) {
      const int e = tid + r * kThreads;
      if (e < dk * kScanCols) {
        const int i = e / kScanCols, c = e % kScanCols;
        float acc = 0.f;
        for (int k = 0; k < dk; ++k) acc = fmaf(sM[i * ldm + k], sX[k * kScanCols + c], acc);
        res[r] = acc;
      }
    }
    __syncthreads();
    if (step > 0) {
      float* op = out + ((size_t)bh * T + (t - 1)) * dk * dv;
#pragma unroll
      for (int r = 0; r < kPer; ++r) {
        const int e = tid + r * kThreads;
        if (e < dk * kScanCols) {
          const int i = e / kScanCols, c = e % kScanCols;
          op[(size_t)i * dv + c0 + c] = res[r];
        }
      }
    }
  }
}

// ---------------------------------------------------------------------------
// readout: one block per (64-row tile, frame).  S = S^f + S^b staged in
// shared memory; thread (ty, tx) owns rows ty + 16a, columns tx + 16b.
// ---------------------------------------------------------------------------
template <typename TIn>
__global__ void __launch_bounds__(kThreads) readout_simt_kernel(
    const TIn* __restrict__ Q, const TIn* __restrict__ G, const float* __restrict__ SF,
    const float* __restrict__ SB, TIn* __restrict__ O, int n, int dk, int dv) {
  extern __shared__ float smem[];
  const int ldq = dk + 1;
  float* sS = smem;               // dk x dv
  float* sQ = smem + dk * dv;     // 64 x ldq
  const int r0 = blockIdx.x * 64;
  const size_t u = blockIdx.y;    // frame unit (b*H + h)*T + t
  const int tid = threadIdx.x, tx = tid % 16, ty = tid / 16;
  const float* sf = SF + u * dk * dv;
  const float* sb = SB + u * dk * dv;
  for (int e = tid; e < dk * dv; e += kThreads) sS[e] = sf[e] + sb[e];
  const TIn* Qp = Q + u * n * dk;
  for (int e = tid; e < 64 * dk; e += kThreads) {
    const int r = e / dk, k = e % dk;
    sQ[r * ldq + k] = (r0 + r < n) ? ld_in(Qp + (size_t)(r0 + r) * dk + k) : 0.f;
  }
  __syncthreads();
  float acc[4][8];
#pragma unroll
  for (int a = 0; a < 4; ++a)
#pragma unroll
    for (int b = 0; b < 8; ++b) acc[a][b] = 0.f;
  const int nb = dv / 16;
  for (int k = 0; k < dk; ++k) {
    float q[4], s[8];
#pragma unroll
    for (int a = 0; a < 4; ++a) q[a] = sQ[(ty + 16 * a) * ldq + k];
#pragma unroll
    for (int b = 0; b < 8; ++b) s[b] = b < nb ? sS[k * dv + tx + 16 * b] : 0.f;
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
      for (int b = 0; b < 8; ++b) acc[a][b] = fmaf(q[a], s[b], acc[a][b]);
  }
  const TIn* Gp = G + u * n * dv;
  TIn* Op = O + u * n * dv;
#pragma unroll
  for (int a = 0; a < 4; ++a) {
    const int r = r0 + ty + 16 * a;
    if (r >= n) continue;
#pragma unroll
    for (int b = 0; b < 8; ++b) {
      if (b >= nb) continue;
      const int c = tx + 16 * b;
      const float g = ld_in(Gp + (size_t)r * dv + c);
      const float gate = 1.f / (1.f + expf(-g));
      st_out(Op + (size_t)r * dv + c, gate * acc[a][b]);
    }
  }
}

}  // namespace

template <typename TIn>
cudaError_t launch_gram_simt(const vda_problem& p, const TIn* K, const TIn* V, const TIn* Kt,
                             const TIn* Vt, float* A, float* Bm, cudaStream_t st) {
  const int tiles = ((p.d_k + 63) / 64) * ((p.d_k + p.d_v + 63) / 64);
  const unsigned slots = (unsigned)(p.B * p.H * (p.T + 1));
  dim3 grid(tiles, slots);
  gram_simt_kernel<TIn><<<grid, kThreads, 0, st>>>(K, V, Kt, Vt, A, Bm, p.T, p.n, p.n_txt, p.d_k,
                                                   p.d_v, p.lambda);
  return cudaGetLastError();
}

cudaError_t launch_scan_simt(const vda_problem& p, const float* M, const float* Bm, float* SF,
                             float* SB, cudaStream_t st) {
  const size_t smem = ((size_t)p.d_k * (p.d_k + 1) + (size_t)p.d_k * kScanCols) * sizeof(float);
  cudaError_t e = cudaFuncSetAttribute(scan_simt_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid(p.d_v / kScanCols, 2, p.B * p.H);
  scan_simt_kernel<<<grid, kThreads, smem, st>>>(M, Bm, SF, SB, p.T, p.d_k, p.d_v, p.lambda);
  return cudaGetLastError();
}

template <typename TIn>
cudaError_t launch_readout_simt(const vda_problem& p, const TIn* Q, const TIn* G,
                                const float* SF, const float* SB, TIn* O, cudaStream_t st) {
  const size_t smem = ((size_t)p.d_k * p.d_v + 64 * (size_t)(p.d_k + 1)) * sizeof(float);
  cudaError_t e = cudaFuncSetAttribute(readout_simt_kernel<TIn>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid((p.n + 63) / 64, p.B * p.H * p.T);
  readout_simt_kernel<TIn><<<grid, kThreads, smem, st>>>(Q, G, SF, SB, O, p.n, p.d_k, p.d_v);
  return cudaGetLastError();
}

template cudaError_t launch_gram_simt<float>(const vda_problem&, const float*, const float*,
                                             const float*, const float*, float*, float*,
                                             cudaStream_t);
template cudaError_t launch_gram_simt<__nv_bfloat16>(const vda_problem&, const __nv_bfloat16*,
                                                     const __nv_bfloat16*, const __nv_bfloat16*,
                                                     const __nv_bfloat16*, float*, float*,
                                                     cudaStream_t);
template cudaError_t launch_readout_simt<float>(const vda_problem&, const float*, const float*,
                                                const float*, const float*, float*, cudaStream_t);
template cudaError_t launch_readout_simt<__nv_bfloat16>(const vda_problem&, const __nv_bfloat16*,
                                                        const __nv_bfloat16*, const float*,
                                                        const float*, __nv_bfloat16*,
                                                        cudaStream_t);

}  // namespace vda
