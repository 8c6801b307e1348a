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
// vda_forward call has just left them in the workspace; the readout's
// backward in one tensor-core pass over the tokens (dQ, dG, E); the scan
// kernel once more for both adjoints (bf16); the 128 x 128 products per
// frame and the text's small chain in one tensor-core kernel
// (vda_bwd_operands_tc.cu); then the Gram products' backward in one
// tensor-core pass over the tokens (dK, dV).  Six launches (four from the
// forward's state), all on the caller's stream; no library calls.
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

int grid_for(size_t count) {
  size_t b = (count + 255) / 256;
  return (int)(b > 148 * 16 ? 148 * 16 : (b ? b : 1));
}

struct BwdLayout {
  Layout fwd;
  size_t Sb, E, GfB, GbB, W, Wt, total;
};

// After the forward's regions (whose M_t, B_t and bf16 states a preceding
// vda_forward leaves in place): frame-indexed blocks ([frames][128][128]),
// and the text's operand image per head.
BwdLayout make_bwd_layout(const vda_problem& p) {
  BwdLayout L;
  L.fwd = make_layout(p);
  const size_t bh = (size_t)p.B * p.H, frames = bh * p.T;
  size_t off = L.fwd.total;
  auto take = [&](size_t bytes) { const size_t o = off; off = align_up(off + bytes, 256); return o; };
  L.Sb = take(frames * kMat * 2);         // S = S^f + S^b, bf16
  L.E = take(frames * kMat * 4);          // E_t = Q_t^T dP_t, float32
  L.GfB = take(frames * kMat * 2);        // the adjoints, bf16
  L.GbB = take(frames * kMat * 2);
  L.W = take(frames * 2 * kMat * 2);      // per frame: W1 | dB, bf16
  L.Wt = take(bh * 2 * kMat * 2);         // per head, the text's
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
  const int frames = p.B * p.H * p.T;
  unsigned* err = reinterpret_cast<unsigned*>(ws + L.fwd.err);
  float* M = reinterpret_cast<float*>(ws + L.fwd.M);
  float* Bm = reinterpret_cast<float*>(ws + L.fwd.C);
  __nv_bfloat16* SFb = reinterpret_cast<__nv_bfloat16*>(ws + L.fwd.SF);
  __nv_bfloat16* SBb = reinterpret_cast<__nv_bfloat16*>(ws + L.fwd.SB);
  __nv_bfloat16* Sb = reinterpret_cast<__nv_bfloat16*>(ws + L.Sb);
  float* E = reinterpret_cast<float*>(ws + L.E);
  __nv_bfloat16* GfB = reinterpret_cast<__nv_bfloat16*>(ws + L.GfB);
  __nv_bfloat16* GbB = reinterpret_cast<__nv_bfloat16*>(ws + L.GbB);
  __nv_bfloat16* W = reinterpret_cast<__nv_bfloat16*>(ws + L.W);
  __nv_bfloat16* Wt = reinterpret_cast<__nv_bfloat16*>(ws + L.Wt);
  cudaError_t e;
#define VDA_TRY(expr, what)                 \
  if ((e = (expr)) != cudaSuccess) {        \
    *where = what;                          \
    return e;                               \
  }

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
  //    direction 1 gives Gf; bf16, the next step's operands.
  VDA_TRY(launch_scan_tc(p, M, E, GbB, GfB, nullptr, nullptr, err, st, /*b_frames=*/true), "adjoint scan launch");

  // 4. W1 = dA + dA^T and dB per frame, and the text's W1_0 | dB_0 per head
  //    (vda_bwd_operands_tc.cu).
  VDA_TRY(launch_bwd_operands_tc(p, GfB, GbB, SFb, SBb, M, Bm, W, Wt, err, st), "operands launch");

  // 5. dK = K W1 + V dB^T, dV = K dB, for the frames and the text, in one
  //    pass over the tokens (vda_gram_bwd_tc.cu).
  VDA_TRY(launch_gram_bwd_tc(p, K, V, W, Kt, Vt, Wt, dK, dV, dKt, dVt, err, st), "gram backward launch");
#undef VDA_TRY
  return cudaSuccess;
}

}  // namespace vda
