// Internal declarations shared by the kernels and the host API of libvda.so.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "vda.h"

namespace vda {

// Bits of the device error word (first 4 bytes of the workspace).
enum : unsigned {
  kDevErrNotSpd = 1u,    // a Cholesky pivot was <= 0 or not finite
  kDevErrTimeout = 2u,   // a bounded wait gave up
};

// Workspace carve-up.  Slots: one per (b, h, t) with t = 0 for the text and
// t = 1..T for the frames, slot = (b * H + h) * (T + 1) + t.
//   err   : 256 bytes, the error word and reserved space
//   M     : per slot, d_k x d_k float  (Gram A_t, then M_t = lambda A_t^{-1})
//   C     : per slot, d_k x d_v float  (B_t = K_t^T V_t)
//   SF,SB : per frame (b, h, t), d_k x d_v float
struct Layout {
  size_t err, M, C, SF, SB, total;
};

inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

inline Layout make_layout(const vda_problem& p) {
  const size_t slots = (size_t)p.B * p.H * (p.T + 1);
  const size_t frames = (size_t)p.B * p.H * p.T;
  Layout L;
  size_t off = 0;
  L.err = off;  off += 256;
  L.M = off;    off = align_up(off + slots * p.d_k * p.d_k * sizeof(float), 256);
  L.C = off;    off = align_up(off + slots * p.d_k * p.d_v * sizeof(float), 256);
  // The states for the readout: float32 on the float32 path; bfloat16 (the
  // readout's MMA operand) on the tensor-core paths (bfloat16 and e4m3 inputs).
  const size_t se = p.dtype != VDA_DTYPE_F32 ? 2 : sizeof(float);
  L.SF = off;   off = align_up(off + frames * p.d_k * p.d_v * se, 256);
  L.SB = off;   off = align_up(off + frames * p.d_k * p.d_v * se, 256);
  L.total = off;
  return L;
}

// Launchers of the float32 SIMT path (vda_simt.cu).  All return the launch
// error (cudaSuccess when enqueued).
template <typename TIn>
cudaError_t launch_gram_simt(const vda_problem& p, const TIn* K, const TIn* V, const TIn* Kt,
                             const TIn* Vt, float* A, float* Bm, cudaStream_t st);
cudaError_t launch_scan_simt(const vda_problem& p, const float* M, const float* Bm, float* SF,
                             float* SB, cudaStream_t st);
template <typename TIn>
cudaError_t launch_readout_simt(const vda_problem& p, const TIn* Q, const TIn* G,
                                const float* SF, const float* SB, TIn* O, cudaStream_t st);

// Factor step of the float32 path (vda_factor.cu): overwrites each slot's A_t
// in M with M_t = lambda A_t^{-1}, float32 row-major.
cudaError_t launch_factor(const vda_problem& p, float* M, unsigned* err, cudaStream_t st);

// Tensor-core scan (vda_scan_tc.cu): bf16 path, d_k = d_v = 128; M in the
// split layout above, B_t float32 in the C region.
// S^f, S^b go to SFb, SBb as bfloat16 ([frames][d_k][d_v], the readout's
// operand); also as float32 to SF, SB when both are non-null.
// b_frames: Bm is [frames][128][128] (no text slots) and the text step adds
// nothing, the form of the backward's adjoint scans.
cudaError_t launch_scan_tc(const vda_problem& p, const float* M, const float* Bm, __nv_bfloat16* SFb,
                           __nv_bfloat16* SBb, float* SF, float* SB, unsigned* err, cudaStream_t st,
                           bool b_frames = false);

// Gram and factor in one kernel (vda_gramfactor_tc.cu): bf16 or e4m3 inputs
// (p.dtype), d_k = d_v = 128.  Writes each slot's M_t into M as bf16 hi and lo halves
// (32 KB each) of the K-major, 128-byte-swizzled image of the scan's MMA A
// operand, and B_t into Bm; A_t stays in TMEM.
cudaError_t launch_gramfactor_tc(const vda_problem& p, const void* K, const void* V, const void* Kt, const void* Vt,
                                 float* M, float* Bm, unsigned* err, cudaStream_t st);

// Tensor-core readout (vda_readout_tc.cu): bf16 or e4m3 Q, G (p.dtype), bf16
// O, d_k = d_v = 128.  SF, SB: the bfloat16 states written by launch_scan_tc.
cudaError_t launch_readout_tc(const vda_problem& p, const void* Q, const void* G, const __nv_bfloat16* SF,
                              const __nv_bfloat16* SB, __nv_bfloat16* O, unsigned* err, cudaStream_t st);

// Backward of the gated readout (vda_readout_bwd_tc.cu): bf16 Q, G, dO and
// S = S^f + S^b ([frames][128][128]); writes dQ and dG (bf16, the tokens'
// layout) and E = Q^T dP (float32, [frames][128][128]).
cudaError_t launch_readout_bwd_tc(const vda_problem& p, const __nv_bfloat16* Q, const __nv_bfloat16* G,
                                  const __nv_bfloat16* dO, const __nv_bfloat16* S, __nv_bfloat16* dQ,
                                  __nv_bfloat16* dG, float* E, unsigned* err, cudaStream_t st);

// Backward of the Gram products (vda_gram_bwd_tc.cu): dK = K W1 + V dB^T and
// dV = K dB per frame (W: [frames][256][128] bf16, W1 rows then dB rows) and
// per head for the text (Wt: [heads][256][128]; skipped when n_txt == 0).
cudaError_t launch_gram_bwd_tc(const vda_problem& p, const __nv_bfloat16* K, const __nv_bfloat16* V,
                               const __nv_bfloat16* W, const __nv_bfloat16* Kt, const __nv_bfloat16* Vt,
                               const __nv_bfloat16* Wt, __nv_bfloat16* dK, __nv_bfloat16* dV, __nv_bfloat16* dKt,
                               __nv_bfloat16* dVt, unsigned* err, cudaStream_t st);

// The backward's per-frame and per-text operands (vda_bwd_operands_tc.cu):
// from the bf16 adjoints Gf, Gb and states S^f, S^b ([frames][128][128]),
// W = [frames][256][128] bf16, W1 = -(Gf S^f^T + S^f Gf^T + Gb S^b^T + S^b
// Gb^T) rows then dB = Gf + Gb rows; and, when n_txt > 0, Wt = [heads][256]
// [128] bf16 for the text from M_0 (the M image of slot 0), B_0 and X_0 =
// Gf_1 + Gb_T.
cudaError_t launch_bwd_operands_tc(const vda_problem& p, const __nv_bfloat16* Gf, const __nv_bfloat16* Gb,
                                   const __nv_bfloat16* SF, const __nv_bfloat16* SB, const float* M, const float* Bm,
                                   __nv_bfloat16* W, __nv_bfloat16* Wt, unsigned* err, cudaStream_t st);

// Backward (vda_backward.cu): bf16 inputs, d_k = d_v = 128.  Workspace bytes,
// and the whole backward enqueued on `st` (on failure *where names the step);
// from_forward: the workspace holds what a vda_forward call with the same
// problem and inputs left there (M_t, B_t, bf16 states), not recomputed.
size_t backward_workspace_bytes(const vda_problem& p);
cudaError_t run_backward(const vda_problem& p, const __nv_bfloat16* Q, const __nv_bfloat16* K,
                         const __nv_bfloat16* V, const __nv_bfloat16* G, const __nv_bfloat16* Kt,
                         const __nv_bfloat16* Vt, const __nv_bfloat16* dO, __nv_bfloat16* dQ, __nv_bfloat16* dK,
                         __nv_bfloat16* dV, __nv_bfloat16* dG, __nv_bfloat16* dKt, __nv_bfloat16* dVt, char* ws,
                         cudaStream_t st, const char** where, bool from_forward);

// TMA descriptor of a [items][rows][128] bf16 tensor, boxes of 64 features x
// box_rows rows with the 128-byte swizzle (vda_tma.cu).  False on failure.
bool make_bf16_rows_map(CUtensorMap* m, const void* ptr, int rows, int items, int box_rows);
// The same [items][rows][128] bf16 tensor with boxes of box_cols features x
// box_rows rows and the swizzle whose span is one box row (box_cols * 2 bytes:
// 32, 64 or 128) (vda_tma.cu).  False on failure.
bool make_bf16_box_map(CUtensorMap* m, const void* ptr, int rows, int items, int box_cols, int box_rows,
                       int swizzle_bytes);

// TMA descriptor of a [rows][cols] bf16 matrix (row stride cols * 2 bytes, a
// multiple of 16), boxes of 64 columns x box_rows rows with the 128-byte
// swizzle (vda_tma.cu).  False on failure.
bool make_bf16_2d_map(CUtensorMap* m, const void* ptr, long long rows, long long cols, int box_cols, int box_rows);

// The branch merge (vda_merge_tc.cu): Y = O_lin W_lin (+ O_sm W_sm when O_sm
// is not null), bf16 [tokens][K] x [K][D] -> [tokens][D], K a multiple of 64.
cudaError_t launch_merge_tc(long long tokens, int K, int D, const __nv_bfloat16* O_lin, const __nv_bfloat16* W_lin,
                            const __nv_bfloat16* O_sm, const __nv_bfloat16* W_sm, __nv_bfloat16* Y, unsigned* err,
                            cudaStream_t st, int stall = 0);

// The local softmax branch (vda_local_softmax_tc.cu): bf16 Q, K, V, G, O in
// the problem's layout, the text's K_txt, V_txt (skipped when n_txt == 0).
cudaError_t launch_local_softmax_tc(const vda_problem& p, const __nv_bfloat16* Q, const __nv_bfloat16* K,
                                    const __nv_bfloat16* V, const __nv_bfloat16* G, const __nv_bfloat16* Kt,
                                    const __nv_bfloat16* Vt, __nv_bfloat16* O, unsigned* err, cudaStream_t st);

// TMA descriptor of a token tensor (128 features of elem_bytes each: 2 for
// bf16, 1 for e4m3) in either layout: layout 0 [B][H][T][rows][128], layout
// 1 [B][T][rows][H][128] (T = 1 for the text's [B][H][n_txt][128] /
// [B][n_txt][H][128]).  Layout 0 is a 3-D map (c, r, unit); layout 1 has five
// dimensions in increasing stride order, (c, h, r, t, b).  Boxes of one
// box_bytes row per token (by default 128 bytes: 64 bf16 or 128 e4m3
// features) x box_rows tokens of one unit, with the swizzle of that span, so
// a box lands in shared memory the same way in both layouts (vda_tma.cu).
bool make_tok_map(CUtensorMap* m, const void* ptr, int layout, int B, int H, int T, int rows, int box_rows,
                  int elem_bytes = 2, int box_bytes = 128);

// TMA descriptor of a [rows][128] float32 matrix, boxes of 32 columns x
// box_rows rows with the 128-byte swizzle (vda_tma.cu).  False on failure.
bool make_f32_rows_map(CUtensorMap* m, const void* ptr, long long rows, int box_rows);

// Replaces the thread-local message vda_last_error() returns (vda_api.cu).
void set_error_message(const char* msg);

}  // namespace vda
