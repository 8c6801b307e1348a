/*
 * vda.h -- C ABI of libvda.so: Video Delta Attention (VDA) forward on B200.
 *
 * What is computed.  VDA is the linear branch of the VDN-H3 hybrid video
 * attention.  The pages describe it in words only:
 *   - "VDN-MiniMax-H3" (aiezz.com), section 03 (technical principles), item
 *     "Video Delta Attention", and the same item in section 技术原理 of
 *     "VDN-MiniMax-H3 OpenVDN 开源的视频生成加速方案" (laicaila.com): the
 *     token-wise delta rule becomes a frame-wise joint solve through the
 *     normal equations; non-expansive; no frame-size scaling.
 *   - same sections, item "text dual-branch injection": the text is written
 *     once, at initialisation, into both directional states.
 *   - same sections, item "gate fusion": a content-dependent sigmoid gate.
 *   - "VDN-H3: ..." (comfyui-wiki.com), section on how Video DeltaNet speeds
 *     up H3: a bidirectional linear branch with a constant-size state.
 * The concrete form this library computes, per (batch b, head h):
 *     A_t = K_t^T K_t + lambda I,   B_t = K_t^T V_t            (t = 1..T)
 *     S_0 = A_txt^{-1} B_txt        (S_0 = 0 when n_txt == 0)
 *     S^f_t = A_t^{-1} (lambda S^f_{t-1} + B_t),  S^f_0 = S_0   (t = 1..T)
 *     S^b_t = A_t^{-1} (lambda S^b_{t+1} + B_t),  S^b_{T+1} = S_0 (t = T..1)
 *     O_t   = sigmoid(G_t) * (Q_t S^f_t + Q_t S^b_t)            (element-wise)
 *
 * Layout.  Every tensor is dense, row-major, contiguous.  With
 * vda_problem.layout = VDA_LAYOUT_BHTND (0, the default):
 *     Q, K : [B, H, T, n, d_k]      V, G, O : [B, H, T, n, d_v]
 *     K_txt: [B, H, n_txt, d_k]     V_txt   : [B, H, n_txt, d_v]
 * With VDA_LAYOUT_BTNHD (1; bfloat16 or e4m3), the token-major layout of a
 * video transformer's attention, heads inside tokens:
 *     Q, K : [B, T*n, H, d_k]       V, G, O : [B, T*n, H, d_v]
 *     K_txt: [B, n_txt, H, d_k]     V_txt   : [B, n_txt, H, d_v]
 * The gradients of vda_backward* take the layout of their inputs.  In both:
 *     S_fwd, S_bwd (states)          : [B, H, T, d_k, d_v], float32
 * Inputs and O share one element type, vda_problem.dtype: float32 or
 * bfloat16; with e4m3 inputs (per-tensor scales) O is bfloat16.  The state
 * recurrence and every accumulation are float32; O is rounded to its type
 * with round-to-nearest-even.  With bfloat16 inputs the
 * readout takes the two states as bfloat16 operands (O = sigmoid(G) *
 * (Q S^f + Q S^b) with S^f, S^b rounded to bfloat16, accumulated in
 * float32); the states returned by vda_forward_states are the float32 ones.
 *
 * Ownership.  The caller owns every buffer.  Device pointers must be CUDA
 * device memory of the current device, 16-byte aligned.  The library
 * allocates nothing and keeps no per-call state between calls; calls on one
 * stream are ordered, calls on different streams must use different
 * workspaces.  Every call that takes a stream only enqueues work on it
 * (asynchronous), except where stated.  `stream` is a cudaStream_t passed as
 * void* (NULL = the legacy default stream).
 *
 * Errors.  Argument errors are found on the host before anything is
 * enqueued and return VDA_ERR_INVALID_ARG / VDA_ERR_UNSUPPORTED /
 * VDA_ERR_WORKSPACE; nothing runs in that case.  A launch failure returns
 * VDA_ERR_CUDA.  Conditions found on the device (a non-positive Cholesky
 * pivot, which exact arithmetic rules out for lambda > 0; a bounded wait
 * that ran out) are written to an error word in the workspace, which every
 * vda_forward* call clears first; vda_sync_status() reads it.  There is no
 * CPU fallback: without a usable device the calls fail.
 */
#ifndef VDA_H_
#define VDA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum vda_status {
  VDA_OK = 0,
  VDA_ERR_INVALID_ARG = 1,  /* bad size, lambda, null or misaligned pointer */
  VDA_ERR_UNSUPPORTED = 2,  /* valid, but outside what the kernels support  */
  VDA_ERR_WORKSPACE = 3,    /* workspace missing, too small or misaligned   */
  VDA_ERR_CUDA = 4,         /* a CUDA runtime call or launch failed         */
  VDA_ERR_NOT_SPD = 5,      /* device: a Cholesky pivot was not positive    */
  VDA_ERR_TIMEOUT = 6       /* device: a bounded wait gave up               */
} vda_status;

/* Element type of the inputs.  VDA_DTYPE_E4M3: Q, K, V, G, K_txt and V_txt
 * are 8-bit floats (OCP E4M3: 1 sign, 4 exponent, 3 mantissa bits, bias 7,
 * largest finite 448, no infinities), each tensor with a per-tensor scale in
 * vda_problem; O is bfloat16.  The forward only. */
typedef enum vda_dtype { VDA_DTYPE_F32 = 0, VDA_DTYPE_BF16 = 1, VDA_DTYPE_E4M3 = 2 } vda_dtype;

typedef enum vda_layout { VDA_LAYOUT_BHTND = 0, VDA_LAYOUT_BTNHD = 1 } vda_layout;

/* Problem sizes.  B, H, T, n >= 1; n_txt >= 0.
 * float32: d_k, d_v multiples of 16 in [16, 128].
 * bfloat16, e4m3: d_k = d_v = 128.
 * lambda: the ridge weight of every frame-wise solve, finite and > 0, one
 * value shared by all batches, heads, frames and the text (the pages name no
 * such parameter; one scalar per call is the plainest reading). */
typedef struct vda_problem {
  int32_t B, H, T, n, n_txt, d_k, d_v;
  int32_t dtype; /* vda_dtype */
  float lambda;
  int32_t layout; /* vda_layout; VDA_LAYOUT_BTNHD needs bfloat16 or e4m3 */
  int32_t test_stall; /* testing hook, VDA_TEST_STALL_*; 0 in normal use */
  /* e4m3 inputs only (ignored otherwise): the value an element stands for is
   * scale times its stored e4m3 value, one scale per tensor (K_txt takes
   * scale_k, V_txt scale_v); each finite and > 0. */
  float scale_q, scale_k, scale_v, scale_g;
} vda_problem;

/* Testing hook for the device timeout path (vda_problem.test_stall).  Every
 * wait inside the tensor-core kernels is bounded (2 s of the GPU's global
 * timer); a wait that runs out sets VDA_ERR_TIMEOUT in the error word and the
 * kernel winds down: its other warps stop at their next decision point, the
 * copies and MMAs it has issued complete, its tensor memory is released, and
 * the kernels after it on the stream still end.  A nonzero test_stall names
 * one wait below; in one CTA of the kernel that holds it (the first, unless
 * the site says otherwise), that wait is made on a barrier nothing ever
 * signals, so it runs out
 * exactly as a wait on a lost signal would.  The call then returns VDA_OK
 * (enqueued), vda_sync_status() reports VDA_ERR_TIMEOUT, and later calls run
 * normally.  A site that the problem's sizes never reach (for example the
 * text chunk when n_txt == 0) leaves the call unchanged.  The sites apply to
 * the bfloat16 path (the float32 path has no bounded waits). */
enum {
  VDA_TEST_STALL_NONE = 0,
  VDA_TEST_STALL_GRAM_STAGE = 1,     /* Gram+factor: the MMA thread's wait for its first token chunk   */
  VDA_TEST_STALL_FACTOR_UPDATE = 2,  /* Gram+factor: factor group 0's wait for its first block update  */
  VDA_TEST_STALL_SERVICE_GRAM = 3,   /* Gram+factor: the service warps' wait for the first Gram chain  */
  VDA_TEST_STALL_SCAN_OPERAND = 4,   /* scan: the MMA thread's wait for the second step's operand      */
  VDA_TEST_STALL_SCAN_PRODUCT = 5,   /* scan: the row warps' wait for the second step's product        */
  VDA_TEST_STALL_READOUT_TILE = 6,   /* readout: the MMA thread's wait for the first Q tile            */
  VDA_TEST_STALL_READOUT_GATE = 7,   /* readout: the epilogue's wait for the second G tile             */
  VDA_TEST_STALL_READOUT_STATE = 8,  /* readout: the state warps' wait for the second frame's states   */
  VDA_TEST_STALL_RBWD_TILE = 9,      /* readout backward: the MMA thread's wait for the first Q tile   */
  VDA_TEST_STALL_RBWD_DQ = 10,       /* readout backward: the epilogue's wait for the first dQ         */
  VDA_TEST_STALL_GBWD_TILE = 11,     /* Gram backward: the MMA thread's wait for the first K, V tile   */
  VDA_TEST_STALL_GBWD_STORE = 12,    /* Gram backward: the epilogue's wait for the second dK, dV       */
  VDA_TEST_STALL_OPERANDS = 13,      /* backward operands: the MMA thread's wait for its first frame,
                                        in the kernel's last CTA (the first may have no frames)       */
  VDA_TEST_STALL_MERGE = 14,         /* vda_merge_project: the MMA thread's wait for its first K block */
  VDA_TEST_STALL_SOFTMAX = 15,       /* vda_local_softmax: the softmax warps' wait for the first scores */
  VDA_TEST_STALL_MAX = 15
};

/* Bytes of device workspace vda_forward needs for `p` (written to *bytes).
 * Host only, enqueues nothing.  Errors: INVALID_ARG / UNSUPPORTED as for
 * vda_forward. */
vda_status vda_workspace_size(const vda_problem* p, size_t* bytes);

/* O = VDA(Q, K, V, G, K_txt, V_txt; lambda), the whole forward (both scan
 * directions and the gated readout), enqueued on `stream`.
 * Q, K, V, G, O: device pointers, layout above, element type p->dtype.
 * K_txt, V_txt: device pointers, or NULL when p->n_txt == 0.
 * workspace: device memory of at least vda_workspace_size() bytes, 256-byte
 * aligned; its contents on entry do not matter and on return are the
 * intermediates plus the error word.  Returns once the work is enqueued. */
vda_status vda_forward(const vda_problem* p, const void* Q, const void* K, const void* V,
                       const void* G, const void* K_txt, const void* V_txt, void* O,
                       void* workspace, size_t workspace_bytes, void* stream);

/* As vda_forward, and also writes the per-frame states S^f_t and S^b_t
 * (float32, [B, H, T, d_k, d_v]) to the device buffers S_fwd, S_bwd.  Used to
 * check the scan stage on its own. */
vda_status vda_forward_states(const vda_problem* p, const void* Q, const void* K, const void* V,
                              const void* G, const void* K_txt, const void* V_txt, void* O,
                              void* workspace, size_t workspace_bytes, void* stream,
                              float* S_fwd, float* S_bwd);

/* As vda_forward, and records CUDA events on `stream` around the stages so
 * a caller can time each kernel on the stream that runs it.  `events` holds
 * `n_events` cudaEvent_t handles (passed as void*), created by the caller;
 * events[0] is recorded before the first kernel and events[i] after stage i
 * (1 = Gram, 2 = factor-and-solve, 3 = scan, 4 = readout).  n_events must be
 * VDA_TIMED_EVENTS; elapsed time between events i-1 and i is stage i.  With
 * bf16 inputs the Gram and the factor run as one kernel: stage 1 times both
 * and events 1 and 2 are recorded back to back (stage 2 is empty). */
#define VDA_TIMED_EVENTS 5
vda_status vda_forward_timed(const vda_problem* p, const void* Q, const void* K, const void* V,
                             const void* G, const void* K_txt, const void* V_txt, void* O,
                             void* workspace, size_t workspace_bytes, void* stream,
                             void* const* events, int n_events);

/* Bytes of device workspace vda_forward_host needs: room for the inputs and
 * O on the device plus vda_workspace_size(). */
vda_status vda_host_workspace_size(const vda_problem* p, size_t* bytes);

/* End-to-end call on HOST buffers: copies the inputs host -> device into the
 * workspace (one cudaMemcpyAsync per tensor), runs vda_forward, copies O
 * device -> host, all on `stream`, then synchronises `stream` and returns the
 * device status (as vda_sync_status).  Host buffers should be pinned
 * (cudaHostAlloc / page-locked) for the copies to be asynchronous.  The same
 * pointer rules hold, with host pointers in place of device ones. */
vda_status vda_forward_host(const vda_problem* p, const void* Q, const void* K, const void* V,
                            const void* G, const void* K_txt, const void* V_txt, void* O,
                            void* workspace, size_t workspace_bytes, void* stream);

/* Forward for callers that cannot allocate device memory.  Some callers own
 * no device allocator of their own or may not call one: code running under a
 * framework whose memory manager owns the whole device (a caching allocator,
 * or a fixed per-process budget that cudaMalloc would overrun), and callers on
 * a latency-critical path, where cudaMalloc/cudaFree would synchronise the
 * device.  They can neither hand vda_forward a workspace nor let the library
 * allocate one.
 * This call computes exactly what vda_forward computes, but its workspace is
 * a scratch array inside the library: a file-scope device array of
 * VDA_NOALLOC_SCRATCH_BYTES (64 MiB) that every GPU which loads the library
 * holds until the process exits.  It allocates nothing: no cudaMalloc, no
 * cudaFree, no allocating library routine.  The caller still owns Q, K, V, G,
 * K_txt, V_txt and O (device pointers, same rules as vda_forward).
 * Limits and caveats:
 *   - problems whose vda_workspace_size() exceeds the scratch are rejected
 *     with VDA_ERR_WORKSPACE before anything is enqueued (for example the
 *     mid workload, 8 heads x 16 frames, fits; 32 heads x 45 frames does not);
 *   - the scratch's device address belongs to the CUDA context current on
 *     the calling thread; the first call in each context (the device's
 *     primary context, one a driver-API caller made current, or the new
 *     primary context after a cudaDeviceReset) looks that address up and
 *     caches it under the context's unique ID; make that first call before
 *     any stream capture;
 *   - every call on a device shares the one scratch, which keeps the last
 *     call's contents (each call clears what must start at zero): calls that
 *     overlap on the GPU, on different streams or from different threads,
 *     race and give wrong results;
 *   - the device error word lives in the scratch, so device-side conditions
 *     (VDA_ERR_NOT_SPD, VDA_ERR_TIMEOUT) are not reported by this call: a
 *     caller that needs them must validate O itself (for example, that it
 *     is finite) or use vda_forward with vda_sync_status; host-side argument
 *     errors are reported, as for vda_forward.
 * The pages describe no such entry point: it has no counterpart there. */
#define VDA_NOALLOC_SCRATCH_BYTES (64u * 1024u * 1024u)
vda_status vda_forward_noalloc(const vda_problem* p, const void* Q, const void* K, const void* V,
                               const void* G, const void* K_txt, const void* V_txt, void* O,
                               void* stream);

/* Backward of vda_forward: the gradients of L = sum(dO * O) with respect to
 * Q, K, V, G, K_txt and V_txt (lambda held fixed).  The pages give the
 * forward only; this is its exact derivative (the chain rule through the
 * gate, the readout, both scans, the text state and the normal equations).
 * bfloat16 inputs with d_k = d_v = 128 only (VDA_ERR_UNSUPPORTED otherwise).
 * dO, dQ, dK, dV, dG have the shapes of O, Q, K, V, G; dK_txt, dV_txt those
 * of K_txt, V_txt (ignored, may be NULL, when n_txt == 0); all bfloat16,
 * device memory, 16-byte aligned, written, not accumulated into.  The call
 * recomputes the forward's transitions and states in `workspace` (at least
 * vda_backward_workspace_size() bytes, 256-byte aligned); its device error
 * word is read by vda_sync_status() as for vda_forward.  Asynchronous on
 * `stream`: every step is one of the library's kernels, enqueued on that
 * stream only (no library calls, no other streams, no allocation). */
vda_status vda_backward_workspace_size(const vda_problem* p, size_t* bytes);
vda_status vda_backward(const vda_problem* p, const void* Q, const void* K, const void* V,
                        const void* G, const void* K_txt, const void* V_txt, const void* dO,
                        void* dQ, void* dK, void* dV, void* dG, void* dK_txt, void* dV_txt,
                        void* workspace, size_t workspace_bytes, void* stream);

/* The same gradients without recomputing the forward: `workspace` (at least
 * vda_backward_workspace_size() bytes) must hold what a vda_forward call with
 * the same problem and the same Q, K, V, G, K_txt, V_txt left there, enqueued
 * before this call in stream order, with nothing written to the workspace in
 * between (vda_forward's own workspace layout is a prefix of the backward's).
 * The library does not check this precondition: other contents give wrong
 * gradients, not an error.  The error word is not cleared, so a failure of
 * that forward (VDA_ERR_NOT_SPD, VDA_ERR_TIMEOUT) still reaches
 * vda_sync_status().  Arguments, layout and errors as for vda_backward. */
vda_status vda_backward_from_forward(const vda_problem* p, const void* Q, const void* K, const void* V,
                                     const void* G, const void* K_txt, const void* V_txt, const void* dO,
                                     void* dQ, void* dK, void* dV, void* dG, void* dK_txt, void* dV_txt,
                                     void* workspace, size_t workspace_bytes, void* stream);

/* The local softmax branch of the hybrid attention, the linear branch's
 * partner ("VDN-MiniMax-H3" (aiezz.com), section 03, local softmax branch
 * item, restated in the laicaila.com page, section 技术原理; the "VDN-H3"
 * page (comfyui-wiki.com) on the boundary anchors): frames form blocks of 5
 * and a query token of frame t attends to every token of the frames of
 * blocks t/5 - 1, t/5 and t/5 + 1 (those that exist), to every token of the
 * first and last frames (the anchors, visible from every frame), and to every
 * text token (text dual-branch injection item); the branch's own sigmoid gate
 * (gate fusion item) is applied to its output:
 *     O_t = sigmoid(G_t) * softmax(Q_t K_S^T / sqrt(d)) V_S     (per b, h, t)
 * with S the tokens above.  The problem's sizes and layout as for vda_forward
 * (bfloat16, d_k = d_v = 128; Q, K, V, G, O in the tokens' layout; K_txt,
 * V_txt the text's keys and values, NULL when n_txt == 0); lambda is not
 * read.  Scores, softmax and accumulation in float32; O rounded to bf16.
 * workspace: at least 256 bytes of device memory (256-byte aligned) holding
 * the device error word, which the call clears and vda_sync_status() reads.
 * Asynchronous on `stream`.  Errors on the host, before anything is enqueued:
 * vda_forward's size and pointer checks (VDA_ERR_INVALID_ARG,
 * VDA_ERR_UNSUPPORTED), VDA_ERR_UNSUPPORTED for float32 or e4m3 problems,
 * VDA_ERR_WORKSPACE for a missing, misaligned or short workspace; on the
 * device, VDA_ERR_TIMEOUT through vda_sync_status(). */
vda_status vda_local_softmax(const vda_problem* p, const void* Q, const void* K, const void* V, const void* G,
                             const void* K_txt, const void* V_txt, void* O, void* workspace, size_t workspace_bytes,
                             void* stream);

/* The merge of the hybrid attention's two branches ("VDN-MiniMax-H3"
 * (aiezz.com), section 03, gate fusion item, restated in the laicaila.com
 * page, section 技术原理): each branch has its own content-dependent sigmoid
 * gate and its own output projection, and the projected branches are summed.
 * With each gate applied by its branch (vda_forward applies the linear
 * branch's), this computes
 *     Y = O_lin W_lin + O_sm W_sm      (float32 accumulation, Y rounded to bf16)
 * O_lin, O_sm: [tokens, K] bfloat16, row-major (a token's heads concatenated:
 * the [B, T*n, H, d_v] output of the token-major layout is [B*T*n, H*d_v]);
 * W_lin, W_sm: [K, D] bfloat16, row-major; Y: [tokens, D] bfloat16.  O_sm and
 * W_sm are both NULL when there is no softmax branch (Y = O_lin W_lin).
 * tokens >= 1; K a multiple of 64; D a multiple of 8 (>= 8).  Device
 * pointers, 16-byte aligned.  workspace: at least 256 bytes of device memory
 * (256-byte aligned) holding the device error word, which the call clears
 * and vda_sync_status() reads.  Asynchronous on `stream`.  Errors on the host,
 * before anything is enqueued: VDA_ERR_INVALID_ARG for a NULL problem, tokens
 * out of [1, 2^31 - 256], a NULL or misaligned pointer, O_sm or W_sm given
 * alone, an unknown test_stall or a nonzero reserved field;
 * VDA_ERR_UNSUPPORTED for K or D off the grid above; VDA_ERR_WORKSPACE for a
 * missing, misaligned or short workspace; on the device, VDA_ERR_TIMEOUT
 * through vda_sync_status(). */
typedef struct vda_merge_problem {
  int64_t tokens;
  int32_t K, D;
  int32_t test_stall; /* testing hook as in vda_problem; 0 in normal use */
  int32_t reserved;   /* 0 */
} vda_merge_problem;
vda_status vda_merge_project(const vda_merge_problem* p, const void* O_lin, const void* W_lin, const void* O_sm,
                             const void* W_sm, void* Y, void* workspace, size_t workspace_bytes, void* stream);

/* Synchronises `stream`, then reads and clears the device error word of
 * `workspace`: VDA_OK, VDA_ERR_NOT_SPD or VDA_ERR_TIMEOUT (first one set),
 * or VDA_ERR_CUDA if the stream reports an error.  Blocking. */
vda_status vda_sync_status(void* workspace, void* stream);

/* A static, human-readable name for a status code. */
const char* vda_status_string(vda_status s);

/* A thread-local message describing the last error returned on this host
 * thread ("" if none).  Valid until the next call on the same thread. */
const char* vda_last_error(void);

#ifdef __cplusplus
}
#endif

#endif /* VDA_H_ */
