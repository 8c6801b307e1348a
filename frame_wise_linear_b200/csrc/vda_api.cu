// Host side of the C ABI declared in include/vda.h: argument checks,
// workspace carve-up and the launch sequence.  No compute happens here.
#include <math.h>
#include <stdarg.h>
#include <stdio.h>
#include <string.h>

#include <type_traits>

#include "vda_internal.cuh"

namespace {

thread_local char g_msg[512] = "";

vda_status fail(vda_status s, const char* fmt, ...) __attribute__((format(printf, 2, 3)));
vda_status fail(vda_status s, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_msg, sizeof(g_msg), fmt, ap);
  va_end(ap);
  return s;
}

vda_status cuda_fail(cudaError_t e, const char* where) {
  return fail(VDA_ERR_CUDA, "%s: %s", where, cudaGetErrorString(e));
}

bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }

vda_status check_problem(const vda_problem* p) {
  if (!p) return fail(VDA_ERR_INVALID_ARG, "problem is NULL");
  if (p->B < 1 || p->H < 1 || p->T < 1 || p->n < 1)
    return fail(VDA_ERR_INVALID_ARG, "B, H, T, n must be >= 1 (got %d, %d, %d, %d)", p->B, p->H,
                p->T, p->n);
  if (p->n_txt < 0) return fail(VDA_ERR_INVALID_ARG, "n_txt must be >= 0 (got %d)", p->n_txt);
  if (p->d_k < 1 || p->d_v < 1)
    return fail(VDA_ERR_INVALID_ARG, "d_k, d_v must be >= 1 (got %d, %d)", p->d_k, p->d_v);
  if (!(p->lambda > 0.f) || !isfinite(p->lambda))
    return fail(VDA_ERR_INVALID_ARG, "lambda must be finite and > 0 (got %g)", (double)p->lambda);
  if (p->dtype != VDA_DTYPE_F32 && p->dtype != VDA_DTYPE_BF16 && p->dtype != VDA_DTYPE_E4M3)
    return fail(VDA_ERR_INVALID_ARG, "unknown dtype %d", p->dtype);
  if (p->dtype == VDA_DTYPE_E4M3) {
    const float sc[4] = {p->scale_q, p->scale_k, p->scale_v, p->scale_g};
    for (float v : sc)
      if (!(v > 0.f) || !isfinite(v))
        return fail(VDA_ERR_INVALID_ARG, "e4m3 scales must be finite and > 0 (got %g, %g, %g, %g)",
                    (double)sc[0], (double)sc[1], (double)sc[2], (double)sc[3]);
  }
  if (p->layout != VDA_LAYOUT_BHTND && p->layout != VDA_LAYOUT_BTNHD)
    return fail(VDA_ERR_INVALID_ARG, "unknown layout %d", p->layout);
  if (p->test_stall < 0 || p->test_stall > VDA_TEST_STALL_MAX)
    return fail(VDA_ERR_INVALID_ARG, "unknown test_stall site %d", p->test_stall);
  if (p->layout == VDA_LAYOUT_BTNHD && p->dtype == VDA_DTYPE_F32)
    return fail(VDA_ERR_UNSUPPORTED, "the token-major layout is supported for bfloat16 and e4m3 inputs only");
  if (p->dtype == VDA_DTYPE_F32) {
    if (p->d_k % 16 || p->d_v % 16 || p->d_k > 128 || p->d_v > 128)
      return fail(VDA_ERR_UNSUPPORTED,
                  "float32 path supports d_k, d_v multiples of 16 up to 128 (got %d, %d)", p->d_k,
                  p->d_v);
  } else {
    if (p->d_k != 128 || p->d_v != 128)
      return fail(VDA_ERR_UNSUPPORTED, "%s path supports d_k = d_v = 128 (got %d, %d)",
                  p->dtype == VDA_DTYPE_E4M3 ? "e4m3" : "bfloat16", p->d_k, p->d_v);
  }
  // Index arithmetic in the kernels: slots and frames fit 32 bits, element
  // offsets are 64-bit.
  const long long slots = (long long)p->B * p->H * (p->T + 1);
  if (slots > 65535LL * 64)
    return fail(VDA_ERR_UNSUPPORTED, "B*H*(T+1) = %lld is above the supported 4194240", slots);
  if ((long long)p->B * p->H > 65535)
    return fail(VDA_ERR_UNSUPPORTED, "B*H = %lld is above 65535", (long long)p->B * p->H);
  if ((long long)p->B * p->H * p->T > 65535LL * 1024)
    return fail(VDA_ERR_UNSUPPORTED, "B*H*T is too large");
  if (p->n > (1 << 24) || p->n_txt > (1 << 24))
    return fail(VDA_ERR_UNSUPPORTED, "n and n_txt must be <= 2^24");
  return VDA_OK;
}

// Bytes of one input element, and of one element of O (bfloat16 for e4m3 inputs).
size_t elem_size(const vda_problem& p) {
  return p.dtype == VDA_DTYPE_E4M3 ? 1 : p.dtype == VDA_DTYPE_BF16 ? 2 : 4;
}
size_t out_elem_size(const vda_problem& p) { return p.dtype == VDA_DTYPE_F32 ? 4 : 2; }

struct Sizes {
  size_t q, k, v, g, kt, vt, o;
};

Sizes tensor_bytes(const vda_problem& p) {
  const size_t es = elem_size(p);
  const size_t fr = (size_t)p.B * p.H * p.T * p.n;
  const size_t tx = (size_t)p.B * p.H * p.n_txt;
  return Sizes{fr * p.d_k * es, fr * p.d_k * es, fr * p.d_v * es, fr * p.d_v * es,
               tx * p.d_k * es, tx * p.d_v * es, fr * p.d_v * out_elem_size(p)};
}

vda_status check_pointers(const vda_problem& p, const void* Q, const void* K, const void* V,
                          const void* G, const void* Kt, const void* Vt, const void* O) {
  const void* req[5] = {Q, K, V, G, O};
  const char* names[5] = {"Q", "K", "V", "G", "O"};
  for (int i = 0; i < 5; ++i) {
    if (!req[i]) return fail(VDA_ERR_INVALID_ARG, "%s is NULL", names[i]);
    if (!aligned16(req[i])) return fail(VDA_ERR_INVALID_ARG, "%s is not 16-byte aligned", names[i]);
  }
  if (p.n_txt > 0) {
    if (!Kt || !Vt) return fail(VDA_ERR_INVALID_ARG, "K_txt / V_txt NULL with n_txt = %d", p.n_txt);
    if (!aligned16(Kt) || !aligned16(Vt))
      return fail(VDA_ERR_INVALID_ARG, "K_txt / V_txt not 16-byte aligned");
  }
  return VDA_OK;
}

// The float32 path: SIMT Gram, the register-blocked factor, SIMT scan and
// readout; every state and product in float32.
vda_status run_forward_f32(const vda_problem& p, const float* q, const float* k, const float* v, const float* g,
                           const float* kt, const float* vt, float* O, char* ws, cudaStream_t st, float* S_fwd,
                           float* S_bwd, cudaEvent_t const* ev) {
  const vda::Layout L = vda::make_layout(p);
  unsigned* err = reinterpret_cast<unsigned*>(ws + L.err);
  float* M = reinterpret_cast<float*>(ws + L.M);
  float* C = reinterpret_cast<float*>(ws + L.C);
  // The states live in the workspace unless the caller wants them.
  float* SF = S_fwd ? S_fwd : reinterpret_cast<float*>(ws + L.SF);
  float* SB = S_bwd ? S_bwd : reinterpret_cast<float*>(ws + L.SB);
  cudaError_t e = cudaMemsetAsync(err, 0, 256, st);
  if (e != cudaSuccess) return cuda_fail(e, "clearing the error word");
  auto mark = [&](int i) -> cudaError_t { return ev ? cudaEventRecord(ev[i], st) : cudaSuccess; };
  if ((e = mark(0)) != cudaSuccess) return cuda_fail(e, "event record");
  if ((e = vda::launch_gram_simt<float>(p, k, v, kt, vt, M, C, st)) != cudaSuccess) return cuda_fail(e, "gram launch");
  if ((e = mark(1)) != cudaSuccess) return cuda_fail(e, "event record");
  if ((e = vda::launch_factor(p, M, err, st)) != cudaSuccess) return cuda_fail(e, "factor launch");
  if ((e = mark(2)) != cudaSuccess) return cuda_fail(e, "event record");
  if ((e = vda::launch_scan_simt(p, M, C, SF, SB, st)) != cudaSuccess) return cuda_fail(e, "scan launch");
  if ((e = mark(3)) != cudaSuccess) return cuda_fail(e, "event record");
  if ((e = vda::launch_readout_simt<float>(p, q, g, SF, SB, O, st)) != cudaSuccess)
    return cuda_fail(e, "readout launch");
  if ((e = mark(4)) != cudaSuccess) return cuda_fail(e, "event record");
  return VDA_OK;
}

// The tensor-core path (bfloat16 or e4m3 inputs, d = 128): the fused
// Gram+factor kernel (A_t never leaves TMEM), the scan, the readout.  The
// workspace holds bf16 states for the readout; the caller's float32 state
// buffers, if any, are written besides.
vda_status run_forward_tc(const vda_problem& p, const void* q, const void* k, const void* v, const void* g,
                          const void* kt, const void* vt, void* O, char* ws, cudaStream_t st, float* S_fwd,
                          float* S_bwd, cudaEvent_t const* ev) {
  const vda::Layout L = vda::make_layout(p);
  unsigned* err = reinterpret_cast<unsigned*>(ws + L.err);
  float* M = reinterpret_cast<float*>(ws + L.M);
  float* C = reinterpret_cast<float*>(ws + L.C);
  __nv_bfloat16* SFb = reinterpret_cast<__nv_bfloat16*>(ws + L.SF);
  __nv_bfloat16* SBb = reinterpret_cast<__nv_bfloat16*>(ws + L.SB);
  cudaError_t e = cudaMemsetAsync(err, 0, 256, st);
  if (e != cudaSuccess) return cuda_fail(e, "clearing the error word");
  auto mark = [&](int i) -> cudaError_t { return ev ? cudaEventRecord(ev[i], st) : cudaSuccess; };
  if ((e = mark(0)) != cudaSuccess) return cuda_fail(e, "event record");
  // Gram and factor in one kernel: the factor interval between events 1 and
  // 2 is empty on this path.
  if ((e = vda::launch_gramfactor_tc(p, k, v, kt, vt, M, C, err, st)) != cudaSuccess)
    return cuda_fail(e, "gram+factor launch");
  if ((e = mark(1)) != cudaSuccess) return cuda_fail(e, "event record");
  if ((e = mark(2)) != cudaSuccess) return cuda_fail(e, "event record");
  if ((e = vda::launch_scan_tc(p, M, C, SFb, SBb, S_fwd, S_bwd, err, st)) != cudaSuccess)
    return cuda_fail(e, "scan launch");
  if ((e = mark(3)) != cudaSuccess) return cuda_fail(e, "event record");
  if ((e = vda::launch_readout_tc(p, q, g, SFb, SBb, static_cast<__nv_bfloat16*>(O), err, st)) != cudaSuccess)
    return cuda_fail(e, "readout launch");
  if ((e = mark(4)) != cudaSuccess) return cuda_fail(e, "event record");
  return VDA_OK;
}

vda_status forward_impl(const vda_problem* p, const void* Q, const void* K, const void* V,
                        const void* G, const void* Kt, const void* Vt, void* O, void* workspace,
                        size_t workspace_bytes, void* stream, float* S_fwd, float* S_bwd,
                        cudaEvent_t const* ev = nullptr) {
  g_msg[0] = 0;
  vda_status s = check_problem(p);
  if (s != VDA_OK) return s;
  if ((s = check_pointers(*p, Q, K, V, G, Kt, Vt, O)) != VDA_OK) return s;
  const vda::Layout L = vda::make_layout(*p);
  if (!workspace) return fail(VDA_ERR_WORKSPACE, "workspace is NULL");
  if ((uintptr_t)workspace & 255u) return fail(VDA_ERR_WORKSPACE, "workspace not 256-byte aligned");
  if (workspace_bytes < L.total)
    return fail(VDA_ERR_WORKSPACE, "workspace has %zu bytes, needs %zu", workspace_bytes, L.total);
  if ((S_fwd && !aligned16(S_fwd)) || (S_bwd && !aligned16(S_bwd)))
    return fail(VDA_ERR_INVALID_ARG, "S_fwd / S_bwd not 16-byte aligned");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  char* ws = static_cast<char*>(workspace);
  if (p->dtype != VDA_DTYPE_F32) return run_forward_tc(*p, Q, K, V, G, Kt, Vt, O, ws, st, S_fwd, S_bwd, ev);
  auto f = [](const void* x) { return static_cast<const float*>(x); };
  return run_forward_f32(*p, f(Q), f(K), f(V), f(G), f(Kt), f(Vt), static_cast<float*>(O), ws, st, S_fwd, S_bwd, ev);
}

}  // namespace

namespace vda {
void set_error_message(const char* msg) { snprintf(g_msg, sizeof(g_msg), "%s", msg); }
}  // namespace vda

extern "C" {

vda_status vda_workspace_size(const vda_problem* p, size_t* bytes) {
  g_msg[0] = 0;
  vda_status s = check_problem(p);
  if (s != VDA_OK) return s;
  if (!bytes) return fail(VDA_ERR_INVALID_ARG, "bytes is NULL");
  *bytes = vda::make_layout(*p).total;
  return VDA_OK;
}

vda_status vda_forward(const vda_problem* p, const void* Q, const void* K, const void* V,
                       const void* G, const void* K_txt, const void* V_txt, void* O,
                       void* workspace, size_t workspace_bytes, void* stream) {
  return forward_impl(p, Q, K, V, G, K_txt, V_txt, O, workspace, workspace_bytes, stream, nullptr,
                      nullptr);
}

vda_status vda_forward_states(const vda_problem* p, const void* Q, const void* K, const void* V,
                              const void* G, const void* K_txt, const void* V_txt, void* O,
                              void* workspace, size_t workspace_bytes, void* stream,
                              float* S_fwd, float* S_bwd) {
  if (!S_fwd || !S_bwd) return fail(VDA_ERR_INVALID_ARG, "S_fwd / S_bwd is NULL");
  return forward_impl(p, Q, K, V, G, K_txt, V_txt, O, workspace, workspace_bytes, stream, S_fwd,
                      S_bwd);
}

vda_status vda_forward_timed(const vda_problem* p, const void* Q, const void* K, const void* V,
                             const void* G, const void* K_txt, const void* V_txt, void* O,
                             void* workspace, size_t workspace_bytes, void* stream,
                             void* const* events, int n_events) {
  if (!events || n_events != VDA_TIMED_EVENTS)
    return fail(VDA_ERR_INVALID_ARG, "events must hold %d cudaEvent_t handles", VDA_TIMED_EVENTS);
  for (int i = 0; i < n_events; ++i)
    if (!events[i]) return fail(VDA_ERR_INVALID_ARG, "events[%d] is NULL", i);
  return forward_impl(p, Q, K, V, G, K_txt, V_txt, O, workspace, workspace_bytes, stream, nullptr,
                      nullptr, reinterpret_cast<cudaEvent_t const*>(events));
}

vda_status vda_host_workspace_size(const vda_problem* p, size_t* bytes) {
  g_msg[0] = 0;
  vda_status s = check_problem(p);
  if (s != VDA_OK) return s;
  if (!bytes) return fail(VDA_ERR_INVALID_ARG, "bytes is NULL");
  const Sizes z = tensor_bytes(*p);
  size_t off = 0;
  const size_t parts[7] = {z.q, z.k, z.v, z.g, z.kt, z.vt, z.o};
  for (size_t b : parts) off = vda::align_up(off + b, 256);
  *bytes = off + vda::make_layout(*p).total;
  return VDA_OK;
}

vda_status vda_forward_host(const vda_problem* p, const void* Q, const void* K, const void* V,
                            const void* G, const void* K_txt, const void* V_txt, void* O,
                            void* workspace, size_t workspace_bytes, void* stream) {
  g_msg[0] = 0;
  vda_status s = check_problem(p);
  if (s != VDA_OK) return s;
  if ((s = check_pointers(*p, Q, K, V, G, K_txt, V_txt, O)) != VDA_OK) return s;
  size_t need = 0;
  vda_host_workspace_size(p, &need);
  if (!workspace) return fail(VDA_ERR_WORKSPACE, "workspace is NULL");
  if ((uintptr_t)workspace & 255u) return fail(VDA_ERR_WORKSPACE, "workspace not 256-byte aligned");
  if (workspace_bytes < need)
    return fail(VDA_ERR_WORKSPACE, "workspace has %zu bytes, needs %zu", workspace_bytes, need);
  const Sizes z = tensor_bytes(*p);
  char* base = static_cast<char*>(workspace);
  const void* src[6] = {Q, K, V, G, K_txt, V_txt};
  const size_t len[6] = {z.q, z.k, z.v, z.g, z.kt, z.vt};
  void* dev[7];
  size_t off = 0;
  for (int i = 0; i < 6; ++i) {
    dev[i] = base + off;
    off = vda::align_up(off + len[i], 256);
  }
  dev[6] = base + off;
  off = vda::align_up(off + z.o, 256);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  for (int i = 0; i < 6; ++i) {
    if (len[i] == 0) continue;
    cudaError_t e = cudaMemcpyAsync(dev[i], src[i], len[i], cudaMemcpyHostToDevice, st);
    if (e != cudaSuccess) return cuda_fail(e, "host-to-device copy");
  }
  s = forward_impl(p, dev[0], dev[1], dev[2], dev[3], p->n_txt ? dev[4] : nullptr,
                   p->n_txt ? dev[5] : nullptr, dev[6], base + off, workspace_bytes - off, stream,
                   nullptr, nullptr);
  if (s != VDA_OK) return s;
  cudaError_t e = cudaMemcpyAsync(O, dev[6], z.o, cudaMemcpyDeviceToHost, st);
  if (e != cudaSuccess) return cuda_fail(e, "device-to-host copy");
  return vda_sync_status(base + off, stream);
}

vda_status vda_backward_workspace_size(const vda_problem* p, size_t* bytes) {
  g_msg[0] = 0;
  vda_status s = check_problem(p);
  if (s != VDA_OK) return s;
  if (p->dtype != VDA_DTYPE_BF16)
    return fail(VDA_ERR_UNSUPPORTED, "the backward supports bfloat16 inputs only");
  if (!bytes) return fail(VDA_ERR_INVALID_ARG, "bytes is NULL");
  *bytes = vda::backward_workspace_bytes(*p);
  return VDA_OK;
}

namespace {

vda_status backward_impl(const vda_problem* p, const void* Q, const void* K, const void* V, const void* G,
                         const void* K_txt, const void* V_txt, const void* dO, void* dQ, void* dK, void* dV,
                         void* dG, void* dK_txt, void* dV_txt, void* workspace, size_t workspace_bytes, void* stream,
                         bool from_forward) {
  size_t need = 0;
  vda_status s = vda_backward_workspace_size(p, &need);
  if (s != VDA_OK) return s;
  if ((s = check_pointers(*p, Q, K, V, G, K_txt, V_txt, dO)) != VDA_OK) return s;
  const void* outs[4] = {dQ, dK, dV, dG};
  const char* names[4] = {"dQ", "dK", "dV", "dG"};
  for (int i = 0; i < 4; ++i) {
    if (!outs[i]) return fail(VDA_ERR_INVALID_ARG, "%s is NULL", names[i]);
    if (!aligned16(outs[i])) return fail(VDA_ERR_INVALID_ARG, "%s is not 16-byte aligned", names[i]);
  }
  if (p->n_txt > 0 && (!dK_txt || !dV_txt || !aligned16(dK_txt) || !aligned16(dV_txt)))
    return fail(VDA_ERR_INVALID_ARG, "dK_txt / dV_txt NULL or not 16-byte aligned with n_txt = %d", p->n_txt);
  if (!workspace) return fail(VDA_ERR_WORKSPACE, "workspace is NULL");
  if ((uintptr_t)workspace & 255u) return fail(VDA_ERR_WORKSPACE, "workspace not 256-byte aligned");
  if (workspace_bytes < need)
    return fail(VDA_ERR_WORKSPACE, "workspace has %zu bytes, needs %zu", workspace_bytes, need);
  using bf = __nv_bfloat16;
  const char* where = "";
  cudaError_t e = vda::run_backward(*p, static_cast<const bf*>(Q), static_cast<const bf*>(K),
                                    static_cast<const bf*>(V), static_cast<const bf*>(G),
                                    static_cast<const bf*>(K_txt), static_cast<const bf*>(V_txt),
                                    static_cast<const bf*>(dO), static_cast<bf*>(dQ), static_cast<bf*>(dK),
                                    static_cast<bf*>(dV), static_cast<bf*>(dG), static_cast<bf*>(dK_txt),
                                    static_cast<bf*>(dV_txt), static_cast<char*>(workspace),
                                    static_cast<cudaStream_t>(stream), &where, from_forward);
  if (e != cudaSuccess) return cuda_fail(e, where);
  return VDA_OK;
}

}  // namespace

vda_status vda_backward(const vda_problem* p, const void* Q, const void* K, const void* V, const void* G,
                        const void* K_txt, const void* V_txt, const void* dO, void* dQ, void* dK, void* dV,
                        void* dG, void* dK_txt, void* dV_txt, void* workspace, size_t workspace_bytes,
                        void* stream) {
  return backward_impl(p, Q, K, V, G, K_txt, V_txt, dO, dQ, dK, dV, dG, dK_txt, dV_txt, workspace, workspace_bytes,
                       stream, false);
}

vda_status vda_backward_from_forward(const vda_problem* p, const void* Q, const void* K, const void* V,
                                     const void* G, const void* K_txt, const void* V_txt, const void* dO, void* dQ,
                                     void* dK, void* dV, void* dG, void* dK_txt, void* dV_txt, void* workspace,
                                     size_t workspace_bytes, void* stream) {
  return backward_impl(p, Q, K, V, G, K_txt, V_txt, dO, dQ, dK, dV, dG, dK_txt, dV_txt, workspace, workspace_bytes,
                       stream, true);
}

vda_status vda_local_softmax(const vda_problem* p, const void* Q, const void* K, const void* V, const void* G,
                             const void* K_txt, const void* V_txt, void* O, void* workspace, size_t workspace_bytes,
                             void* stream) {
  g_msg[0] = 0;
  if (!p) return fail(VDA_ERR_INVALID_ARG, "problem is NULL");
  vda_problem q = *p;
  q.lambda = 1.f;   // not read by this branch
  vda_status s = check_problem(&q);
  if (s != VDA_OK) return s;
  if (q.dtype != VDA_DTYPE_BF16)
    return fail(VDA_ERR_UNSUPPORTED, "the local softmax branch supports bfloat16 inputs only");
  if ((s = check_pointers(q, Q, K, V, G, K_txt, V_txt, O)) != VDA_OK) return s;
  if (!workspace) return fail(VDA_ERR_WORKSPACE, "workspace is NULL");
  if ((uintptr_t)workspace & 255u) return fail(VDA_ERR_WORKSPACE, "workspace not 256-byte aligned");
  if (workspace_bytes < 256) return fail(VDA_ERR_WORKSPACE, "workspace has %zu bytes, needs 256", workspace_bytes);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaMemsetAsync(workspace, 0, 256, st);
  if (e != cudaSuccess) return cuda_fail(e, "clearing the error word");
  using bf = __nv_bfloat16;
  e = vda::launch_local_softmax_tc(q, static_cast<const bf*>(Q), static_cast<const bf*>(K), static_cast<const bf*>(V),
                                   static_cast<const bf*>(G), static_cast<const bf*>(K_txt),
                                   static_cast<const bf*>(V_txt), static_cast<bf*>(O),
                                   static_cast<unsigned*>(workspace), st);
  if (e != cudaSuccess) return cuda_fail(e, "local softmax launch");
  return VDA_OK;
}

vda_status vda_merge_project(const vda_merge_problem* p, const void* O_lin, const void* W_lin, const void* O_sm,
                             const void* W_sm, void* Y, void* workspace, size_t workspace_bytes, void* stream) {
  g_msg[0] = 0;
  if (!p) return fail(VDA_ERR_INVALID_ARG, "problem is NULL");
  if (p->tokens < 1 || p->tokens > (1LL << 31) - 256)
    return fail(VDA_ERR_INVALID_ARG, "tokens must be in [1, 2^31 - 256] (got %lld)", (long long)p->tokens);
  if (p->K < 64 || p->K % 64) return fail(VDA_ERR_UNSUPPORTED, "K must be a positive multiple of 64 (got %d)", p->K);
  if (p->D < 8 || p->D % 8) return fail(VDA_ERR_UNSUPPORTED, "D must be a positive multiple of 8 (got %d)", p->D);
  if (p->test_stall < 0 || p->test_stall > VDA_TEST_STALL_MAX)
    return fail(VDA_ERR_INVALID_ARG, "unknown test_stall site %d", p->test_stall);
  if (p->reserved != 0) return fail(VDA_ERR_INVALID_ARG, "reserved must be 0 (got %d)", p->reserved);
  const void* req[3] = {O_lin, W_lin, Y};
  const char* names[3] = {"O_lin", "W_lin", "Y"};
  for (int i = 0; i < 3; ++i) {
    if (!req[i]) return fail(VDA_ERR_INVALID_ARG, "%s is NULL", names[i]);
    if (!aligned16(req[i])) return fail(VDA_ERR_INVALID_ARG, "%s is not 16-byte aligned", names[i]);
  }
  if ((O_sm == nullptr) != (W_sm == nullptr))
    return fail(VDA_ERR_INVALID_ARG, "O_sm and W_sm must both be given or both be NULL");
  if (O_sm && (!aligned16(O_sm) || !aligned16(W_sm)))
    return fail(VDA_ERR_INVALID_ARG, "O_sm / W_sm not 16-byte aligned");
  if (!workspace) return fail(VDA_ERR_WORKSPACE, "workspace is NULL");
  if ((uintptr_t)workspace & 255u) return fail(VDA_ERR_WORKSPACE, "workspace not 256-byte aligned");
  if (workspace_bytes < 256) return fail(VDA_ERR_WORKSPACE, "workspace has %zu bytes, needs 256", workspace_bytes);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaMemsetAsync(workspace, 0, 256, st);
  if (e != cudaSuccess) return cuda_fail(e, "clearing the error word");
  using bf = __nv_bfloat16;
  e = vda::launch_merge_tc(p->tokens, p->K, p->D, static_cast<const bf*>(O_lin), static_cast<const bf*>(W_lin),
                           static_cast<const bf*>(O_sm), static_cast<const bf*>(W_sm), static_cast<bf*>(Y),
                           static_cast<unsigned*>(workspace), st, p->test_stall);
  if (e != cudaSuccess) return cuda_fail(e, "merge launch");
  return VDA_OK;
}

vda_status vda_sync_status(void* workspace, void* stream) {
  g_msg[0] = 0;
  if (!workspace) return fail(VDA_ERR_WORKSPACE, "workspace is NULL");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return cuda_fail(e, "stream synchronize");
  unsigned word = 0;
  e = cudaMemcpy(&word, workspace, sizeof(word), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail(e, "reading the error word");
  if (word) {
    e = cudaMemset(workspace, 0, sizeof(word));
    if (e != cudaSuccess) return cuda_fail(e, "clearing the error word");
  }
  if (word & vda::kDevErrNotSpd) return fail(VDA_ERR_NOT_SPD, "a Cholesky pivot was not positive");
  if (word & vda::kDevErrTimeout) return fail(VDA_ERR_TIMEOUT, "a bounded device wait gave up");
  return VDA_OK;
}

const char* vda_status_string(vda_status s) {
  switch (s) {
    case VDA_OK: return "VDA_OK";
    case VDA_ERR_INVALID_ARG: return "VDA_ERR_INVALID_ARG";
    case VDA_ERR_UNSUPPORTED: return "VDA_ERR_UNSUPPORTED";
    case VDA_ERR_WORKSPACE: return "VDA_ERR_WORKSPACE";
    case VDA_ERR_CUDA: return "VDA_ERR_CUDA";
    case VDA_ERR_NOT_SPD: return "VDA_ERR_NOT_SPD";
    case VDA_ERR_TIMEOUT: return "VDA_ERR_TIMEOUT";
  }
  return "VDA_ERR_UNKNOWN";
}

const char* vda_last_error(void) { return g_msg; }

}  // extern "C"
