"""Python binding of libvda.so (include/vda.h): argument marshalling only.

Every function here mirrors one C entry point of the same name; tensors are
passed as torch tensors (device pointers are taken from ``data_ptr()``) or as
raw integer addresses.  All arithmetic runs in the library's CUDA kernels;
nothing here computes any step of VDA, and there is no CPU path: if the
library is missing or no CUDA device is present, the calls raise.

``forward`` is the convenience call a user makes: it allocates O and the
workspace with torch on the inputs' device and runs ``vda_forward`` on the
current torch stream.
"""

from __future__ import annotations

import ctypes
import os
import threading

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libvda.so")

VDA_OK = 0
VDA_ERR_INVALID_ARG = 1
VDA_ERR_UNSUPPORTED = 2
VDA_ERR_WORKSPACE = 3
VDA_ERR_CUDA = 4
VDA_ERR_NOT_SPD = 5
VDA_ERR_TIMEOUT = 6

VDA_DTYPE_F32 = 0
VDA_DTYPE_BF16 = 1
VDA_DTYPE_E4M3 = 2     # 8-bit float inputs with per-tensor scales (uint8 storage); O is bf16
VDA_LAYOUT_BHTND = 0   # Q, K, V, G, O: [B, H, T, n, d]; text [B, H, n_txt, d]
VDA_LAYOUT_BTNHD = 1   # Q, K, V, G, O: [B, T*n, H, d]; text [B, n_txt, H, d] (bf16 only)

# Testing hook for the device timeout path (vda_problem.test_stall): the wait
# named here runs out in the first CTA of its kernel (include/vda.h).
TEST_STALL_SITES = {
    "gram_stage": 1, "factor_update": 2, "service_gram": 3, "scan_operand": 4, "scan_product": 5,
    "readout_tile": 6, "readout_gate": 7, "readout_state": 8, "rbwd_tile": 9, "rbwd_dq": 10,
    "gbwd_tile": 11, "gbwd_store": 12, "operands": 13, "merge": 14, "softmax": 15,
}

SYMBOLS = (
    "vda_workspace_size",
    "vda_forward",
    "vda_forward_states",
    "vda_forward_timed",
    "vda_host_workspace_size",
    "vda_forward_host",
    "vda_forward_noalloc",
    "vda_backward_workspace_size",
    "vda_backward",
    "vda_backward_from_forward",
    "vda_local_softmax",
    "vda_merge_project",
    "vda_sync_status",
    "vda_status_string",
    "vda_last_error",
)


class vda_problem(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int32), ("H", ctypes.c_int32), ("T", ctypes.c_int32),
                ("n", ctypes.c_int32), ("n_txt", ctypes.c_int32), ("d_k", ctypes.c_int32),
                ("d_v", ctypes.c_int32), ("dtype", ctypes.c_int32), ("lambda_", ctypes.c_float),
                ("layout", ctypes.c_int32), ("test_stall", ctypes.c_int32),
                ("scale_q", ctypes.c_float), ("scale_k", ctypes.c_float), ("scale_v", ctypes.c_float),
                ("scale_g", ctypes.c_float)]


class vda_merge_problem(ctypes.Structure):
    _fields_ = [("tokens", ctypes.c_int64), ("K", ctypes.c_int32), ("D", ctypes.c_int32),
                ("test_stall", ctypes.c_int32), ("reserved", ctypes.c_int32)]


class VdaError(RuntimeError):
    def __init__(self, status: int, where: str, msg: str):
        self.status = status
        super().__init__(f"{where}: {_status_name(status)}: {msg}")


_lib = None
_lock = threading.Lock()


def load(path: str | None = None):
    """Loads libvda.so (once).  Raises if it has not been built."""
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        p = path or LIB_PATH
        if not os.path.exists(p):
            raise RuntimeError(f"{p} is missing: build it with `python -m frame_wise_linear_b200.build`")
        lib = ctypes.CDLL(p)
        P = ctypes.POINTER(vda_problem)
        vp = ctypes.c_void_p
        st = ctypes.c_int
        lib.vda_workspace_size.argtypes = [P, ctypes.POINTER(ctypes.c_size_t)]
        lib.vda_workspace_size.restype = st
        lib.vda_host_workspace_size.argtypes = [P, ctypes.POINTER(ctypes.c_size_t)]
        lib.vda_host_workspace_size.restype = st
        fwd = [P, vp, vp, vp, vp, vp, vp, vp, vp, ctypes.c_size_t, vp]
        lib.vda_forward.argtypes = fwd
        lib.vda_forward.restype = st
        lib.vda_forward_host.argtypes = fwd
        lib.vda_forward_host.restype = st
        lib.vda_forward_states.argtypes = fwd + [vp, vp]
        lib.vda_forward_states.restype = st
        lib.vda_forward_timed.argtypes = fwd + [ctypes.POINTER(ctypes.c_void_p), ctypes.c_int]
        lib.vda_forward_timed.restype = st
        lib.vda_forward_noalloc.argtypes = [P, vp, vp, vp, vp, vp, vp, vp, vp]
        lib.vda_forward_noalloc.restype = st
        lib.vda_backward_workspace_size.argtypes = [P, ctypes.POINTER(ctypes.c_size_t)]
        lib.vda_backward_workspace_size.restype = st
        lib.vda_backward.argtypes = [P] + [vp] * 13 + [vp, ctypes.c_size_t, vp]
        lib.vda_backward.restype = st
        lib.vda_backward_from_forward.argtypes = [P] + [vp] * 13 + [vp, ctypes.c_size_t, vp]
        lib.vda_backward_from_forward.restype = st
        lib.vda_local_softmax.argtypes = [P, vp, vp, vp, vp, vp, vp, vp, vp, ctypes.c_size_t, vp]
        lib.vda_local_softmax.restype = st
        lib.vda_merge_project.argtypes = [ctypes.POINTER(vda_merge_problem), vp, vp, vp, vp, vp, vp, ctypes.c_size_t,
                                          vp]
        lib.vda_merge_project.restype = st
        lib.vda_sync_status.argtypes = [vp, vp]
        lib.vda_sync_status.restype = st
        lib.vda_status_string.argtypes = [st]
        lib.vda_status_string.restype = ctypes.c_char_p
        lib.vda_last_error.argtypes = []
        lib.vda_last_error.restype = ctypes.c_char_p
        _lib = lib
        return lib


def _status_name(s: int) -> str:
    try:
        return load().vda_status_string(s).decode()
    except Exception:
        return str(s)


def _check(status: int, where: str):
    if status != VDA_OK:
        raise VdaError(status, where, load().vda_last_error().decode())


def make_problem(B, H, T, n, n_txt, d_k, d_v, dtype, lam, layout=0, test_stall=0, scale_q=1.0, scale_k=1.0,
                 scale_v=1.0, scale_g=1.0) -> vda_problem:
    return vda_problem(int(B), int(H), int(T), int(n), int(n_txt), int(d_k), int(d_v), int(dtype),
                       float(lam), int(layout), int(test_stall), float(scale_q), float(scale_k), float(scale_v),
                       float(scale_g))


def _ptr(x) -> int | None:
    if x is None:
        return None
    if isinstance(x, int):
        return x
    return x.data_ptr()


def _stream(stream) -> int | None:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def vda_workspace_size(problem: vda_problem) -> int:
    out = ctypes.c_size_t(0)
    _check(load().vda_workspace_size(ctypes.byref(problem), ctypes.byref(out)), "vda_workspace_size")
    return out.value


def vda_backward_workspace_size(problem: vda_problem) -> int:
    out = ctypes.c_size_t(0)
    _check(load().vda_backward_workspace_size(ctypes.byref(problem), ctypes.byref(out)),
           "vda_backward_workspace_size")
    return out.value


def vda_backward(problem, Q, K, V, G, K_txt, V_txt, dO, dQ, dK, dV, dG, dK_txt, dV_txt, workspace,
                 stream=None, workspace_bytes=None, check=True) -> int:
    """Gradients of sum(dO * O) into dQ, dK, dV, dG, dK_txt, dV_txt (device buffers)."""
    wb = _nbytes(workspace) if workspace_bytes is None else workspace_bytes
    s = load().vda_backward(ctypes.byref(problem), _ptr(Q), _ptr(K), _ptr(V), _ptr(G), _ptr(K_txt),
                            _ptr(V_txt), _ptr(dO), _ptr(dQ), _ptr(dK), _ptr(dV), _ptr(dG), _ptr(dK_txt),
                            _ptr(dV_txt), _ptr(workspace), wb, _stream(stream))
    if check:
        _check(s, "vda_backward")
    return s


def vda_backward_from_forward(problem, Q, K, V, G, K_txt, V_txt, dO, dQ, dK, dV, dG, dK_txt, dV_txt, workspace,
                              stream=None, workspace_bytes=None, check=True) -> int:
    """As vda_backward, reusing what a preceding vda_forward left in `workspace` (same problem and inputs)."""
    wb = _nbytes(workspace) if workspace_bytes is None else workspace_bytes
    s = load().vda_backward_from_forward(ctypes.byref(problem), _ptr(Q), _ptr(K), _ptr(V), _ptr(G), _ptr(K_txt),
                                         _ptr(V_txt), _ptr(dO), _ptr(dQ), _ptr(dK), _ptr(dV), _ptr(dG),
                                         _ptr(dK_txt), _ptr(dV_txt), _ptr(workspace), wb, _stream(stream))
    if check:
        _check(s, "vda_backward_from_forward")
    return s


def vda_host_workspace_size(problem: vda_problem) -> int:
    out = ctypes.c_size_t(0)
    _check(load().vda_host_workspace_size(ctypes.byref(problem), ctypes.byref(out)),
           "vda_host_workspace_size")
    return out.value


def _nbytes(x) -> int:
    if isinstance(x, int):
        return 1 << 62
    return x.numel() * x.element_size()


def vda_forward(problem, Q, K, V, G, K_txt, V_txt, O, workspace, stream=None, workspace_bytes=None,
                check=True) -> int:
    wb = _nbytes(workspace) if workspace_bytes is None else workspace_bytes
    s = load().vda_forward(ctypes.byref(problem), _ptr(Q), _ptr(K), _ptr(V), _ptr(G), _ptr(K_txt),
                           _ptr(V_txt), _ptr(O), _ptr(workspace), wb, _stream(stream))
    if check:
        _check(s, "vda_forward")
    return s


def vda_forward_states(problem, Q, K, V, G, K_txt, V_txt, O, workspace, S_fwd, S_bwd, stream=None,
                       workspace_bytes=None, check=True) -> int:
    wb = _nbytes(workspace) if workspace_bytes is None else workspace_bytes
    s = load().vda_forward_states(ctypes.byref(problem), _ptr(Q), _ptr(K), _ptr(V), _ptr(G),
                                  _ptr(K_txt), _ptr(V_txt), _ptr(O), _ptr(workspace), wb,
                                  _stream(stream), _ptr(S_fwd), _ptr(S_bwd))
    if check:
        _check(s, "vda_forward_states")
    return s


VDA_TIMED_EVENTS = 5
STAGES = ("gram", "factor", "scan", "readout")   # the intervals between the 5 events
# Kernels one forward launches.  With bf16 inputs the Gram and the factor are
# one kernel (the "factor" interval is then empty).
LAUNCHES_PER_FORWARD = {VDA_DTYPE_F32: 4, VDA_DTYPE_BF16: 3, VDA_DTYPE_E4M3: 3}


def vda_forward_timed(problem, Q, K, V, G, K_txt, V_txt, O, workspace, events, stream=None,
                      workspace_bytes=None, check=True) -> int:
    """vda_forward with cudaEvents recorded between the stages (torch.cuda.Event list)."""
    wb = _nbytes(workspace) if workspace_bytes is None else workspace_bytes
    handles = (ctypes.c_void_p * len(events))(*[e.cuda_event if hasattr(e, "cuda_event") else e
                                                for e in events])
    s = load().vda_forward_timed(ctypes.byref(problem), _ptr(Q), _ptr(K), _ptr(V), _ptr(G),
                                 _ptr(K_txt), _ptr(V_txt), _ptr(O), _ptr(workspace), wb,
                                 _stream(stream), handles, len(events))
    if check:
        _check(s, "vda_forward_timed")
    return s


def vda_forward_host(problem, Q, K, V, G, K_txt, V_txt, O, workspace, stream=None,
                     workspace_bytes=None, check=True) -> int:
    """Host buffers in, host O out; copies inside the call; returns after a sync."""
    wb = _nbytes(workspace) if workspace_bytes is None else workspace_bytes
    s = load().vda_forward_host(ctypes.byref(problem), _ptr(Q), _ptr(K), _ptr(V), _ptr(G),
                                _ptr(K_txt), _ptr(V_txt), _ptr(O), _ptr(workspace), wb,
                                _stream(stream))
    if check:
        _check(s, "vda_forward_host")
    return s


VDA_NOALLOC_SCRATCH_BYTES = 64 * 1024 * 1024


def vda_forward_noalloc(problem, Q, K, V, G, K_txt, V_txt, O, stream=None, check=True) -> int:
    """Forward on the library's own static scratch, for callers that cannot allocate.

    Same results as vda_forward; no workspace argument.  Problems needing more
    than VDA_NOALLOC_SCRATCH_BYTES of workspace are rejected; calls that
    overlap on the GPU share the scratch and race.
    """
    s = load().vda_forward_noalloc(ctypes.byref(problem), _ptr(Q), _ptr(K), _ptr(V), _ptr(G),
                                   _ptr(K_txt), _ptr(V_txt), _ptr(O), _stream(stream))
    if check:
        _check(s, "vda_forward_noalloc")
    return s


def vda_local_softmax(problem, Q, K, V, G, K_txt, V_txt, O, workspace, stream=None, workspace_bytes=None,
                      check=True) -> int:
    """The local softmax branch: O = sigmoid(G) * windowed softmax attention (bf16 device buffers)."""
    wb = _nbytes(workspace) if workspace_bytes is None else workspace_bytes
    s = load().vda_local_softmax(ctypes.byref(problem), _ptr(Q), _ptr(K), _ptr(V), _ptr(G), _ptr(K_txt),
                                 _ptr(V_txt), _ptr(O), _ptr(workspace), wb, _stream(stream))
    if check:
        _check(s, "vda_local_softmax")
    return s


def vda_merge_project(tokens, K, D, O_lin, W_lin, O_sm, W_sm, Y, workspace, stream=None, workspace_bytes=None,
                      check=True, test_stall=0) -> int:
    """Y = O_lin W_lin + O_sm W_sm (bf16 device buffers; O_sm, W_sm may be None)."""
    p = vda_merge_problem(int(tokens), int(K), int(D), int(test_stall), 0)
    wb = _nbytes(workspace) if workspace_bytes is None else workspace_bytes
    s = load().vda_merge_project(ctypes.byref(p), _ptr(O_lin), _ptr(W_lin), _ptr(O_sm), _ptr(W_sm), _ptr(Y),
                                 _ptr(workspace), wb, _stream(stream))
    if check:
        _check(s, "vda_merge_project")
    return s


def vda_sync_status(workspace, stream=None, check=True) -> int:
    s = load().vda_sync_status(_ptr(workspace), _stream(stream))
    if check:
        _check(s, "vda_sync_status")
    return s


def vda_status_string(status: int) -> str:
    return load().vda_status_string(int(status)).decode()


def vda_last_error() -> str:
    return load().vda_last_error().decode()


# ---------------------------------------------------------------------------
# Convenience layer (torch tensors in, torch tensor out)
# ---------------------------------------------------------------------------

def problem_for(Q, K, V, G, K_txt, V_txt, lam, scales=None) -> vda_problem:
    """The problem of torch tensors in the [B, H, T, n, d] layout.  float32 and
    bfloat16 tensors take their type; uint8 tensors are E4M3 bit patterns and
    need `scales` = (scale_q, scale_k, scale_v, scale_g)."""
    import torch
    sc = (1.0, 1.0, 1.0, 1.0)
    if Q.dtype == torch.bfloat16:
        dt = VDA_DTYPE_BF16
    elif Q.dtype == torch.float32:
        dt = VDA_DTYPE_F32
    elif Q.dtype in (torch.uint8, torch.float8_e4m3fn):
        dt = VDA_DTYPE_E4M3
        if scales is None:
            raise ValueError("E4M3 inputs need scales=(scale_q, scale_k, scale_v, scale_g)")
        sc = tuple(float(x) for x in scales)
    else:
        raise TypeError(f"unsupported dtype {Q.dtype}")
    for name, x in (("K", K), ("V", V), ("G", G)):
        if x.dtype != Q.dtype:
            raise TypeError(f"{name} has dtype {x.dtype}, Q has {Q.dtype}")
    Bn, Hn, T, n, d_k = Q.shape
    d_v = V.shape[-1]
    n_txt = 0 if K_txt is None else K_txt.shape[2]
    if tuple(K.shape) != (Bn, Hn, T, n, d_k) or tuple(V.shape) != (Bn, Hn, T, n, d_v) \
            or tuple(G.shape) != (Bn, Hn, T, n, d_v):
        raise ValueError("Q, K, V, G shapes disagree")
    if n_txt and (tuple(K_txt.shape) != (Bn, Hn, n_txt, d_k) or tuple(V_txt.shape) != (Bn, Hn, n_txt, d_v)):
        raise ValueError("K_txt, V_txt shapes disagree")
    for x in (Q, K, V, G) + ((K_txt, V_txt) if n_txt else ()):
        if not x.is_cuda or not x.is_contiguous():
            raise ValueError("tensors must be contiguous CUDA tensors")
    return make_problem(Bn, Hn, T, n, n_txt, d_k, d_v, dt, lam, scale_q=sc[0], scale_k=sc[1], scale_v=sc[2],
                        scale_g=sc[3])


def forward(Q, K, V, G, K_txt, V_txt, lam: float, stream=None, workspace=None, out=None, check=False,
            scales=None):
    """O = VDA(Q, K, V, G, K_txt, V_txt; lam) on the inputs' device.

    The call is enqueued on `stream` (default: the current torch stream).  A
    workspace allocated here is allocated on that stream and marked as used by
    it, so torch's caching allocator does not hand its memory to another
    stream while the kernels still run.  check=True synchronises the stream
    and raises on a device-side condition (VDA_ERR_NOT_SPD, VDA_ERR_TIMEOUT).
    """
    import torch
    prob = problem_for(Q, K, V, G, K_txt, V_txt, lam, scales)
    ws_bytes = vda_workspace_size(prob)
    s = torch.cuda.current_stream(Q.device) if stream is None else stream
    if not isinstance(s, torch.cuda.Stream):
        raise TypeError("stream must be a torch.cuda.Stream (or None for the current stream)")
    with torch.cuda.stream(s):
        if workspace is None or _nbytes(workspace) < ws_bytes:
            workspace = torch.empty(ws_bytes, dtype=torch.uint8, device=Q.device)
        odt = torch.bfloat16 if prob.dtype == VDA_DTYPE_E4M3 else G.dtype
        O = out if out is not None else torch.empty(G.shape, dtype=odt, device=G.device)
    txt = prob.n_txt > 0
    vda_forward(prob, Q, K, V, G, K_txt if txt else None, V_txt if txt else None, O, workspace,
                stream=s)
    workspace.record_stream(s)
    O.record_stream(s)
    if check:
        vda_sync_status(workspace, stream=s)
    return O
