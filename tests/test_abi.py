"""The C ABI on the host: symbols, argument checks, error codes (no GPU needed).

Every call here fails its host-side checks before anything is enqueued, so no
device pointer is ever dereferenced; the single call that passes the checks
runs only where no CUDA device exists and must then fail loudly.
"""
import ctypes
import os
import re

import pytest

from frame_wise_linear_b200 import build, vda

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    build.build()
    return vda.load()


def _declared_symbols():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            txt = open(os.path.join(ROOT, "include", fn)).read()
            txt = re.sub(r"/\*.*?\*/", "", txt, flags=re.S)
            names |= set(re.findall(r"\b(vda_[a-z_0-9]+)\s*\(", txt))
    return names


def test_every_declared_symbol_is_exported(lib):
    declared = _declared_symbols()
    assert declared, "no entry points found in include/*.h"
    for name in declared:
        assert hasattr(lib, name), f"{name} declared in include/ but not exported"
    assert declared == set(vda.SYMBOLS) | (declared - set(vda.SYMBOLS))
    for name in vda.SYMBOLS:
        assert name in declared, f"binding exposes {name}, which include/ does not declare"


def test_problem_struct_layout():
    # the header's vda_problem: 15 int32 / float fields, no padding; in a
    # zeroed struct the fields added after lambda (layout, test_stall, and
    # the e4m3 scales, which only e4m3 problems read) mean the defaults
    assert ctypes.sizeof(vda.vda_problem) == 60
    assert vda.vda_problem.test_stall.offset == 40
    assert vda.vda_problem.scale_q.offset == 44 and vda.vda_problem.scale_g.offset == 56
    txt = open(os.path.join(ROOT, "include", "vda.h")).read()
    assert "VDA_TEST_STALL_MAX = %d" % max(vda.TEST_STALL_SITES.values()) in txt
    for name, v in vda.TEST_STALL_SITES.items():
        assert "VDA_TEST_STALL_%s = %d" % (name.upper(), v) in txt


def test_merge_problem_struct_layout():
    # the header's vda_merge_problem: int64 tokens, int32 K, D, test_stall, reserved
    assert ctypes.sizeof(vda.vda_merge_problem) == 24
    assert vda.vda_merge_problem.test_stall.offset == 16


def test_merge_bad_problem_rejected(lib):
    ok = 1 << 20
    s = vda.vda_merge_project(128, 128, 64, ok, ok, None, None, ok, ok, stream=0, check=False, test_stall=99)
    assert s == vda.VDA_ERR_INVALID_ARG, vda.vda_last_error()
    s = vda.vda_merge_project(128, 128, 64, ok, ok, None, None, ok, ok, stream=0, check=False, test_stall=-1)
    assert s == vda.VDA_ERR_INVALID_ARG, vda.vda_last_error()


def test_noalloc_refuses_problems_above_its_scratch(lib):
    # the size check comes before anything touches the device: the 768p problem needs about 287 MB
    from frame_wise_linear_b200 import synth
    ok = 1 << 20
    big = vda.make_problem(**synth.WORKLOADS["768p"].problem())
    assert vda.vda_workspace_size(big) > 64 << 20
    s = vda.vda_forward_noalloc(big, *([ok] * 7), stream=0, check=False)
    assert s == vda.VDA_ERR_WORKSPACE
    assert "scratch" in vda.vda_last_error()
    bad = _p(lam=-1.0)
    assert vda.vda_forward_noalloc(bad, *([ok] * 7), stream=0, check=False) == vda.VDA_ERR_INVALID_ARG


def test_backward_refuses_e4m3_and_f32(lib):
    # the backward is built for bf16 inputs (d = 128); other types are refused on the host
    ok = 1 << 20
    for kw in (dict(dtype=vda.VDA_DTYPE_E4M3), dict(dtype=vda.VDA_DTYPE_F32)):
        p = _p(**kw)
        out = ctypes.c_size_t(0)
        assert lib.vda_backward_workspace_size(ctypes.byref(p), ctypes.byref(out)) == vda.VDA_ERR_UNSUPPORTED
        s = vda.vda_backward(p, *([ok] * 7), *([ok] * 6), ok, stream=0, workspace_bytes=1 << 40, check=False)
        assert s == vda.VDA_ERR_UNSUPPORTED, vda.vda_last_error()


def test_local_softmax_bad_arguments_rejected(lib):
    # rejected on the host before any CUDA call; lambda is not read by this branch
    ok = 1 << 20
    args = [ok] * 7
    p = _p(lam=0.0)
    assert vda.vda_local_softmax(p, *args, None, stream=0, workspace_bytes=256, check=False) == vda.VDA_ERR_WORKSPACE
    assert vda.vda_local_softmax(_p(), *args, ok, stream=0, workspace_bytes=255, check=False) == vda.VDA_ERR_WORKSPACE
    assert vda.vda_local_softmax(_p(), *args, ok + 16, stream=0, workspace_bytes=256, check=False) == vda.VDA_ERR_WORKSPACE
    assert vda.vda_local_softmax(_p(dtype=vda.VDA_DTYPE_F32), *args, ok, stream=0, workspace_bytes=256,
                                 check=False) == vda.VDA_ERR_UNSUPPORTED
    assert vda.vda_local_softmax(_p(dtype=vda.VDA_DTYPE_E4M3), *args, ok, stream=0, workspace_bytes=256,
                                 check=False) == vda.VDA_ERR_UNSUPPORTED
    bad = list(args)
    bad[0] = 0
    assert vda.vda_local_softmax(_p(), *bad, ok, stream=0, workspace_bytes=256, check=False) == vda.VDA_ERR_INVALID_ARG
    assert vda.vda_local_softmax(_p(T=0), *args, ok, stream=0, workspace_bytes=256, check=False) == vda.VDA_ERR_INVALID_ARG


def _p(**kw):
    base = dict(B=1, H=2, T=3, n=64, n_txt=8, d_k=128, d_v=128, dtype=vda.VDA_DTYPE_BF16, lam=1.0)
    base.update(kw)
    return vda.make_problem(**base)


@pytest.mark.parametrize("dtype,state_bytes", [(vda.VDA_DTYPE_BF16, 2), (vda.VDA_DTYPE_F32, 4)])
def test_workspace_size_valid(lib, dtype, state_bytes):
    # error word, M and B_t per slot (float32), S^f and S^b per frame (bf16 on
    # the bf16 path, where they are the readout's operands; float32 otherwise)
    p = _p(dtype=dtype)
    nb = vda.vda_workspace_size(p)
    slots, frames = 1 * 2 * 4, 1 * 2 * 3
    assert nb >= 256 + slots * 128 * 128 * 4 * 2 + frames * 128 * 128 * state_bytes * 2
    assert nb < 256 + slots * 128 * 128 * 4 * 2 + frames * 128 * 128 * state_bytes * 2 + 5 * 256
    assert vda.vda_host_workspace_size(p) > nb


@pytest.mark.parametrize("kw,status", [
    (dict(lam=0.0), vda.VDA_ERR_INVALID_ARG),
    (dict(lam=-1.0), vda.VDA_ERR_INVALID_ARG),
    (dict(lam=float("nan")), vda.VDA_ERR_INVALID_ARG),
    (dict(lam=float("inf")), vda.VDA_ERR_INVALID_ARG),
    (dict(B=0), vda.VDA_ERR_INVALID_ARG),
    (dict(T=0), vda.VDA_ERR_INVALID_ARG),
    (dict(n=0), vda.VDA_ERR_INVALID_ARG),
    (dict(n_txt=-1), vda.VDA_ERR_INVALID_ARG),
    (dict(dtype=7), vda.VDA_ERR_INVALID_ARG),
    (dict(d_k=64, d_v=64), vda.VDA_ERR_UNSUPPORTED),            # bf16 needs 128
    (dict(dtype=vda.VDA_DTYPE_F32, d_k=24), vda.VDA_ERR_UNSUPPORTED),
    (dict(dtype=vda.VDA_DTYPE_F32, d_k=256), vda.VDA_ERR_UNSUPPORTED),
    (dict(B=70000), vda.VDA_ERR_UNSUPPORTED),
    (dict(test_stall=-1), vda.VDA_ERR_INVALID_ARG),
    (dict(dtype=vda.VDA_DTYPE_E4M3, scale_q=0.0), vda.VDA_ERR_INVALID_ARG),
    (dict(dtype=vda.VDA_DTYPE_E4M3, scale_v=float("inf")), vda.VDA_ERR_INVALID_ARG),
    (dict(dtype=vda.VDA_DTYPE_E4M3, scale_k=-1.0), vda.VDA_ERR_INVALID_ARG),
    (dict(dtype=vda.VDA_DTYPE_E4M3, d_k=64, d_v=64), vda.VDA_ERR_UNSUPPORTED),
    (dict(test_stall=16), vda.VDA_ERR_INVALID_ARG),
])
def test_bad_problem_rejected(lib, kw, status):
    p = _p(**kw)
    out = ctypes.c_size_t(0)
    s = lib.vda_workspace_size(ctypes.byref(p), ctypes.byref(out))
    assert s == status, vda.vda_last_error()
    assert vda.vda_last_error()
    # and vda_forward rejects it before enqueuing anything
    s = vda.vda_forward(p, 16, 16, 16, 16, 16, 16, 16, 256, stream=0, workspace_bytes=1 << 40, check=False)
    assert s == status


def test_null_and_misaligned_pointers(lib):
    p = _p()
    ok = 1 << 20
    args = [ok] * 7
    for i in range(7):
        a = list(args)
        a[i] = 0
        s = vda.vda_forward(p, *a, ok, stream=0, workspace_bytes=1 << 40, check=False)
        assert s == vda.VDA_ERR_INVALID_ARG, (i, vda.vda_last_error())
        a[i] = ok + 8
        s = vda.vda_forward(p, *a, ok, stream=0, workspace_bytes=1 << 40, check=False)
        assert s == vda.VDA_ERR_INVALID_ARG, (i, vda.vda_last_error())


def test_text_pointers_may_be_null_without_text(lib):
    p = _p(n_txt=0)
    ok = 1 << 20
    # passes the pointer checks, fails on the workspace size instead
    s = vda.vda_forward(p, ok, ok, ok, ok, None, None, ok, ok, stream=0, workspace_bytes=16, check=False)
    assert s == vda.VDA_ERR_WORKSPACE


def test_workspace_checks(lib):
    p = _p()
    ok = 1 << 20
    need = vda.vda_workspace_size(p)
    s = vda.vda_forward(p, *([ok] * 7), None, stream=0, workspace_bytes=need, check=False)
    assert s == vda.VDA_ERR_WORKSPACE
    s = vda.vda_forward(p, *([ok] * 7), ok + 16, stream=0, workspace_bytes=need, check=False)
    assert s == vda.VDA_ERR_WORKSPACE
    s = vda.vda_forward(p, *([ok] * 7), ok, stream=0, workspace_bytes=need - 1, check=False)
    assert s == vda.VDA_ERR_WORKSPACE
    s = vda.vda_forward_states(p, *([ok] * 7), ok, None, ok, stream=0, workspace_bytes=need, check=False)
    assert s == vda.VDA_ERR_INVALID_ARG
    need_h = vda.vda_host_workspace_size(p)
    s = vda.vda_forward_host(p, *([ok] * 7), ok, stream=0, workspace_bytes=need_h - 1, check=False)
    assert s == vda.VDA_ERR_WORKSPACE


def test_status_strings(lib):
    for code in range(7):
        assert vda.vda_status_string(code).startswith("VDA_")
    assert vda.vda_status_string(99) == "VDA_ERR_UNKNOWN"


def _has_cuda():
    try:
        import torch
        return torch.cuda.is_available()
    except Exception:
        return False


@pytest.mark.skipif(_has_cuda(), reason="only meaningful where no CUDA device exists")
def test_no_device_fails_loudly(lib):
    """With every check passed and no GPU, the call reports a CUDA error: no CPU fallback."""
    p = _p()
    ok = 1 << 20
    need = vda.vda_workspace_size(p)
    s = vda.vda_forward(p, *([ok] * 7), ok, stream=0, workspace_bytes=need, check=False)
    assert s == vda.VDA_ERR_CUDA


@pytest.mark.skipif(_has_cuda(), reason="only meaningful where no CUDA device exists")
@pytest.mark.parametrize("entry", ["vda_backward", "vda_backward_from_forward"])
def test_backward_entry_points_checked_and_fail_loudly(lib, entry):
    """Both backward entry points: bf16 only, pointer and workspace checks, then a CUDA error with no GPU."""
    import ctypes
    fn = getattr(vda, entry)
    size = ctypes.c_size_t(0)
    p32 = _p(dtype=vda.VDA_DTYPE_F32)
    assert lib.vda_backward_workspace_size(ctypes.byref(p32), ctypes.byref(size)) == vda.VDA_ERR_UNSUPPORTED
    p = _p()
    need = vda.vda_backward_workspace_size(p)
    ok = 1 << 20
    args = [ok] * 13
    assert fn(p32, *args, ok, stream=0, workspace_bytes=need, check=False) == vda.VDA_ERR_UNSUPPORTED
    bad = list(args)
    bad[7] = 0                                  # dQ
    assert fn(p, *bad, ok, stream=0, workspace_bytes=need, check=False) == vda.VDA_ERR_INVALID_ARG
    assert fn(p, *args, ok, stream=0, workspace_bytes=need - 1, check=False) == vda.VDA_ERR_WORKSPACE
    assert fn(p, *args, ok, stream=0, workspace_bytes=need, check=False) == vda.VDA_ERR_CUDA


def test_layout_checked(lib):
    """An unknown layout is an argument error; the token-major layout needs bf16."""
    import ctypes
    size = ctypes.c_size_t(0)
    bad = _p(layout=2)
    assert lib.vda_workspace_size(ctypes.byref(bad), ctypes.byref(size)) == vda.VDA_ERR_INVALID_ARG
    f32 = _p(dtype=vda.VDA_DTYPE_F32, layout=vda.VDA_LAYOUT_BTNHD)
    assert lib.vda_workspace_size(ctypes.byref(f32), ctypes.byref(size)) == vda.VDA_ERR_UNSUPPORTED
    ok = _p(layout=vda.VDA_LAYOUT_BTNHD)
    assert vda.vda_workspace_size(ok) == vda.vda_workspace_size(_p())
    assert vda.vda_backward_workspace_size(ok) == vda.vda_backward_workspace_size(_p())


@pytest.mark.parametrize("layout", [0, 1])
def test_backward_workspace_extends_the_forward_one(lib, layout):
    """vda_backward_from_forward reads the forward's regions at the forward's offsets, so the backward
    workspace is the forward's plus more (the forward's layout is its prefix)."""
    for kw in (dict(), dict(n_txt=0), dict(T=1), dict(B=2, H=3, T=5, n=1008, n_txt=256)):
        p = _p(layout=layout, **kw)
        assert vda.vda_backward_workspace_size(p) > vda.vda_workspace_size(p)
