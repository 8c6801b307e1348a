"""Parity of the GPU backward (vda_backward) with the float64 oracle's.

Every gradient (dQ, dK, dV, dG, dK_txt, dV_txt) is compared element by
element with ``vda_head_backward`` on the same seeded bf16 inputs and dO, as
a relative Frobenius error per tensor.  Small workloads are compared whole;
the 768p workload runs whole on the device and is compared on sampled heads.
"""
import numpy as np
import pytest

from frame_wise_linear_b200 import synth

pytestmark = pytest.mark.gpu

# bf16 inputs and gradients: the same bar as the forward's O.
BWD_TOL = 2e-2

BF = synth.DTYPE_BF16
SMALL = {
    "bwd_small": synth.Workload("bwd_small", B=1, H=2, T=4, n=200, n_txt=20, d_k=128, d_v=128, dtype=BF, lam=0.5),
    "bwd_no_text": synth.Workload("bwd_no_text", B=2, H=1, T=3, n=130, n_txt=0, d_k=128, d_v=128, dtype=BF, lam=1.0),
    "bwd_one_frame": synth.Workload("bwd_one_frame", B=1, H=2, T=1, n=64, n_txt=8, d_k=128, d_v=128, dtype=BF,
                                    lam=1.0),
    "bwd_tail": synth.Workload("bwd_tail", B=1, H=1, T=2, n=1008, n_txt=256, d_k=128, d_v=128, dtype=BF, lam=1.0),
}
NAMES = ("dQ", "dK", "dV", "dG", "dK_txt", "dV_txt")


def _run_gpu(w, seed=0, from_forward=False, raw=False):
    import torch
    from frame_wise_linear_b200 import vda
    from vda_testutil import from_device
    d = synth.make_inputs_torch(w, seed=seed, device="cuda")
    dO = synth.grad_out_torch(w, seed=seed, device="cuda")
    prob = vda.make_problem(w.B, w.H, w.T, w.n, w.n_txt, w.d_k, w.d_v, w.dtype, w.lam)
    ws = torch.empty(vda.vda_backward_workspace_size(prob), dtype=torch.uint8, device="cuda")
    out = {"dQ": torch.empty_like(d["Q"]), "dK": torch.empty_like(d["K"]), "dV": torch.empty_like(d["V"]),
           "dG": torch.empty_like(d["G"])}
    txt = w.n_txt > 0
    out["dK_txt"] = torch.empty_like(d["K_txt"]) if txt else None
    out["dV_txt"] = torch.empty_like(d["V_txt"]) if txt else None
    args = (prob, d["Q"], d["K"], d["V"], d["G"], d["K_txt"] if txt else None, d["V_txt"] if txt else None)
    if from_forward:
        # The forward's own output, then the backward on what it left in the workspace.
        O = torch.empty_like(d["G"])
        vda.vda_forward(*args, O, ws)
        vda.vda_backward_from_forward(*args, dO, out["dQ"], out["dK"], out["dV"], out["dG"], out["dK_txt"],
                                      out["dV_txt"], ws)
    else:
        vda.vda_backward(*args, dO, out["dQ"], out["dK"], out["dV"], out["dG"], out["dK_txt"], out["dV_txt"], ws)
    vda.vda_sync_status(ws)
    if raw:
        return out
    return {k: (from_device(v) if v is not None else None) for k, v in out.items()}


def _oracle(w, b, h, seed=0):
    from oracle import vda_oracle as vo
    f = synth.head_widened(w, b, h, seed)
    txt = w.n_txt > 0
    return vo.vda_head_backward(f["Q"], f["K"], f["V"], f["G"], f["K_txt"] if txt else None,
                                f["V_txt"] if txt else None, w.lam, synth.head_grad_out_widened(w, b, h, seed))


def _compare(w, got, heads):
    from vda_testutil import rel_fro
    errs = {}
    for b, h in heads:
        ref = _oracle(w, b, h)
        for k in NAMES:
            if ref[k] is None:
                assert w.n_txt == 0
                continue
            errs[(b, h, k)] = rel_fro(got[k][b, h], ref[k])
    return errs


@pytest.mark.parametrize("name", list(SMALL))
def test_backward_small(name):
    w = SMALL[name]
    got = _run_gpu(w)
    errs = _compare(w, got, [(b, h) for b in range(w.B) for h in range(w.H)])
    assert max(errs.values()) <= BWD_TOL, errs
    for k in ("dQ", "dK", "dV", "dG"):
        assert np.isfinite(got[k]).all(), k


def test_backward_768p_sampled_heads():
    w = synth.WORKLOADS["768p"]
    got = _run_gpu(w)
    errs = _compare(w, got, [(0, 0), (0, 17)])
    assert max(errs.values()) <= BWD_TOL, errs


@pytest.mark.parametrize("name", ["bwd_small", "bwd_no_text", "bwd_tail"])
def test_backward_from_forward_small(name):
    """vda_backward_from_forward after vda_forward: the oracle's gradients, and bit for bit the recomputing call's."""
    import torch
    w = SMALL[name]
    got = _run_gpu(w, from_forward=True)
    errs = _compare(w, got, [(b, h) for b in range(w.B) for h in range(w.H)])
    assert max(errs.values()) <= BWD_TOL, errs
    a = _run_gpu(w, raw=True)
    b = _run_gpu(w, from_forward=True, raw=True)
    for k in NAMES:
        if a[k] is not None:
            assert torch.equal(a[k], b[k]), k


def test_backward_from_forward_768p_equals_recompute():
    import torch
    w = synth.WORKLOADS["768p"]
    a = _run_gpu(w, raw=True)
    b = _run_gpu(w, from_forward=True, raw=True)
    for k in NAMES:
        assert torch.equal(a[k], b[k]), k
