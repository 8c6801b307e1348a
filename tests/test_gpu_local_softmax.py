"""The local softmax branch (vda_local_softmax) against the float64 oracle.

"VDN-MiniMax-H3" (aiezz.com), section 03, local softmax branch item: blocks of
5 frames attending to their neighbouring blocks, the first and last frames
as anchors, the whole text, and the branch's sigmoid gate.  The oracle
(oracle/softmax_oracle.py) computes on the exact widened bf16 inputs, so the
comparison measures the kernel's float32 scores and softmax, its bf16 P
operand and the bf16 rounding of O: held to the bf16 bar, 2e-2 relative
Frobenius error.
"""
import numpy as np
import pytest

from frame_wise_linear_b200 import synth
from vda_testutil import TOL, from_device, rel_fro, to_device

pytestmark = pytest.mark.gpu
W = synth.WORKLOADS


def _run(w, inp, layout=0):
    import torch
    from frame_wise_linear_b200 import vda
    d = to_device(inp)
    if layout:
        d = {k: synth.token_major(v) for k, v in d.items()}
    prob = vda.make_problem(**w.problem(), layout=layout)
    O = torch.full_like(d["G"], float("nan"))
    ws = torch.empty(256, dtype=torch.uint8, device="cuda")
    txt = w.n_txt > 0
    vda.vda_local_softmax(prob, d["Q"], d["K"], d["V"], d["G"], d["K_txt"] if txt else None,
                          d["V_txt"] if txt else None, O, ws)
    vda.vda_sync_status(ws)
    return from_device(O)


def _oracle(w, inp, heads=None, frames=None):
    from oracle import softmax_oracle as so
    out = {}
    for b, h in heads or [(b, h) for b in range(w.B) for h in range(w.H)]:
        x = {k: inp.widened(k, (b, h)) for k in ("Q", "K", "V", "G", "K_txt", "V_txt")}
        out[(b, h)] = so.local_softmax_head(x["Q"], x["K"], x["V"], x["G"], x["K_txt"] if w.n_txt else None,
                                            x["V_txt"] if w.n_txt else None)
    return out


CASES = {
    "ragged_text": synth.Workload("ls_ragged", B=1, H=2, T=12, n=200, n_txt=40, d_k=128, d_v=128,
                                  dtype=synth.DTYPE_BF16, lam=1.0),
    "short_no_text": synth.Workload("ls_short", B=2, H=1, T=7, n=128, n_txt=0, d_k=128, d_v=128,
                                    dtype=synth.DTYPE_BF16, lam=1.0),
    "anchors": synth.Workload("ls_anchor", B=1, H=1, T=30, n=64, n_txt=16, d_k=128, d_v=128,
                              dtype=synth.DTYPE_BF16, lam=1.0),
    "one_frame_one_token": synth.Workload("ls_1x1", B=1, H=2, T=1, n=1, n_txt=3, d_k=128, d_v=128,
                                          dtype=synth.DTYPE_BF16, lam=1.0),
    "tail_tile": synth.Workload("ls_tail", B=1, H=1, T=11, n=1008, n_txt=256, d_k=128, d_v=128,
                                dtype=synth.DTYPE_BF16, lam=1.0),
}


@pytest.mark.parametrize("name", list(CASES))
def test_local_softmax_whole_tensor(name):
    w = CASES[name]
    inp = synth.make_inputs(w, seed=6)
    O = _run(w, inp)
    assert np.all(np.isfinite(O))
    ref = _oracle(w, inp)
    for (b, h), r in ref.items():
        assert rel_fro(O[b, h], r) <= TOL[synth.DTYPE_BF16], (name, b, h, rel_fro(O[b, h], r))


def test_local_softmax_token_major_layout_is_the_same_arithmetic():
    w = CASES["ragged_text"].replace(B=2, H=3)
    inp = synth.make_inputs(w, seed=8)
    ref = _run(w, inp)
    got = _run(w, inp, layout=1).reshape(w.B, w.T, w.n, w.H, w.d_v).transpose(0, 3, 1, 2, 4)
    assert np.array_equal(got, ref)


@pytest.mark.slow
def test_local_softmax_768p_sampled_frames():
    """The 768p clip's shapes, every head computed; head (0, 5), frames 0, 22 and 44 against the oracle."""
    import torch
    from frame_wise_linear_b200 import vda
    from oracle import softmax_oracle as so
    w = W["768p"]
    d = synth.make_inputs_torch(w, seed=0, device="cuda")
    prob = vda.make_problem(**w.problem())
    O = torch.empty_like(d["G"])
    ws = torch.empty(256, dtype=torch.uint8, device="cuda")
    vda.vda_local_softmax(prob, d["Q"], d["K"], d["V"], d["G"], d["K_txt"], d["V_txt"], O, ws)
    vda.vda_sync_status(ws)
    x = synth.head_widened(w, 0, 5, seed=0)
    got = O[0, 5].float().cpu().numpy().astype(np.float64)
    for t in (0, 22, 44):
        ref = so.local_softmax_frame(x["Q"], x["K"], x["V"], x["G"], x["K_txt"], x["V_txt"], t)
        assert rel_fro(got[t], ref) <= TOL[synth.DTYPE_BF16], (t, rel_fro(got[t], ref))
