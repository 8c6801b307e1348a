"""The token-major layout ([B, T*n, H, d], text [B, n_txt, H, d]) on the GPU.

The same seeded inputs run in both layouts; the kernels do the same
arithmetic per tile, so O and every gradient must agree bit for bit after
the permutation (the default layout is held to the oracle elsewhere).
"""
import pytest

from frame_wise_linear_b200 import synth

pytestmark = pytest.mark.gpu

BF = synth.DTYPE_BF16
CASES = {
    "small_text": synth.Workload("lay_small", B=2, H=3, T=4, n=200, n_txt=20, d_k=128, d_v=128, dtype=BF, lam=0.5),
    "no_text": synth.Workload("lay_no_text", B=1, H=2, T=3, n=130, n_txt=0, d_k=128, d_v=128, dtype=BF, lam=1.0),
    "tail": synth.Workload("lay_tail", B=1, H=2, T=2, n=1008, n_txt=256, d_k=128, d_v=128, dtype=BF, lam=1.0),
}


def _untok(x, w, text=False):
    if x is None:
        return None
    if text:
        return x.permute(0, 2, 1, 3).contiguous()
    return x.reshape(w.B, w.T, w.n, w.H, 128).permute(0, 3, 1, 2, 4).contiguous()


def _forward(w, d, layout):
    import torch
    from frame_wise_linear_b200 import vda
    prob = vda.make_problem(**w.problem(), layout=layout)
    ws = torch.empty(vda.vda_workspace_size(prob), dtype=torch.uint8, device="cuda")
    O = torch.empty_like(d["G"])
    txt = w.n_txt > 0
    vda.vda_forward(prob, d["Q"], d["K"], d["V"], d["G"], d["K_txt"] if txt else None, d["V_txt"] if txt else None,
                    O, ws)
    vda.vda_sync_status(ws)
    return O


def _backward(w, d, dO, layout):
    import torch
    from frame_wise_linear_b200 import vda
    prob = vda.make_problem(**w.problem(), layout=layout)
    ws = torch.empty(vda.vda_backward_workspace_size(prob), dtype=torch.uint8, device="cuda")
    txt = w.n_txt > 0
    out = [torch.empty_like(d[k]) for k in ("Q", "K", "V", "G")]
    tout = [torch.empty_like(d["K_txt"]), torch.empty_like(d["V_txt"])] if txt else [None, None]
    vda.vda_backward(prob, d["Q"], d["K"], d["V"], d["G"], d["K_txt"] if txt else None,
                     d["V_txt"] if txt else None, dO, *out, *tout, ws)
    vda.vda_sync_status(ws)
    return out + tout


def _inputs(w):
    d = synth.make_inputs_torch(w, seed=0, device="cuda")
    dO = synth.grad_out_torch(w, seed=0, device="cuda")
    dt = {k: synth.token_major(v) if v is not None else None for k, v in d.items()}
    return d, dO, dt, synth.token_major(dO)


@pytest.mark.parametrize("name", list(CASES))
def test_token_major_forward_bitwise(name):
    import torch
    w = CASES[name]
    d, _, dt, _ = _inputs(w)
    O0 = _forward(w, d, 0)
    O1 = _forward(w, dt, 1)
    assert O1.shape == (w.B, w.T * w.n, w.H, 128)
    assert torch.equal(_untok(O1, w), O0)


@pytest.mark.parametrize("name", list(CASES))
def test_token_major_backward_bitwise(name):
    import torch
    w = CASES[name]
    d, dO, dt, dOt = _inputs(w)
    g0 = _backward(w, d, dO, 0)
    g1 = _backward(w, dt, dOt, 1)
    for i, k in enumerate(("dQ", "dK", "dV", "dG")):
        assert torch.equal(_untok(g1[i], w), g0[i]), k
    if w.n_txt > 0:
        for i, k in ((4, "dK_txt"), (5, "dV_txt")):
            assert torch.equal(_untok(g1[i], w, text=True), g0[i]), k


def test_token_major_768p_forward_bitwise():
    import torch
    w = synth.WORKLOADS["768p"]
    d = synth.make_inputs_torch(w, seed=0, device="cuda")
    O0 = _forward(w, d, 0)
    dt = {k: synth.token_major(v) for k, v in d.items()}
    del d
    O1 = _forward(w, dt, 1)
    assert torch.equal(_untok(O1, w), O0)
