"""E4M3 (8-bit float) inputs against the float64 oracle, element by element.

The pages' model runs its linear layers in FP8 ("OpenVDN/vdn-minimax-h3"
(agentlenshq.com), quick-start: the 8nfe_tuned_fp8 inference script; "VDN-H3"
(comfyui-wiki.com), ComfyUI section: FP8 linear layers), so the attention
inputs arrive as 8-bit floats.  Here Q, K, V, G and the text are E4M3 bit
patterns with one scale per tensor; the oracle computes on their exact
widened values (scale times the 8-bit value), so the comparison measures the
kernels' arithmetic, not the 8-bit rounding of the inputs.  O is bfloat16 and
is held to the bfloat16 bar, 2e-2 relative Frobenius error; the float32
states to 2e-3.
"""
import numpy as np
import pytest

from frame_wise_linear_b200 import synth
from vda_testutil import TOL, from_device, oracle, out_like, rel_fro, run_gpu, to_device

pytestmark = pytest.mark.gpu

E8 = synth.DTYPE_E4M3
STATE_TOL = 2e-3
W = synth.WORKLOADS
SMALL = {
    "mid": W["mid"].replace(name="mid_fp8", dtype=E8),
    "ragged_no_text": synth.Workload("fp8_ragged", B=2, H=2, T=3, n=200, n_txt=0, d_k=128, d_v=128, dtype=E8, lam=2.0),
    "one_frame_one_token": synth.Workload("fp8_1x1", B=1, H=3, T=1, n=1, n_txt=1, d_k=128, d_v=128, dtype=E8,
                                          lam=1.0),
    "tail_tile": synth.Workload("fp8_tail", B=1, H=2, T=6, n=1008, n_txt=256, d_k=128, d_v=128, dtype=E8, lam=1.0),
    "ill_small": W["illcond"].replace(name="fp8_ill", dtype=E8, H=2, T=12),
    "text_tail": synth.Workload("fp8_text_tail", B=1, H=2, T=3, n=130, n_txt=200, d_k=128, d_v=128, dtype=E8,
                                lam=0.5),
}


@pytest.mark.parametrize("name", list(SMALL))
def test_fp8_small_workload_whole_tensor(name):
    w = SMALL[name]
    inp = synth.make_inputs(w, seed=0)
    O, SF, SB = run_gpu(inp, states=True)
    Oref, SFref, SBref = oracle(inp, states=True)
    assert np.all(np.isfinite(O))
    e_o = rel_fro(O, Oref.reshape(O.shape))
    e_f = rel_fro(SF, SFref.reshape(SF.shape))
    e_b = rel_fro(SB, SBref.reshape(SB.shape))
    assert e_o <= TOL[E8], (name, e_o)
    assert e_f <= STATE_TOL, (name, e_f)
    assert e_b <= STATE_TOL, (name, e_b)


def test_fp8_scales_enter_as_stated():
    """Doubling a tensor's scale is the same as doubling its values: checked against the oracle."""
    w = synth.Workload("fp8_scales", B=1, H=2, T=4, n=256, n_txt=32, d_k=128, d_v=128, dtype=E8, lam=0.7)
    inp = synth.make_inputs(w, seed=2)
    import torch
    from frame_wise_linear_b200 import vda
    from oracle import vda_oracle as vo
    d = to_device(inp)
    sc = w.scales()
    for which in ("q", "k", "v", "g"):
        kw = dict(w.problem())
        kw["scale_" + which] *= 2.0
        prob = vda.make_problem(**kw)
        ws = torch.empty(vda.vda_workspace_size(prob), dtype=torch.uint8, device="cuda")
        O = out_like(w, d["G"])
        vda.vda_forward(prob, d["Q"], d["K"], d["V"], d["G"], d["K_txt"], d["V_txt"], O, ws)
        vda.vda_sync_status(ws)
        got = from_device(O)
        owner = {"Q": "q", "K": "k", "K_txt": "k", "V": "v", "V_txt": "v", "G": "g"}   # the text takes K's, V's
        mult = {k: 2.0 if owner[k] == which else 1.0 for k in sc}
        for b in range(w.B):
            for h in range(w.H):
                x = {k: synth.widen(getattr(inp, k)[b, h], E8, sc[k] * mult[k]) for k in sc}
                ref = vo.vda_head(x["Q"], x["K"], x["V"], x["G"], x["K_txt"], x["V_txt"], w.lam)
                assert rel_fro(got[b, h], ref) <= TOL[E8], (which, b, h)


@pytest.mark.slow
def test_fp8_768p_sampled_heads():
    import torch
    from frame_wise_linear_b200 import vda
    from oracle import vda_oracle as vo
    w = W["768p_fp8"]
    d = synth.make_inputs_torch(w, seed=0, device="cuda")
    O = vda.forward(d["Q"], d["K"], d["V"], d["G"], d["K_txt"], d["V_txt"], w.lam,
                    scales=tuple(w.scales()[k] for k in ("Q", "K", "V", "G")))
    torch.cuda.synchronize()
    assert O.dtype == torch.bfloat16
    errs = []
    for b, h in [(0, 0), (0, 17), (0, 31)]:
        x = synth.head_widened(w, b, h, seed=0)
        ref = vo.vda_head(x["Q"], x["K"], x["V"], x["G"], x["K_txt"], x["V_txt"], w.lam)
        errs.append(rel_fro(O[b, h].float().cpu().numpy().astype(np.float64), ref))
    assert max(errs) <= TOL[E8], errs


def test_fp8_token_major_layout_is_the_same_arithmetic():
    """[B, T*n, H, d] inputs give O bit-equal (after the permutation) to the [B, H, T, n, d] call."""
    import torch
    from frame_wise_linear_b200 import vda
    w = synth.Workload("fp8_layout", B=2, H=3, T=3, n=300, n_txt=40, d_k=128, d_v=128, dtype=E8, lam=1.0)
    inp = synth.make_inputs(w, seed=5)
    ref = run_gpu(inp)
    d = {k: synth.token_major(v) for k, v in to_device(inp).items()}
    prob = vda.make_problem(**w.problem(), layout=vda.VDA_LAYOUT_BTNHD)
    ws = torch.empty(vda.vda_workspace_size(prob), dtype=torch.uint8, device="cuda")
    O = torch.empty(d["G"].shape, dtype=torch.bfloat16, device="cuda")
    vda.vda_forward(prob, d["Q"], d["K"], d["V"], d["G"], d["K_txt"], d["V_txt"], O, ws)
    vda.vda_sync_status(ws)
    got = from_device(O).reshape(w.B, w.T, w.n, w.H, w.d_v).transpose(0, 3, 1, 2, 4)
    assert np.array_equal(got, ref)
