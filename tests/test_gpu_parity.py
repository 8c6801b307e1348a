"""CUDA path against the float64 oracle, element by element, on seeded inputs.

Tolerances (relative Frobenius error of O over the tensor compared): 1e-4 for
float32 inputs, 2e-2 for bfloat16 inputs.  The per-frame states, which carry
no output rounding, are held to 1e-4 (float32) and 2e-3 (bfloat16).
Full-size workloads run whole on the device, in the launch configuration the
benchmark times, and are compared on sampled heads (every frame and element
of those heads).
"""
import numpy as np
import pytest

from frame_wise_linear_b200 import synth
from vda_testutil import TOL, oracle, rel_fro, run_gpu

pytestmark = pytest.mark.gpu

STATE_TOL = {synth.DTYPE_F32: 1e-4, synth.DTYPE_BF16: 2e-3}

W = synth.WORKLOADS
SMALL = {
    "tiny": W["tiny"],
    "mid": W["mid"],
    "f32_ragged": synth.Workload("f32_ragged", B=2, H=3, T=5, n=200, n_txt=0, d_k=48, d_v=80,
                                 dtype=synth.DTYPE_F32, lam=0.7),
    "f32_single_token": synth.Workload("f32_single_token", B=1, H=2, T=1, n=1, n_txt=3, d_k=16, d_v=32,
                                       dtype=synth.DTYPE_F32, lam=0.3),
    "f32_d128": synth.Workload("f32_d128", B=1, H=2, T=4, n=300, n_txt=20, d_k=128, d_v=128,
                               dtype=synth.DTYPE_F32, lam=1.0),
    "bf16_ragged": synth.Workload("bf16_ragged", B=2, H=2, T=3, n=200, n_txt=0, d_k=128, d_v=128,
                                  dtype=synth.DTYPE_BF16, lam=2.0),
    "bf16_one_frame_one_token": synth.Workload("bf16_1x1", B=1, H=3, T=1, n=1, n_txt=1, d_k=128, d_v=128,
                                               dtype=synth.DTYPE_BF16, lam=1.0),
    "bf16_tail_tile": synth.Workload("bf16_tail", B=1, H=2, T=6, n=1008, n_txt=256, d_k=128, d_v=128,
                                     dtype=synth.DTYPE_BF16, lam=1.0),
    "bf16_ill_small": W["illcond"].replace(name="ill_small", H=2, T=12),
}


@pytest.mark.parametrize("name", list(SMALL))
def test_small_workload_whole_tensor(name):
    w = SMALL[name]
    inp = synth.make_inputs(w, seed=0)
    O, SF, SB = run_gpu(inp, states=True)
    Oref, SFref, SBref = oracle(inp, states=True)
    Oref = Oref.reshape(O.shape)
    SFref = SFref.reshape(SF.shape)
    SBref = SBref.reshape(SB.shape)
    assert np.all(np.isfinite(O))
    e_o = rel_fro(O, Oref)
    e_f = rel_fro(SF, SFref)
    e_b = rel_fro(SB, SBref)
    assert e_o <= TOL[w.dtype], (name, e_o)
    assert e_f <= STATE_TOL[w.dtype], (name, e_f)
    assert e_b <= STATE_TOL[w.dtype], (name, e_b)


def _sampled(name, heads):
    import torch
    from frame_wise_linear_b200 import vda
    w = W[name]
    d = synth.make_inputs_torch(w, seed=0, device="cuda")
    O = vda.forward(d["Q"], d["K"], d["V"], d["G"], d["K_txt"], d["V_txt"], w.lam)
    torch.cuda.synchronize()
    assert bool(torch.isfinite(O.float()).all())
    errs = []
    for b, h in heads:
        x = synth.head_widened(w, b, h, seed=0)
        from oracle import vda_oracle as vo
        ref = vo.vda_head(x["Q"], x["K"], x["V"], x["G"], x["K_txt"], x["V_txt"], w.lam)
        got = O[b, h].float().cpu().numpy().astype(np.float64)
        errs.append(rel_fro(got, ref))
    del d, O
    torch.cuda.empty_cache()
    return errs


@pytest.mark.slow
def test_768p_sampled_heads():
    errs = _sampled("768p", [(0, 0), (0, 13), (0, 31)])
    assert max(errs) <= TOL[synth.DTYPE_BF16], errs


@pytest.mark.slow
def test_ill_conditioned_sampled_heads():
    errs = _sampled("illcond", [(0, 0), (0, 9), (0, 22), (0, 31)])
    assert max(errs) <= TOL[synth.DTYPE_BF16], errs


@pytest.mark.slow
@pytest.mark.parametrize("name", ["long45", "long90", "long180"])
def test_long_clip_sampled_heads(name):
    """The long-clip sweep (B = 2): the first head of batch 0 and the last head of batch 1, every frame."""
    errs = _sampled(name, [(0, 0), (1, 31)])
    assert max(errs) <= TOL[synth.DTYPE_BF16], (name, errs)


def test_repeat_is_bitwise_identical():
    inp = synth.make_inputs(W["mid"], seed=3)
    a = run_gpu(inp)
    b = run_gpu(inp)
    assert np.array_equal(a, b)


@pytest.mark.parametrize("dtype", [synth.DTYPE_F32, synth.DTYPE_BF16])
def test_overflowing_keys_report_not_spd_then_clear(dtype):
    """K^T K overflows float32: the Cholesky pivot is not finite; the device error word says so."""
    import torch
    from frame_wise_linear_b200 import vda
    w = synth.Workload("overflow", B=1, H=1, T=2, n=64, n_txt=4, d_k=128, d_v=128, dtype=dtype, lam=1.0)
    inp = synth.make_inputs(w, seed=0)
    from vda_testutil import to_device
    d = to_device(inp)
    d["K"][0, 0, 1].mul_(1e20)
    prob = vda.make_problem(**{k: v for k, v in w.problem().items()})
    ws = torch.empty(vda.vda_workspace_size(prob), dtype=torch.uint8, device="cuda")
    O = torch.empty_like(d["G"])
    vda.vda_forward(prob, d["Q"], d["K"], d["V"], d["G"], d["K_txt"], d["V_txt"], O, ws)
    assert vda.vda_sync_status(ws, check=False) == vda.VDA_ERR_NOT_SPD
    assert vda.vda_sync_status(ws, check=False) == vda.VDA_OK  # read clears it
    d2 = to_device(inp)
    vda.vda_forward(prob, d2["Q"], d2["K"], d2["V"], d2["G"], d2["K_txt"], d2["V_txt"], O, ws)
    assert vda.vda_sync_status(ws, check=False) == vda.VDA_OK


def test_non_default_stream_and_host_entry_point():
    import torch
    from frame_wise_linear_b200 import vda
    w = W["mid"].replace(H=2, T=5)
    inp = synth.make_inputs(w, seed=1)
    ref = run_gpu(inp)
    from vda_testutil import from_device, to_device
    d = to_device(inp)
    prob = vda.make_problem(**w.problem())
    s = torch.cuda.Stream()
    ws = torch.empty(vda.vda_workspace_size(prob), dtype=torch.uint8, device="cuda")
    O = torch.empty_like(d["G"])
    with torch.cuda.stream(s):
        vda.vda_forward(prob, d["Q"], d["K"], d["V"], d["G"], d["K_txt"], d["V_txt"], O, ws, stream=s)
    vda.vda_sync_status(ws, stream=s)
    assert np.array_equal(from_device(O), ref)
    # host buffers through vda_forward_host
    host = {k: v.cpu().pin_memory() for k, v in d.items()}
    Oh = torch.empty_like(host["G"]).pin_memory()
    wsh = torch.empty(vda.vda_host_workspace_size(prob), dtype=torch.uint8, device="cuda")
    vda.vda_forward_host(prob, host["Q"], host["K"], host["V"], host["G"], host["K_txt"], host["V_txt"],
                         Oh, wsh, stream=s)
    assert np.array_equal(from_device(Oh), ref)
