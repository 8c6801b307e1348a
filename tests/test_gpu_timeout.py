"""Device timeout path: a bounded wait that runs out ends the call with VDA_ERR_TIMEOUT.

Every wait inside the tensor-core kernels gives up after 2 s of the GPU's
global timer; the kernel then sets the timeout bit of the error word and
winds down (its other warps stop at their next decision point, its copies and
MMAs complete, its tensor memory is released).  The testing hook
``vda_problem.test_stall`` makes one named wait, in one CTA of its kernel
(the first, or for the operands site the last), wait on a barrier that nothing
signals, so it runs out exactly as a
wait on a lost signal would.  Nothing faults: the hook only chooses which
barrier a bounded wait watches.

Each case checks that the stalled call is enqueued, that the stream finishes
within a bound, that vda_sync_status() reports VDA_ERR_TIMEOUT and clears it,
and that a normal call afterwards on the same workspace returns VDA_OK with
the same outputs, bit for bit, as a call made before the stalled one (the
device and the library stay usable).
"""
import time

import numpy as np
import pytest

from frame_wise_linear_b200 import synth
from vda_testutil import from_device, to_device

pytestmark = pytest.mark.gpu

# 320 frames of one 128-token tile over 148 CTAs: the first CTA of every
# persistent kernel gets two tiles (two frames), and the Gram+factor kernel's
# first CTA starts with a text slot of 16 tokens, so every site is reached.
W = synth.Workload("stall", B=1, H=4, T=80, n=128, n_txt=16, d_k=128, d_v=128, dtype=synth.DTYPE_BF16, lam=1.0)
FORWARD_SITES = ["gram_stage", "factor_update", "service_gram", "scan_operand", "scan_product",
                 "readout_tile", "readout_gate", "readout_state"]
BACKWARD_SITES = ["rbwd_tile", "rbwd_dq", "operands", "gbwd_tile", "gbwd_store"]
OTHER_SITES = ["merge", "softmax"]
BOUND_S = 30.0   # a stalled call ends within a few 2 s wait limits


def _setup():
    import torch
    from frame_wise_linear_b200 import vda
    d = to_device(synth.make_inputs(W, seed=4))
    dO = synth.grad_out_torch(W, seed=4, device="cuda")
    prob = vda.make_problem(**W.problem())
    ws = torch.empty(vda.vda_backward_workspace_size(prob), dtype=torch.uint8, device="cuda")
    return d, dO, prob, ws


def _forward(d, prob, ws):
    import torch
    from frame_wise_linear_b200 import vda
    O = torch.empty_like(d["G"])
    vda.vda_forward(prob, d["Q"], d["K"], d["V"], d["G"], d["K_txt"], d["V_txt"], O, ws)
    return O


def _backward(d, dO, prob, ws):
    import torch
    from frame_wise_linear_b200 import vda
    outs = [torch.empty_like(d[k]) for k in ("Q", "K", "V", "G", "K_txt", "V_txt")]
    vda.vda_backward(prob, d["Q"], d["K"], d["V"], d["G"], d["K_txt"], d["V_txt"], dO, *outs, ws)
    return outs


def _stalled(run, site):
    """Runs `run(problem)` with the wait at `site` made to run out; returns (status, seconds)."""
    import torch
    from frame_wise_linear_b200 import vda
    prob = vda.make_problem(**W.problem(), test_stall=vda.TEST_STALL_SITES[site])
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    ws = run(prob)
    status = vda.vda_sync_status(ws, check=False)
    if status not in (vda.VDA_OK, vda.VDA_ERR_TIMEOUT):
        print("stalled call at", site, ":", vda.vda_status_string(status), vda.vda_last_error())
    return status, time.perf_counter() - t0


@pytest.mark.parametrize("site", FORWARD_SITES)
def test_forward_wait_that_runs_out_reports_timeout(site):
    from frame_wise_linear_b200 import vda
    d, _, prob, ws = _setup()
    ref = from_device(_forward(d, prob, ws))
    assert vda.vda_sync_status(ws, check=False) == vda.VDA_OK
    status, dt = _stalled(lambda pr: (_forward(d, pr, ws), ws)[1], site)
    assert status == vda.VDA_ERR_TIMEOUT, (site, vda.vda_status_string(status))
    assert dt < BOUND_S, (site, dt)
    assert vda.vda_sync_status(ws, check=False) == vda.VDA_OK     # the read cleared it
    again = _forward(d, prob, ws)
    assert vda.vda_sync_status(ws, check=False) == vda.VDA_OK
    assert np.array_equal(from_device(again), ref), site


@pytest.mark.parametrize("site", BACKWARD_SITES)
def test_backward_wait_that_runs_out_reports_timeout(site):
    from frame_wise_linear_b200 import vda
    d, dO, prob, ws = _setup()
    ref = [from_device(t) for t in _backward(d, dO, prob, ws)]
    assert vda.vda_sync_status(ws, check=False) == vda.VDA_OK
    status, dt = _stalled(lambda pr: (_backward(d, dO, pr, ws), ws)[1], site)
    assert status == vda.VDA_ERR_TIMEOUT, (site, vda.vda_status_string(status))
    assert dt < BOUND_S, (site, dt)
    again = [from_device(t) for t in _backward(d, dO, prob, ws)]
    assert vda.vda_sync_status(ws, check=False) == vda.VDA_OK
    for a, b in zip(again, ref):
        assert np.array_equal(a, b), site


W8 = W.replace(name="stall_e4m3", dtype=synth.DTYPE_E4M3)


@pytest.mark.parametrize("site", ["gram_stage", "factor_update", "service_gram", "readout_tile", "readout_gate",
                                  "readout_state"])
def test_e4m3_forward_wait_that_runs_out_reports_timeout(site):
    """The e4m3 variants of the Gram+factor and readout kernels (their own loads, widening and epilogue)."""
    import torch
    from frame_wise_linear_b200 import vda
    from vda_testutil import out_like
    d = to_device(synth.make_inputs(W8, seed=5))
    prob = vda.make_problem(**W8.problem())
    ws = torch.empty(vda.vda_workspace_size(prob), dtype=torch.uint8, device="cuda")

    def fwd(pr):
        O = out_like(W8, d["G"])
        vda.vda_forward(pr, d["Q"], d["K"], d["V"], d["G"], d["K_txt"], d["V_txt"], O, ws)
        return O

    ref = from_device(fwd(prob))
    assert vda.vda_sync_status(ws, check=False) == vda.VDA_OK
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    fwd(vda.make_problem(**W8.problem(), test_stall=vda.TEST_STALL_SITES[site]))
    status = vda.vda_sync_status(ws, check=False)
    dt = time.perf_counter() - t0
    assert status == vda.VDA_ERR_TIMEOUT, (site, vda.vda_status_string(status), vda.vda_last_error())
    assert dt < BOUND_S, (site, dt)
    again = from_device(fwd(prob))
    assert vda.vda_sync_status(ws, check=False) == vda.VDA_OK
    assert np.array_equal(again, ref), site


def _merge(ws, stall=0):
    """One merge of 4096 tokens (32 row tiles, so the first CTA has one), K = 128, D = 256, both branches."""
    import torch
    from frame_wise_linear_b200 import vda
    g = torch.Generator(device="cuda").manual_seed(11)
    O, P = (torch.randn(4096, 128, device="cuda", generator=g).to(torch.bfloat16) for _ in range(2))
    Wl, Ws = (torch.randn(128, 256, device="cuda", generator=g).mul_(0.09).to(torch.bfloat16) for _ in range(2))
    Y = torch.empty(4096, 256, dtype=torch.bfloat16, device="cuda")
    vda.vda_merge_project(4096, 128, 256, O, Wl, P, Ws, Y, ws, test_stall=stall)
    return Y


def _softmax(d, prob, ws):
    import torch
    from frame_wise_linear_b200 import vda
    O = torch.empty_like(d["G"])
    vda.vda_local_softmax(prob, d["Q"], d["K"], d["V"], d["G"], d["K_txt"], d["V_txt"], O, ws)
    return O


@pytest.mark.parametrize("site", OTHER_SITES)
def test_merge_and_local_softmax_wait_that_runs_out_reports_timeout(site):
    import torch
    from frame_wise_linear_b200 import vda
    d, _, prob, _ = _setup()
    ws = torch.empty(256, dtype=torch.uint8, device="cuda")
    if site == "merge":
        run = lambda stall: _merge(ws, stall)
    else:
        run = lambda stall: _softmax(d, vda.make_problem(**W.problem(), test_stall=stall), ws)
    ref = from_device(run(0))
    assert vda.vda_sync_status(ws, check=False) == vda.VDA_OK
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    run(vda.TEST_STALL_SITES[site])
    status = vda.vda_sync_status(ws, check=False)
    dt = time.perf_counter() - t0
    assert status == vda.VDA_ERR_TIMEOUT, (site, vda.vda_status_string(status), vda.vda_last_error())
    assert dt < BOUND_S, (site, dt)
    again = from_device(run(0))
    assert vda.vda_sync_status(ws, check=False) == vda.VDA_OK
    assert np.array_equal(again, ref), site


def test_every_site_is_covered():
    from frame_wise_linear_b200 import vda
    assert sorted(FORWARD_SITES + BACKWARD_SITES + OTHER_SITES) == sorted(vda.TEST_STALL_SITES)
