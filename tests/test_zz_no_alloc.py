"""vda_forward_noalloc: the forward for callers that cannot allocate device memory.

Such callers (code whose device memory is owned by a framework's allocator or
a fixed budget, or that may not let cudaMalloc synchronise the device) can't
provide a workspace, so the library runs on a static scratch array of its own.
These tests call the entry point through the C ABI and check that it gives
what vda_forward gives with a caller-provided workspace, on two different
calls in a row (the scratch keeps the previous call's contents), and that a
problem too large for the scratch is refused before anything runs.

This file is collected last on purpose, and it also passes alone in a fresh
process.
"""
import numpy as np
import pytest

from frame_wise_linear_b200 import synth
from vda_testutil import from_device, rel_fro, to_device

pytestmark = pytest.mark.gpu


def _reference_and_noalloc(w, seed):
    import torch
    from frame_wise_linear_b200 import vda
    inp = synth.make_inputs(w, seed=seed)
    d = to_device(inp)
    prob = vda.make_problem(**w.problem())
    kt = d["K_txt"] if w.n_txt else None
    vt = d["V_txt"] if w.n_txt else None
    ws = torch.empty(vda.vda_workspace_size(prob), dtype=torch.uint8, device="cuda")
    O_ref = torch.empty_like(d["G"])
    vda.vda_forward(prob, d["Q"], d["K"], d["V"], d["G"], kt, vt, O_ref, ws)
    vda.vda_sync_status(ws)
    O = torch.full_like(d["G"], float("nan"))
    vda.vda_forward_noalloc(prob, d["Q"], d["K"], d["V"], d["G"], kt, vt, O)
    torch.cuda.synchronize()
    return from_device(O), from_device(O_ref)


def test_noalloc_matches_forward_on_two_calls_in_a_row():
    from frame_wise_linear_b200 import vda
    first = synth.WORKLOADS["mid"]
    second = synth.Workload("noalloc_second", B=2, H=3, T=5, n=200, n_txt=0, d_k=128, d_v=128,
                            dtype=synth.DTYPE_BF16, lam=2.0)
    for w, seed in ((first, 0), (second, 7)):
        prob = vda.make_problem(**w.problem())
        assert vda.vda_workspace_size(prob) <= vda.VDA_NOALLOC_SCRATCH_BYTES
        O, O_ref = _reference_and_noalloc(w, seed)
        assert np.all(np.isfinite(O)), w.name
        # The same kernels on the same inputs: any stale scratch content or
        # wrong offset would show up as a difference, so equality is exact.
        assert np.array_equal(O, O_ref), (w.name, rel_fro(O, O_ref))


def test_noalloc_refuses_a_problem_larger_than_its_scratch():
    import torch
    from frame_wise_linear_b200 import vda
    w = synth.WORKLOADS["768p"]
    prob = vda.make_problem(**w.problem())
    assert vda.vda_workspace_size(prob) > vda.VDA_NOALLOC_SCRATCH_BYTES
    buf = torch.empty(1024, dtype=torch.uint8, device="cuda")   # never read: the call is refused first
    s = vda.vda_forward_noalloc(prob, buf, buf, buf, buf, buf, buf, buf, check=False)
    assert s == vda.VDA_ERR_WORKSPACE
    assert "static scratch" in vda.vda_last_error()
