"""Helpers shared by the tests: device upload of seeded inputs, oracle calls, error metrics."""
from __future__ import annotations

import numpy as np

from frame_wise_linear_b200 import synth

# Relative Frobenius tolerance on O, by input dtype: 1e-4 for float32 inputs,
# 2e-2 for bfloat16 inputs; E4M3 inputs produce a bfloat16 O through the same
# bf16 state operands and bf16 output rounding, so they take the bfloat16 bar
# (the comparison is against the oracle on the exact widened 8-bit inputs).
TOL = {synth.DTYPE_F32: 1e-4, synth.DTYPE_BF16: 2e-2, synth.DTYPE_E4M3: 2e-2}


def rel_fro(a, b) -> float:
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


def to_device(inp: synth.Inputs):
    import torch
    dt = {synth.DTYPE_BF16: torch.bfloat16, synth.DTYPE_E4M3: torch.uint8}.get(inp.workload.dtype, torch.float32)

    def up(a):
        t = torch.from_numpy(np.ascontiguousarray(a))
        if dt == torch.bfloat16:
            t = t.view(torch.int16).view(torch.bfloat16)
        return t.cuda()

    return {k: up(getattr(inp, k)) for k in ("Q", "K", "V", "G", "K_txt", "V_txt")}


def from_device(t) -> np.ndarray:
    import torch
    if t.dtype == torch.bfloat16:
        bits = t.view(torch.int16).cpu().numpy().view(np.uint16)
        return synth.bf16_bits_to_f32(bits).astype(np.float64)
    return t.detach().cpu().numpy().astype(np.float64)


def out_like(w: synth.Workload, G):
    """An O buffer for the workload: G's shape, float32 or bfloat16 (bfloat16 for E4M3 inputs)."""
    import torch
    return torch.empty(G.shape, dtype=torch.float32 if w.dtype == synth.DTYPE_F32 else torch.bfloat16,
                       device=G.device)


def run_gpu(inp: synth.Inputs, states: bool = False):
    """Runs the library on a workload's inputs; returns O (float64) and optionally the states."""
    import torch
    from frame_wise_linear_b200 import vda
    w = inp.workload
    d = to_device(inp)
    prob = vda.make_problem(**w.problem())
    ws = torch.empty(vda.vda_workspace_size(prob), dtype=torch.uint8, device="cuda")
    O = out_like(w, d["G"])
    txt = w.n_txt > 0
    kt = d["K_txt"] if txt else None
    vt = d["V_txt"] if txt else None
    if states:
        SF = torch.empty((w.B, w.H, w.T, w.d_k, w.d_v), dtype=torch.float32, device="cuda")
        SB = torch.empty_like(SF)
        vda.vda_forward_states(prob, d["Q"], d["K"], d["V"], d["G"], kt, vt, O, ws, SF, SB)
    else:
        vda.vda_forward(prob, d["Q"], d["K"], d["V"], d["G"], kt, vt, O, ws)
    vda.vda_sync_status(ws)
    out = from_device(O)
    if states:
        return out, SF.cpu().numpy().astype(np.float64), SB.cpu().numpy().astype(np.float64)
    return out


def oracle(inp: synth.Inputs, heads=None, states: bool = False):
    """Float64 oracle on the same inputs (all heads, or a list of (b, h))."""
    from oracle import vda_oracle as vo
    w = inp.workload
    pairs = heads if heads is not None else [(b, h) for b in range(w.B) for h in range(w.H)]
    outs, sfs, sbs = [], [], []
    for b, h in pairs:
        f = lambda k: inp.widened(k, (b, h))  # noqa: E731
        kt = f("K_txt") if w.n_txt else None
        vt = f("V_txt") if w.n_txt else None
        r = vo.vda_head(f("Q"), f("K"), f("V"), f("G"), kt, vt, w.lam, return_states=states)
        if states:
            outs.append(r[0])
            sfs.append(r[1]["SF"])
            sbs.append(r[1]["SB"])
        else:
            outs.append(r)
    if states:
        return np.stack(outs), np.stack(sfs), np.stack(sbs)
    return np.stack(outs)
