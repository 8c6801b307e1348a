"""The branch merge (vda_merge_project) against the float64 oracle.

"VDN-MiniMax-H3" (aiezz.com), section 03, gate fusion item: each branch's
gated output goes through its own output projection and the two are summed,
Y = O_lin W_lin + O_sm W_sm.  Inputs are seeded bf16 tensors; the oracle
computes on their exact widened values, so the comparison measures the
kernel's float32 accumulation and the bf16 rounding of Y (2^-9 relative):
held to the bf16 bar, 2e-2 relative Frobenius error, per row block or over
sampled rows at full size.
"""
import numpy as np
import pytest

from frame_wise_linear_b200 import synth
from vda_testutil import TOL, from_device, rel_fro

pytestmark = pytest.mark.gpu


def _bf16(rng, shape, std=1.0):
    import torch
    bits = synth.to_bf16_bits((rng.standard_normal(shape) * std).astype(np.float32))
    return torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).cuda(), synth.bf16_bits_to_f32(bits).astype(np.float64)


def _run(tokens, K, D, two, seed, rows=None):
    import torch
    from frame_wise_linear_b200 import vda
    from oracle import merge_oracle as mo
    rng = np.random.default_rng(seed)
    O, On = _bf16(rng, (tokens, K))
    W, Wn = _bf16(rng, (K, D), 1.0 / np.sqrt(K))
    if two:
        P, Pn = _bf16(rng, (tokens, K))
        Ws, Wsn = _bf16(rng, (K, D), 1.0 / np.sqrt(K))
    else:
        P = Pn = Ws = Wsn = None
    Y = torch.full((tokens, D), float("nan"), dtype=torch.bfloat16, device="cuda")
    ws = torch.empty(256, dtype=torch.uint8, device="cuda")
    vda.vda_merge_project(tokens, K, D, O, W, P, Ws, Y, ws)
    vda.vda_sync_status(ws)
    got = from_device(Y)
    idx = np.arange(tokens) if rows is None else rows
    ref = mo.merge_project(On[idx], Wn, None if Pn is None else Pn[idx], Wsn)
    return got[idx], ref


@pytest.mark.parametrize("tokens,K,D,two", [
    (300, 128, 200, True),      # ragged rows, columns short of one 256-wide tile
    (128, 64, 8, False),        # one tile, the narrowest output, one branch
    (1000, 512, 768, True),
    (257, 256, 520, False),     # one row and eight columns past the tiles
])
def test_merge_small_whole(tokens, K, D, two):
    got, ref = _run(tokens, K, D, two, seed=tokens + K)
    assert np.all(np.isfinite(got))
    assert rel_fro(got, ref) <= TOL[synth.DTYPE_BF16], rel_fro(got, ref)


@pytest.mark.slow
def test_merge_768p_sampled_rows():
    """The 768p clip's tokens (45 x 1008), 32 heads x 128 features, D = 4096, both branches."""
    rows = np.random.default_rng(9).choice(45 * 1008, size=96, replace=False)
    rows = np.concatenate([rows, [0, 45 * 1008 - 1]])
    got, ref = _run(45 * 1008, 4096, 4096, True, seed=3, rows=rows)
    assert np.all(np.isfinite(got))
    assert rel_fro(got, ref) <= TOL[synth.DTYPE_BF16], rel_fro(got, ref)


def test_merge_refuses_bad_sizes_before_launch():
    import torch
    from frame_wise_linear_b200 import vda
    buf = torch.empty(1 << 16, dtype=torch.uint8, device="cuda")
    assert vda.vda_merge_project(128, 100, 64, buf, buf, None, None, buf, buf, check=False) == vda.VDA_ERR_UNSUPPORTED
    assert vda.vda_merge_project(128, 128, 12, buf, buf, None, None, buf, buf, check=False) == vda.VDA_ERR_UNSUPPORTED
    assert vda.vda_merge_project(128, 128, 64, buf, buf, buf, None, buf, buf, check=False) == vda.VDA_ERR_INVALID_ARG
