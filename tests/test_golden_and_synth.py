"""Oracle regression fixture and the seeded input generators (CPU only)."""
import os

import numpy as np

from frame_wise_linear_b200 import synth

HERE = os.path.dirname(os.path.abspath(__file__))


def _load_golden():
    rows = {"frob_SF": {}, "frob_SB": {}, "O": {}}
    with open(os.path.join(HERE, "golden", "tiny_oracle.txt")) as fh:
        for line in fh:
            if line.startswith("#"):
                continue
            p = line.split()
            if p[0] == "frob_O":
                rows["frob_O"] = float(p[1])
            elif p[0] in ("frob_SF", "frob_SB"):
                rows[p[0]][int(p[1])] = float(p[2])
            else:
                rows["O"][tuple(int(x) for x in p[1:-1])] = float(p[-1])
    return rows


def test_oracle_matches_stored_fixture():
    import sys
    sys.path.insert(0, os.path.join(HERE, "golden"))
    import make_golden
    O, st, idx = make_golden.compute()
    g = _load_golden()
    assert abs(np.linalg.norm(O) - g["frob_O"]) <= 1e-12 * g["frob_O"]
    for t, v in g["frob_SF"].items():
        assert abs(np.linalg.norm(st["SF"][t]) - v) <= 1e-12 * v
    for t, v in g["frob_SB"].items():
        assert abs(np.linalg.norm(st["SB"][t]) - v) <= 1e-12 * v
    for i, v in g["O"].items():
        assert abs(O[i] - v) <= 1e-12 * max(1.0, abs(v))


def test_generator_is_deterministic_and_normalised():
    a = synth.make_inputs("tiny", seed=0)
    b = synth.make_inputs("tiny", seed=0)
    c = synth.make_inputs("tiny", seed=1)
    for k in ("Q", "K", "V", "G", "K_txt", "V_txt"):
        assert np.array_equal(getattr(a, k), getattr(b, k))
        assert not np.array_equal(getattr(a, k), getattr(c, k))
    for k in ("Q", "K", "K_txt"):
        nrm = np.linalg.norm(a.widened(k), axis=-1)
        assert np.allclose(nrm, 1.0, atol=1e-6)
    assert a.Q.dtype == np.float32 and a.Q.shape == (1, 1, 8, 64, 64)


def test_bf16_rounding_is_nearest_even():
    x = np.array([1.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -2.5, 3.0e38, 1e-40], dtype=np.float32)
    bits = synth.to_bf16_bits(x)
    back = synth.bf16_bits_to_f32(bits)
    # ties go to even: 1 + 2^-8 -> 1, 1 + 3*2^-8 -> 1 + 2^-6
    assert back[0] == 1.0 and back[1] == 1.0 and back[2] == np.float32(1.0 + 2 ** -6)
    assert back[3] == -2.5
    rng = np.random.default_rng(0)
    y = rng.standard_normal(10000).astype(np.float32)
    yb = synth.bf16_bits_to_f32(synth.to_bf16_bits(y))
    assert np.max(np.abs(yb - y) / np.abs(y)) <= 2 ** -8


def test_mid_workload_statistics():
    w = synth.WORKLOADS["mid"].replace(H=2)
    inp = synth.make_inputs(w, seed=0)
    assert inp.Q.dtype == np.uint16 and inp.Q.shape == (1, 2, 16, 256, 128)
    G = inp.widened("G")
    assert abs(G.var() - 2.0) < 0.05          # G ~ N(0, 2): variance 2
    V = inp.widened("V")
    assert abs(V.var() - 1.0) < 0.05


def test_ill_conditioned_keys_are_nearly_low_rank():
    w = synth.WORKLOADS["illcond"].replace(H=1, T=2)
    inp = synth.make_inputs(w, seed=0)
    K = inp.widened("K")[0, 0, 0]
    s = np.linalg.svd(K, compute_uv=False)
    assert s[7] ** 2 > 50 and s[8] ** 2 < 0.05     # 8 dominant directions, the rest noise


def test_token_major_permutation_is_the_documented_layout():
    """synth.token_major: element (b, h, t, r, c) of [B, H, T, n, d] lands at (b, t*n + r, h, c); the
    text's (b, h, r, c) at (b, r, h, c)."""
    import torch
    B, H, T, n, d, nt = 2, 3, 4, 5, 6, 7
    x = torch.arange(B * H * T * n * d, dtype=torch.float32).reshape(B, H, T, n, d)
    y = synth.token_major(x)
    assert y.shape == (B, T * n, H, d) and y.is_contiguous()
    for b in range(B):
        for h in range(H):
            for t in range(T):
                for r in range(n):
                    assert torch.equal(y[b, t * n + r, h], x[b, h, t, r])
    xt = torch.arange(B * H * nt * d, dtype=torch.float32).reshape(B, H, nt, d)
    yt = synth.token_major(xt)
    assert yt.shape == (B, nt, H, d)
    for b in range(B):
        for h in range(H):
            for r in range(nt):
                assert torch.equal(yt[b, r, h], xt[b, h, r])
    assert synth.token_major(None) is None


def test_e4m3_codec_against_an_independent_implementation():
    """The 8-bit input format (OCP E4M3): every code decodes as torch's float8_e4m3fn does, and the
    encoder rounds to nearest with ties to even (saturating at 448) as torch's conversion does."""
    import torch
    codes = np.arange(256, dtype=np.uint8)
    mine = synth.e4m3_bits_to_f64(codes)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    assert np.array_equal(np.isnan(mine), np.isnan(ref))
    assert np.array_equal(mine[~np.isnan(ref)], ref[~np.isnan(ref)])
    rng = np.random.default_rng(0)
    x = rng.standard_normal(20000) * np.exp(rng.uniform(-14, 7, 20000))
    mids = (synth._E4M3_POS[1:] + synth._E4M3_POS[:-1]) / 2          # exact ties
    x = np.concatenate([x, synth._E4M3_POS, -synth._E4M3_POS, mids, -mids])
    got = synth.to_e4m3_bits(x)
    want = torch.from_numpy(np.clip(x, -448.0, 448.0)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(got, want)
    assert list(synth.to_e4m3_bits(np.array([460.0, 1e9, -1e9]))) == [0x7E, 0x7E, 0xFE]   # saturation
    # a few values by hand: 1 = 0 0111 000, 0.5 = 0 0110 000, -2.25 = 1 1000 001, 2^-9 = 0 0000 001
    assert list(synth.to_e4m3_bits(np.array([1.0, 0.5, -2.25, 2.0 ** -9]))) == [0x38, 0x30, 0xC1, 0x01]


def test_e4m3_workload_values_are_scale_times_codes():
    w = synth.WORKLOADS["768p_fp8"].replace(H=1, T=1, n=16, n_txt=4)
    raw = synth.head_inputs(w, 0, 0)
    wide = synth.head_widened(w, 0, 0)
    f = synth.head_f32(w, 0, 0)
    for k, sc in w.scales().items():
        assert raw[k].dtype == np.uint8
        np.testing.assert_array_equal(wide[k], sc * synth.e4m3_bits_to_f64(raw[k]))
        # the stored value is within half an 8-bit step (2^-4 relative) of the drawn one
        big = np.abs(f[k]) > 2.0 ** -6 * sc
        assert np.all(np.abs(wide[k] - f[k])[big] <= 2.0 ** -4 * np.abs(f[k])[big] + 1e-30)
