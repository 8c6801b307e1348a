"""Pins of the oracle's backward (vda_head_backward), on the CPU.

The backward is the exact derivative of the forward oracle for
L = sum(dO * O).  It is pinned by central finite differences of the forward
oracle itself (a route that shares none of the backward's algebra), by
linearity in dO, and by planted mistakes in its source, each of which the
finite-difference check must catch.
"""
import inspect
import textwrap

import numpy as np
import pytest

from oracle import vda_oracle as vo


def _case(seed, T=3, n=5, d_k=4, d_v=3, n_txt=2, lam=0.7):
    rng = np.random.default_rng(seed)
    c = dict(Q=rng.standard_normal((T, n, d_k)), K=rng.standard_normal((T, n, d_k)),
             V=rng.standard_normal((T, n, d_v)), G=rng.standard_normal((T, n, d_v)),
             K_txt=rng.standard_normal((n_txt, d_k)) if n_txt else None,
             V_txt=rng.standard_normal((n_txt, d_v)) if n_txt else None,
             dO=rng.standard_normal((T, n, d_v)))
    return c, lam


def _loss(c, lam, **repl):
    a = {**c, **repl}
    O = vo.vda_head(a["Q"], a["K"], a["V"], a["G"], a["K_txt"], a["V_txt"], lam)
    return float(np.sum(c["dO"] * O))


def _fd_errors(c, lam, grads, samples=6, h=1e-6, seed=1):
    """Max relative error of the gradients against central differences, per input."""
    rng = np.random.default_rng(seed)
    out = {}
    for name, key in (("Q", "dQ"), ("K", "dK"), ("V", "dV"), ("G", "dG"), ("K_txt", "dK_txt"), ("V_txt", "dV_txt")):
        arr = c[name]
        if arr is None:
            continue
        worst = 0.0
        for _ in range(samples):
            idx = tuple(int(rng.integers(0, s)) for s in arr.shape)
            up, dn = arr.copy(), arr.copy()
            up[idx] += h
            dn[idx] -= h
            fd = (_loss(c, lam, **{name: up}) - _loss(c, lam, **{name: dn})) / (2 * h)
            worst = max(worst, abs(fd - grads[key][idx]) / max(1.0, abs(fd)))
        out[name] = worst
    return out


CASES = {
    "base": dict(),
    "no_text": dict(n_txt=0),
    "one_frame": dict(T=1),
    "square": dict(d_k=4, d_v=4),
    "rank_deficient": dict(n=2, d_k=5, d_v=3),     # n < d_k: K_t^T K_t singular, lam keeps A SPD
    "small_lambda": dict(lam=0.05),
    "long": dict(T=6, n=3),
}


@pytest.mark.parametrize("name", list(CASES))
def test_backward_matches_finite_differences(name):
    c, lam = _case(11, **CASES[name])
    g = vo.vda_head_backward(c["Q"], c["K"], c["V"], c["G"], c["K_txt"], c["V_txt"], lam, c["dO"])
    errs = _fd_errors(c, lam, g)
    assert max(errs.values()) < 1e-6, errs
    if c["K_txt"] is None:
        assert g["dK_txt"] is None and g["dV_txt"] is None


def test_backward_is_linear_in_dO():
    c, lam = _case(3)
    rng = np.random.default_rng(4)
    dO2 = rng.standard_normal(c["dO"].shape)
    args = (c["Q"], c["K"], c["V"], c["G"], c["K_txt"], c["V_txt"], lam)
    g1 = vo.vda_head_backward(*args, c["dO"])
    g2 = vo.vda_head_backward(*args, dO2)
    g3 = vo.vda_head_backward(*args, 2.0 * c["dO"] + dO2)
    for k in g1:
        np.testing.assert_allclose(g3[k], 2.0 * g1[k] + g2[k], rtol=1e-10, atol=1e-12)


def test_backward_layout_wrapper_matches_heads():
    rng = np.random.default_rng(5)
    B, H, T, n, d_k, d_v, nt = 2, 2, 2, 3, 3, 2, 2
    t = lambda *s: rng.standard_normal(s)  # noqa: E731
    Q, K, V, G, dO = t(B, H, T, n, d_k), t(B, H, T, n, d_k), t(B, H, T, n, d_v), t(B, H, T, n, d_v), t(B, H, T, n, d_v)
    Kt, Vt = t(B, H, nt, d_k), t(B, H, nt, d_v)
    full = vo.vda_backward(Q, K, V, G, Kt, Vt, 0.5, dO)
    for b in range(B):
        for h in range(H):
            one = vo.vda_head_backward(Q[b, h], K[b, h], V[b, h], G[b, h], Kt[b, h], Vt[b, h], 0.5, dO[b, h])
            for k in one:
                np.testing.assert_array_equal(full[k][b, h], one[k])
    some = vo.vda_backward(Q, K, V, G, Kt, Vt, 0.5, dO, heads=[(1, 0)])
    np.testing.assert_array_equal(some["dV"][0], full["dV"][1, 0])


# Plausible mistakes, planted in the backward's source (on the CPU); the
# finite-difference check must fail for every one.
MUTATIONS = {
    "dropped lambda in the forward scan's adjoint": ("E[t] + lam * nxt", "E[t] + nxt"),
    "dropped lambda in the backward scan's adjoint": ("E[t] + lam * prv", "E[t] + prv"),
    "adjoint of the forward scan run forward in time": ("range(T - 1, -1, -1)", "range(T)"),
    "dA not symmetrised": ("K[t] @ (dA + dA.T)", "K[t] @ (2.0 * dA)"),
    "wrong sign of dA": ("dA = -(Gf[t] @ SF[t].T + Gb[t] @ SB[t].T)", "dA = (Gf[t] @ SF[t].T + Gb[t] @ SB[t].T)"),
    "text seeded from the wrong ends": ("lam * (Gf[0] + Gb[T - 1])", "lam * (Gf[T - 1] + Gb[0])"),
    "sigmoid derivative sign": ("gate[t] * (1.0 - gate[t])", "gate[t] * (1.0 + gate[t])"),
    "dB from one direction only": ("dB = Gf[t] + Gb[t]", "dB = Gf[t]"),
}


def _mutant(old, new):
    src = textwrap.dedent(inspect.getsource(vo.vda_head_backward))
    assert src.count(old) == 1, old
    ns = dict(vars(vo))
    exec(src.replace(old, new), ns)  # noqa: S102 -- a planted mistake in the oracle, CPU only
    return ns["vda_head_backward"]


@pytest.mark.parametrize("name", list(MUTATIONS))
def test_planted_mistake_is_caught(name):
    c, lam = _case(21, T=3, d_k=4, d_v=3)
    bad = _mutant(*MUTATIONS[name])
    g = bad(c["Q"], c["K"], c["V"], c["G"], c["K_txt"], c["V_txt"], lam, c["dO"])
    errs = _fd_errors(c, lam, g, samples=8)
    assert max(errs.values()) > 1e-4, (name, errs)
