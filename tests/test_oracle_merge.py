"""Pins of the branch-merge oracle (oracle/merge_oracle.py), each by a route that
does not retype its formula: element sums written out, special cases that
reduce to one branch, linearity, and the gate's fixed values."""
import numpy as np

from oracle import merge_oracle as mo


def _case(rng, t=5, k=6, d=4):
    f = lambda *s: rng.standard_normal(s)  # noqa: E731
    return f(t, k), f(k, d), f(t, k), f(t, k), f(k, d)


def test_every_element_is_the_written_out_sum():
    """Y[i, j] = sum_k sigmoid(G_lin) P_lin W_lin + sigmoid(G_sm) P_sm W_sm, by explicit loops and exp."""
    rng = np.random.default_rng(0)
    Pl, Wl, P, G, Ws = _case(rng)
    Gl = rng.standard_normal(Pl.shape)
    Y = mo.merge_project(mo.gated(Gl, Pl), Wl, mo.gated(G, P), Ws)
    for i in range(Pl.shape[0]):
        for j in range(Wl.shape[1]):
            s = 0.0
            for k in range(Pl.shape[1]):
                s += Pl[i, k] / (1.0 + np.exp(-Gl[i, k])) * Wl[k, j] + P[i, k] / (1.0 + np.exp(-G[i, k])) * Ws[k, j]
            assert abs(Y[i, j] - s) <= 1e-12 * (1 + abs(s))


def test_without_a_softmax_branch_it_is_the_projected_linear_output():
    rng = np.random.default_rng(1)
    O, Wl, P, G, Ws = _case(rng)
    ref = np.array([[sum(O[i, k] * Wl[k, j] for k in range(O.shape[1])) for j in range(Wl.shape[1])]
                    for i in range(O.shape[0])])
    np.testing.assert_allclose(mo.merge_project(O, Wl, None, None), ref, atol=1e-13)
    np.testing.assert_allclose(mo.merge_project(O, Wl, 0 * P, Ws), ref, atol=1e-13)
    # a gate driven far negative closes the softmax branch, far positive passes it whole
    np.testing.assert_allclose(mo.merge_project(O, Wl, mo.gated(np.full_like(G, -800.0), P), Ws), ref, atol=1e-13)
    np.testing.assert_allclose(mo.merge_project(0 * O, Wl, mo.gated(np.full_like(G, 800.0), P), Ws),
                               mo.merge_project(P, Ws, None, None), atol=1e-12)


def test_zero_logits_halve_a_branch():
    rng = np.random.default_rng(2)
    O, Wl, P, G, Ws = _case(rng)
    np.testing.assert_allclose(mo.merge_project(O, Wl, mo.gated(0 * G, P), Ws),
                               mo.merge_project(O, Wl, 0.5 * P, Ws), atol=1e-12)


def test_linear_in_each_projection_and_symmetric_in_the_branches():
    rng = np.random.default_rng(3)
    O, Wl, P, _, Ws = _case(rng)
    _, Wl2, _, _, Ws2 = _case(rng)
    a = mo.merge_project(O, Wl + 2 * Wl2, P, Ws - Ws2)
    b = mo.merge_project(O, Wl, P, Ws) + 2 * mo.merge_project(O, Wl2, None, None) - mo.merge_project(P, Ws2, None, None)
    np.testing.assert_allclose(a, b, atol=1e-11)
    np.testing.assert_allclose(mo.merge_project(P, Ws, O, Wl), mo.merge_project(O, Wl, P, Ws), atol=1e-11)
    # the same as one product over the concatenated features
    np.testing.assert_allclose(mo.merge_project(O, Wl, P, Ws), np.hstack([O, P]) @ np.vstack([Wl, Ws]), atol=1e-11)


def test_planted_mistakes_fail_a_pin():
    """A transposed projection, a dropped branch, or the branches' projections swapped each change the result."""
    rng = np.random.default_rng(4)
    O, Wl, P, _, Ws = _case(rng, t=6, k=6, d=6)
    good = mo.merge_project(O, Wl, P, Ws)
    bad = [O @ Wl.T + P @ Ws, O @ Wl, O @ Ws + P @ Wl]
    for b in bad:
        assert np.max(np.abs(b - good)) > 1e-3
