"""The oracle against what the pages and mathematics fix (CPU only).

Also plants plausible mistakes in the oracle (on the CPU, through
monkeypatching) and checks that some pin catches each one.
"""

import numpy as np
import pytest
from scipy.linalg import solve_triangular

import oracle_pins as P
from oracle import vda_oracle as vo


@pytest.mark.parametrize("pin", P.ALL_PINS, ids=lambda p: p.__name__)
def test_pin(pin):
    assert pin(), pin.__doc__


def _bad_normal_no_lambda(K, V, lam):
    K = np.asarray(K, float)
    V = np.asarray(V, float)
    return K.T @ K, K.T @ V


def _bad_normal_frame_scaled(K, V, lam):
    K = np.asarray(K, float)
    V = np.asarray(V, float)
    n = max(K.shape[0], 1)
    return K.T @ K / n + lam * np.eye(K.shape[1]), K.T @ V / n


def _bad_update_no_lambda(S, K, V, lam):
    A, B = vo.normal_equations(K, V, lam)
    return vo.spd_solve(A, S + B)


def _bad_update_sign(S, K, V, lam):
    A, B = vo.normal_equations(K, V, lam)
    return vo.spd_solve(A, lam * S - B)


def _bad_solve_wrong_transpose(A, R):
    L = np.linalg.cholesky(A)
    Y = solve_triangular(L, R, lower=True)
    return solve_triangular(L, Y, lower=True)


def _bad_backward_zero_seed(S0, K, V, lam):
    return _orig_backward(np.zeros_like(S0), K, V, lam)


def _bad_backward_exclusive(S0, K, V, lam):
    T = K.shape[0]
    out = np.empty((T,) + S0.shape)
    S = S0
    for t in range(T - 1, -1, -1):
        out[t] = S
        S = vo.frame_update(S, K[t], V[t], lam)
    return out


def _bad_forward_off_by_one(S0, K, V, lam):
    T = K.shape[0]
    out = np.empty((T,) + S0.shape)
    S = S0
    for t in range(T):
        S = vo.frame_update(S, K[min(t + 1, T - 1)], V[min(t + 1, T - 1)], lam)
        out[t] = S
    return out


def _bad_sigmoid(g):
    return 1.0 / (1.0 + np.exp(np.asarray(g, float)))


def _bad_text_unsolved(K_txt, V_txt, lam, d_k, d_v):
    if K_txt is None or np.asarray(K_txt).shape[0] == 0:
        return np.zeros((d_k, d_v))
    return vo.normal_equations(K_txt, V_txt, lam)[1]


_orig_backward = vo.scan_backward
_orig_head = vo.vda_head


def _bad_head_forward_only(Q, K, V, G, K_txt, V_txt, lam, return_states=False):
    d_k, d_v = K.shape[2], V.shape[2]
    S0 = vo.text_state(K_txt, V_txt, lam, d_k, d_v)
    SF = vo.scan_forward(S0, np.asarray(K, float), np.asarray(V, float), lam)
    O = np.stack([vo.sigmoid(G[t]) * (2 * Q[t] @ SF[t]) for t in range(K.shape[0])])
    if return_states:
        return O, {"S0": S0, "SF": SF, "SB": SF}
    return O


def _bad_head_transposed_read(Q, K, V, G, K_txt, V_txt, lam, return_states=False):
    O, st = _orig_head(Q, K, V, G, K_txt, V_txt, lam, return_states=True)
    gate = vo.sigmoid(G)
    O = np.stack([gate[t] * (Q[t] @ (st["SF"][t] + st["SB"][t]).T) if st["SF"][t].shape[0] == st["SF"][t].shape[1]
                  else O[t] * np.nan for t in range(K.shape[0])])
    if return_states:
        return O, st
    return O


MUTATIONS = {
    "normal_equations drops lam I": ("normal_equations", _bad_normal_no_lambda),
    "normal_equations divides by n": ("normal_equations", _bad_normal_frame_scaled),
    "update drops lam on S_prev": ("frame_update", _bad_update_no_lambda),
    "update flips the sign of B": ("frame_update", _bad_update_sign),
    "solve uses L instead of L^T": ("spd_solve", _bad_solve_wrong_transpose),
    "backward scan seeded with zero": ("scan_backward", _bad_backward_zero_seed),
    "backward scan exclusive of frame t": ("scan_backward", _bad_backward_exclusive),
    "forward scan reads the next frame": ("scan_forward", _bad_forward_off_by_one),
    "sigmoid sign flipped": ("sigmoid", _bad_sigmoid),
    "text state not solved": ("text_state", _bad_text_unsolved),
    "readout drops the backward state": ("vda_head", _bad_head_forward_only),
    "readout transposes the state": ("vda_head", _bad_head_transposed_read),
}


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_pins_catch_planted_mistake(name, monkeypatch):
    attr, bad = MUTATIONS[name]
    monkeypatch.setattr(vo, attr, bad)
    results = P.run_all()
    failed = [k for k, ok in results.items() if not ok]
    assert failed, f"no pin caught the planted mistake: {name}"


def test_unmutated_oracle_passes_every_pin():
    results = P.run_all()
    assert all(results.values()), results


def _layout_case(seed, B=2, H=3, T=3, n=4, d_k=3, d_v=2, n_txt=2):
    rng = np.random.default_rng(seed)
    t = lambda *s: rng.standard_normal(s)  # noqa: E731
    Q, K, V, G = t(B, H, T, n, d_k), t(B, H, T, n, d_k), t(B, H, T, n, d_v), t(B, H, T, n, d_v)
    Kt, Vt = (t(B, H, n_txt, d_k), t(B, H, n_txt, d_v)) if n_txt else (None, None)
    return Q, K, V, G, Kt, Vt


def test_forward_layout_wrapper_matches_heads():
    """The [B, H] wrapper is the per-head function applied to head (b, h) and put back at [b, h].

    Heads and batch entries are independent problems ("VDN-MiniMax-H3", section 03:
    the linear branch is per attention head).  Every head gets different data and a
    non-square d_k x d_v, so a swapped (b, h) index, a transposed reshape or a
    misordered head selection fails the element-wise equality.
    """
    Q, K, V, G, Kt, Vt = _layout_case(11)
    B, H = Q.shape[:2]
    O, states = vo.vda_forward(Q, K, V, G, Kt, Vt, 0.7, return_states=True)
    assert O.shape == G.shape
    assert len(states) == B * H
    for b in range(B):
        for h in range(H):
            o1, s1 = vo.vda_head(Q[b, h], K[b, h], V[b, h], G[b, h], Kt[b, h], Vt[b, h], 0.7, return_states=True)
            np.testing.assert_array_equal(O[b, h], o1)
            for k in ("S0", "SF", "SB"):
                np.testing.assert_array_equal(states[b * H + h][k], s1[k])
    # distinct heads really differ, so the equality above can tell them apart
    assert not np.allclose(O[0, 1], O[1, 0])
    assert np.array_equal(vo.vda_forward(Q, K, V, G, Kt, Vt, 0.7), O)
    # a selection returns exactly those heads, stacked in the order asked for
    sel = [(1, 2), (0, 0), (1, 0)]
    some, some_states = vo.vda_forward(Q, K, V, G, Kt, Vt, 0.7, heads=sel, return_states=True)
    assert some.shape == (len(sel),) + G.shape[2:]
    for i, (b, h) in enumerate(sel):
        np.testing.assert_array_equal(some[i], O[b, h])
        np.testing.assert_array_equal(some_states[i]["SF"], states[b * H + h]["SF"])


def test_forward_layout_wrapper_without_text():
    """n_txt = 0 (no text tensors) gives S_0 = 0 in every head ("VDN-MiniMax-H3", section 03, text injection)."""
    Q, K, V, G, _, _ = _layout_case(12, n_txt=0)
    B, H = Q.shape[:2]
    O, states = vo.vda_forward(Q, K, V, G, None, None, 1.3, return_states=True)
    for b in range(B):
        for h in range(H):
            np.testing.assert_array_equal(O[b, h], vo.vda_head(Q[b, h], K[b, h], V[b, h], G[b, h], None, None, 1.3))
            assert not np.any(states[b * H + h]["S0"])
