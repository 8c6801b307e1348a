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
