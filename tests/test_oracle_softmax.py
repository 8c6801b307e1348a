"""Pins of the local softmax branch's oracle (oracle/softmax_oracle.py): a
second route through a dense masked score matrix, reductions to full
attention, softmax invariants, and which frames reach which queries."""
import numpy as np
import pytest

from oracle import softmax_oracle as so


def _inputs(rng, T=12, n=3, d=4, dv=5, nt=2):
    f = lambda *s: rng.standard_normal(s)  # noqa: E731
    return f(T, n, d), f(T, n, d), f(T, n, dv), f(T, n, dv), (f(nt, d) if nt else None), (f(nt, dv) if nt else None)


def test_key_frames_by_hand():
    # blocks of 5: frame 12 is in block 2 (frames 10..14), neighbours blocks 1 and 3 (5..19), anchors 0 and 29
    assert so.key_frames(12, 30) == [0] + list(range(5, 20)) + [29]
    assert so.key_frames(0, 30) == list(range(0, 10)) + [29]        # first block: itself and the next
    assert so.key_frames(29, 30) == [0] + list(range(20, 30))      # last block: itself and the one before
    assert so.key_frames(3, 7) == list(range(7))                    # everything is in reach
    # density added by the anchors at the 768p clip's 45 frames: 70 frame pairs of 45^2 (3.5 %)
    window = lambda t: {f for f in range(45) if abs(f // 5 - t // 5) <= 1}  # noqa: E731
    assert sum(len(set(so.key_frames(t, 45)) - window(t)) for t in range(45)) == 70


@pytest.mark.parametrize("T,nt", [(12, 2), (30, 0), (7, 3), (1, 0)])
def test_the_two_routes_agree(T, nt):
    rng = np.random.default_rng(T + nt)
    args = _inputs(rng, T=T, nt=nt)
    np.testing.assert_allclose(so.local_softmax_head(*args), so.local_softmax_dense(*args), rtol=1e-12, atol=1e-13)


def test_short_clip_is_full_attention_by_explicit_sums():
    """T <= 10 keeps every frame in reach of every query: plain softmax attention, written out with exp."""
    rng = np.random.default_rng(1)
    Q, K, V, G, Kt, Vt = _inputs(rng, T=4, n=2, d=3, dv=2, nt=1)
    O = so.local_softmax_head(Q, K, V, G, Kt, Vt)
    keys = [(K[f, j], V[f, j]) for f in range(4) for j in range(2)] + [(Kt[0], Vt[0])]
    for t in range(4):
        for i in range(2):
            w = [np.exp(Q[t, i] @ k / np.sqrt(3)) for k, _ in keys]
            out = sum(wi * v for wi, (_, v) in zip(w, keys)) / sum(w)
            np.testing.assert_allclose(O[t, i], out / (1 + np.exp(-G[t, i])), rtol=1e-12)


def test_softmax_invariants():
    rng = np.random.default_rng(2)
    Q, K, V, G, Kt, Vt = _inputs(rng, T=20)
    base = so.local_softmax_head(Q, K, V, G, Kt, Vt)
    # a common shift of all keys adds the same q . u to every score of a row: no change
    u = rng.standard_normal(K.shape[-1])
    np.testing.assert_allclose(so.local_softmax_head(Q, K + u, V, G, Kt + u, Vt), base, atol=1e-12)
    # equal value rows everywhere give that row back (times the gate)
    v = rng.standard_normal(V.shape[-1])
    out = so.local_softmax_head(Q, K, 0 * V + v, G, Kt, 0 * Vt + v)
    np.testing.assert_allclose(out, 1 / (1 + np.exp(-G)) * v, atol=1e-12)
    # permuting the tokens of a frame permutes its queries' rows and leaves the others
    perm = rng.permutation(Q.shape[1])
    Qp, Kp, Vp, Gp = Q.copy(), K.copy(), V.copy(), G.copy()
    Qp[7], Kp[7], Vp[7], Gp[7] = Q[7][perm], K[7][perm], V[7][perm], G[7][perm]
    outp = so.local_softmax_head(Qp, Kp, Vp, Gp, Kt, Vt)
    np.testing.assert_allclose(outp[7], base[7][perm], atol=1e-12)
    np.testing.assert_allclose(np.delete(outp, 7, 0), np.delete(base, 7, 0), atol=1e-12)


def test_which_frames_reach_which_queries():
    """Perturbing frame f's values changes exactly the queries whose key frames include f."""
    rng = np.random.default_rng(3)
    T = 30
    Q, K, V, G, Kt, Vt = _inputs(rng, T=T)
    base = so.local_softmax_head(Q, K, V, G, Kt, Vt)
    for f in (0, 13, 22, T - 1):
        V2 = V.copy()
        V2[f] += 1.0
        changed = np.abs(so.local_softmax_head(Q, K, V2, G, Kt, Vt) - base).max(axis=(1, 2)) > 1e-12
        want = np.array([f in so.key_frames(t, T) for t in range(T)])
        assert np.array_equal(changed, want), f
    # the text reaches every query
    Vt2 = Vt + 1.0
    assert np.all(np.abs(so.local_softmax_head(Q, K, V, G, Kt, Vt2) - base).max(axis=(1, 2)) > 1e-12)


def test_planted_mistakes_fail_a_pin():
    """No anchors, a window of +-1 frame, no text, or a wrong scale each change the result."""
    rng = np.random.default_rng(4)
    T = 30
    Q, K, V, G, Kt, Vt = _inputs(rng, T=T)
    good = so.local_softmax_head(Q, K, V, G, Kt, Vt)
    orig = so.key_frames
    try:
        so.key_frames = lambda t, T, block=5: [f for f in orig(t, T, block) if abs(f // block - t // block) <= 1]
        assert np.abs(so.local_softmax_head(Q, K, V, G, Kt, Vt) - good).max() > 1e-3
        so.key_frames = lambda t, T, block=5: [f for f in range(T) if abs(f - t) <= 1]
        assert np.abs(so.local_softmax_head(Q, K, V, G, Kt, Vt) - good).max() > 1e-3
    finally:
        so.key_frames = orig
    assert np.abs(so.local_softmax_head(Q, K, V, G, None, None) - good).max() > 1e-3
    assert np.abs(so.local_softmax_head(Q, K, V, G, Kt, Vt, scale=1.0) - good).max() > 1e-3
