"""Pins for the float64 oracle: facts fixed by the pages and by mathematics.

Each pin computes its expected value by a route that does not go through the
oracle's own arithmetic (a closed form, another algorithm, exact rational
arithmetic or an invariant), so that a dropped term, a wrong sign, a wrong
index or a transposed operand in the oracle fails at least one of them.
Every pin returns True when the oracle agrees.

Sources for what the method is: aiezz.com "VDN-MiniMax-H3", section 03
(technical principles): Video Delta Attention (token-wise delta rule lifted to
a frame-wise joint solve through the normal equations; non-expansive; no
frame-size scaling), text dual-branch injection (text written once into both
directional states), gate fusion (content-dependent sigmoid gate);
comfyui-wiki.com "VDN-H3" news page, section on how Video DeltaNet speeds up
H3 (bidirectional linear branch, constant-size recurrent state).
"""

from __future__ import annotations

from fractions import Fraction

import numpy as np

from oracle import vda_oracle as vo

TOL = 1e-10


def _rng(seed):
    return np.random.default_rng(seed)


def _rel(a, b):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    den = max(np.linalg.norm(b), 1e-300)
    return float(np.linalg.norm(a - b) / den)


def _rand_head(rng, T, n, d_k, d_v, n_txt, normalise=True):
    Q = rng.standard_normal((T, n, d_k))
    K = rng.standard_normal((T, n, d_k))
    if normalise:
        Q /= np.linalg.norm(Q, axis=-1, keepdims=True)
        K /= np.linalg.norm(K, axis=-1, keepdims=True)
    V = rng.standard_normal((T, n, d_v))
    G = rng.standard_normal((T, n, d_v))
    Kt = rng.standard_normal((n_txt, d_k))
    Vt = rng.standard_normal((n_txt, d_v))
    return Q, K, V, G, Kt, Vt


# ---------------------------------------------------------------------------
# a1 + a2: one frame-wise step
# ---------------------------------------------------------------------------

def pin_single_token_delta_rule() -> bool:
    """n = 1 reduces to the normalised token delta rule.

    With one token (k, v) the joint solve is a rank-one update; by
    Sherman-Morrison, S_t = S + k (v^T - k^T S) / (lam + |k|^2).  The pages say
    VDA extends the token-wise delta rule, so this must hold.  d_k != d_v
    exposes transposed operands.
    """
    rng = _rng(1)
    ok = True
    for lam in (0.3, 1.0, 4.0):
        d_k, d_v = 5, 3
        S = rng.standard_normal((d_k, d_v))
        for _ in range(4):
            k = rng.standard_normal(d_k)
            v = rng.standard_normal(d_v)
            expect = S + np.outer(k, v - k @ S) / (lam + k @ k)
            got = vo.frame_update(S, k[None, :], v[None, :], lam)
            ok &= _rel(got, expect) < TOL
            S = expect
    return bool(ok)


def pin_woodbury_token_space() -> bool:
    """The token-space (Woodbury) form of the same step.

    S_t = S + K^T (K K^T + lam I_n)^{-1} (V - K S), an n x n solve instead of a
    d_k x d_k one.  Checked with n below and above d_k.
    """
    rng = _rng(2)
    ok = True
    for n in (3, 11):
        d_k, d_v, lam = 7, 4, 0.7
        K = rng.standard_normal((n, d_k))
        V = rng.standard_normal((n, d_v))
        S = rng.standard_normal((d_k, d_v))
        expect = S + K.T @ np.linalg.solve(K @ K.T + lam * np.eye(n), V - K @ S)
        got = vo.frame_update(S, K, V, lam)
        ok &= _rel(got, expect) < TOL
    return bool(ok)


def pin_stacked_least_squares() -> bool:
    """Brute force by another algorithm: the step as a stacked least-squares problem.

    argmin_S |K S - V|^2 + lam |S - S_prev|^2 equals the least-squares solution
    of [K; sqrt(lam) I] S = [V; sqrt(lam) S_prev], solved with an SVD-based
    routine that never forms the normal equations.
    """
    rng = _rng(3)
    ok = True
    for n, d_k, d_v, lam in ((6, 4, 5, 0.5), (2, 6, 3, 2.0), (9, 9, 9, 1e-3)):
        K = rng.standard_normal((n, d_k))
        V = rng.standard_normal((n, d_v))
        S = rng.standard_normal((d_k, d_v))
        Ast = np.vstack([K, np.sqrt(lam) * np.eye(d_k)])
        Bst = np.vstack([V, np.sqrt(lam) * S])
        expect = np.linalg.lstsq(Ast, Bst, rcond=None)[0]
        got = vo.frame_update(S, K, V, lam)
        ok &= _rel(got, expect) < 1e-9
    return bool(ok)


def pin_non_expansive() -> bool:
    """|lam A_t^{-1}|_2 = lam / (lam + sigma_min(K_t)^2) <= 1.

    Equality holds exactly when K_t is column-rank deficient (n < d_k), as for
    a short text segment.  Checked on M from ``transition`` against the SVD of
    K, and on the spectral norm.
    """
    rng = _rng(4)
    ok = True
    for n, d_k, lam in ((40, 8, 1.0), (5, 8, 0.05), (100, 16, 0.01)):
        K = rng.standard_normal((n, d_k))
        V = rng.standard_normal((n, 3))
        M, _ = vo.transition(K, V, lam)
        sig = np.linalg.svd(K, compute_uv=False)
        smin2 = sig[-1] ** 2 if n >= d_k else 0.0
        expect = lam / (lam + smin2)
        got = np.linalg.norm(M, 2)
        ok &= abs(got - expect) < 1e-9 and got <= 1 + 1e-12
        ok &= np.allclose(M, M.T, atol=1e-12)
    return bool(ok)


def pin_transition_consistent() -> bool:
    """The affine form M S + C reproduces the step for an arbitrary S."""
    rng = _rng(5)
    K = rng.standard_normal((12, 6))
    V = rng.standard_normal((12, 4))
    S = rng.standard_normal((6, 4))
    M, C = vo.transition(K, V, 0.8)
    # M S + C must equal the stacked least-squares answer (independent route)
    Ast = np.vstack([K, np.sqrt(0.8) * np.eye(6)])
    Bst = np.vstack([V, np.sqrt(0.8) * S])
    expect = np.linalg.lstsq(Ast, Bst, rcond=None)[0]
    return _rel(M @ S + C, expect) < 1e-9


def pin_least_squares_limit() -> bool:
    """As lam -> 0 with full column rank K_t, S_t -> argmin |K_t S - V_t|."""
    rng = _rng(6)
    K = rng.standard_normal((30, 6))
    V = rng.standard_normal((30, 4))
    S = rng.standard_normal((6, 4)) * 10
    expect = np.linalg.lstsq(K, V, rcond=None)[0]
    errs = [_rel(vo.frame_update(S, K, V, lam), expect) for lam in (1e-2, 1e-4, 1e-6, 1e-8)]
    return errs[-1] < 1e-7 and all(errs[i + 1] < errs[i] for i in range(len(errs) - 1))


def pin_no_frame_size_scaling() -> bool:
    """Duplicating every token of a frame equals doubling K^T K and K^T V.

    No frame-size scaling: a frame with each token repeated twice solves
    (2 K^T K + lam I) S = 2 K^T V + lam S_prev, which is the step for
    (sqrt(2) K, sqrt(2) V).  A per-token average (division by n) would make
    the duplicated frame identical to the original one instead.
    """
    rng = _rng(7)
    K = rng.standard_normal((5, 4))
    V = rng.standard_normal((5, 3))
    S = rng.standard_normal((4, 3))
    dup = vo.frame_update(S, np.vstack([K, K]), np.vstack([V, V]), 0.9)
    expect = vo.frame_update(S, np.sqrt(2) * K, np.sqrt(2) * V, 0.9)
    once = vo.frame_update(S, K, V, 0.9)
    return _rel(dup, expect) < TOL and _rel(dup, once) > 1e-3


def pin_normal_equations() -> bool:
    """A = K^T K + lam I and B = K^T V, checked entry by entry as token sums."""
    rng = _rng(8)
    K = rng.standard_normal((7, 3))
    V = rng.standard_normal((7, 2))
    A, B = vo.normal_equations(K, V, 0.25)
    ok = True
    for i in range(3):
        for j in range(3):
            s = sum(K[r, i] * K[r, j] for r in range(7)) + (0.25 if i == j else 0.0)
            ok &= abs(A[i, j] - s) < 1e-12
        for j in range(2):
            s = sum(K[r, i] * V[r, j] for r in range(7))
            ok &= abs(B[i, j] - s) < 1e-12
    return bool(ok)


# ---------------------------------------------------------------------------
# a3: the two scans and the text seeding
# ---------------------------------------------------------------------------

def pin_orthonormal_closed_form() -> bool:
    """K_t with orthonormal columns and a constant frame: geometric closed form.

    With K^T K = I, S_t = (lam S_{t-1} + K^T V) / (1 + lam), whose solution is
    S_t = C + (lam / (1 + lam))^t (S_0 - C) with C = K^T V.  Checks the scan's
    indexing (the exponent) and the lam placement, in both directions.
    """
    rng = _rng(9)
    d, T, lam = 6, 7, 0.6
    Kq, _ = np.linalg.qr(rng.standard_normal((d, d)))
    V = rng.standard_normal((d, 4))
    S0 = rng.standard_normal((d, 4))
    Kall = np.broadcast_to(Kq, (T, d, d)).copy()
    Vall = np.broadcast_to(V, (T, d, 4)).copy()
    C = Kq.T @ V
    r = lam / (1 + lam)
    SF = vo.scan_forward(S0, Kall, Vall, lam)
    SB = vo.scan_backward(S0, Kall, Vall, lam)
    ok = True
    for t in range(1, T + 1):
        expect_f = C + r ** t * (S0 - C)
        expect_b = C + r ** (T - t + 1) * (S0 - C)
        ok &= _rel(SF[t - 1], expect_f) < TOL
        ok &= _rel(SB[t - 1], expect_b) < TOL
    return bool(ok)


def pin_text_seeds_both_directions() -> bool:
    """S_0 = A_txt^{-1} B_txt seeds frame 1 forward and frame T backward.

    S_0 is checked as a least-squares solution with ridge lam (SVD route), and
    the first forward / first backward states as single steps from S_0.
    With no text tokens S_0 = 0.
    """
    rng = _rng(10)
    T, n, d_k, d_v, n_txt, lam = 4, 6, 5, 3, 3, 0.4
    Q, K, V, G, Kt, Vt = _rand_head(rng, T, n, d_k, d_v, n_txt)
    Ast = np.vstack([Kt, np.sqrt(lam) * np.eye(d_k)])
    Bst = np.vstack([Vt, np.zeros((d_k, d_v))])
    S0 = np.linalg.lstsq(Ast, Bst, rcond=None)[0]
    got0 = vo.text_state(Kt, Vt, lam, d_k, d_v)
    _, st = vo.vda_head(Q, K, V, G, Kt, Vt, lam, return_states=True)
    ok = _rel(got0, S0) < 1e-9 and _rel(st["S0"], S0) < 1e-9
    # first forward step and first backward step both start from S_0
    sm = lambda S, k, v: S + k.T @ np.linalg.solve(k @ k.T + lam * np.eye(k.shape[0]), v - k @ S)  # noqa: E731
    ok &= _rel(st["SF"][0], sm(S0, K[0], V[0])) < 1e-9
    ok &= _rel(st["SB"][T - 1], sm(S0, K[T - 1], V[T - 1])) < 1e-9
    z = vo.text_state(np.zeros((0, d_k)), np.zeros((0, d_v)), lam, d_k, d_v)
    ok &= z.shape == (d_k, d_v) and not np.any(z)
    return bool(ok)


def pin_scan_inclusive_causal() -> bool:
    """S^fwd_t depends on frames 1..t only; S^bwd_t on frames t..T only.

    Both include frame t.  Perturbing frame j changes S^fwd_t exactly for
    t >= j and S^bwd_t exactly for t <= j.
    """
    rng = _rng(11)
    T, n, d_k, d_v = 6, 5, 4, 3
    Q, K, V, G, Kt, Vt = _rand_head(rng, T, n, d_k, d_v, 2)
    _, st = vo.vda_head(Q, K, V, G, Kt, Vt, 0.5, return_states=True)
    ok = True
    for j in range(T):
        V2 = V.copy()
        V2[j] += 1.0
        _, st2 = vo.vda_head(Q, K, V2, G, Kt, Vt, 0.5, return_states=True)
        for t in range(T):
            df = np.abs(st2["SF"][t] - st["SF"][t]).max()
            db = np.abs(st2["SB"][t] - st["SB"][t]).max()
            ok &= (df > 1e-9) == (t >= j)
            ok &= (db > 1e-9) == (t <= j)
    return bool(ok)


def pin_time_reversal() -> bool:
    """Reversing Q, K, V, G along time reverses O (the two directions swap)."""
    rng = _rng(12)
    Q, K, V, G, Kt, Vt = _rand_head(rng, 5, 6, 4, 4, 3)
    O = vo.vda_head(Q, K, V, G, Kt, Vt, 0.8)
    Or = vo.vda_head(Q[::-1], K[::-1], V[::-1], G[::-1], Kt, Vt, 0.8)
    return _rel(Or[::-1], O) < TOL


def pin_fixed_point() -> bool:
    """If every frame and the text are consistent with one S*, all states equal S*.

    V_t = K_t S*, V_txt = K_txt S*: then S_0 = S* only if K_txt has full column
    rank, and each step keeps S*, so O_t = 2 sigmoid(G_t) * (Q_t S*).
    """
    rng = _rng(13)
    T, n, d_k, d_v, n_txt, lam = 5, 8, 4, 3, 40, 0.3
    Q, K, _, G, Kt, _ = _rand_head(rng, T, n, d_k, d_v, n_txt)
    Ss = rng.standard_normal((d_k, d_v))
    V = K @ Ss
    # The text is exact too; with lam > 0 the text state shrinks toward 0, so
    # a consistent text alone does not give S*: give the text an enormous
    # weight instead (scale K_txt, V_txt by c, lam fixed) -> S_0 -> S*.
    c = 1e4
    Kt2 = c * Kt
    Vt2 = Kt2 @ Ss
    O = vo.vda_head(Q, K, V, G, Kt2, Vt2, lam)
    gate = 1.0 / (1.0 + np.exp(-G))
    expect = 2.0 * gate * (Q @ Ss)
    return _rel(O, expect) < 1e-7


def pin_single_frame() -> bool:
    """T = 1: both directions see the same frame, so O = 2 sigmoid(G) * (Q S_1)."""
    rng = _rng(14)
    Q, K, V, G, Kt, Vt = _rand_head(rng, 1, 7, 5, 4, 3)
    _, st = vo.vda_head(Q, K, V, G, Kt, Vt, 0.9, return_states=True)
    O = vo.vda_head(Q, K, V, G, Kt, Vt, 0.9)
    S1 = st["SF"][0]
    gate = 1.0 / (1.0 + np.exp(-G[0]))
    ok = _rel(st["SB"][0], S1) < TOL
    ok &= _rel(O[0], 2 * gate * (Q[0] @ S1)) < TOL
    return bool(ok)


# ---------------------------------------------------------------------------
# a4 and whole-pipeline invariants
# ---------------------------------------------------------------------------

def pin_sigmoid_values() -> bool:
    """sigmoid(0) = 1/2, sigmoid(ln 3) = 3/4, sigmoid(-g) = 1 - sigmoid(g), no overflow."""
    g = np.array([0.0, np.log(3.0), -np.log(3.0), 800.0, -800.0, 30.0, -30.0])
    s = vo.sigmoid(g)
    ok = abs(s[0] - 0.5) < 1e-15 and abs(s[1] - 0.75) < 1e-15 and abs(s[2] - 0.25) < 1e-15
    ok &= s[3] == 1.0 and 0.0 <= s[4] < 1e-300 and np.all(np.isfinite(s))
    ok &= abs(s[5] + s[6] - 1.0) < 1e-15
    x = np.linspace(-20, 20, 81)
    ok &= np.max(np.abs(vo.sigmoid(x) + vo.sigmoid(-x) - 1)) < 1e-15
    ok &= np.max(np.abs(vo.sigmoid(x) - 0.5 * (1 + np.tanh(x / 2)))) < 1e-15
    return bool(ok)


def pin_token_permutation() -> bool:
    """Permuting the tokens of one frame permutes the rows of that frame's O."""
    rng = _rng(15)
    Q, K, V, G, Kt, Vt = _rand_head(rng, 3, 9, 4, 5, 2)
    O = vo.vda_head(Q, K, V, G, Kt, Vt, 0.7)
    p = rng.permutation(9)
    Q2, K2, V2, G2 = Q.copy(), K.copy(), V.copy(), G.copy()
    Q2[1], K2[1], V2[1], G2[1] = Q[1][p], K[1][p], V[1][p], G[1][p]
    O2 = vo.vda_head(Q2, K2, V2, G2, Kt, Vt, 0.7)
    ok = _rel(O2[1], O[1][p]) < TOL and _rel(O2[0], O[0]) < TOL and _rel(O2[2], O[2]) < TOL
    return bool(ok)


def pin_linearity_in_values() -> bool:
    """O / sigmoid(G) is linear in (V, V_txt) jointly."""
    rng = _rng(16)
    Q, K, V, G, Kt, Vt = _rand_head(rng, 4, 6, 4, 3, 3)
    V2 = rng.standard_normal(V.shape)
    Vt2 = rng.standard_normal(Vt.shape)
    a, b = 0.7, -1.9
    O1 = vo.vda_head(Q, K, V, G, Kt, Vt, 0.6)
    O2 = vo.vda_head(Q, K, V2, G, Kt, Vt2, 0.6)
    O3 = vo.vda_head(Q, K, a * V + b * V2, G, Kt, a * Vt + b * Vt2, 0.6)
    return _rel(O3, a * O1 + b * O2) < 1e-9


def pin_scale_invariance() -> bool:
    """(K, K_txt, lam) -> (cK, cK_txt, c^2 lam) with V -> cV leaves every state unchanged."""
    rng = _rng(17)
    Q, K, V, G, Kt, Vt = _rand_head(rng, 4, 6, 4, 3, 3)
    c = 3.0
    _, s1 = vo.vda_head(Q, K, V, G, Kt, Vt, 0.5, return_states=True)
    _, s2 = vo.vda_head(Q, c * K, c * V, G, c * Kt, c * Vt, c * c * 0.5, return_states=True)
    return _rel(s2["SF"], s1["SF"]) < TOL and _rel(s2["SB"], s1["SB"]) < TOL


# ---------------------------------------------------------------------------
# Exact rational brute force on a hand-sized example
# ---------------------------------------------------------------------------

def _frac_solve(A, R):
    """Gauss-Jordan elimination in exact rationals: A^{-1} R."""
    n = len(A)
    m = len(R[0])
    M = [list(A[i]) + list(R[i]) for i in range(n)]
    for c in range(n):
        p = next(r for r in range(c, n) if M[r][c] != 0)
        M[c], M[p] = M[p], M[c]
        piv = M[c][c]
        M[c] = [x / piv for x in M[c]]
        for r in range(n):
            if r != c and M[r][c] != 0:
                f = M[r][c]
                M[r] = [x - f * y for x, y in zip(M[r], M[c])]
    return [row[n:n + m] for row in M]


def _frac_mm(X, Y):
    return [[sum(X[i][k] * Y[k][j] for k in range(len(Y))) for j in range(len(Y[0]))] for i in range(len(X))]


def _frac_T(X):
    return [list(r) for r in zip(*X)]


def exact_rational_head(Q, K, V, Kt, Vt, lam):
    """Whole forward with G = 0 (gate exactly 1/2), in exact rational arithmetic.

    Each step minimises |K S - V|^2 + lam |S - S_prev|^2; its stationarity
    condition (K^T K + lam I) S = K^T V + lam S_prev is solved by Gauss-Jordan
    over the rationals.  Returns O as a nested list of Fractions.
    """
    lam = Fraction(lam)
    d_k = len(K[0][0])
    d_v = len(V[0][0])

    def step(S, Kf, Vf):
        KT = _frac_T(Kf)
        A = _frac_mm(KT, Kf)
        for i in range(d_k):
            A[i][i] += lam
        R = _frac_mm(KT, Vf)
        R = [[R[i][j] + lam * S[i][j] for j in range(d_v)] for i in range(d_k)]
        return _frac_solve(A, R)

    zero = [[Fraction(0)] * d_v for _ in range(d_k)]
    S0 = step(zero, Kt, Vt) if len(Kt) else zero
    T = len(K)
    SF, SB = [None] * T, [None] * T
    S = S0
    for t in range(T):
        S = step(S, K[t], V[t])
        SF[t] = S
    S = S0
    for t in range(T - 1, -1, -1):
        S = step(S, K[t], V[t])
        SB[t] = S
    O = []
    for t in range(T):
        Ssum = [[SF[t][i][j] + SB[t][i][j] for j in range(d_v)] for i in range(d_k)]
        P = _frac_mm(Q[t], Ssum)
        O.append([[x / 2 for x in row] for row in P])
    return O


def exact_example():
    """A hand-sized example: d_k = 3, d_v = 2, n = 2 tokens, T = 3 frames, one text token."""
    K = [[[1, 2, 0], [0, 1, -1]], [[2, 0, 1], [1, 1, 1]], [[0, -1, 2], [3, 0, 0]]]
    V = [[[1, 0], [2, -1]], [[0, 3], [1, 1]], [[-2, 1], [0, 2]]]
    Q = [[[1, 0, 1], [0, 2, -1]], [[1, 1, 1], [-1, 0, 2]], [[0, 1, 0], [2, -1, 1]]]
    Kt = [[1, -1, 1]]
    Vt = [[2, 1]]
    lam = Fraction(1, 2)
    F = lambda x: [[[Fraction(v) for v in row] for row in m] for m in x]  # noqa: E731
    return F(Q), F(K), F(V), [[Fraction(v) for v in r] for r in Kt], [[Fraction(v) for v in r] for r in Vt], lam


def pin_exact_rational() -> bool:
    """The oracle agrees with exact rational arithmetic on a hand-sized example."""
    Qf, Kf, Vf, Ktf, Vtf, lam = exact_example()
    O_exact = exact_rational_head(Qf, Kf, Vf, Ktf, Vtf, lam)
    f = lambda x: np.array([[[float(v) for v in r] for r in m] for m in x])  # noqa: E731
    Q, K, V = f(Qf), f(Kf), f(Vf)
    Kt = np.array([[float(v) for v in r] for r in Ktf])
    Vt = np.array([[float(v) for v in r] for r in Vtf])
    G = np.zeros((3, 2, 2))
    O = vo.vda_head(Q, K, V, G, Kt, Vt, float(lam))
    return _rel(O, f(O_exact)) < 1e-13


ALL_PINS = [
    pin_single_token_delta_rule,
    pin_woodbury_token_space,
    pin_stacked_least_squares,
    pin_non_expansive,
    pin_transition_consistent,
    pin_least_squares_limit,
    pin_no_frame_size_scaling,
    pin_normal_equations,
    pin_orthonormal_closed_form,
    pin_text_seeds_both_directions,
    pin_scan_inclusive_causal,
    pin_time_reversal,
    pin_fixed_point,
    pin_single_frame,
    pin_sigmoid_values,
    pin_token_permutation,
    pin_linearity_in_values,
    pin_scale_invariance,
    pin_exact_rational,
]


def run_all() -> dict:
    out = {}
    for p in ALL_PINS:
        try:
            out[p.__name__] = bool(p())
        except Exception:  # a planted mistake may also raise
            out[p.__name__] = False
    return out
