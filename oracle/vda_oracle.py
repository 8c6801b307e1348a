"""Float64 CPU oracle for the Video Delta Attention (VDA) linear branch:
forward, and the backward (the gradients of the forward).

TEST INFRASTRUCTURE ONLY.  Nothing in the product path may import, call or
execute this module: only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` use it.  It shares
no code, constant or helper with the CUDA library; the two meet only through
the seeded input generators, which hold none of the method's arithmetic.

What the method computes, and where it is stated
------------------------------------------------
The pages describe VDA in words only.  The concrete form adopted here is the
plainest reading of those words:

* "VDN-MiniMax-H3" (aiezz.com), section 03 (technical principles), item
  "Video Delta Attention"; restated in "VDN-MiniMax-H3 OpenVDN 开源的视频生成
  加速方案" (laicaila.com), section 技术原理: the token-wise delta rule is
  lifted to a frame-wise joint solve; all spatial tokens of a frame decide the
  new state together through the normal equations; the update is therefore
  non-expansive and needs no frame-size scaling.  Read as: per head, with
  state S (d_k x d_v),

      A_t = K_t^T K_t + lam * I,   B_t = K_t^T V_t,
      S_t = A_t^{-1} (lam * S_{t-1} + B_t),

  the minimiser of ||K_t S - V_t||_F^2 + lam * ||S - S_{t-1}||_F^2.
  B_t is not divided by the token count (no frame-size scaling).

* Same pages, item "text dual-branch injection" (テキストの二分岐注入 /
  文本双分支注入): the text is written once, at initialisation, into both
  directional states.  Read as S_0 = A_txt^{-1} B_txt (the same update from a
  zero prior), shared by the forward and the backward scan.  No text tokens
  means S_0 = 0.

* "VDN-H3: ..." (comfyui-wiki.com), section "Video DeltaNetがH3を高速化する
  仕組み": a bidirectional linear-attention branch carries long-range context
  through a constant-size recurrent state.  Read as a forward scan over frames
  1..T and a backward scan over frames T..1, both inclusive of frame t.

* aiezz.com section 03, item "gate fusion" (ゲート融合機構): each branch has a
  content-dependent sigmoid gate.  Read as
  O_t = sigmoid(G_t) * (Q_t S^fwd_t + Q_t S^bwd_t), element-wise, with G_t of
  the same shape as O_t.

Everything is float64.  BF16 inputs reach this module already widened exactly
to float64, so both sides see identical input values.
"""

from __future__ import annotations

import numpy as np
from scipy.linalg import solve_triangular

__all__ = [
    "normal_equations",
    "spd_solve",
    "text_state",
    "frame_update",
    "transition",
    "scan_forward",
    "scan_backward",
    "sigmoid",
    "vda_head",
    "vda_forward",
    "vda_head_backward",
    "vda_backward",
]


def normal_equations(K: np.ndarray, V: np.ndarray, lam: float):
    """Normal equations of one frame's joint solve.

    ``K`` is (n, d_k), ``V`` is (n, d_v).  Returns ``A = K^T K + lam I``
    (d_k x d_k) and ``B = K^T V`` (d_k x d_v).  Source: aiezz.com
    "VDN-MiniMax-H3" section 03, Video Delta Attention item (normal equations
    over all spatial tokens of a frame; no frame-size scaling, so B is not
    divided by n).
    """
    K = np.asarray(K, dtype=np.float64)
    V = np.asarray(V, dtype=np.float64)
    d_k = K.shape[1]
    A = K.T @ K + lam * np.eye(d_k)
    B = K.T @ V
    return A, B


def spd_solve(A: np.ndarray, R: np.ndarray) -> np.ndarray:
    """X = A^{-1} R for symmetric positive definite A.

    Cholesky factor A = L L^T, then L Y = R and L^T X = Y.  A is SPD whenever
    lam > 0, so the factor exists and the answer is unique.
    """
    L = np.linalg.cholesky(A)
    Y = solve_triangular(L, R, lower=True)
    return solve_triangular(L.T, Y, lower=False)


def text_state(K_txt: np.ndarray, V_txt: np.ndarray, lam: float, d_k: int, d_v: int):
    """S_0: the text written once into the state, from a zero prior.

    Source: aiezz.com section 03, text dual-branch injection item; laicaila.com
    技术原理, 文本双分支注入.  With no text tokens S_0 = 0.
    """
    if K_txt is None or np.asarray(K_txt).shape[0] == 0:
        return np.zeros((d_k, d_v))
    A, B = normal_equations(K_txt, V_txt, lam)
    return spd_solve(A, B)


def frame_update(S_prev: np.ndarray, K_t: np.ndarray, V_t: np.ndarray, lam: float) -> np.ndarray:
    """One frame-wise delta step: S_t = A_t^{-1} (lam S_{t-1} + B_t).

    Source: aiezz.com section 03, Video Delta Attention item.
    """
    A, B = normal_equations(K_t, V_t, lam)
    return spd_solve(A, lam * S_prev + B)


def transition(K_t: np.ndarray, V_t: np.ndarray, lam: float):
    """The affine form of one step, S_t = M_t S_{t-1} + C_t.

    M_t = lam A_t^{-1}, C_t = A_t^{-1} B_t.  Exposed for per-stage parity of
    the factor-and-solve step; ``frame_update`` does not use it.
    """
    A, B = normal_equations(K_t, V_t, lam)
    M = spd_solve(A, lam * np.eye(A.shape[0]))
    C = spd_solve(A, B)
    return M, C


def scan_forward(S0: np.ndarray, K: np.ndarray, V: np.ndarray, lam: float) -> np.ndarray:
    """Forward scan over frames 1..T; returns S^fwd_t for every t, shape (T, d_k, d_v).

    S^fwd_0 = S0 and S^fwd_t includes frame t.  Source: comfyui-wiki.com
    "VDN-H3" page, section on how Video DeltaNet speeds up H3 (bidirectional
    linear branch with a recurrent state).
    """
    T = K.shape[0]
    out = np.empty((T,) + S0.shape)
    S = S0
    for t in range(T):
        S = frame_update(S, K[t], V[t], lam)
        out[t] = S
    return out


def scan_backward(S0: np.ndarray, K: np.ndarray, V: np.ndarray, lam: float) -> np.ndarray:
    """Backward scan over frames T..1; returns S^bwd_t, shape (T, d_k, d_v).

    S^bwd_{T+1} = S0 (the same text state as the forward scan) and S^bwd_t
    includes frame t.
    """
    T = K.shape[0]
    out = np.empty((T,) + S0.shape)
    S = S0
    for t in range(T - 1, -1, -1):
        S = frame_update(S, K[t], V[t], lam)
        out[t] = S
    return out


def sigmoid(g: np.ndarray) -> np.ndarray:
    """Logistic function, evaluated without overflow for either sign of g."""
    g = np.asarray(g, dtype=np.float64)
    out = np.empty_like(g)
    pos = g >= 0
    out[pos] = 1.0 / (1.0 + np.exp(-g[pos]))
    e = np.exp(g[~pos])
    out[~pos] = e / (1.0 + e)
    return out


def vda_head(Q, K, V, G, K_txt, V_txt, lam: float, return_states: bool = False):
    """VDA forward for one (batch, head).

    Q, K: (T, n, d_k); V, G: (T, n, d_v); K_txt: (n_txt, d_k); V_txt:
    (n_txt, d_v).  Returns O (T, n, d_v) and, with ``return_states``, a dict
    holding S0, S^fwd and S^bwd.

    O_t = sigmoid(G_t) * (Q_t S^fwd_t + Q_t S^bwd_t): aiezz.com section 03,
    gate fusion item (content-dependent sigmoid gate per branch).
    """
    Q = np.asarray(Q, dtype=np.float64)
    K = np.asarray(K, dtype=np.float64)
    V = np.asarray(V, dtype=np.float64)
    G = np.asarray(G, dtype=np.float64)
    d_k, d_v = K.shape[2], V.shape[2]
    S0 = text_state(K_txt, V_txt, lam, d_k, d_v)
    SF = scan_forward(S0, K, V, lam)
    SB = scan_backward(S0, K, V, lam)
    T = K.shape[0]
    O = np.empty(G.shape)
    gate = sigmoid(G)
    for t in range(T):
        O[t] = gate[t] * (Q[t] @ SF[t] + Q[t] @ SB[t])
    if return_states:
        return O, {"S0": S0, "SF": SF, "SB": SB}
    return O


def vda_forward(Q, K, V, G, K_txt, V_txt, lam: float, heads=None, return_states: bool = False):
    """VDA forward over the whole [B, H, T, n, d] layout.

    Q, K: [B, H, T, n, d_k]; V, G: [B, H, T, n, d_v]; K_txt: [B, H, n_txt, d_k];
    V_txt: [B, H, n_txt, d_v].  Batch entries and heads are independent.

    ``heads`` optionally restricts the work to a list of (b, h) pairs; the
    result then holds only those heads, in that order, stacked on a leading
    axis.  Returns float64 O (and the per-head states if asked).
    """
    Bn, Hn = np.shape(Q)[0], np.shape(Q)[1]
    pairs = [(b, h) for b in range(Bn) for h in range(Hn)] if heads is None else list(heads)
    outs, states = [], []
    for b, h in pairs:
        kt = None if K_txt is None else K_txt[b, h]
        vt = None if V_txt is None else V_txt[b, h]
        r = vda_head(Q[b, h], K[b, h], V[b, h], G[b, h], kt, vt, lam, return_states=return_states)
        if return_states:
            outs.append(r[0])
            states.append(r[1])
        else:
            outs.append(r)
    if heads is None:
        O = np.stack(outs).reshape((Bn, Hn) + outs[0].shape)
    else:
        O = np.stack(outs)
    if return_states:
        return O, states
    return O


def vda_head_backward(Q, K, V, G, K_txt, V_txt, lam: float, dO):
    """Gradients of one head's VDA forward, for the scalar L = sum(dO * O).

    The pages give no backward; this is the exact derivative of ``vda_head``
    (the reverse-mode chain rule through its steps), lam held fixed.  Inputs
    as ``vda_head``; ``dO`` has O's shape.  Returns a dict of float64 arrays
    dQ, dK, dV, dG, dK_txt, dV_txt (the last two None without text tokens).

    Steps, with S_t = S^fwd_t + S^bwd_t and P_t = Q_t S_t:
      dG_t = dO_t * P_t * s_t (1 - s_t), s_t = sigmoid(G_t);
      dP_t = dO_t * s_t;  dQ_t = dP_t S_t^T;  E_t = Q_t^T dP_t.
      The forward scan's adjoint runs from t = T down to 1:
        Gf_t = A_t^{-1} (E_t + lam Gf_{t+1}),  Gf_{T+1} = 0,
      and the backward scan's from t = 1 up to T:
        Gb_t = A_t^{-1} (E_t + lam Gb_{t-1}),  Gb_0 = 0
      (Gf_t is the gradient of lam S^fwd_{t-1} + B_t, the right-hand side of
      frame t's solve; likewise Gb_t).  S_0 seeds both scans, so
      G_0 = A_txt^{-1} lam (Gf_1 + Gb_T).  Each solve S = A^{-1} R gives
      dR = A^{-1} dS and dA = -dR S^T, hence for t = 1..T
        dB_t = Gf_t + Gb_t,   dA_t = -(Gf_t S^fwd_t^T + Gb_t S^bwd_t^T),
      and for the text dB_0 = G_0, dA_0 = -G_0 S_0^T.  Through the normal
      equations A = K^T K + lam I, B = K^T V:
        dK = K (dA + dA^T) + V dB^T,   dV = K dB.
    """
    Q = np.asarray(Q, dtype=np.float64)
    K = np.asarray(K, dtype=np.float64)
    V = np.asarray(V, dtype=np.float64)
    G = np.asarray(G, dtype=np.float64)
    dO = np.asarray(dO, dtype=np.float64)
    T, _, d_k = K.shape
    d_v = V.shape[2]
    has_text = K_txt is not None and np.asarray(K_txt).shape[0] > 0
    S0 = text_state(K_txt, V_txt, lam, d_k, d_v)
    SF = scan_forward(S0, K, V, lam)
    SB = scan_backward(S0, K, V, lam)
    A = [normal_equations(K[t], V[t], lam)[0] for t in range(T)]

    gate = sigmoid(G)
    dQ = np.empty(Q.shape)
    dG = np.empty(G.shape)
    E = np.empty((T, d_k, d_v))
    for t in range(T):
        S = SF[t] + SB[t]
        P = Q[t] @ S
        dG[t] = dO[t] * P * gate[t] * (1.0 - gate[t])
        dP = dO[t] * gate[t]
        dQ[t] = dP @ S.T
        E[t] = Q[t].T @ dP

    Gf = np.empty((T, d_k, d_v))
    nxt = np.zeros((d_k, d_v))
    for t in range(T - 1, -1, -1):
        Gf[t] = spd_solve(A[t], E[t] + lam * nxt)
        nxt = Gf[t]
    Gb = np.empty((T, d_k, d_v))
    prv = np.zeros((d_k, d_v))
    for t in range(T):
        Gb[t] = spd_solve(A[t], E[t] + lam * prv)
        prv = Gb[t]

    dK = np.empty(K.shape)
    dV = np.empty(V.shape)
    for t in range(T):
        dB = Gf[t] + Gb[t]
        dA = -(Gf[t] @ SF[t].T + Gb[t] @ SB[t].T)
        dK[t] = K[t] @ (dA + dA.T) + V[t] @ dB.T
        dV[t] = K[t] @ dB

    dK_txt = dV_txt = None
    if has_text:
        K_txt = np.asarray(K_txt, dtype=np.float64)
        V_txt = np.asarray(V_txt, dtype=np.float64)
        A0, _ = normal_equations(K_txt, V_txt, lam)
        G0 = spd_solve(A0, lam * (Gf[0] + Gb[T - 1]))
        dA0 = -G0 @ S0.T
        dK_txt = K_txt @ (dA0 + dA0.T) + V_txt @ G0.T
        dV_txt = K_txt @ G0
    return {"dQ": dQ, "dK": dK, "dV": dV, "dG": dG, "dK_txt": dK_txt, "dV_txt": dV_txt}


def vda_backward(Q, K, V, G, K_txt, V_txt, lam: float, dO, heads=None):
    """``vda_head_backward`` over the [B, H, T, n, d] layout (or a list of
    (b, h) pairs, stacked on a leading axis, as ``vda_forward``)."""
    Bn, Hn = np.shape(Q)[0], np.shape(Q)[1]
    pairs = [(b, h) for b in range(Bn) for h in range(Hn)] if heads is None else list(heads)
    res = []
    for b, h in pairs:
        kt = None if K_txt is None else K_txt[b, h]
        vt = None if V_txt is None else V_txt[b, h]
        res.append(vda_head_backward(Q[b, h], K[b, h], V[b, h], G[b, h], kt, vt, lam, dO[b, h]))
    out = {}
    for k in res[0]:
        if res[0][k] is None:
            out[k] = None
            continue
        arr = np.stack([r[k] for r in res])
        out[k] = arr.reshape((Bn, Hn) + arr.shape[1:]) if heads is None else arr
    return out
