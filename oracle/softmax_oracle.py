"""Float64 CPU oracle for the local softmax branch of the hybrid video
attention.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path may import, call or
execute this module: only ``tests/``, ``__graft_entry__.smoke()`` and the CPU
legs of ``bench.py`` use it.  It shares no code, constant or helper with the
CUDA library.

What it computes, and where it is stated
----------------------------------------
* "VDN-MiniMax-H3" (aiezz.com), section 03 (technical principles), item
  "local softmax branch" (局所Softmax分岐), restated in the laicaila.com page,
  section 技术原理 (局部 Softmax 分支): a bidirectional sliding window; the
  frames form groups of 5 and each group attends to its neighbouring blocks;
  the first and the last frame are added as boundary anchors, which raises
  the attention density by only 3.57 % and keeps the clip temporally
  consistent.  "VDN-H3" (comfyui-wiki.com), section on how Video DeltaNet
  speeds up H3: the anchors keep the clip's first and last frames visible
  from every frame.
  Read as: frames t = 0 .. T-1 fall into blocks of 5 (block t // 5); a query
  token of frame t attends to every token of the frames of blocks
  t // 5 - 1, t // 5 and t // 5 + 1 (those that exist), and to every token of
  frames 0 and T - 1.  The anchors are one-way (every frame sees them; they
  do not see every frame): the pages say only that all frames see the first
  and last ones.  (At T = 45 this adds 3.5 % of the T x T frame pairs; the
  pages' 3.57 % is at their own clip length.)
* Same pages, item "text dual-branch injection": in the softmax branch every
  frame attends to the whole text.  Read as: the text tokens' keys and values
  join every query's key set.
* Same pages, item "gate fusion": each branch has its own content-dependent
  sigmoid gate.  Read as O = sigmoid(G) * attention, element-wise, G of O's
  shape (the branch's output projection and the merge are the merge oracle's).
* The attention itself is the standard scaled dot-product softmax of the
  backbone's attention (the branch replaces part of it): per query row,
  softmax over its allowed keys of q . k / sqrt(d), then the weighted sum of
  the values.

Everything is float64.
"""

from __future__ import annotations

import numpy as np

from oracle.vda_oracle import sigmoid

__all__ = ["BLOCK", "key_frames", "local_softmax_frame", "local_softmax_head", "local_softmax_dense"]

BLOCK = 5   # frames per block of the sliding window (the pages' "every 5 frames")


def key_frames(t: int, T: int, block: int = BLOCK) -> list:
    """The frames whose tokens a query of frame t attends to: its block and the two neighbouring blocks, and
    the first and last frames (the anchors), in increasing order."""
    b = t // block
    lo, hi = max(0, (b - 1) * block), min(T, (b + 2) * block)
    return sorted(set(range(lo, hi)) | {0, T - 1})


def _attend(q, Kall, Vall, scale):
    """softmax(q Kall^T * scale) Vall for the rows of q (a stable softmax: the row maximum is subtracted)."""
    s = (q @ Kall.T) * scale
    s = s - s.max(axis=1, keepdims=True)
    e = np.exp(s)
    return (e / e.sum(axis=1, keepdims=True)) @ Vall


def local_softmax_frame(Q, K, V, G, K_txt, V_txt, t: int, block: int = BLOCK, scale: float | None = None):
    """Frame t of one head: O_t = sigmoid(G_t) * softmax(Q_t K_S^T * scale) V_S, with S the tokens of
    key_frames(t) and the text's.  Shapes as local_softmax_head; returns [n, d_v] float64."""
    T, _, d = np.shape(Q)
    scale = 1.0 / np.sqrt(d) if scale is None else scale
    fr = key_frames(t, T, block)
    Kall = np.concatenate([np.asarray(K[f], np.float64) for f in fr] +
                          ([np.asarray(K_txt, np.float64)] if K_txt is not None else []))
    Vall = np.concatenate([np.asarray(V[f], np.float64) for f in fr] +
                          ([np.asarray(V_txt, np.float64)] if V_txt is not None else []))
    return sigmoid(np.asarray(G[t], np.float64)) * _attend(np.asarray(Q[t], np.float64), Kall, Vall, scale)


def local_softmax_head(Q, K, V, G, K_txt, V_txt, block: int = BLOCK, scale: float | None = None):
    """One head: Q, K: [T, n, d]; V, G: [T, n, d_v]; K_txt: [n_txt, d]; V_txt: [n_txt, d_v] (or None).
    Returns O = sigmoid(G) * attention, [T, n, d_v] float64; the keys of frame t are those of
    key_frames(t) and the text's; scale defaults to 1 / sqrt(d)."""
    return np.stack([local_softmax_frame(Q, K, V, G, K_txt, V_txt, t, block, scale) for t in range(np.shape(Q)[0])])


def local_softmax_dense(Q, K, V, G, K_txt, V_txt, block: int = BLOCK, scale: float | None = None):
    """The same result by another route: all T*n (+ n_txt) keys at once, with the window written as a
    boolean mask over the full [T*n, T*n + n_txt] score matrix and excluded scores set to -inf."""
    Q, K, V, G = (np.asarray(x, dtype=np.float64) for x in (Q, K, V, G))
    T, n, d = Q.shape
    scale = 1.0 / np.sqrt(d) if scale is None else scale
    nt = 0 if K_txt is None else len(K_txt)
    Kf = K.reshape(T * n, d)
    Vf = V.reshape(T * n, -1)
    if nt:
        Kf = np.concatenate([Kf, np.asarray(K_txt, np.float64)])
        Vf = np.concatenate([Vf, np.asarray(V_txt, np.float64)])
    qf = np.repeat(np.arange(T), n)                       # frame of each query row
    kf = np.concatenate([np.repeat(np.arange(T), n), np.full(nt, -1)])   # frame of each key (-1: text)
    qb, kb = qf[:, None] // block, kf[None, :] // block
    allowed = (np.abs(qb - kb) <= 1) | (kf[None, :] == 0) | (kf[None, :] == T - 1) | (kf[None, :] < 0)
    s = np.where(allowed, (Q.reshape(T * n, d) @ Kf.T) * scale, -np.inf)
    s = s - s.max(axis=1, keepdims=True)
    e = np.exp(s)
    A = (e / e.sum(axis=1, keepdims=True)) @ Vf
    return sigmoid(G) * A.reshape(G.shape)
