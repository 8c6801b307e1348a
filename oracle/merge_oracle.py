"""Float64 CPU oracle for the branch merge of the hybrid attention: each
branch's gated output through its own output projection, summed.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path may import, call or
execute this module: only ``tests/``, ``__graft_entry__.smoke()`` and the CPU
legs of ``bench.py`` use it.  It shares no code, constant or helper with the
CUDA library.

What it computes, and where it is stated
----------------------------------------
"VDN-MiniMax-H3" (aiezz.com), section 03 (technical principles), item "gate
fusion" (ゲート融合機構), restated in "VDN-MiniMax-H3 OpenVDN ..."
(laicaila.com), section 技术原理, item 门控融合机制: the two branches' outputs
have different scales, so each branch gets its own content-dependent sigmoid
gate and its own output projection, and the results are then merged.  Read as,
per token (a row), with the heads' outputs concatenated (H * d_v features):

    Y = (sigmoid(G_lin) * P_lin) W_lin + (sigmoid(G_sm) * P_sm) W_sm
      = O_lin W_lin + O_sm W_sm

where P_lin, P_sm are the linear (VDA) and local softmax branches' outputs
before their gates, O_lin, O_sm the gated outputs, W_lin and W_sm
[H * d_v, D] projections and Y is [tokens, D].  The merge is a sum: the pages
name no other combination, and the separate gates and projections already
scale each branch.  Each gate belongs to its branch (the VDA forward applies
the linear one itself), so the merge takes the two gated outputs.

Everything is float64.
"""

from __future__ import annotations

import numpy as np

from oracle.vda_oracle import sigmoid

__all__ = ["gated", "merge_project"]


def gated(G: np.ndarray, P: np.ndarray) -> np.ndarray:
    """A branch's gated output, sigmoid(G) * P element-wise (the gate fusion item)."""
    return sigmoid(np.asarray(G, dtype=np.float64)) * np.asarray(P, dtype=np.float64)


def merge_project(O_lin, W_lin, O_sm, W_sm) -> np.ndarray:
    """Y = O_lin W_lin + O_sm W_sm.

    O_lin, O_sm: [tokens, K] the two branches' gated outputs (heads
    concatenated); W_lin, W_sm: [K, D].  O_sm and W_sm may be None (no softmax
    branch).  Returns [tokens, D] float64.
    """
    Y = np.asarray(O_lin, dtype=np.float64) @ np.asarray(W_lin, dtype=np.float64)
    if O_sm is not None:
        Y = Y + np.asarray(O_sm, dtype=np.float64) @ np.asarray(W_sm, dtype=np.float64)
    return Y
