"""Seeded synthetic inputs for VDA forward.

This module holds no step of the method: it only draws random tensors,
normalises key/query rows, rounds to BF16 and widens BF16 bits back to
float64.  Both the CUDA path and the float64 oracle are fed from here, so both
see identical input values.

Workloads.  The pages measure a 768p, 14.4 s clip (the performance tables of
the agentlenshq.com project summary and the comfyui-wiki.com news page); no
dataset is involved.  The shapes below stand in for that clip's attention
inputs: a 24 x 42 latent grid (n = 1008 tokens per frame), T = 45 latent
frames, 32 heads of width 128 and 256 text tokens.

Recipe (per tensor and per (b, h), an independent stream
``PCG64(SeedSequence(seed, spawn_key=(tensor index, b, h)))``, so that any head
can be drawn alone):
  Q, K, K_txt : rows L2-normalised from N(0, 1)
  V, V_txt, G : N(0, 1)  (G ~ N(0, 2), i.e. variance 2, for the mid config)
  ill-conditioned keys: K_t = L2norm(U_t W + 0.05 E), U_t ~ N(0,1) (n x 8,
  fresh per frame), W ~ N(0,1) (8 x d_k, one per (b, h)), E ~ N(0,1).
Values are drawn in float32, normalised in float32, then rounded to BF16
(round to nearest even) for BF16 workloads.  E4M3 workloads store each tensor
x as the 8-bit float nearest to x / s (round to nearest even, saturating at
+-448), with one power-of-two scale s per tensor kind chosen from the
distribution (2^-8 for the unit-norm Q, K rows, 2^-6 for the N(0, 1) V and
G, 2^-5 for a G of larger spread): the values the device and the oracle see
are s times the stored 8-bit floats.
"""

from __future__ import annotations

import dataclasses
import math

import numpy as np

# Stream index of every tensor; fixed so that a tensor's values do not depend
# on which other tensors a workload draws.
_STREAM = {"Q": 0, "K": 1, "V": 2, "G": 3, "K_txt": 4, "V_txt": 5, "U": 6, "W": 7, "E": 8, "dO": 9}

DTYPE_F32 = 0
DTYPE_BF16 = 1
DTYPE_E4M3 = 2


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    T: int
    n: int
    n_txt: int
    d_k: int
    d_v: int
    dtype: int
    lam: float
    g_std: float = 1.0
    ill_conditioned: bool = False
    rank: int = 8
    noise: float = 0.05

    def scales(self) -> dict:
        """Per-tensor scales of an E4M3 workload (1 for the other types); the text takes K's and V's."""
        if self.dtype != DTYPE_E4M3:
            return dict(Q=1.0, K=1.0, V=1.0, G=1.0, K_txt=1.0, V_txt=1.0)
        qk, v = 2.0 ** -8, 2.0 ** -6
        g = 2.0 ** -6 if self.g_std <= 1.0 else 2.0 ** -5
        return dict(Q=qk, K=qk, V=v, G=g, K_txt=qk, V_txt=v)

    @property
    def units(self) -> int:
        """(frame, head) units, the metric's counting unit."""
        return self.B * self.H * self.T

    def problem(self) -> dict:
        d = dict(B=self.B, H=self.H, T=self.T, n=self.n, n_txt=self.n_txt,
                 d_k=self.d_k, d_v=self.d_v, dtype=self.dtype, lam=self.lam)
        if self.dtype == DTYPE_E4M3:
            sc = self.scales()
            d.update(scale_q=sc["Q"], scale_k=sc["K"], scale_v=sc["V"], scale_g=sc["G"])
        return d

    def replace(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


WORKLOADS = {
    "tiny": Workload("tiny", B=1, H=1, T=8, n=64, n_txt=16, d_k=64, d_v=64, dtype=DTYPE_F32, lam=1.0),
    "mid": Workload("mid", B=1, H=8, T=16, n=256, n_txt=128, d_k=128, d_v=128, dtype=DTYPE_BF16,
                    lam=0.5, g_std=math.sqrt(2.0)),
    "768p": Workload("768p", B=1, H=32, T=45, n=1008, n_txt=256, d_k=128, d_v=128, dtype=DTYPE_BF16, lam=1.0),
    # The 768p shapes with 8 heads: 372 MB of inputs (above L2) for profiler captures.
    "768p_h8": Workload("768p_h8", B=1, H=8, T=45, n=1008, n_txt=256, d_k=128, d_v=128, dtype=DTYPE_BF16, lam=1.0),
    "illcond": Workload("illcond", B=1, H=32, T=45, n=1008, n_txt=256, d_k=128, d_v=128, dtype=DTYPE_BF16,
                        lam=0.05, ill_conditioned=True),
    "long45": Workload("long45", B=2, H=32, T=45, n=1008, n_txt=256, d_k=128, d_v=128, dtype=DTYPE_BF16, lam=1.0),
    "long90": Workload("long90", B=2, H=32, T=90, n=1008, n_txt=256, d_k=128, d_v=128, dtype=DTYPE_BF16, lam=1.0),
    "long180": Workload("long180", B=2, H=32, T=180, n=1008, n_txt=256, d_k=128, d_v=128, dtype=DTYPE_BF16,
                        lam=1.0),
    # The 768p clip with 8-bit (E4M3) Q, K, V, G and text, per-tensor scales, bf16 O.
    "768p_fp8": Workload("768p_fp8", B=1, H=32, T=45, n=1008, n_txt=256, d_k=128, d_v=128, dtype=DTYPE_E4M3,
                         lam=1.0),
    "768p_fp8_h8": Workload("768p_fp8_h8", B=1, H=8, T=45, n=1008, n_txt=256, d_k=128, d_v=128,
                            dtype=DTYPE_E4M3, lam=1.0),
}


def _rng(seed: int, name: str, b: int, h: int) -> np.random.Generator:
    ss = np.random.SeedSequence(seed, spawn_key=(_STREAM[name], b, h))
    return np.random.Generator(np.random.PCG64(ss))


def _l2norm_rows(x: np.ndarray) -> np.ndarray:
    nrm = np.sqrt(np.einsum("...i,...i->...", x, x, dtype=np.float32))
    nrm = np.maximum(nrm, np.float32(1e-30))
    return (x / nrm[..., None]).astype(np.float32)


def to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """float32 -> BF16 bit patterns (uint16), round to nearest even."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    r = (u + np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))) >> np.uint32(16)
    return r.astype(np.uint16)


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


E4M3_MAX = 448.0


def e4m3_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    """OCP E4M3 (1 sign, 4 exponent, 3 mantissa bits, bias 7; no infinities,
    0x7F / 0xFF are NaN) bit patterns to their exact float64 values."""
    b = np.asarray(bits, dtype=np.uint8).astype(np.int64)
    sign = np.where(b & 0x80, -1.0, 1.0)
    e = (b >> 3) & 0xF
    m = (b & 0x7).astype(np.float64)
    mag = np.where(e == 0, m * 2.0 ** -9, (1.0 + m / 8.0) * np.exp2(e.astype(np.float64) - 7.0))
    mag = np.where((b & 0x7F) == 0x7F, np.nan, mag)
    return sign * mag


# The 127 finite non-negative E4M3 values, increasing with their codes 0x00 .. 0x7E.
_E4M3_POS = e4m3_bits_to_f64(np.arange(0x7F, dtype=np.uint8))


def to_e4m3_bits(x: np.ndarray) -> np.ndarray:
    """Values to the nearest E4M3 bit patterns (ties to the even code, which is
    the even mantissa), saturating at +-448; NaN maps to 0x7F."""
    x = np.asarray(x, dtype=np.float64)
    a = np.minimum(np.abs(x), E4M3_MAX)
    hi = np.clip(np.searchsorted(_E4M3_POS, a, side="left"), 0, 0x7E)
    lo = np.clip(hi - 1, 0, 0x7E)
    d_hi = _E4M3_POS[hi] - a
    d_lo = a - _E4M3_POS[lo]
    pick_hi = (d_hi < d_lo) | ((d_hi == d_lo) & (hi % 2 == 0))
    code = np.where(pick_hi, hi, lo).astype(np.uint8)
    code = np.where(np.signbit(x), code | np.uint8(0x80), code)
    code = np.where(np.isnan(x), np.uint8(0x7F), code)
    return code.astype(np.uint8)


def widen(x: np.ndarray, dtype: int, scale: float = 1.0) -> np.ndarray:
    """Exact float64 view of an input tensor as stored (BF16 bits, E4M3 bits
    times the tensor's scale, or float32)."""
    if dtype == DTYPE_BF16:
        return bf16_bits_to_f32(x).astype(np.float64)
    if dtype == DTYPE_E4M3:
        return scale * e4m3_bits_to_f64(x)
    return np.asarray(x, dtype=np.float32).astype(np.float64)


@dataclasses.dataclass
class Inputs:
    """Host copies of one workload's inputs, as stored on the device.

    BF16 tensors are uint16 bit patterns; FP32 tensors are float32.
    """
    workload: Workload
    Q: np.ndarray
    K: np.ndarray
    V: np.ndarray
    G: np.ndarray
    K_txt: np.ndarray
    V_txt: np.ndarray

    def widened(self, name: str, index=None) -> np.ndarray:
        a = getattr(self, name)
        if index is not None:
            a = a[index]
        return widen(a, self.workload.dtype, self.workload.scales()[name])

    def nbytes_in(self) -> int:
        return sum(getattr(self, k).nbytes for k in ("Q", "K", "V", "G", "K_txt", "V_txt"))


def _normal(seed: int, name: str, b: int, h: int, shape, std: float = 1.0) -> np.ndarray:
    x = _rng(seed, name, b, h).standard_normal(size=shape, dtype=np.float32)
    if std != 1.0:
        x *= np.float32(std)
    return x


NAMES = ("Q", "K", "V", "G", "K_txt", "V_txt")


def head_f32(w: Workload, b: int, h: int, seed: int = 0) -> dict:
    """One (b, h)'s inputs in float32, before any BF16 rounding."""
    sh_k = (w.T, w.n, w.d_k)
    sh_v = (w.T, w.n, w.d_v)
    Q = _l2norm_rows(_normal(seed, "Q", b, h, sh_k))
    if w.ill_conditioned:
        U = _normal(seed, "U", b, h, (w.T, w.n, w.rank))
        W = _normal(seed, "W", b, h, (w.rank, w.d_k))
        E = _normal(seed, "E", b, h, sh_k)
        K = _l2norm_rows(np.matmul(U, W) + np.float32(w.noise) * E)
    else:
        K = _l2norm_rows(_normal(seed, "K", b, h, sh_k))
    V = _normal(seed, "V", b, h, sh_v)
    G = _normal(seed, "G", b, h, sh_v, std=w.g_std)
    K_txt = _l2norm_rows(_normal(seed, "K_txt", b, h, (w.n_txt, w.d_k)))
    V_txt = _normal(seed, "V_txt", b, h, (w.n_txt, w.d_v))
    return dict(Q=Q, K=K, V=V, G=G, K_txt=K_txt, V_txt=V_txt)


def head_inputs(w: Workload | str, b: int, h: int, seed: int = 0) -> dict:
    """One (b, h)'s inputs in storage form (BF16 bits as uint16, E4M3 bits as
    uint8 of the values over their scale, or float32)."""
    if isinstance(w, str):
        w = WORKLOADS[w]
    f = head_f32(w, b, h, seed)
    if w.dtype == DTYPE_BF16:
        return {k: to_bf16_bits(v) for k, v in f.items()}
    if w.dtype == DTYPE_E4M3:
        sc = w.scales()
        return {k: to_e4m3_bits(v.astype(np.float64) / sc[k]) for k, v in f.items()}
    return {k: np.ascontiguousarray(v, dtype=np.float32) for k, v in f.items()}


def head_widened(w: Workload | str, b: int, h: int, seed: int = 0) -> dict:
    """One (b, h)'s inputs as the exact float64 values the device sees."""
    if isinstance(w, str):
        w = WORKLOADS[w]
    sc = w.scales()
    return {k: widen(v, w.dtype, sc[k]) for k, v in head_inputs(w, b, h, seed).items()}


def make_inputs(w: Workload | str, seed: int = 0) -> Inputs:
    """All of a workload's inputs as host numpy arrays (storage dtype)."""
    if isinstance(w, str):
        w = WORKLOADS[w]
    st = {DTYPE_BF16: np.uint16, DTYPE_E4M3: np.uint8}.get(w.dtype, np.float32)
    shapes = dict(Q=(w.T, w.n, w.d_k), K=(w.T, w.n, w.d_k), V=(w.T, w.n, w.d_v), G=(w.T, w.n, w.d_v),
                  K_txt=(w.n_txt, w.d_k), V_txt=(w.n_txt, w.d_v))
    out = {k: np.empty((w.B, w.H) + s, dtype=st) for k, s in shapes.items()}
    for b in range(w.B):
        for h in range(w.H):
            for k, v in head_inputs(w, b, h, seed).items():
                out[k][b, h] = v
    return Inputs(w, **out)


def make_inputs_torch(w: Workload | str, seed: int = 0, device="cuda", pin: bool = False) -> dict:
    """All inputs as torch tensors on `device` (or pinned host memory), drawn head by head.

    BF16 workloads give torch.bfloat16 tensors holding exactly the bits of
    ``head_inputs``; the host never holds more than one head at a time
    unless ``device`` is "cpu".
    """
    import torch
    if isinstance(w, str):
        w = WORKLOADS[w]
    tdt = {DTYPE_BF16: torch.bfloat16, DTYPE_E4M3: torch.uint8}.get(w.dtype, torch.float32)
    shapes = dict(Q=(w.T, w.n, w.d_k), K=(w.T, w.n, w.d_k), V=(w.T, w.n, w.d_v), G=(w.T, w.n, w.d_v),
                  K_txt=(w.n_txt, w.d_k), V_txt=(w.n_txt, w.d_v))
    kw = dict(pin_memory=True) if (pin and str(device) == "cpu") else {}
    out = {k: torch.empty((w.B, w.H) + s, dtype=tdt, device=device, **kw) for k, s in shapes.items()}
    for b in range(w.B):
        for h in range(w.H):
            for k, v in head_inputs(w, b, h, seed).items():
                t = torch.from_numpy(v)
                if tdt == torch.bfloat16:
                    t = t.view(torch.int16).view(torch.bfloat16)
                out[k][b, h].copy_(t)
    return out


def head_grad_out(w: Workload | str, b: int, h: int, seed: int = 0) -> np.ndarray:
    """One (b, h)'s output gradient dO for the backward, N(0, 1) of O's shape,
    in storage form (BF16 bits as uint16, or float32); its own stream."""
    if isinstance(w, str):
        w = WORKLOADS[w]
    x = _rng(seed, "dO", b, h).standard_normal((w.T, w.n, w.d_v), dtype=np.float32)
    return to_bf16_bits(x) if w.dtype == DTYPE_BF16 else x


def head_grad_out_widened(w: Workload | str, b: int, h: int, seed: int = 0) -> np.ndarray:
    """``head_grad_out`` as the exact float64 values the device sees."""
    if isinstance(w, str):
        w = WORKLOADS[w]
    return widen(head_grad_out(w, b, h, seed), w.dtype)


def grad_out_torch(w: Workload | str, seed: int = 0, device="cuda"):
    """dO for every (b, h) as a [B, H, T, n, d_v] torch tensor on `device`."""
    import torch
    if isinstance(w, str):
        w = WORKLOADS[w]
    tdt = torch.bfloat16 if w.dtype == DTYPE_BF16 else torch.float32
    out = torch.empty((w.B, w.H, w.T, w.n, w.d_v), dtype=tdt, device=device)
    for b in range(w.B):
        for h in range(w.H):
            t = torch.from_numpy(head_grad_out(w, b, h, seed))
            if tdt == torch.bfloat16:
                t = t.view(torch.int16).view(torch.bfloat16)
            out[b, h].copy_(t)
    return out


def token_major(x):
    """A tensor of the [B, H, T, n, d] layout as [B, T*n, H, d] (text [B, H, n_txt, d] as
    [B, n_txt, H, d]), contiguous: the inputs of the token-major layout, same values."""
    if x is None:
        return None
    if x.dim() == 5:
        B, H, T, n, d = x.shape
        return x.permute(0, 2, 3, 1, 4).reshape(B, T * n, H, d).contiguous()
    return x.permute(0, 2, 1, 3).contiguous()
