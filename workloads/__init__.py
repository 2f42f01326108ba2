"""Seeded synthetic inputs for the LUT binary GEMV, shared by the CUDA path's
tests/bench and by the oracle's tests.

This module only draws random numbers and stores them in plain interchange
formats. It holds none of the method's arithmetic: no dequantisation, no
lookup tables, no GEMV.

Interchange formats (the contract both sides read):

* ``sign_bits``: uint8 ``[K][M][N/8]``, canonical row-major bit planes. Bit
  ``t`` (LSB first) of byte ``j`` in row ``i`` is column ``8j+t``; a set bit
  means the sign +1, a clear bit means -1.
* ``alpha_r``: float32 ``[K][M]``; ``alpha_c``: float32 ``[K][N]`` or ``None``
  (meaning all ones).
* ``s_idx``: uint32 ``[nS]`` salient columns, strictly ascending.
* ``s_sign_bits``: uint8 ``[Ks][M][nS_pad/8]`` over the *compact* salient
  columns ``t = 0..nS-1`` (``nS_pad = roundup(nS, 32)``; pad bits are 0).
* ``s_alpha_r``: float32 ``[Ks][M]``; ``s_alpha_c``: float32 ``[Ks][nS]``.
* ``x``: ``[batch][N]`` as float32, float16, or bfloat16 held as its uint16
  bit pattern (numpy has no bfloat16).

The five workloads follow the FluxBin page's evaluation setting (batch-1
decode of LLaMA-shaped linear layers on one GPU, "Experimental results"
section) and the ternary weights of the FlashLM v6 page ("Ternary weights and
hardware efficiency" section). No trained weights exist here, so every tensor
is drawn from the stated distributions.

Draw order inside one matrix: B, alpha_r, alpha_c, S, Bs, alpha_r^s,
alpha_c^s, x.
"""

from __future__ import annotations

import dataclasses
from typing import Iterator, List, Optional, Tuple

import numpy as np

X_DTYPES = ("f32", "f16", "bf16")


def round_up(a: int, b: int) -> int:
    return (a + b - 1) // b * b


def salient_count(p: float, n: int) -> int:
    """Round half up: the number of salient columns for a fraction p of N."""
    return int(np.floor(p * n + 0.5))


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round float32 to bfloat16 (nearest, ties to even) and return the bits."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32).astype(np.uint64)
    lsb = (u >> 16) & 1
    r = ((u + 0x7FFF + lsb) >> 16).astype(np.uint16)
    return r


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (b.astype(np.uint32) << 16).view(np.float32)


def x_as_f32(x: np.ndarray, dtype: str) -> np.ndarray:
    """Widen stored activations to float32 (exact for all three dtypes)."""
    if dtype == "bf16":
        return bf16_bits_to_f32(x)
    return x.astype(np.float32)


def unpack_signs(bits: np.ndarray, ncols: int) -> np.ndarray:
    """Canonical bit planes -> int8 +/-1 over the first ``ncols`` columns."""
    u = np.unpackbits(bits, axis=-1, bitorder="little")[..., :ncols]
    return (u.astype(np.int8) * 2 - 1).astype(np.int8)


def pack_signs(signs: np.ndarray) -> np.ndarray:
    """int8 +/-1 ``[..., n]`` -> canonical bit planes ``[..., roundup(n,32)/8]``
    (columns past n are 0 bits)."""
    n = signs.shape[-1]
    npad = round_up(max(n, 1), 32)
    b = np.zeros(signs.shape[:-1] + (npad,), dtype=np.uint8)
    b[..., :n] = (signs > 0)
    return np.packbits(b, axis=-1, bitorder="little")


@dataclasses.dataclass
class Problem:
    """One synthetic weight set plus its activations."""

    name: str
    M: int
    N: int
    K: int
    g: int
    nS: int
    Ks: int
    batch: int
    x_dtype: str
    sign_bits: np.ndarray
    alpha_r: np.ndarray
    alpha_c: Optional[np.ndarray]
    s_idx: np.ndarray
    s_sign_bits: np.ndarray
    s_alpha_r: np.ndarray
    s_alpha_c: np.ndarray
    x: np.ndarray
    integer_mode: bool = False
    ternary: Optional[np.ndarray] = None  # int8 [M][N] in {-1,0,+1}, ternary inputs only

    @property
    def nS_pad(self) -> int:
        return round_up(self.nS, 32) if self.nS else 0

    def signs(self, rows: Optional[np.ndarray] = None) -> np.ndarray:
        b = self.sign_bits if rows is None else self.sign_bits[:, rows]
        return unpack_signs(b, self.N)

    def s_signs(self, rows: Optional[np.ndarray] = None) -> np.ndarray:
        b = self.s_sign_bits if rows is None else self.s_sign_bits[:, rows]
        return unpack_signs(b, self.nS)

    def x_f32(self) -> np.ndarray:
        return x_as_f32(self.x, self.x_dtype)

    def algorithmic_bytes(self) -> int:
        """Bytes the method itself must move for one call (weights, scales,
        salient data, activations, outputs); dense weights are not counted."""
        xb = {"f32": 4, "f16": 2, "bf16": 2}[self.x_dtype]
        b = self.K * self.M * self.N // 8 + 4 * self.K * self.M
        if self.alpha_c is not None:
            b += 4 * self.K * self.N
        b += self.batch * self.N * xb + 4 * self.batch * self.M
        if self.nS:
            b += (self.Ks * self.M * self.nS + 7) // 8 + 4 * self.Ks * self.M
            b += 4 * self.Ks * self.nS + 4 * self.nS
        return b


def _alpha(rng: np.random.Generator, shape, dist: str, integer_mode: bool,
           row_scale: bool) -> np.ndarray:
    if integer_mode:
        if row_scale:
            return rng.choice(np.array([0.5, 1.0, 1.5, 2.0], np.float32), size=shape)
        return rng.integers(1, 5, size=shape).astype(np.float32)
    if dist == "unit":   # |N(0,1)| + 0.1
        return (np.abs(rng.standard_normal(shape)) + 0.1).astype(np.float32)
    if dist == "small":  # |N(0,0.02)| + 1e-3
        return (np.abs(rng.normal(0.0, 0.02, shape)) + 1e-3).astype(np.float32)
    raise ValueError(dist)


def _x(rng: np.random.Generator, batch: int, n: int, dtype: str,
       integer_mode: bool) -> np.ndarray:
    if integer_mode:
        v = rng.integers(-4, 5, size=(batch, n)).astype(np.float32)
    else:
        v = rng.standard_normal((batch, n)).astype(np.float32)
    if dtype == "f32":
        return v
    if dtype == "f16":
        return v.astype(np.float16)
    if dtype == "bf16":
        return f32_to_bf16_bits(v)
    raise ValueError(dtype)


def group_row_scales(K: int, M: int, ngroups: int, *, seed, alpha_dist: str = "small",
                     integer_mode: bool = False) -> np.ndarray:
    """Row scales of the group-wise format, one per (base, row, group of
    input columns): float32 [K][M][ngroups], drawn like the per-row scales
    (same distributions, same integer-mode values) from their own seed."""
    rng = np.random.default_rng(seed)
    return _alpha(rng, (K, M, ngroups), alpha_dist, integer_mode, row_scale=True)


def make_problem(M: int, N: int, K: int, *, g: int = 4, nS: int = 0, Ks: int = 2,
                 batch: int = 1, x_dtype: str = "f32", alpha_dist: str = "small",
                 seed=0, integer_mode: bool = False, ternary: bool = False,
                 alpha_c_ones: bool = False, name: str = "custom") -> Problem:
    """Draw one weight set. ``ternary`` draws T in {-1,0,+1} (p=1/3 each) and
    stores it as two +/-1 bases (+1->(+1,+1), -1->(-1,-1), 0->(+1,-1)) whose
    row scales are both 0.5*alpha_r; alpha_c is then all ones (``None``)."""
    if N % 32:
        raise ValueError("N must be a multiple of 32")
    rng = np.random.default_rng(seed)
    tern = None
    if ternary:
        if K != 2:
            raise ValueError("ternary weights use exactly two bases")
        tern = rng.integers(-1, 2, size=(M, N), dtype=np.int8)
        b0 = np.where(tern >= 0, 1, -1).astype(np.int8)
        b1 = np.where(tern > 0, 1, -1).astype(np.int8)
        sign_bits = pack_signs(np.stack([b0, b1]))
        if integer_mode:
            ar = rng.choice(np.array([1.0, 2.0, 4.0], np.float32), size=M)
        else:
            ar = np.abs(rng.normal(0.0, 0.02, M)).astype(np.float32)
        alpha_r = np.stack([0.5 * ar, 0.5 * ar]).astype(np.float32)
        alpha_c = None
    else:
        sign_bits = rng.integers(0, 256, size=(K, M, N // 8), dtype=np.uint8)
        alpha_r = _alpha(rng, (K, M), alpha_dist, integer_mode, True)
        if alpha_c_ones:
            alpha_c = None
        else:
            alpha_c = _alpha(rng, (K, N), alpha_dist, integer_mode, False)
    if nS:
        if nS > N:
            raise ValueError("nS > N")
        s_idx = np.sort(rng.choice(N, size=nS, replace=False)).astype(np.uint32)
        nS_pad = round_up(nS, 32)
        sb = rng.integers(0, 256, size=(Ks, M, nS_pad // 8), dtype=np.uint8)
        # clear the pad bits so the compact planes hold exactly nS columns
        mask = np.zeros(nS_pad, np.uint8)
        mask[:nS] = 1
        sb &= np.packbits(mask, bitorder="little")[None, None, :]
        s_alpha_r = _alpha(rng, (Ks, M), alpha_dist, integer_mode, True)
        s_alpha_c = _alpha(rng, (Ks, nS), alpha_dist, integer_mode, False)
    else:
        s_idx = np.zeros(0, np.uint32)
        sb = np.zeros((Ks, M, 0), np.uint8)
        s_alpha_r = np.zeros((Ks, M), np.float32)
        s_alpha_c = np.zeros((Ks, 0), np.float32)
    x = _x(rng, batch, N, x_dtype, integer_mode)
    return Problem(name=name, M=M, N=N, K=K, g=g, nS=nS, Ks=Ks, batch=batch,
                   x_dtype=x_dtype, sign_bits=sign_bits, alpha_r=alpha_r,
                   alpha_c=alpha_c, s_idx=s_idx, s_sign_bits=sb,
                   s_alpha_r=s_alpha_r, s_alpha_c=s_alpha_c, x=x,
                   integer_mode=integer_mode, ternary=tern)


# ---------------------------------------------------------------------------
# The five named workloads.

def tiny(integer_mode: bool = False) -> Problem:
    """256x256, K=2, g=4, no salient columns, batch 1, fp32 x ~ N(0,1),
    alpha ~ |N(0,1)|+0.1; seed 0."""
    return make_problem(256, 256, 2, g=4, nS=0, x_dtype="f32", alpha_dist="unit",
                        seed=0, integer_mode=integer_mode, name="tiny_256")


def layer4096(integer_mode: bool = False, seed=1) -> Problem:
    """4096x4096, K=2, g=4, 128 salient columns with 2 extra bases, batch 1,
    fp16 x ~ N(0,1), alpha ~ |N(0,0.02)|+1e-3; seed 1."""
    return make_problem(4096, 4096, 2, g=4, nS=128, Ks=2, x_dtype="f16",
                        alpha_dist="small", seed=seed, integer_mode=integer_mode,
                        name="layer_4096x4096_k2")


def ternary11008(integer_mode: bool = False) -> Problem:
    """11008x4096 ternary weights (p=1/3 each) as two bases with 0.5*alpha_r,
    alpha_r ~ |N(0,0.02)| per row, alpha_c = 1, bf16 x ~ N(0,1); seed 2.
    The group width is not stated for this workload; g=4 is used, as for the
    other batch-1 layers."""
    return make_problem(11008, 4096, 2, g=4, nS=0, x_dtype="bf16", seed=2,
                        integer_mode=integer_mode, ternary=True,
                        name="ternary_11008x4096")


STEP7B_MATRICES: Tuple[Tuple[str, int, int], ...] = (
    ("q", 4096, 4096), ("k", 4096, 4096), ("v", 4096, 4096), ("o", 4096, 4096),
    ("gate", 11008, 4096), ("up", 11008, 4096), ("down", 4096, 11008),
)
STEP7B_LAYERS = 32


def step7b_matrix(layer: int, m: int, integer_mode: bool = False) -> Problem:
    """One GEMV of the 7B-shaped decode step: K=2, g=4, 3% salient columns
    (123 of 4096, 330 of 11008) with 2 extra bases, fp16 x drawn fresh per GEMV,
    alpha ~ |N(0,0.02)|+1e-3; seed 1000 + 7*layer + m."""
    name, M, N = STEP7B_MATRICES[m]
    return make_problem(M, N, 2, g=4, nS=salient_count(0.03, N), Ks=2,
                        x_dtype="f16", alpha_dist="small",
                        seed=1000 + 7 * layer + m, integer_mode=integer_mode,
                        name=f"7b_l{layer}_{name}")


def step7b(layers: int = STEP7B_LAYERS) -> Iterator[Problem]:
    for layer in range(layers):
        for m in range(len(STEP7B_MATRICES)):
            yield step7b_matrix(layer, m)


SHAPES70B: Tuple[Tuple[int, int], ...] = ((8192, 8192), (28672, 8192), (8192, 28672))
BATCHES70B: Tuple[int, ...] = (1, 4, 16)


def layer70b(shape_index: int, batch: int, integer_mode: bool = False) -> Problem:
    """70B-shaped layer: K=3, g=8, 5% salient columns (410 of 8192, 1434 of
    28672) with 2 extra bases, fp16 x ~ N(0,1) for ``batch`` tokens; alpha as
    in the 4096 layer. Seed (4, shape_index, batch)."""
    M, N = SHAPES70B[shape_index]
    return make_problem(M, N, 3, g=8, nS=salient_count(0.05, N), Ks=2,
                        batch=batch, x_dtype="f16", alpha_dist="small",
                        seed=(4, shape_index, batch), integer_mode=integer_mode,
                        name=f"70b_{M}x{N}_b{batch}")


def all_named() -> List[str]:
    return ["tiny", "layer4096", "ternary11008", "step7b", "layer70b"]


@dataclasses.dataclass
class FitInputs:
    """A dense matrix to decompose and calibration activations for the
    saliency proxy (inputs of the fitter, the step before the GEMV)."""

    W: np.ndarray   # float32 [M][N]
    X: np.ndarray   # float32 [T][N]


def fit_inputs(M: int, N: int, T: int = 64, seed=7) -> FitInputs:
    """A dense LLaMA-like layer W ~ N(0, 0.02^2) and activations with outlier
    channels: X[t][j] = s_j * N(0, 1), s_j = exp(N(0, 1)) (a few columns carry
    much larger activations, which is what makes some columns salient).  Draw
    order: W, s, X."""
    rng = np.random.default_rng(seed)
    W = rng.normal(0.0, 0.02, size=(M, N)).astype(np.float32)
    s = np.exp(rng.normal(0.0, 1.0, size=N))
    X = (rng.normal(0.0, 1.0, size=(T, N)) * s).astype(np.float32)
    return FitInputs(W=W, X=X)
