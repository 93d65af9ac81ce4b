"""Seeded synthetic inputs for the low-rank transformer hot path.

This module only draws numbers: factor matrices, activations, token ids and
norm gains.  It contains none of the arithmetic of the inference path itself
(no products, norms, attention or activations), so both the CPU oracle tests
and the CUDA path can take their inputs from here without sharing any of the
method's code.

All random draws use numpy ``Generator(PCG64(seed))``.  Values are drawn in
float32 and stored as bfloat16 bit patterns (``uint16``), rounded to nearest
even, which is the storage format of every weight and activation on the GPU
path ("bf16 cached execution", FlashSVD v1.5 explainer, Technical Summary,
Significance and Claims).

Shape conventions (row-major, last dimension contiguous):
  U [d_in x r], V [r x d_out]: one factorized linear y = (x U) V.
  U_gu [d x 2 r_f]: input-side gate and up factors packed along the rank axis,
      gate columns first (FlashSVD v1.5, Methodology 3, "Offline Prepacking").
  V_gu [2 r_f x f]: V_g stacked on V_u.
"""
from __future__ import annotations

import numpy as np

__all__ = [
    "rng_for", "f32_to_bf16", "normal_bf16", "rank_for_ratio", "svd_factors",
    "decoder_layer_weights", "bert_layer_weights", "tokens",
]


def rng_for(seed: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(seed))


def f32_to_bf16(a) -> np.ndarray:
    """Round float32 values to bfloat16 (round to nearest, ties to even).

    Returns the bit patterns as uint16.  NaN is not produced by the
    generators, so it is not special-cased.
    """
    a = np.ascontiguousarray(np.asarray(a, dtype=np.float32))
    bits = a.view(np.uint32).astype(np.uint64)
    lsb = (bits >> 16) & 1
    rounded = (bits + 0x7FFF + lsb) >> 16
    return rounded.astype(np.uint16)


def normal_bf16(rng: np.random.Generator, shape, std: float = 1.0,
                mean: float = 0.0) -> np.ndarray:
    x = rng.standard_normal(size=shape, dtype=np.float32) * np.float32(std)
    if mean:
        x = x + np.float32(mean)
    return f32_to_bf16(x)


def rank_for_ratio(rho: float, d_in: int, d_out: int, multiple: int = 64) -> int:
    """Rank that keeps a fraction ``rho`` of the d_in*d_out dense parameters.

    A rank-r factor pair holds r*(d_in+d_out) parameters; the rank is rounded
    to a multiple of 64 (a tile-friendly choice).  For 4096x4096 this gives
    832/1216/1664 at rho=0.4/0.6/0.8, and 1216/1792/2368 for 4096x11008.
    """
    exact = rho * d_in * d_out / (d_in + d_out)
    return int(multiple * round(exact / multiple))


def mixed_rho(seed: int, layers: int, choices=(0.4, 0.6, 0.8)) -> tuple:
    """One retention ratio per layer, drawn uniformly from ``choices`` in
    layer order with a seeded PCG64 generator (mixed-rank model)."""
    rng = rng_for(seed)
    return tuple(float(choices[i]) for i in rng.integers(0, len(choices), size=layers))


def _haar_columns(rng: np.random.Generator, n: int, k: int) -> np.ndarray:
    """n x k matrix with orthonormal columns, Haar distributed (QR of a
    Gaussian with the signs of R's diagonal folded into Q)."""
    g = rng.standard_normal(size=(n, k))
    q, r = np.linalg.qr(g)
    s = np.sign(np.diag(r))
    s[s == 0] = 1.0
    return q * s


def svd_factors(rng: np.random.Generator, d_in: int, d_out: int, r: int,
                decay: float = 0.5, full_rank: int | None = None):
    """Truncated-SVD factors of a synthetic W = P diag(sigma) Q^T.

    P [d_in x k] and Q [d_out x k] have Haar-orthonormal columns,
    k = full_rank or min(d_in, d_out), and sigma_i = i^(-decay), i = 1..k.
    The rank-r factors split sigma evenly: U = P_r diag(sqrt sigma_r),
    V = diag(sqrt sigma_r) Q_r^T.

    Returns (U_bf16, V_bf16, (P, sigma, Q)) where P, sigma, Q are float64 so a
    test can rebuild W exactly.
    """
    k = full_rank or min(d_in, d_out)
    if r > k:
        raise ValueError("rank exceeds the rank of W")
    P = _haar_columns(rng, d_in, k)
    Q = _haar_columns(rng, d_out, k)
    sigma = np.arange(1, k + 1, dtype=np.float64) ** (-decay)
    root = np.sqrt(sigma[:r])
    U = (P[:, :r] * root[None, :]).astype(np.float32)
    V = (root[:, None] * Q[:, :r].T).astype(np.float32)
    return f32_to_bf16(U), f32_to_bf16(V), (P, sigma, Q)


def decoder_layer_weights(rng: np.random.Generator, d: int, f: int,
                          r_attn: int, r_ffn: int, r_down: int | None = None,
                          gain_jitter: float = 0.0) -> dict:
    """Random-init factors of one pre-norm SwiGLU decoder layer.

    U ~ N(0, 1/d_in), V ~ N(0, 1/r); norm gains are 1 (optionally jittered by
    N(0, gain_jitter^2) so that tests exercise the multiply).
    """
    r_down = r_down or r_ffn
    w = {}
    for name in ("q", "k", "v", "o"):
        w["U_" + name] = normal_bf16(rng, (d, r_attn), std=d ** -0.5)
        w["V_" + name] = normal_bf16(rng, (r_attn, d), std=r_attn ** -0.5)
    w["U_gu"] = normal_bf16(rng, (d, 2 * r_ffn), std=d ** -0.5)
    w["V_gu"] = normal_bf16(rng, (2 * r_ffn, f), std=r_ffn ** -0.5)
    w["U_dn"] = normal_bf16(rng, (f, r_down), std=f ** -0.5)
    w["V_dn"] = normal_bf16(rng, (r_down, d), std=r_down ** -0.5)
    for name in ("g1", "g2"):
        if gain_jitter:
            w[name] = normal_bf16(rng, (d,), std=gain_jitter, mean=1.0)
        else:
            w[name] = f32_to_bf16(np.ones(d, dtype=np.float32))
    w["dims"] = dict(d=d, f=f, r_attn=r_attn, r_ffn=r_ffn, r_down=r_down)
    return w


def bert_layer_weights(rng: np.random.Generator, d: int, f: int, r: int,
                       bias_std: float = 0.0, gain_jitter: float = 0.0) -> dict:
    """Random-init factors of one post-LN GELU encoder layer (every linear at
    rank r, each with a bias; biases are 0 unless bias_std > 0)."""
    w = {}
    shapes = {"q": (d, d), "k": (d, d), "v": (d, d), "o": (d, d),
              "up": (d, f), "dn": (f, d)}
    for name, (di, do) in shapes.items():
        w["U_" + name] = normal_bf16(rng, (di, r), std=di ** -0.5)
        w["V_" + name] = normal_bf16(rng, (r, do), std=r ** -0.5)
        if bias_std:
            w["b_" + name] = normal_bf16(rng, (do,), std=bias_std)
        else:
            w["b_" + name] = f32_to_bf16(np.zeros(do, dtype=np.float32))
    for name in ("ln1", "ln2"):
        if gain_jitter:
            w[name + "_g"] = normal_bf16(rng, (d,), std=gain_jitter, mean=1.0)
            w[name + "_b"] = normal_bf16(rng, (d,), std=gain_jitter)
        else:
            w[name + "_g"] = f32_to_bf16(np.ones(d, dtype=np.float32))
            w[name + "_b"] = f32_to_bf16(np.zeros(d, dtype=np.float32))
    w["dims"] = dict(d=d, f=f, r=r)
    return w


def tokens(rng: np.random.Generator, shape, vocab: int) -> np.ndarray:
    return rng.integers(0, vocab, size=shape, dtype=np.int64).astype(np.int32)
