"""CPU oracle for the low-rank (SVD-factorized) transformer inference path.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path imports this module:
only the tests, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` may call it.  It shares no code with
the CUDA library (``rank_transformer_b200/csrc``) and imports nothing from it.

Every function is the plain mathematical definition of one step, written out
in float64 with numpy (a matmul or ``erf`` from a library serves as a step;
nothing is blocked, fused or reordered).  Inputs are the same bfloat16 bit
patterns the GPU receives, widened exactly with :func:`from_bf16`.

Sources (cited by page title and section):
  [v1.5]  "FlashSVD v1.5: Making Low-Rank Transformers Inference Actually
          Fast" (gist.science explainer, English), Technical Summary:
          Problem Statement; Methodology 1-4; Significance and Claims.
  [v1]    "FlashSVD: Memory-Efficient Inference with Streaming for Low-Rank
          Models" (abstract).
Where the pages are silent (norm epsilons, RoPE convention, head split,
attention scale) the plainest reading is taken and named in the docstring.

Pins: every function here is checked against closed forms, invariants,
special cases and tiny worked examples in ``tests/test_oracle.py``; none is
left unpinned.
"""
from __future__ import annotations

import math

import numpy as np
from scipy.special import erf as _erf

RMS_EPS = 1e-5      # reading: RMSNorm epsilon of Llama-family decoders
LN_EPS = 1e-12      # reading: LayerNorm epsilon of BERT-family encoders
ROPE_BASE = 10000.0  # reading: rotary base of Llama-family decoders


# ---------------------------------------------------------------- storage --

def from_bf16(bits) -> np.ndarray:
    """Widen bfloat16 bit patterns (uint16) exactly to float64."""
    b = np.ascontiguousarray(np.asarray(bits, dtype=np.uint16))
    return (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


# --------------------------------------------------------------- linears --

def lowrank_linear(x, U, V, bias=None):
    """Factorized linear y = (x U) V (+ bias).

    [v1] abstract: the truncated factors of W ~ U_r V_r are applied as two
    chained products whose rank-r intermediate z = x U is reduced on the fly;
    [v1.5] Methodology 1: every supported checkpoint is mapped to this common
    factorized representation.  x [M x d], U [d x r], V [r x n] -> [M x n].
    """
    z = np.asarray(x, np.float64) @ np.asarray(U, np.float64)
    y = z @ np.asarray(V, np.float64)
    if bias is not None:
        y = y + np.asarray(bias, np.float64)
    return y


def dense_linear(x, W, bias=None):
    """Dense y = x W (+ bias), for the output head (not factorized)."""
    y = np.asarray(x, np.float64) @ np.asarray(W, np.float64)
    if bias is not None:
        y = y + np.asarray(bias, np.float64)
    return y


# ----------------------------------------------------------- activations --

def silu(x):
    """SiLU(x) = x * sigmoid(x) = x / (1 + exp(-x))."""
    x = np.asarray(x, np.float64)
    return x / (1.0 + np.exp(-x))


def gelu(x):
    """Exact (erf) GELU(x) = x/2 * (1 + erf(x / sqrt 2))."""
    x = np.asarray(x, np.float64)
    return 0.5 * x * (1.0 + _erf(x / math.sqrt(2.0)))


# ------------------------------------------------------------------ MLPs --

def packed_gateup_mlp(x, U_gu, V_gu, U_dn, V_dn, r_f):
    """Packed gate|up low-rank SwiGLU MLP.

    [v1.5] Methodology 3 (Packed MLP Execution): the input-side factors of the
    gate and up branches are packed offline into one tensor
    U_gu = [U_g | U_u] (gate columns first); at run time one wide projection
    z = x U_gu is taken and its rank activations are split; each half goes
    through its own output factor (V_gu = V_g stacked on V_u).  The result is
    the exact low-rank MLP:
        h = SiLU(z_g V_g) * (z_u V_u),   y = (h U_dn) V_dn.
    """
    z = np.asarray(x, np.float64) @ np.asarray(U_gu, np.float64)
    z_g, z_u = z[:, :r_f], z[:, r_f:2 * r_f]
    V_gu = np.asarray(V_gu, np.float64)
    g = z_g @ V_gu[:r_f]
    u = z_u @ V_gu[r_f:2 * r_f]
    h = silu(g) * u
    return lowrank_linear(h, U_dn, V_dn)


def unpacked_gateup_mlp(x, U_g, U_u, V_g, V_u, U_dn, V_dn):
    """The same MLP with the gate and up branches run separately (the path
    that packing replaces, [v1.5] Methodology 3)."""
    g = lowrank_linear(x, U_g, V_g)
    u = lowrank_linear(x, U_u, V_u)
    return lowrank_linear(silu(g) * u, U_dn, V_dn)


def gateup_swiglu(x, U_gu, V_gu, r_f):
    """First two stages of the packed MLP only: h = SiLU(z_g V_g) * (z_u V_u),
    [M x f] (the shape measured in the isolated gate|up sweep)."""
    z = np.asarray(x, np.float64) @ np.asarray(U_gu, np.float64)
    V_gu = np.asarray(V_gu, np.float64)
    g = z[:, :r_f] @ V_gu[:r_f]
    u = z[:, r_f:2 * r_f] @ V_gu[r_f:2 * r_f]
    return silu(g) * u


# ----------------------------------------------------------------- norms --

def rmsnorm(x, g, eps=RMS_EPS):
    """RMSNorm over the last axis: x * g / sqrt(mean(x^2) + eps)."""
    x = np.asarray(x, np.float64)
    ms = np.mean(x * x, axis=-1, keepdims=True)
    return x / np.sqrt(ms + eps) * np.asarray(g, np.float64)


def layernorm(x, g, b, eps=LN_EPS):
    """LayerNorm over the last axis: (x - mean) / sqrt(var + eps) * g + b,
    with the biased (population) variance."""
    x = np.asarray(x, np.float64)
    mu = np.mean(x, axis=-1, keepdims=True)
    var = np.mean((x - mu) ** 2, axis=-1, keepdims=True)
    return (x - mu) / np.sqrt(var + eps) * np.asarray(g, np.float64) + \
        np.asarray(b, np.float64)


# ------------------------------------------------------------------ RoPE --

def rope(x, positions, base=ROPE_BASE):
    """Rotary position embedding, rotate-half convention (a reading; the
    pages name none).  x [..., T, D] with positions [T] (0-based): for
    i < D/2, with theta = pos * base^(-2i/D),
        (x_i, x_{i+D/2}) -> (x_i cos - x_{i+D/2} sin, x_{i+D/2} cos + x_i sin).
    """
    x = np.asarray(x, np.float64)
    D = x.shape[-1]
    half = D // 2
    inv = base ** (-2.0 * np.arange(half, dtype=np.float64) / D)
    ang = np.asarray(positions, np.float64)[:, None] * inv[None, :]
    c, s = np.cos(ang), np.sin(ang)
    a, b = x[..., :half], x[..., half:]
    return np.concatenate([a * c - b * s, b * c + a * s], axis=-1)


# ------------------------------------------------------------- attention --

def attention(q, k, v, causal=False, q_offset=0):
    """Scaled dot-product attention for one head, two-pass softmax.

    q [Tq x D], k [Tk x D], v [Tk x D]; scores s = q k^T / sqrt(D).  With
    ``causal`` query i (absolute position q_offset + i) sees keys j <= that
    position.  For each query: m = max_j s_j, p_j = exp(s_j - m) / sum exp,
    o = sum_j p_j v_j.
    """
    q = np.asarray(q, np.float64)
    k = np.asarray(k, np.float64)
    v = np.asarray(v, np.float64)
    s = (q @ k.T) / math.sqrt(q.shape[-1])
    if causal:
        qi = q_offset + np.arange(q.shape[0])[:, None]
        kj = np.arange(k.shape[0])[None, :]
        s = np.where(kj <= qi, s, -np.inf)
    m = np.max(s, axis=-1, keepdims=True)
    p = np.exp(s - m)
    p = p / np.sum(p, axis=-1, keepdims=True)
    return p @ v


def _split_heads(x, H):
    T, HD = x.shape
    return x.reshape(T, H, HD // H)


# -------------------------------------------------------- decoder layer --

def decoder_layer_prefill(x, w, H, positions=None, eps=RMS_EPS):
    """One pre-norm SwiGLU decoder layer over a whole sequence (prefill).

        n1 = rmsnorm(x, g1)
        q, k, v = lowrank(n1, U_q, V_q), lowrank(n1, U_k, V_k), lowrank(n1, U_v, V_v)
        q, k = rope(q), rope(k)          (heads = contiguous D-slices)
        a = causal attention per head
        h = x + lowrank(a, U_o, V_o)
        y = h + packed_gateup_mlp(rmsnorm(h, g2))

    x [S x d] (float64).  Returns y [S x d] and the rotated keys and the
    values [S x H x D] that prefill writes into the dense KV cache ([v1.5]
    Methodology 2: prefill runs over the full sequence and keeps its own
    attention; decode later reads this cache).
    """
    x = np.asarray(x, np.float64)
    S, d = x.shape
    pos = np.arange(S) if positions is None else np.asarray(positions)
    n1 = rmsnorm(x, w["g1"], eps)
    q = _split_heads(lowrank_linear(n1, w["U_q"], w["V_q"]), H)
    k = _split_heads(lowrank_linear(n1, w["U_k"], w["V_k"]), H)
    v = _split_heads(lowrank_linear(n1, w["U_v"], w["V_v"]), H)
    q = np.stack([rope(q[:, h], pos) for h in range(H)], axis=1)
    k = np.stack([rope(k[:, h], pos) for h in range(H)], axis=1)
    a = np.stack([attention(q[:, h], k[:, h], v[:, h], causal=True,
                            q_offset=int(pos[0]))
                  for h in range(H)], axis=1).reshape(S, d)
    h_res = x + lowrank_linear(a, w["U_o"], w["V_o"])
    r_f = w["U_gu"].shape[1] // 2
    y = h_res + packed_gateup_mlp(rmsnorm(h_res, w["g2"], eps), w["U_gu"],
                                  w["V_gu"], w["U_dn"], w["V_dn"], r_f)
    return y, k, v


def decoder_layer_decode(x, w, H, k_hist, v_hist, pos, eps=RMS_EPS):
    """One decode step of the same layer for B sequences.

    [v1.5] Methodology 2 ("reconstruct the present, read the past
    contiguously"): dense q, k, v are formed for the current token only,
    through the low-rank projections; the history is read from a dense
    contiguous KV cache.  The new (rotated) key and value are appended at
    index pos[b] and the query attends over keys 0..pos[b] inclusive.

    x [B x d]; k_hist, v_hist [B x >=pos[b] x H x D] (rows beyond pos[b] are
    ignored); pos [B] int.  Returns y [B x d], k_new [B x H x D], v_new.
    """
    x = np.asarray(x, np.float64)
    B, d = x.shape
    n1 = rmsnorm(x, w["g1"], eps)
    q = lowrank_linear(n1, w["U_q"], w["V_q"]).reshape(B, H, -1)
    k = lowrank_linear(n1, w["U_k"], w["V_k"]).reshape(B, H, -1)
    v = lowrank_linear(n1, w["U_v"], w["V_v"]).reshape(B, H, -1)
    a = np.empty((B, H, d // H))
    k_new = np.empty_like(k)
    for b in range(B):
        p = int(pos[b])
        qb = rope(q[b], np.full(H, p))          # [H x D], all at position p
        kb = rope(k[b], np.full(H, p))
        k_new[b] = kb
        for h in range(H):
            keys = np.concatenate([np.asarray(k_hist[b, :p, h], np.float64),
                                   kb[h][None]], axis=0)
            vals = np.concatenate([np.asarray(v_hist[b, :p, h], np.float64),
                                   v[b, h][None]], axis=0)
            a[b, h] = attention(qb[h][None], keys, vals)[0]
    h_res = x + lowrank_linear(a.reshape(B, d), w["U_o"], w["V_o"])
    r_f = w["U_gu"].shape[1] // 2
    y = h_res + packed_gateup_mlp(rmsnorm(h_res, w["g2"], eps), w["U_gu"],
                                  w["V_gu"], w["U_dn"], w["V_dn"], r_f)
    return y, k_new, v


# ------------------------------------------------------------ encoder FFN --

def lowrank_gelu_ffn(x, U_up, V_up, b_up, U_dn, V_dn, b_dn):
    """Low-rank GELU FFN of an encoder layer ([v1] abstract: the FFN of
    BERT-class encoders with both projections factorized; its intermediate
    activation is what the streamed kernel never materialises):

        y = lowrank(GELU(lowrank(x, U_up, V_up, b_up)), U_dn, V_dn, b_dn)
    """
    return lowrank_linear(gelu(lowrank_linear(x, U_up, V_up, b_up)), U_dn, V_dn, b_dn)


# --------------------------------------------------------- encoder layer --

def bert_layer(x, w, H, eps=LN_EPS):
    """One post-LN GELU encoder layer, bidirectional attention, every linear
    factorized with a bias ([v1] abstract: low-rank projections in both the
    self-attention and the FFN of BERT-Base-class encoders):

        h = LN1(x + lowrank_o(attn(lowrank_q(x), lowrank_k(x), lowrank_v(x))))
        y = LN2(h + lowrank_dn(GELU(lowrank_up(h))))
    """
    x = np.asarray(x, np.float64)
    S, d = x.shape
    q = _split_heads(lowrank_linear(x, w["U_q"], w["V_q"], w["b_q"]), H)
    k = _split_heads(lowrank_linear(x, w["U_k"], w["V_k"], w["b_k"]), H)
    v = _split_heads(lowrank_linear(x, w["U_v"], w["V_v"], w["b_v"]), H)
    a = np.stack([attention(q[:, h], k[:, h], v[:, h]) for h in range(H)],
                 axis=1).reshape(S, d)
    h = layernorm(x + lowrank_linear(a, w["U_o"], w["V_o"], w["b_o"]),
                  w["ln1_g"], w["ln1_b"], eps)
    f = lowrank_gelu_ffn(h, w["U_up"], w["V_up"], w["b_up"], w["U_dn"], w["V_dn"], w["b_dn"])
    return layernorm(h + f, w["ln2_g"], w["ln2_b"], eps)


# ------------------------------------------------------------ model head --

def lm_head(x, g_final, W_lm, eps=RMS_EPS):
    """Final RMSNorm then the dense output projection: logits [B x vocab]."""
    return dense_linear(rmsnorm(x, g_final, eps), W_lm)


def greedy(logits):
    """Greedy next token: argmax, ties to the lowest index."""
    return np.argmax(np.asarray(logits), axis=-1).astype(np.int64)


def decoder_model_prefill(tokens, emb, layers, g_final, W_lm, H):
    """Whole decoder over one prompt: embeddings -> layers -> head.
    Returns logits [S x vocab] and the per-layer (k, v) cache entries."""
    x = np.asarray(emb, np.float64)[np.asarray(tokens)]
    cache = []
    for w in layers:
        x, k, v = decoder_layer_prefill(x, w, H)
        cache.append((k, v))
    return lm_head(x, g_final, W_lm), cache


def widen_layer(w_bf16: dict) -> dict:
    """Widen every bf16 array of a weight dict to float64 (other entries are
    passed through)."""
    out = {}
    for k, v in w_bf16.items():
        if isinstance(v, np.ndarray) and v.dtype == np.uint16:
            out[k] = from_bf16(v)
        else:
            out[k] = v
    return out
