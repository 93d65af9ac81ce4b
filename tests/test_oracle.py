"""Pins for the CPU oracle: closed forms, invariants, special cases and tiny
worked examples that hold independently of the oracle's own code.

Every pin is a function of the oracle module ``o`` so that
``test_pins_catch_planted_mistakes`` can run the same pins against copies of
the oracle with one plausible mistake planted (on the CPU) and show that each
mistake is caught.
"""
import importlib.util
import json
import math
import os

import numpy as np
import pytest
from scipy.stats import norm

from oracle import flashsvd_oracle as oracle
from rank_transformer_b200 import synth

HERE = os.path.dirname(os.path.abspath(__file__))


def _rng(seed=0):
    return np.random.default_rng(seed)


def _close(a, b, tol=1e-12):
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    assert a.shape == b.shape, (a.shape, b.shape)
    scale = max(1.0, float(np.max(np.abs(b))) if b.size else 1.0)
    err = float(np.max(np.abs(a - b))) if a.size else 0.0
    assert err <= tol * scale, f"max err {err} > {tol * scale}"


def _tiny_layer(rng, d=32, H=4, f=48, r=8, gain_jitter=True):
    w = {}
    for n in ("q", "k", "v", "o"):
        w["U_" + n] = rng.standard_normal((d, r)) / math.sqrt(d)
        w["V_" + n] = rng.standard_normal((r, d)) / math.sqrt(r)
    w["U_gu"] = rng.standard_normal((d, 2 * r)) / math.sqrt(d)
    w["V_gu"] = rng.standard_normal((2 * r, f)) / math.sqrt(r)
    w["U_dn"] = rng.standard_normal((f, r)) / math.sqrt(f)
    w["V_dn"] = rng.standard_normal((r, d)) / math.sqrt(r)
    w["g1"] = 1 + (0.1 * rng.standard_normal(d) if gain_jitter else 0)
    w["g2"] = 1 + (0.1 * rng.standard_normal(d) if gain_jitter else 0)
    return w


# ------------------------------------------------------------ pins ------

def pin_lowrank_worked_example(o):
    # Hand-computed: Z = X U = [[3, 2], [-1, 0]]; Y = Z V.
    X = np.array([[1., 0., 2.], [0., 1., -1.]])
    U = np.array([[1., 0.], [0., 1.], [1., 1.]])
    V = np.array([[1., 2., 0., 1.], [0., 1., 1., -1.]])
    _close(o.lowrank_linear(X, U, V), [[3., 8., 2., 1.], [-1., -2., 0., -1.]])
    b = np.array([1., 0., -1., 0.5])
    _close(o.lowrank_linear(X, U, V, b), [[4., 8., 1., 1.5], [0., -2., -1., -0.5]])


def pin_lowrank_associativity(o):
    rng = _rng(1)
    for (M, d, r, n) in ((3, 5, 2, 7), (16, 24, 8, 40)):
        X, U, V = (rng.standard_normal(s) for s in ((M, d), (d, r), (r, n)))
        _close(o.lowrank_linear(X, U, V), X @ (U @ V), 1e-12)


def pin_lowrank_identity_factor(o):
    # r = d and U = I: the factorized linear is the plain product X V.
    rng = _rng(2)
    X, V = rng.standard_normal((5, 6)), rng.standard_normal((6, 9))
    _close(o.lowrank_linear(X, np.eye(6), V), np.matmul(X, V))


def pin_svd_reconstruction(o):
    # W = P diag(sigma) Q^T from the generator; at full rank U V rebuilds W,
    # and at rank r the squared Frobenius error is sum_{i>r} sigma_i^2
    # (Eckart-Young).  Factors are kept in float64 here.
    d, n = 24, 40
    _, _, (P, sigma, Q) = synth.svd_factors(synth.rng_for(0), d, n, r=d)
    W = (P * sigma) @ Q.T
    for r in (d, 10, 3):
        root = np.sqrt(sigma[:r])
        U, V = P[:, :r] * root, root[:, None] * Q[:, :r].T
        W_r = o.lowrank_linear(np.eye(d), U, V)
        if r == d:
            _close(W_r, W, 1e-12)
        err2 = float(np.sum((W - W_r) ** 2))
        assert abs(err2 - float(np.sum(sigma[r:] ** 2))) <= 1e-10 * max(1.0, err2)


def pin_activations(o):
    x = np.array([0.0, 1.0, -1.0, 2.5, -3.0, 30.0])
    # SiLU(1) = 1/(1+e^-1); SiLU(x) - SiLU(-x) = x.
    _close(o.silu(np.array([0.0, 1.0, -1.0])),
           [0.0, 0.7310585786300049, -0.2689414213699951])
    _close(o.silu(x) - o.silu(-x), x)
    # GELU(x) = x Phi(x), Phi the standard normal CDF.
    _close(o.gelu(x), x * norm.cdf(x))
    _close(o.gelu(np.array([1.0])), [0.8413447460685429])


def pin_packed_equals_unpacked(o):
    rng = _rng(3)
    M, d, r, f, r_dn = 4, 16, 5, 12, 6
    U_g, U_u = rng.standard_normal((d, r)), rng.standard_normal((d, r))
    V_g, V_u = rng.standard_normal((r, f)), rng.standard_normal((r, f))
    U_dn, V_dn = rng.standard_normal((f, r_dn)), rng.standard_normal((r_dn, d))
    X = rng.standard_normal((M, d))
    packed = o.packed_gateup_mlp(X, np.concatenate([U_g, U_u], 1),
                                 np.concatenate([V_g, V_u], 0), U_dn, V_dn, r)
    _close(packed, o.unpacked_gateup_mlp(X, U_g, U_u, V_g, V_u, U_dn, V_dn), 1e-12)


def pin_packed_mlp_closed_form(o):
    # U_gu = [I | I], V_gu = [diag(a); I], U_dn = V_dn = I:
    # gate = a*x, up = x, so y = SiLU(a*x) * x elementwise.
    rng = _rng(4)
    d = 6
    a = rng.standard_normal(d)
    X = rng.standard_normal((3, d))
    I = np.eye(d)
    y = o.packed_gateup_mlp(X, np.concatenate([I, I], 1),
                            np.concatenate([np.diag(a), I], 0), I, I, d)
    _close(y, (a * X) / (1 + np.exp(-(a * X))) * X)
    _close(o.gateup_swiglu(X, np.concatenate([I, I], 1),
                           np.concatenate([np.diag(a), I], 0), d), y)


def pin_rmsnorm(o):
    # [3, 4]: mean square 12.5.
    _close(o.rmsnorm(np.array([[3.0, 4.0]]), np.ones(2), eps=0.0),
           [[3 / math.sqrt(12.5), 4 / math.sqrt(12.5)]])
    rng = _rng(5)
    x = rng.standard_normal((4, 32))
    g = rng.standard_normal(32)
    y = o.rmsnorm(x, np.ones(32))
    ms = np.mean(x * x, 1)
    _close(np.sqrt(np.mean(y * y, 1)), np.sqrt(ms / (ms + o.RMS_EPS)))
    _close(o.rmsnorm(x, g), y * g)
    _close(o.rmsnorm(7.5 * x, g, eps=0.0), o.rmsnorm(x, g, eps=0.0))


def pin_layernorm(o):
    # [1, 2, 3, 4]: mean 2.5, population variance 1.25.
    s = math.sqrt(1.25)
    _close(o.layernorm(np.array([[1., 2., 3., 4.]]), np.ones(4), np.zeros(4), eps=0.0),
           [[-1.5 / s, -0.5 / s, 0.5 / s, 1.5 / s]])
    rng = _rng(6)
    x = 3 + 2 * rng.standard_normal((5, 64))
    y = o.layernorm(x, np.ones(64), np.zeros(64), eps=0.0)
    _close(np.mean(y, 1), np.zeros(5))
    _close(np.mean(y * y, 1), np.ones(5))
    g, b = rng.standard_normal(64), rng.standard_normal(64)
    _close(o.layernorm(x + 11.0, g, b, eps=0.0), y * g + b)


def pin_rope(o):
    p = np.array([0.3, 5.0, 123.0])
    # D = 2: a plane rotation by angle pos.
    _close(o.rope(np.tile([1.0, 0.0], (3, 1)), p), np.stack([np.cos(p), np.sin(p)], 1))
    _close(o.rope(np.tile([0.0, 1.0], (3, 1)), p), np.stack([-np.sin(p), np.cos(p)], 1))
    # D = 4: pair (0,2) turns at rate 1, pair (1,3) at rate base^(-1/2) = 0.01.
    y = o.rope(np.array([[0.0, 1.0, 0.0, 0.0]]), np.array([100.0]))
    _close(y, [[0.0, math.cos(1.0), 0.0, math.sin(1.0)]])
    rng = _rng(7)
    x = rng.standard_normal((6, 16))
    _close(o.rope(x, np.zeros(6)), x)                                  # identity
    _close(np.linalg.norm(o.rope(x, np.arange(6) * 7.0), axis=1),
           np.linalg.norm(x, axis=1))                                   # isometry
    a, b = np.arange(6) * 3.0, np.arange(6) * 5.0 + 1
    _close(o.rope(o.rope(x, a), b), o.rope(x, a + b))                   # composition
    q, k = rng.standard_normal((1, 16)), rng.standard_normal((1, 16))
    dots = [float((o.rope(q, [m + 4.0]) @ o.rope(k, [m]).T)[0, 0]) for m in (0, 9, 40)]
    _close(dots, [dots[0]] * 3)                                         # relative


def pin_attention(o):
    rng = _rng(8)
    q, k, v = (rng.standard_normal((1, 8)) for _ in range(3))
    _close(o.attention(q, k, v), v)                                     # one key
    vs = rng.standard_normal((5, 8))
    _close(o.attention(q, np.tile(k, (5, 1)), vs), vs.mean(0, keepdims=True))
    _close(o.attention(np.zeros((1, 8)), rng.standard_normal((5, 8)), vs),
           vs.mean(0, keepdims=True))
    # D = 4 (scale 1/2): scores 0 and ln 3 -> weights 1/4, 3/4.
    qq = np.array([[2 * math.log(3.0), 0, 0, 0]])
    kk = np.array([[0.0, 0, 0, 0], [1.0, 0, 0, 0]])
    vv = np.array([[4.0, 0, 8, 1], [0.0, 4, -4, 1]])
    _close(o.attention(qq, kk, vv), [[1.0, 3.0, -1.0, 1.0]])
    # Shifting every key by c moves every score by q.c: output unchanged.
    Q, K, V = (rng.standard_normal((6, 8)) for _ in range(3))
    _close(o.attention(Q, K + rng.standard_normal(8), V), o.attention(Q, K, V))
    # Causal: row i ignores keys > i; row 0 returns v_0.
    out = o.attention(Q, K, V, causal=True)
    K2, V2 = K.copy(), V.copy()
    K2[4:] += 10.0
    V2[4:] -= 3.0
    _close(o.attention(Q, K2, V2, causal=True)[:4], out[:4])
    _close(out[0], V[0])
    _close(out[5], o.attention(Q[5:6], K, V)[0])
    # With q_offset = 5 a single query sees all 6 keys.
    _close(o.attention(Q[5:6], K, V, causal=True, q_offset=5), o.attention(Q[5:6], K, V))


def pin_decode_matches_prefill(o):
    # "Reconstruct the present, read the past contiguously": decoding token t
    # against the cache written by prefill of tokens < t must give prefill's
    # row t, and the appended key/value must be prefill's cache row t.
    rng = _rng(9)
    H, S = 4, 6
    w = _tiny_layer(rng)
    x = rng.standard_normal((S, 32))
    y, k, v = o.decoder_layer_prefill(x, w, H)
    for t in range(S):
        yt, kt, vt = o.decoder_layer_decode(x[t:t + 1], w, H, k[None], v[None], [t])
        _close(yt[0], y[t], 1e-11)
        _close(kt[0], k[t], 1e-11)
        _close(vt[0], v[t], 1e-11)


def pin_decoder_layer_special_cases(o):
    rng = _rng(10)
    H, d = 4, 32
    w = _tiny_layer(rng)
    x = rng.standard_normal((5, d))
    w0 = dict(w, V_o=np.zeros_like(w["V_o"]), V_dn=np.zeros_like(w["V_dn"]))
    _close(o.decoder_layer_prefill(x, w0, H)[0], x)          # pure residual
    # One token attends to itself only: y = x + ((n1 U_v V_v) U_o V_o) when
    # the MLP is switched off.
    w1 = dict(w, V_dn=np.zeros_like(w["V_dn"]))
    x1 = x[:1]
    n1 = x1 / np.sqrt(np.mean(x1 * x1) + o.RMS_EPS) * w["g1"]
    expect = x1 + ((((n1 @ w["U_v"]) @ w["V_v"]) @ w["U_o"]) @ w["V_o"])
    _close(o.decoder_layer_prefill(x1, w1, H)[0], expect, 1e-11)


def pin_bert_layer(o):
    rng = _rng(11)
    S, d, H, f, r = 6, 16, 2, 24, 4
    w = {}
    for n, (di, do) in {"q": (d, d), "k": (d, d), "v": (d, d), "o": (d, d),
                        "up": (d, f), "dn": (f, d)}.items():
        w["U_" + n] = rng.standard_normal((di, r)) / math.sqrt(di)
        w["V_" + n] = rng.standard_normal((r, do)) / math.sqrt(r)
        w["b_" + n] = 0.1 * rng.standard_normal(do)
    for n in ("ln1", "ln2"):
        w[n + "_g"], w[n + "_b"] = np.ones(d), np.zeros(d)
    x = rng.standard_normal((S, d))
    y = o.bert_layer(x, w, H)
    _close(np.mean(y, 1), np.zeros(S), 1e-10)
    _close(np.mean(y * y, 1), np.ones(S), 1e-6)
    # Bidirectional, no positions: permuting tokens permutes the output.
    perm = np.array([3, 0, 5, 1, 4, 2])
    _close(o.bert_layer(x[perm], w, H), y[perm], 1e-11)
    # All output factors and biases zero: y = LN(LN(x)).
    wz = dict(w)
    for n in ("o", "dn"):
        wz["V_" + n] = np.zeros_like(w["V_" + n])
        wz["b_" + n] = np.zeros_like(w["b_" + n])
    ln = lambda t: (t - t.mean(1, keepdims=True)) / np.sqrt(t.var(1, keepdims=True) + o.LN_EPS)
    _close(o.bert_layer(x, wz, H), ln(ln(x)), 1e-10)


def pin_head_and_greedy(o):
    rng = _rng(12)
    x, g = rng.standard_normal((3, 8)), rng.standard_normal(8)
    _close(o.lm_head(x, g, np.eye(8)), o.rmsnorm(x, g))
    assert list(o.greedy(np.array([[1.0, 3.0, 3.0, -1.0], [0.0, 0.0, 0.0, 0.0]]))) == [1, 0]
    emb = rng.standard_normal((10, 8))
    toks = np.array([3, 7, 3])
    logits, cache = o.decoder_model_prefill(toks, emb, [], np.ones(8), np.eye(8), H=2)
    assert cache == []
    _close(logits, o.rmsnorm(emb[toks], np.ones(8)))


def _two_token_case(eps=0.0):
    """Hand-worked two-token, two-head decoder example (d = 4, H = 2, D = 2,
    every factor the identity, RMSNorm with g = 1, MLP off).

    x0 = [1, 1, 1, 1] and x1 = [sqrt2, 0, 0, sqrt2] both have mean square 1,
    so n1 = c x with c = 1 / sqrt(1 + eps), and q = k = v = n1.  Head 0 holds
    dims (0, 1), head 1 dims (2, 3).  RoPE at position 0 is the identity; at
    position 1 it turns each head's pair by 1 radian.  Token 0 sees only
    itself: a0 = v0.  Token 1, head 0: q = c sqrt2 [cos 1, sin 1]; its
    scores (scale 1/sqrt2) to k0 = c [1, 1] and to itself are
    c^2 (cos 1 + sin 1) and c^2 sqrt2.  Head 1: q = c sqrt2 [-sin 1, cos 1],
    scores c^2 (cos 1 - sin 1) and c^2 sqrt2.  The values are not rotated.
    """
    s2, c1, s1 = math.sqrt(2.0), math.cos(1.0), math.sin(1.0)
    c = 1.0 / math.sqrt(1.0 + eps)
    x = np.array([[1.0, 1.0, 1.0, 1.0], [s2, 0.0, 0.0, s2]])
    I = np.eye(4)
    w = {n: I for n in ("U_q", "V_q", "U_k", "V_k", "U_v", "V_v", "U_o", "V_o")}
    w.update(U_gu=np.concatenate([I, I], 1), V_gu=np.concatenate([I, I], 0),
             U_dn=I, V_dn=np.zeros((4, 4)), g1=np.ones(4), g2=np.ones(4))

    def two_key(a, b):          # softmax weight of the first of two scores
        return 1.0 / (1.0 + math.exp(b - a))
    p_h0 = two_key(c * c * (c1 + s1), c * c * s2)
    p_h1 = two_key(c * c * (c1 - s1), c * c * s2)
    a1 = c * np.array([p_h0 * 1 + (1 - p_h0) * s2, p_h0 * 1 + (1 - p_h0) * 0,
                       p_h1 * 1 + (1 - p_h1) * 0, p_h1 * 1 + (1 - p_h1) * s2])
    y = np.stack([x[0] + c * x[0], x[1] + a1])
    k_rot = c * np.array([[[1.0, 1.0], [1.0, 1.0]],
                          [[s2 * c1, s2 * s1], [-s2 * s1, s2 * c1]]])
    return x, w, y, k_rot


def pin_decoder_layer_worked_example(o):
    # Prefill over both tokens, and decode of token 1 against a cache that
    # holds only token 0 (written out by hand), give the hand-worked rows.
    x, w, y, k_rot = _two_token_case()
    yp, kp, vp = o.decoder_layer_prefill(x, w, 2, eps=0.0)
    _close(yp, y)
    _close(kp, k_rot)
    _close(vp, x.reshape(2, 2, 2))
    k_hist = np.array([[[[1.0, 1.0], [1.0, 1.0]]]])
    v_hist = k_hist.copy()
    yd, kd, vd = o.decoder_layer_decode(x[1:], w, 2, k_hist, v_hist, [1], eps=0.0)
    _close(yd[0], y[1])
    _close(kd[0], k_rot[1])
    _close(vd[0], x[1].reshape(2, 2))


def pin_decoder_mlp_branch(o):
    # Attention branch off (V_o = 0): h = x.  Closed-form MLP factors
    # U_gu = [I | I], V_gu = [diag(a); I], U_dn = V_dn = I make the branch
    # SiLU(a * n2) * n2 with n2 = rmsnorm(x) under the SECOND gain g2, which
    # differs from g1 here; y = x + that.  Prefill and decode alike.
    rng = _rng(13)
    d, H = 8, 2
    I = np.eye(d)
    a = rng.standard_normal(d)
    w = _tiny_layer(rng, d=d, H=H, f=d, r=d)
    w.update(V_o=np.zeros((d, d)), U_gu=np.concatenate([I, I], 1),
             V_gu=np.concatenate([np.diag(a), I], 0), U_dn=I, V_dn=I,
             g2=1.0 + 0.5 * rng.standard_normal(d))
    x = rng.standard_normal((3, d))
    ms = np.mean(x * x, axis=1, keepdims=True)
    n2 = x / np.sqrt(ms + o.RMS_EPS) * w["g2"]
    expect = x + (a * n2) / (1.0 + np.exp(-a * n2)) * n2
    _close(o.decoder_layer_prefill(x, w, H)[0], expect, 1e-11)
    D = d // H
    hist = rng.standard_normal((3, 4, H, D))
    yd = o.decoder_layer_decode(x, w, H, hist, hist, [4, 2, 0])[0]
    _close(yd, expect, 1e-11)


def pin_bert_layer_closed_form(o):
    # Query factor and bias zero: every score is 0, so each token averages
    # the values of ALL tokens (bidirectional).  With U_v = V_v = U_o =
    # V_o = I:  h = LN1(x + mean_t(x) + b_v + b_o).
    # FFN with U_up = I, V_up = diag(a), U_dn = V_dn = I:
    #   y = LN2(h + GELU(a * h + b_up) + b_dn),  GELU(t) = t * Phi(t).
    rng = _rng(14)
    S, d, H = 5, 8, 2
    I = np.eye(d)
    a = rng.standard_normal(d)
    w = {"U_q": np.zeros((d, d)), "V_q": I, "b_q": np.zeros(d),
         "U_k": rng.standard_normal((d, d)), "V_k": I, "b_k": rng.standard_normal(d),
         "U_v": I, "V_v": I, "b_v": rng.standard_normal(d),
         "U_o": I, "V_o": I, "b_o": rng.standard_normal(d),
         "U_up": I, "V_up": np.diag(a), "b_up": rng.standard_normal(d),
         "U_dn": I, "V_dn": I, "b_dn": rng.standard_normal(d)}
    for n in ("ln1", "ln2"):
        w[n + "_g"] = 1.0 + 0.3 * rng.standard_normal(d)
        w[n + "_b"] = 0.3 * rng.standard_normal(d)
    x = rng.standard_normal((S, d))

    def ln(t, g, b):
        mu = t.mean(axis=1, keepdims=True)
        var = ((t - mu) ** 2).mean(axis=1, keepdims=True)
        return (t - mu) / np.sqrt(var + o.LN_EPS) * g + b
    h = ln(x + x.mean(axis=0, keepdims=True) + w["b_v"] + w["b_o"], w["ln1_g"], w["ln1_b"])
    t = a * h + w["b_up"]
    y = ln(h + t * norm.cdf(t) + w["b_dn"], w["ln2_g"], w["ln2_b"])
    _close(o.bert_layer(x, w, H), y, 1e-10)


def pin_encoder_ffn(o):
    # U_up = I, V_up = diag(a), U_dn = V_dn = I: y = GELU(a x + b_up) + b_dn
    # elementwise, GELU(t) = t Phi(t).  With a rank-3 pair and zero biases,
    # y = GELU(x (U_up V_up)) (U_dn V_dn) with the products formed first.
    rng = _rng(15)
    d = 6
    I = np.eye(d)
    a, b_up, b_dn = (rng.standard_normal(d) for _ in range(3))
    x = rng.standard_normal((4, d))
    t = a * x + b_up
    _close(o.lowrank_gelu_ffn(x, I, np.diag(a), b_up, I, I, b_dn), t * norm.cdf(t) + b_dn)
    f, r = 10, 3
    U1, V1 = rng.standard_normal((d, r)), rng.standard_normal((r, f))
    U2, V2 = rng.standard_normal((f, r)), rng.standard_normal((r, d))
    h = x @ (U1 @ V1)
    _close(o.lowrank_gelu_ffn(x, U1, V1, None, U2, V2, None), (h * norm.cdf(h)) @ (U2 @ V2), 1e-11)


def pin_model_and_head(o):
    # Output head with a square, non-symmetric W (a transposed W changes the
    # result): rows of mean square 1, g = 1, eps = 0 give logits = x W.
    x = np.array([[1.0, -1.0, 1.0, -1.0], [2.0, 0.0, 0.0, 0.0]])
    W = np.array([[1.0, 2.0, 0.0, 0.0], [0.0, 1.0, 0.0, 5.0],
                  [3.0, 0.0, 1.0, 0.0], [0.0, 0.0, 7.0, 1.0]])
    _close(o.lm_head(x, np.ones(4), W, eps=0.0), [[4.0, 1.0, -6.0, -6.0], [2.0, 4.0, 0.0, 0.0]])
    # One-layer model over the worked two-token example: embedding rows
    # chosen so emb[tokens] = x; logits = rmsnorm(y) W; the cache holds the
    # rotated keys and the plain values.
    eps = o.RMS_EPS
    xs, w, y, k_rot = _two_token_case(eps)
    emb = np.zeros((5, 4))
    emb[3], emb[1] = xs[0], xs[1]
    logits, cache = o.decoder_model_prefill(np.array([3, 1]), emb, [w], np.ones(4), W, H=2)
    yn = y / np.sqrt(np.mean(y * y, axis=1, keepdims=True) + eps)
    _close(logits, yn @ W)
    assert len(cache) == 1
    _close(cache[0][0], k_rot)
    _close(cache[0][1], xs.reshape(2, 2, 2) / math.sqrt(1.0 + eps))


def pin_from_bf16(o):
    bits = np.array([0x3F80, 0xBF80, 0x4049, 0x0000, 0x8000, 0x7F7F, 0x0001], np.uint16)
    want = [1.0, -1.0, 3.140625, 0.0, -0.0, 3.3895313892515355e38, 9.183549615799121e-41]
    _close(o.from_bf16(bits), want, 0.0)


PINS = [pin_lowrank_worked_example, pin_lowrank_associativity,
        pin_lowrank_identity_factor, pin_svd_reconstruction, pin_activations,
        pin_packed_equals_unpacked, pin_packed_mlp_closed_form, pin_rmsnorm,
        pin_layernorm, pin_rope, pin_attention, pin_decode_matches_prefill,
        pin_decoder_layer_special_cases, pin_bert_layer, pin_head_and_greedy,
        pin_from_bf16, pin_decoder_layer_worked_example, pin_decoder_mlp_branch,
        pin_bert_layer_closed_form, pin_model_and_head, pin_encoder_ffn]


@pytest.mark.parametrize("pin", PINS, ids=[p.__name__ for p in PINS])
def test_oracle_pin(pin):
    pin(oracle)


# ------------------------------------------------- planted mistakes ------

def _fresh_oracle():
    path = os.path.join(os.path.dirname(HERE), "oracle", "flashsvd_oracle.py")
    spec = importlib.util.spec_from_file_location("_oracle_mutant", path)
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _mut_rope_sign(m):
    def rope(x, positions, base=m.ROPE_BASE):
        x = np.asarray(x, np.float64)
        D = x.shape[-1]
        half = D // 2
        inv = base ** (-2.0 * np.arange(half) / D)
        ang = np.asarray(positions, np.float64)[:, None] * inv[None, :]
        c, s = np.cos(ang), np.sin(ang)
        a, b = x[..., :half], x[..., half:]
        return np.concatenate([a * c + b * s, b * c - a * s], axis=-1)
    m.rope = rope


def _mut_rope_interleaved(m):
    def rope(x, positions, base=m.ROPE_BASE):
        x = np.asarray(x, np.float64)
        D = x.shape[-1]
        inv = base ** (-2.0 * np.arange(D // 2) / D)
        ang = np.asarray(positions, np.float64)[:, None] * inv[None, :]
        c, s = np.cos(ang), np.sin(ang)
        a, b = x[..., 0::2], x[..., 1::2]
        out = np.empty_like(x)
        out[..., 0::2], out[..., 1::2] = a * c - b * s, b * c + a * s
        return out
    m.rope = rope


def _mut_attention_noscale(m):
    orig = m.attention
    m.attention = lambda q, k, v, causal=False, q_offset=0: orig(
        np.asarray(q) * math.sqrt(np.asarray(q).shape[-1]), k, v, causal, q_offset)


def _mut_attention_causal_strict(m):
    def attention(q, k, v, causal=False, q_offset=0):
        s = (q @ k.T) / math.sqrt(q.shape[-1])
        if causal:
            qi = q_offset + np.arange(q.shape[0])[:, None]
            kj = np.arange(k.shape[0])[None, :]
            s = np.where(kj < qi, s, -np.inf)
            s[np.all(np.isinf(s), axis=1), 0] = 0.0
        p = np.exp(s - s.max(-1, keepdims=True))
        return (p / p.sum(-1, keepdims=True)) @ v
    m.attention = attention


def _mut_swiglu_swapped(m):
    def packed(x, U_gu, V_gu, U_dn, V_dn, r_f):
        z = x @ U_gu
        g, u = z[:, :r_f] @ V_gu[:r_f], z[:, r_f:] @ V_gu[r_f:]
        return m.lowrank_linear(m.silu(u) * g, U_dn, V_dn)
    m.packed_gateup_mlp = packed


def _mut_rmsnorm_nosquare(m):
    m.rmsnorm = lambda x, g, eps=m.RMS_EPS: np.asarray(x) / np.sqrt(
        np.abs(np.mean(x, -1, keepdims=True)) + eps) * g


def _mut_layernorm_unbiased(m):
    def ln(x, g, b, eps=m.LN_EPS):
        mu = x.mean(-1, keepdims=True)
        var = x.var(-1, keepdims=True, ddof=1)
        return (x - mu) / np.sqrt(var + eps) * g + b
    m.layernorm = ln


def _mut_lowrank_drops_bias(m):
    m.lowrank_linear = lambda x, U, V, bias=None: (np.asarray(x) @ U) @ V


def _mut_decode_forgets_current(m):
    orig = m.attention

    def attention(q, k, v, causal=False, q_offset=0):
        if q.shape[0] == 1 and k.shape[0] > 1 and not causal:
            return orig(q, k[:-1], v[:-1])
        return orig(q, k, v, causal, q_offset)
    m.attention = attention


def _mut_gelu_tanh(m):
    m.gelu = lambda x: 0.5 * x * (1 + np.tanh(math.sqrt(2 / math.pi) * (x + 0.044715 * x ** 3)))


def _mut_silu_sigmoid_only(m):
    m.silu = lambda x: 1.0 / (1.0 + np.exp(-np.asarray(x, np.float64)))


def _mut_bert_causal(m):
    orig = m.attention
    m.attention = lambda q, k, v, causal=False, q_offset=0: orig(q, k, v, True, q_offset)



def _source_mutant(old, new, name):
    """A mistake planted by editing the oracle's source text: every
    occurrence of ``old`` becomes ``new`` and the edited source is executed
    in the fresh module's namespace."""
    def mutate(m):
        src = open(m.__file__).read()
        assert old in src, f"mutation anchor missing: {old!r}"
        exec(compile(src.replace(old, new), m.__file__, "exec"), m.__dict__)
    mutate.__name__ = name
    return mutate


_mut_second_norm_uses_g1 = _source_mutant(
    'rmsnorm(h_res, w["g2"], eps)', 'rmsnorm(h_res, w["g1"], eps)', "_mut_second_norm_uses_g1")
_mut_bert_drops_b_up = _source_mutant(
    'w["V_up"], w["b_up"]', 'w["V_up"], None', "_mut_bert_drops_b_up")
_mut_rope_on_values = _source_mutant(
    "    k = np.stack([rope(k[:, h], pos) for h in range(H)], axis=1)\n",
    "    k = np.stack([rope(k[:, h], pos) for h in range(H)], axis=1)\n"
    "    v = np.stack([rope(v[:, h], pos) for h in range(H)], axis=1)\n",
    "_mut_rope_on_values")
_mut_heads_interleaved = _source_mutant(
    "return x.reshape(T, H, HD // H)", "return x.reshape(T, HD // H, H).transpose(0, 2, 1)",
    "_mut_heads_interleaved")
_mut_decode_position_shift = _source_mutant(
    "np.full(H, p)", "np.full(H, p + 1)", "_mut_decode_position_shift")
_mut_head_transposed = _source_mutant(
    "y = np.asarray(x, np.float64) @ np.asarray(W, np.float64)",
    "y = np.asarray(x, np.float64) @ np.asarray(W, np.float64).T", "_mut_head_transposed")
_mut_model_skips_final_norm = _source_mutant(
    "return dense_linear(rmsnorm(x, g_final, eps), W_lm)", "return dense_linear(x, W_lm)",
    "_mut_model_skips_final_norm")

MUTANTS = [_mut_rope_sign, _mut_rope_interleaved, _mut_attention_noscale,
           _mut_attention_causal_strict, _mut_swiglu_swapped,
           _mut_rmsnorm_nosquare, _mut_layernorm_unbiased,
           _mut_lowrank_drops_bias, _mut_decode_forgets_current,
           _mut_gelu_tanh, _mut_silu_sigmoid_only, _mut_bert_causal,
           _mut_second_norm_uses_g1, _mut_bert_drops_b_up, _mut_rope_on_values,
           _mut_heads_interleaved, _mut_decode_position_shift, _mut_head_transposed,
           _mut_model_skips_final_norm]


@pytest.mark.parametrize("mutate", MUTANTS, ids=[f.__name__ for f in MUTANTS])
def test_pins_catch_planted_mistakes(mutate):
    m = _fresh_oracle()
    mutate(m)
    caught = []
    for pin in PINS:
        try:
            with np.errstate(all="ignore"):
                pin(m)
        except (AssertionError, ValueError, FloatingPointError):
            caught.append(pin.__name__)
    assert caught, f"no pin catches {mutate.__name__}"


# ------------------------------------------------------ golden values ----

def test_golden_tiny_layer_regression():
    """Stored oracle outputs for the tiny decoder layer (written by
    tests/golden/make_golden.py, which calls only the oracle and the input
    generator) must not drift."""
    from tests.golden.make_golden import tiny_layer_case
    with open(os.path.join(HERE, "golden", "tiny_layer_seed0.json")) as fh:
        gold = json.load(fh)
    got = tiny_layer_case()
    for key, ref in gold["values"].items():
        _close(np.asarray(got[key]), np.asarray(ref), 1e-12)
