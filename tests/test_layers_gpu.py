"""GPU parity of full-sequence attention and of whole layers (decoder
prefill, decode after prefill, encoder) against the CPU oracle."""
import math

import numpy as np
import pytest

from oracle import flashsvd_oracle as oracle
from rank_transformer_b200 import synth
from tests.gpu_util import assert_parity, dev_bf16, host_bits, host_f64

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module")
def fs():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from rank_transformer_b200 import flashsvd
    flashsvd.init(0, max_tokens=4096, max_rank=4096, max_hidden=4096, max_ffn=11008)
    return flashsvd


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("S", [64, 200])
def test_prefill_attention(fs, D, causal, S):
    rng = synth.rng_for(6000 + D + S + causal)
    B, H, S_max = 2, 3, 256
    q = synth.normal_bf16(rng, (B, S, H, D))
    kc = synth.normal_bf16(rng, (B, S_max, H, D))
    vc = synth.normal_bf16(rng, (B, S_max, H, D))
    out = torch.empty((B, S, H, D), dtype=torch.bfloat16, device="cuda")
    fs.prefill_attn(dev_bf16(q), dev_bf16(kc), dev_bf16(vc), out, B, S, H, D, S_max, causal,
                    1.0 / math.sqrt(D))
    torch.cuda.synchronize()
    Q, K, V = oracle.from_bf16(q), oracle.from_bf16(kc), oracle.from_bf16(vc)
    ref = np.zeros((B, S, H, D))
    for b in range(B):
        for h in range(H):
            ref[b, :, h] = oracle.attention(Q[b, :, h], K[b, :S, h], V[b, :S, h], causal=causal)
    assert_parity(host_f64(out), ref, f"prefill attn D={D} causal={causal} S={S}")


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("causal", [True, False])
def test_prefill_attention_many_items(fs, D, causal):
    """More (query tile, batch row, head) items than SMs, so that every
    persistent CTA walks several items (barrier phases carried across
    items); the oracle checks a sample of (batch row, head) pairs, the
    last query tile ragged."""
    rng = synth.rng_for(6100 + D + causal)
    B, H, S, S_max = 3, 64, 330, 384
    q = synth.normal_bf16(rng, (B, S, H, D))
    kc = synth.normal_bf16(rng, (B, S_max, H, D))
    vc = synth.normal_bf16(rng, (B, S_max, H, D))
    out = torch.empty((B, S, H, D), dtype=torch.bfloat16, device="cuda")
    fs.prefill_attn(dev_bf16(q), dev_bf16(kc), dev_bf16(vc), out, B, S, H, D, S_max, causal,
                    1.0 / math.sqrt(D))
    torch.cuda.synchronize()
    got = host_f64(out)
    Q, K, V = oracle.from_bf16(q), oracle.from_bf16(kc), oracle.from_bf16(vc)
    for b, h in [(0, 0), (0, 63), (1, 17), (2, 40), (2, 63), (1, 1)]:
        ref = oracle.attention(Q[b, :, h], K[b, :S, h], V[b, :S, h], causal=causal)
        assert_parity(got[b, :, h], ref, f"prefill attn D={D} causal={causal} b={b} h={h}")


def _decoder_struct(fs, w, d, H, D, f, cos_t, sin_t):
    dev = {k: dev_bf16(v) for k, v in w.items() if isinstance(v, np.ndarray)}
    L = fs.Layer()
    L.kind = fs.DECODER
    L.d, L.H, L.D, L.f = d, H, D, f
    L.norm_eps = 1e-5
    L.norm1_g, L.norm2_g = dev["g1"].data_ptr(), dev["g2"].data_ptr()
    for name in ("q", "k", "v", "o"):
        F = getattr(L, name)
        F.U, F.V, F.bias, F.r = dev["U_" + name].data_ptr(), dev["V_" + name].data_ptr(), None, \
            w["U_" + name].shape[1]
    L.U_gu, L.V_gu, L.r_f = dev["U_gu"].data_ptr(), dev["V_gu"].data_ptr(), w["U_gu"].shape[1] // 2
    L.down.U, L.down.V, L.down.bias, L.down.r = dev["U_dn"].data_ptr(), dev["V_dn"].data_ptr(), None, \
        w["U_dn"].shape[1]
    L.rope_cos, L.rope_sin = cos_t.data_ptr(), sin_t.data_ptr()
    return L, dev


def _rope(fs, S_max, D):
    c = torch.empty((S_max, D // 2), dtype=torch.float32, device="cuda")
    s = torch.empty_like(c)
    fs.rope_table(c, s, S_max, D, 10000.0)
    return c, s


@pytest.mark.parametrize("B", [1, 2])
def test_decoder_layer_prefill_then_decode(fs, B):
    """Tiny decoder layer: prefill of 128 tokens (cache rows 0..127), then
    16 decode steps on the cache the prefill wrote.  Prefill output and cache
    rows are compared with the oracle's prefill; each decode step with the
    oracle's decode over the GPU cache; and decoding token t after a prefill
    of t tokens must match prefill row t of the longer sequence."""
    d, H, D, f, r, S, steps = 256, 4, 64, 688, 64, 128, 16
    S_max = S + steps
    rng = synth.rng_for(0)
    w = synth.decoder_layer_weights(rng, d, f, r, r, gain_jitter=0.1)
    cos_t, sin_t = _rope(fs, S_max, D)
    L, dev = _decoder_struct(fs, w, d, H, D, f, cos_t, sin_t)
    wf = oracle.widen_layer(w)
    xs = synth.normal_bf16(rng, (B, S + steps, d))

    kc = torch.zeros((B, S_max, H, D), dtype=torch.bfloat16, device="cuda")
    vc = torch.zeros_like(kc)
    x = dev_bf16(xs[:, :S].reshape(B * S, d))
    fs.layer_forward(L, x, kc, vc, None, B, S, S_max, fs.PREFILL_CAUSAL)
    torch.cuda.synchronize()
    for b in range(B):
        y, k, v = oracle.decoder_layer_prefill(oracle.from_bf16(xs[b, :S]), wf, H)
        assert_parity(host_f64(x).reshape(B, S, d)[b], y, f"prefill y b={b}")
        assert_parity(host_f64(kc)[b, :S], k, f"prefill k cache b={b}")
        assert_parity(host_f64(vc)[b, :S], v, f"prefill v cache b={b}")

    seq = torch.full((B,), S, dtype=torch.int32, device="cuda")
    for t in range(steps):
        hk, hv = host_f64(kc), host_f64(vc)
        xt = dev_bf16(xs[:, S + t])
        fs.layer_forward(L, xt, kc, vc, seq, B, 1, S_max, fs.DECODE)
        fs.advance_seqlens(seq, B)
        torch.cuda.synchronize()
        y, kn, vn = oracle.decoder_layer_decode(oracle.from_bf16(xs[:, S + t]), wf, H, hk, hv,
                                                [S + t] * B)
        assert_parity(host_f64(xt), y, f"decode after prefill step {t}")

    # decode of token S after prefill of S tokens == prefill of S+1 tokens, row S
    x_long = dev_bf16(xs[:, :S + 1].reshape(B * (S + 1), d))
    kc2 = torch.zeros_like(kc)
    vc2 = torch.zeros_like(vc)
    fs.layer_forward(L, x_long, kc2, vc2, None, B, S + 1, S_max, fs.PREFILL_CAUSAL)
    kc3 = torch.zeros_like(kc)
    vc3 = torch.zeros_like(vc)
    x_pre = dev_bf16(xs[:, :S].reshape(B * S, d))
    fs.layer_forward(L, x_pre, kc3, vc3, None, B, S, S_max, fs.PREFILL_CAUSAL)
    seq = torch.full((B,), S, dtype=torch.int32, device="cuda")
    x_dec = dev_bf16(xs[:, S])
    fs.layer_forward(L, x_dec, kc3, vc3, seq, B, 1, S_max, fs.DECODE)
    torch.cuda.synchronize()
    long_rows = host_f64(x_long).reshape(B, S + 1, d)[:, S]
    assert_parity(host_f64(x_dec), long_rows, "decode(t) vs prefill row t")


def _encoder_struct(fs, w, d, H, f):
    dev = {k: dev_bf16(v) for k, v in w.items() if isinstance(v, np.ndarray)}
    L = fs.Layer()
    L.kind = fs.ENCODER
    L.d, L.H, L.D, L.f = d, H, d // H, f
    L.norm_eps = 1e-12
    L.norm1_g, L.norm1_b = dev["ln1_g"].data_ptr(), dev["ln1_b"].data_ptr()
    L.norm2_g, L.norm2_b = dev["ln2_g"].data_ptr(), dev["ln2_b"].data_ptr()
    for n, field in (("q", "q"), ("k", "k"), ("v", "v"), ("o", "o"), ("up", "up"), ("dn", "down")):
        F = getattr(L, field)
        F.U, F.V, F.bias, F.r = dev["U_" + n].data_ptr(), dev["V_" + n].data_ptr(), \
            dev["b_" + n].data_ptr(), w["U_" + n].shape[1]
    return L, dev


@pytest.mark.parametrize("B,S", [(2, 128), (1, 200)])
def test_encoder_layer(fs, B, S):
    d, H, f, r = 768, 12, 3072, 192
    rng = synth.rng_for(7000 + S)
    w = synth.bert_layer_weights(rng, d, f, r, bias_std=0.02, gain_jitter=0.1)
    L, dev = _encoder_struct(fs, w, d, H, f)
    x_bits = synth.normal_bf16(rng, (B, S, d))
    x = dev_bf16(x_bits.reshape(B * S, d))
    kb = torch.empty((B, S, H, d // H), dtype=torch.bfloat16, device="cuda")
    vb = torch.empty_like(kb)
    fs.layer_forward(L, x, kb, vb, None, B, S, S, fs.ENCODER_BIDIR)
    torch.cuda.synchronize()
    wf = oracle.widen_layer(w)
    got = host_f64(x).reshape(B, S, d)
    for b in range(B):
        ref = oracle.bert_layer(oracle.from_bf16(x_bits[b]), wf, H)
        assert_parity(got[b], ref, f"encoder layer b={b}")
