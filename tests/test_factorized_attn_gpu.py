"""GPU parity of the factorized prefill attention (the query formed inside the
attention kernel from the rank activation: q = rope(z_q V_q)) against the
CPU oracle, called through the C ABI; and a check that the decoder layer's
prefill takes this path (the query's second-stage projection is never
launched, so dense q is not materialised)."""
import math

import numpy as np
import pytest

from oracle import flashsvd_oracle as oracle
from rank_transformer_b200 import synth
from tests.gpu_util import assert_parity, dev_bf16, host_f64

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module")
def fs():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from rank_transformer_b200 import flashsvd
    flashsvd.init(0, max_tokens=4096, max_rank=4096, max_hidden=4096, max_ffn=11008)
    return flashsvd


def _run(fs, B, S, H, D, r, causal, seed, heads=None, S_max=None):
    S_max = S_max or S + 16
    rng = synth.rng_for(seed)
    zq = synth.normal_bf16(rng, (B * S, r))
    Vq = synth.normal_bf16(rng, (r, H * D), r ** -0.5)
    kc = synth.normal_bf16(rng, (B, S_max, H, D))
    vc = synth.normal_bf16(rng, (B, S_max, H, D))
    cos_t = torch.empty((S_max, D // 2), dtype=torch.float32, device="cuda")
    sin_t = torch.empty_like(cos_t)
    fs.rope_table(cos_t, sin_t, S_max, D, 10000.0)
    out = torch.empty((B, S, H, D), dtype=torch.bfloat16, device="cuda")
    fs.prefill_attn_factorized(dev_bf16(zq), dev_bf16(Vq), cos_t, sin_t, dev_bf16(kc), dev_bf16(vc),
                               out, B, S, H, D, S_max, r, causal, 1.0 / math.sqrt(D))
    torch.cuda.synchronize()
    fs.check_device_status()
    got = host_f64(out)
    Q = oracle.from_bf16(zq) @ oracle.from_bf16(Vq)          # [B*S x H*D]
    K, V = oracle.from_bf16(kc), oracle.from_bf16(vc)
    for b in range(B):
        for h in (heads if heads is not None else range(H)):
            qh = oracle.rope(Q[b * S:(b + 1) * S, h * D:(h + 1) * D], np.arange(S))
            ref = oracle.attention(qh, K[b, :S, h], V[b, :S, h], causal=causal)
            assert_parity(got[b, :, h], ref, f"factorized attn B={B} S={S} D={D} r={r} b={b} h={h}")


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("S,r", [(200, 64), (330, 192), (128, 128)])
def test_factorized_prefill_attention(fs, D, causal, S, r):
    _run(fs, 2, S, 3, D, r, causal, seed=9300 + D + S + r + causal)


def test_factorized_prefill_attention_many_items(fs):
    """More (query tile, batch row, head) items than SMs: every persistent
    CTA forms several query tiles, with the ring shared between the query
    formation and the key/value tiles across items."""
    _run(fs, 3, 330, 64, 64, 320, True, seed=9400, heads=[0, 17, 40, 63])


def test_factorized_prefill_attention_7b(fs):
    """7B shapes: 2048 tokens, 32 heads of 128, rank 1216 (sampled heads)."""
    _run(fs, 1, 2048, 32, 128, 1216, True, seed=9500, heads=[0, 15, 31], S_max=2048)


def test_decoder_prefill_forms_q_in_attention(fs):
    """With the factorized prefill attention selected, the decoder layer's
    prefill launches it, and the second-stage projection (one grouped
    launch) covers only k and v, which the decode path reads from the
    cache: dense q is never written."""
    from tests.test_decode_gpu import _layer_struct
    d, H, D, f, r, S = 512, 4, 128, 1376, 128, 256
    rng = synth.rng_for(9600)
    w = synth.decoder_layer_weights(rng, d, f, r, r, gain_jitter=0.1)
    cos_t = torch.empty((S, D // 2), dtype=torch.float32, device="cuda")
    sin_t = torch.empty_like(cos_t)
    fs.rope_table(cos_t, sin_t, S, D, 10000.0)
    L, dev = _layer_struct(fs, w, d, H, D, f, r, r, cos_t, sin_t, pack=False)
    xs = synth.normal_bf16(rng, (S, d))
    x = dev_bf16(xs)
    kc = torch.zeros((1, S, H, D), dtype=torch.bfloat16, device="cuda")
    vc = torch.zeros_like(kc)
    torch.cuda.synchronize()
    fs.set_prefill_attention(1)
    fs.profile_enable(True)
    try:
        fs.layer_forward(L, x, kc, vc, None, 1, S, S, fs.PREFILL_CAUSAL)
        prof = fs.profile_report(reset=True)
    finally:
        fs.profile_enable(False)
        fs.set_prefill_attention(0)
    assert prof.get("attn_prefill_causal_qf", {}).get("launches") == 1, prof
    assert prof.get("attn_prefill_causal", {}).get("launches", 0) == 0, prof
    # one grouped second-stage launch that projects k and v only (its
    # algorithmic FLOPs are those of two d-wide products, not three)
    g = prof.get("tc_stage2_qkv_grouped", {})
    assert g.get("launches") == 1, prof
    assert abs(g.get("flops", 0.0) / (2.0 * S * (2 * d) * r) - 1.0) < 1e-6, prof
    assert prof.get("tc_stage2_qkv_rope", {}).get("launches", 0) == 0, prof
    y, k, v = oracle.decoder_layer_prefill(oracle.from_bf16(xs), oracle.widen_layer(w), H)
    assert_parity(host_f64(x), y, "layer prefill with in-kernel q")
    assert_parity(host_f64(kc)[0], k, "k cache")
