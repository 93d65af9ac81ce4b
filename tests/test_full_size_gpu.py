"""GPU parity at the workloads' full sizes and at edge values, against the
CPU oracle, called through the C ABI.

* Prefill and decode attention with scores far above the running maximum
  of earlier key tiles or chunks, so that the prefill kernel's output
  rescale in tensor memory and the decode kernels' partial merges across
  very different maxima are taken.
* Prefill linears at 2048 and 8192 rows and the ranks of the mixed-rank
  7B-shaped model (up to r_f = 2368), checked on sampled rows (rows of a
  linear are independent, so the oracle computes only those).
* Causal prefill attention at 2048 tokens (sampled heads), one 7B-shaped
  decoder prefill layer at 512 tokens.
* The whole decoder through the public model driver: prefill, graph-replayed
  decode steps, final norm, output head and greedy pick, with the GPU's own
  tokens fed to the oracle (teacher forcing) and the logits of every step
  compared.
"""
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
    flashsvd.init(0, max_tokens=8192, max_rank=4096, max_hidden=4096, max_ffn=11008)
    return flashsvd


def _sample_rows(M, seed, extra=24):
    rng = np.random.default_rng(seed)
    fixed = [0, 1, 127, 128, 129, M // 2, M - 129, M - 128, M - 2, M - 1]
    rows = set(r for r in fixed if 0 <= r < M)
    rows.update(int(v) for v in rng.integers(0, M, size=extra))
    return np.array(sorted(rows))


# ------------------------------------------------- attention edge values --

@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("big_tile", [1, 2])
def test_prefill_attention_rescale_branch(fs, D, causal, big_tile):
    """Keys of one 128-key tile scaled by 8 (scores there ~8x larger, tens
    of log2 units above the maxima of the tiles before): the kernel must
    rescale its running output when that tile arrives."""
    rng = synth.rng_for(6500 + D + 2 * causal + big_tile)
    B, H, S, S_max = 1, 3, 330, 384
    q = synth.normal_bf16(rng, (B, S, H, D), std=2.0)
    kc = synth.normal_bf16(rng, (B, S_max, H, D))
    vc = synth.normal_bf16(rng, (B, S_max, H, D))
    lo, hi = 128 * big_tile, min(128 * big_tile + 128, S)
    K = oracle.from_bf16(kc)
    K[:, lo:hi] *= 8.0
    kc = synth.f32_to_bf16(K.astype(np.float32))   # exact: a power-of-two scale
    out = torch.empty((B, S, H, D), dtype=torch.bfloat16, device="cuda")
    fs.prefill_attn(dev_bf16(q), dev_bf16(kc), dev_bf16(vc), out, B, S, H, D, S_max, causal,
                    1.0 / math.sqrt(D))
    torch.cuda.synchronize()
    fs.check_device_status()
    Q, K, V = oracle.from_bf16(q), oracle.from_bf16(kc), oracle.from_bf16(vc)
    got = host_f64(out)
    for h in range(H):
        ref = oracle.attention(Q[0, :, h], K[0, :S, h], V[0, :S, h], causal=causal)
        assert_parity(got[0, :, h], ref, f"rescale D={D} causal={causal} tile={big_tile} h={h}")


def test_decode_attention_extreme_chunks(fs):
    """Standalone dense-KV decode attention: one 64-key chunk per row holds
    keys scaled by 8 (a middle chunk in row 0, the first chunk in row 1), so
    the split-sequence partials carry very different maxima when merged."""
    rng = synth.rng_for(6600)
    B, H, D, S_max = 2, 4, 128, 2048
    pos = [1500, 700]
    q = synth.normal_bf16(rng, (B, H, D), std=2.0)
    kn = synth.normal_bf16(rng, (B, H, D))
    vn = synth.normal_bf16(rng, (B, H, D))
    K = oracle.from_bf16(synth.normal_bf16(rng, (B, S_max, H, D)))
    K[0, 640:704] *= 8.0
    K[1, 0:64] *= 8.0
    kc = synth.f32_to_bf16(K.astype(np.float32))
    vc = synth.normal_bf16(rng, (B, S_max, H, D))
    dk, dv = dev_bf16(kc), dev_bf16(vc)
    seq = torch.tensor(pos, dtype=torch.int32, device="cuda")
    out = torch.empty((B, H, D), dtype=torch.bfloat16, device="cuda")
    fs.dense_kv_decode_attn(dev_bf16(q), dev_bf16(kn), dev_bf16(vn), dk, dv, seq, out, B, H, D,
                            S_max, 1.0 / math.sqrt(D))
    torch.cuda.synchronize()
    got = host_f64(out)
    Q, Kn, Vn, V = (oracle.from_bf16(a) for a in (q, kn, vn, vc))
    for b in range(B):
        p = pos[b]
        for h in range(H):
            keys = np.concatenate([K[b, :p, h], Kn[b, h][None]], 0)
            vals = np.concatenate([V[b, :p, h], Vn[b, h][None]], 0)
            ref = oracle.attention(Q[b, h][None], keys, vals)[0]
            assert_parity(got[b, h], ref, f"decode attn extreme b={b} h={h}")


@pytest.mark.parametrize("fused", [True, False])
def test_decode_layer_extreme_history(fs, fused):
    """A decode step of a layer (fused kernel and per-stage kernels) over a
    cache whose keys are scaled by 8 in one chunk per row, so that the
    attention partials merged across CTAs differ by tens of log2 units."""
    from tests.test_decode_gpu import _layer_struct
    d, H, D, f, r = 2048, 16, 128, 1376, 128
    pos = [1500, 700]
    B, S_max = 2, 1536
    rng = synth.rng_for(6700)
    w = synth.decoder_layer_weights(rng, d, f, r, r, gain_jitter=0.1)
    cos_t = torch.empty((S_max, D // 2), dtype=torch.float32, device="cuda")
    sin_t = torch.empty_like(cos_t)
    fs.rope_table(cos_t, sin_t, S_max, D, 10000.0)
    L, dev = _layer_struct(fs, w, d, H, D, f, r, r, cos_t, sin_t)
    K = oracle.from_bf16(synth.normal_bf16(rng, (B, S_max, H, D)))
    K[0, 1024:1088] *= 8.0
    K[1, 0:64] *= 8.0
    kc0 = synth.f32_to_bf16(K.astype(np.float32))
    vc0 = synth.normal_bf16(rng, (B, S_max, H, D))
    xt = synth.normal_bf16(rng, (B, d))
    y, kn, vn = oracle.decoder_layer_decode(oracle.from_bf16(xt), oracle.widen_layer(w), H,
                                            K, oracle.from_bf16(vc0), pos)
    fs.set_decode_path(fused)
    try:
        kc, vc = dev_bf16(kc0), dev_bf16(vc0)
        seq = torch.tensor(pos, dtype=torch.int32, device="cuda")
        x = dev_bf16(xt)
        fs.layer_forward(L, x, kc, vc, seq, B, 1, S_max, fs.DECODE)
        torch.cuda.synchronize()
        fs.check_device_status()
    finally:
        fs.set_decode_path(True)
    assert_parity(host_f64(x), y, f"extreme-history decode fused={fused}")


# ------------------------------------------------------ full-size linears --

@pytest.mark.parametrize("M,d,r,n", [(2048, 4096, 1216, 4096), (8192, 4096, 1664, 4096),
                                     (2048, 11008, 2368, 4096)])
def test_prefill_lowrank_full_size(fs, M, d, r, n):
    rng = synth.rng_for(6800 + M + r)
    x = synth.normal_bf16(rng, (M, d))
    U = synth.normal_bf16(rng, (d, r), d ** -0.5)
    V = synth.normal_bf16(rng, (r, n), r ** -0.5)
    b = synth.normal_bf16(rng, (n,), 0.02)
    y = torch.empty((M, n), dtype=torch.bfloat16, device="cuda")
    fs.lowrank_linear(dev_bf16(x), dev_bf16(U), dev_bf16(V), dev_bf16(b), y, M, d, r, n)
    torch.cuda.synchronize()
    fs.check_device_status()
    rows = _sample_rows(M, M + r)
    ref = oracle.lowrank_linear(oracle.from_bf16(x[rows]), oracle.from_bf16(U),
                                oracle.from_bf16(V), oracle.from_bf16(b))
    assert_parity(host_f64(y)[rows], ref, f"prefill lowrank M={M} r={r}")


@pytest.mark.parametrize("M", [2048, 4])
def test_packed_mlp_rank_2368(fs, M):
    """Packed gate|up MLP at the mixed-rank model's largest rank (r_f =
    r_dn = 2368): prefill (tcgen05) at 2048 rows on sampled rows, decode
    (split-K GEMV) at 4 rows."""
    d, f, r = 4096, 11008, 2368
    rng = synth.rng_for(6900 + M)
    w = synth.decoder_layer_weights(rng, d, f, 64, r)
    x = synth.normal_bf16(rng, (M, d))
    y = torch.empty((M, d), dtype=torch.bfloat16, device="cuda")
    dw = {k: dev_bf16(w[k]) for k in ("U_gu", "V_gu", "U_dn", "V_dn")}
    fs.packed_gateup_mlp(dev_bf16(x), dw["U_gu"], dw["V_gu"], dw["U_dn"], dw["V_dn"], y, M, d, r,
                         f, r)
    torch.cuda.synchronize()
    fs.check_device_status()
    rows = _sample_rows(M, 77) if M > 32 else np.arange(M)
    wf = oracle.widen_layer(w)
    ref = oracle.packed_gateup_mlp(oracle.from_bf16(x[rows]), wf["U_gu"], wf["V_gu"], wf["U_dn"],
                                   wf["V_dn"], r)
    assert_parity(host_f64(y)[rows], ref, f"packed mlp r_f=2368 M={M}")


# ------------------------------------------------- full-size attention ----

def test_prefill_attention_2048_causal(fs):
    rng = synth.rng_for(7100)
    B, H, D, S = 1, 32, 128, 2048
    q = synth.normal_bf16(rng, (B, S, H, D))
    kc = synth.normal_bf16(rng, (B, S, H, D))
    vc = synth.normal_bf16(rng, (B, S, H, D))
    out = torch.empty((B, S, H, D), dtype=torch.bfloat16, device="cuda")
    fs.prefill_attn(dev_bf16(q), dev_bf16(kc), dev_bf16(vc), out, B, S, H, D, S, True,
                    1.0 / math.sqrt(D))
    torch.cuda.synchronize()
    fs.check_device_status()
    got = host_f64(out)
    Q, K, V = oracle.from_bf16(q), oracle.from_bf16(kc), oracle.from_bf16(vc)
    for h in (0, 13, 31):
        ref = oracle.attention(Q[0, :, h], K[0, :, h], V[0, :, h], causal=True)
        assert_parity(got[0, :, h], ref, f"causal attention S=2048 h={h}")


@pytest.mark.parametrize("qf", [0, 1])
def test_decoder_prefill_layer_7b_512(fs, qf):
    """One Llama-2-7B-shaped low-rank decoder layer (ranks 1216 / 1792)
    over a 512-token prompt: output rows and the cache rows it writes, with
    the query projected densely (0) or formed inside the attention kernel
    (1)."""
    from tests.test_decode_gpu import _layer_struct
    d, H, D, f, r, r_f, S = 4096, 32, 128, 11008, 1216, 1792, 512
    rng = synth.rng_for(7200)
    w = synth.decoder_layer_weights(rng, d, f, r, r_f, gain_jitter=0.1)
    cos_t = torch.empty((S, D // 2), dtype=torch.float32, device="cuda")
    sin_t = torch.empty_like(cos_t)
    fs.rope_table(cos_t, sin_t, S, D, 10000.0)
    L, dev = _layer_struct(fs, w, d, H, D, f, r, r_f, cos_t, sin_t, pack=False)
    xs = synth.normal_bf16(rng, (S, d))
    x = dev_bf16(xs)
    kc = torch.zeros((1, S, H, D), dtype=torch.bfloat16, device="cuda")
    vc = torch.zeros_like(kc)
    fs.set_prefill_attention(qf)
    try:
        fs.layer_forward(L, x, kc, vc, None, 1, S, S, fs.PREFILL_CAUSAL)
        torch.cuda.synchronize()
    finally:
        fs.set_prefill_attention(0)
    fs.check_device_status()
    y, k, v = oracle.decoder_layer_prefill(oracle.from_bf16(xs), oracle.widen_layer(w), H)
    assert_parity(host_f64(x), y, f"7B prefill layer S=512 qf={qf}")
    assert_parity(host_f64(kc)[0], k, "7B prefill k cache")
    assert_parity(host_f64(vc)[0], v, "7B prefill v cache")


# ------------------------------------------------------------ whole model --

def test_decoder_model_teacher_forced(fs):
    """Three low-rank decoder layers (hidden 1024, 8 heads of 128, SwiGLU
    2752, retention 0.6: ranks 320 / 448), vocabulary 32000, through the
    public driver: a 256-token prefill then 8 decode steps replayed as one
    CUDA graph per step (embedding, one fused launch of all layers, final
    norm, head, greedy pick).  The oracle runs the same model on the GPU's
    tokens; the logits after the prefill and after every decode step must
    match.  Token agreement with the oracle's own argmax is reported."""
    import dataclasses
    from rank_transformer_b200.model import LLAMA7B, DecoderModel
    cfg = dataclasses.replace(LLAMA7B, layers=3, d=1024, H=8, D=128, f=2752)
    S, steps, B = 256, 8, 1
    r_a, r_f = cfg.ranks(0)
    assert (r_a, r_f) == (320, 448)
    rng = synth.rng_for(7300)
    ws = [synth.decoder_layer_weights(rng, cfg.d, cfg.f, r_a, r_f, gain_jitter=0.1)
          for _ in range(cfg.layers)]
    emb = synth.normal_bf16(rng, (cfg.vocab, cfg.d))
    g_final = synth.normal_bf16(rng, (cfg.d,), std=0.1, mean=1.0)
    W_lm = synth.normal_bf16(rng, (cfg.d, cfg.vocab), cfg.d ** -0.5)
    prompt = synth.tokens(rng, (B, S), cfg.vocab)
    dev_layers = [{k: dev_bf16(v) for k, v in w.items() if isinstance(v, np.ndarray)} for w in ws]
    head = {"emb": dev_bf16(emb), "g_final": dev_bf16(g_final), "W_lm": dev_bf16(W_lm)}
    model = DecoderModel(cfg, B, S + steps, weights=dev_layers, head=head)
    assert model.plan is not None, "every layer should decode through the fused plan"
    stream = torch.cuda.Stream()
    model.capture(stream)
    logits, toks = [], []
    with torch.cuda.stream(stream):
        model.prefill(torch.from_numpy(prompt).cuda(), stream)
        stream.synchronize()
        logits.append(model.logits.double().cpu().numpy()[0])
        toks.append(int(model.tokens.cpu()[0]))
        for _ in range(steps):
            model.decode_step(stream)
            stream.synchronize()
            logits.append(model.logits.double().cpu().numpy()[0])
            toks.append(int(model.tokens.cpu()[0]))
    model.release_graphs()
    fs.check_device_status(stream)

    wf = [oracle.widen_layer(w) for w in ws]
    E, G, W = oracle.from_bf16(emb), oracle.from_bf16(g_final), oracle.from_bf16(W_lm)
    ref0, cache = oracle.decoder_model_prefill(prompt[0], E, wf, G, W, cfg.H)
    assert_parity(logits[0], ref0[S - 1], "logits after prefill")
    k_all = [np.zeros((1, S + steps, cfg.H, cfg.D)) for _ in wf]
    v_all = [np.zeros_like(k) for k in k_all]
    for i, (k, v) in enumerate(cache):
        k_all[i][0, :S], v_all[i][0, :S] = k, v
    agree = int(np.argmax(ref0[S - 1]) == toks[0])
    for t in range(steps):
        x = E[[toks[t]]]
        for i, w in enumerate(wf):
            x, kn, vn = oracle.decoder_layer_decode(x, w, cfg.H, k_all[i], v_all[i], [S + t])
            k_all[i][0, S + t], v_all[i][0, S + t] = kn[0], vn[0]
        ref = oracle.lm_head(x, G, W)[0]
        assert_parity(logits[t + 1], ref, f"logits after decode step {t}")
        agree += int(np.argmax(ref) == toks[t + 1])
    print(f"greedy token agreement with the oracle: {agree}/{steps + 1}")


@pytest.mark.parametrize("B", [1, 2, 4])
def test_decode_layer_rank_2368(fs, B):
    """A retention-0.8 7B-shaped layer (ranks 1664 / 2368: the SwiGLU stage
    input is 2 x 2368 values) decoding at context 1024.  At B = 2 and 4 the
    fused kernel takes it (its wider stage-input buffer); at B = 1 the layer
    runs the per-stage kernels.  Both against the oracle."""
    from tests.test_decode_gpu import _layer_struct
    d, H, D, f, r, r_f, P = 4096, 32, 128, 11008, 1664, 2368, 1024
    S_max = P + 4
    rng = synth.rng_for(9900 + B)
    w = synth.decoder_layer_weights(rng, d, f, r, r_f, gain_jitter=0.1)
    cos_t = torch.empty((S_max, D // 2), dtype=torch.float32, device="cuda")
    sin_t = torch.empty_like(cos_t)
    fs.rope_table(cos_t, sin_t, S_max, D, 10000.0)
    L, dev = _layer_struct(fs, w, d, H, D, f, r, r_f, cos_t, sin_t)
    kc0 = synth.normal_bf16(rng, (B, S_max, H, D))
    vc0 = synth.normal_bf16(rng, (B, S_max, H, D))
    xt = synth.normal_bf16(rng, (B, d))
    kc, vc = dev_bf16(kc0), dev_bf16(vc0)
    seq = torch.full((B,), P, dtype=torch.int32, device="cuda")
    x = dev_bf16(xt)
    torch.cuda.synchronize()
    fs.profile_enable(True)
    try:
        fs.layer_forward(L, x, kc, vc, seq, B, 1, S_max, fs.DECODE)
        prof = fs.profile_report(reset=True)
    finally:
        fs.profile_enable(False)
    fs.check_device_status()
    fused = prof.get("decode_layer_fused", {}).get("launches", 0) == 1
    assert fused == (B > 1), prof
    y, kn, vn = oracle.decoder_layer_decode(oracle.from_bf16(xt), oracle.widen_layer(w), H,
                                            oracle.from_bf16(kc0), oracle.from_bf16(vc0), [P] * B)
    assert_parity(host_f64(x), y, f"rank-2368 decode layer B={B}")
    assert_parity(host_f64(kc)[:, P], kn, f"rank-2368 appended k B={B}")
