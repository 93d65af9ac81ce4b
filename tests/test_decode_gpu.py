"""GPU parity of the decode path (M <= 32) against the CPU oracle, called
through the C ABI."""
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


def _rand_factors(rng, d, r, n):
    return (synth.normal_bf16(rng, (d, r), d ** -0.5),
            synth.normal_bf16(rng, (r, n), r ** -0.5))


LINEAR_CASES = [
    (1, 256, 64, 688), (1, 688, 64, 256), (2, 256, 64, 256), (7, 256, 64, 688),
    (8, 4096, 512, 4096), (32, 4096, 1024, 4096), (1, 4096, 2048, 4096),
    (31, 4096, 1216, 4096), (3, 11008, 1792, 4096), (1, 4096, 1792, 11008),
]


@pytest.mark.parametrize("M,d,r,n", LINEAR_CASES)
def test_lowrank_linear_decode(fs, M, d, r, n):
    rng = synth.rng_for(1000 + M + d + r + n)
    U, V = _rand_factors(rng, d, r, n)
    x = synth.normal_bf16(rng, (M, d))
    bias = synth.normal_bf16(rng, (n,), 0.02) if (M % 2) else None
    y = torch.empty((M, n), dtype=torch.bfloat16, device="cuda")
    b_dev = dev_bf16(bias) if bias is not None else None
    fs.lowrank_linear(dev_bf16(x), dev_bf16(U), dev_bf16(V), b_dev, y, M, d, r, n)
    torch.cuda.synchronize()
    ref = oracle.lowrank_linear(oracle.from_bf16(x), oracle.from_bf16(U), oracle.from_bf16(V),
                                None if bias is None else oracle.from_bf16(bias))
    assert_parity(host_f64(y), ref, f"lowrank M={M} d={d} r={r} n={n}")


def test_lowrank_linear_svd_factors(fs):
    # Factors from the truncated SVD of W = P diag(i^-0.5) Q^T (square 4096).
    rng = synth.rng_for(7)
    U, V, _ = synth.svd_factors(rng, 4096, 4096, 512, full_rank=512)
    for M in (1, 8, 32):
        x = synth.normal_bf16(rng, (M, 4096))
        y = torch.empty((M, 4096), dtype=torch.bfloat16, device="cuda")
        fs.lowrank_linear(dev_bf16(x), dev_bf16(U), dev_bf16(V), None, y, M, 4096, 512, 4096)
        torch.cuda.synchronize()
        ref = oracle.lowrank_linear(oracle.from_bf16(x), oracle.from_bf16(U), oracle.from_bf16(V))
        assert_parity(host_f64(y), ref, f"svd M={M}")


@pytest.mark.parametrize("M,d,r_f,f,r_dn", [(1, 256, 64, 688, 64), (5, 256, 64, 688, 64),
                                           (20, 256, 64, 688, 64),
                                           (1, 4096, 1792, 11008, 1792),
                                           (8, 4096, 512, 11008, 1024)])
def test_packed_mlp_decode(fs, M, d, r_f, f, r_dn):
    rng = synth.rng_for(2000 + M + r_f)
    U_gu = synth.normal_bf16(rng, (d, 2 * r_f), d ** -0.5)
    V_gu = synth.normal_bf16(rng, (2 * r_f, f), r_f ** -0.5)
    U_dn, V_dn = _rand_factors(rng, f, r_dn, d)
    x = synth.normal_bf16(rng, (M, d))
    h = torch.empty((M, f), dtype=torch.bfloat16, device="cuda")
    y = torch.empty((M, d), dtype=torch.bfloat16, device="cuda")
    xs, ugs, vgs = dev_bf16(x), dev_bf16(U_gu), dev_bf16(V_gu)
    fs.gateup_swiglu(xs, ugs, vgs, h, M, d, r_f, f)
    fs.packed_gateup_mlp(xs, ugs, vgs, dev_bf16(U_dn), dev_bf16(V_dn), y, M, d, r_f, f, r_dn)
    torch.cuda.synchronize()
    X = oracle.from_bf16(x)
    w = [oracle.from_bf16(a) for a in (U_gu, V_gu, U_dn, V_dn)]
    assert_parity(host_f64(h), oracle.gateup_swiglu(X, w[0], w[1], r_f), "gate|up h")
    assert_parity(host_f64(y), oracle.packed_gateup_mlp(X, *w, r_f), "packed mlp y")


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("append", [False, True])
def test_dense_kv_decode_attention(fs, D, append):
    rng = synth.rng_for(3000 + D + append)
    B, H, S_max = 3, 4, 300
    seqlens = np.array([0, 131, 299], dtype=np.int32)
    kc = synth.normal_bf16(rng, (B, S_max, H, D))
    vc = synth.normal_bf16(rng, (B, S_max, H, D))
    q = synth.normal_bf16(rng, (B, H, D))
    kn = synth.normal_bf16(rng, (B, H, D))
    vn = synth.normal_bf16(rng, (B, H, D))
    kcd, vcd = dev_bf16(kc), dev_bf16(vc)
    out = torch.empty((B, H, D), dtype=torch.bfloat16, device="cuda")
    sl = torch.from_numpy(seqlens).cuda()
    scale = 1.0 / math.sqrt(D)
    fs.dense_kv_decode_attn(dev_bf16(q), dev_bf16(kn) if append else None,
                            dev_bf16(vn) if append else None, kcd, vcd, sl, out, B, H, D,
                            S_max, scale)
    torch.cuda.synchronize()
    K, Vv = oracle.from_bf16(kc), oracle.from_bf16(vc)
    if append:
        for b in range(B):
            K[b, seqlens[b]] = oracle.from_bf16(kn[b])
            Vv[b, seqlens[b]] = oracle.from_bf16(vn[b])
        # the cache row at the current position now holds the new entries
        assert np.array_equal(host_bits(kcd)[np.arange(B), seqlens], kn)
        assert np.array_equal(host_bits(vcd)[np.arange(B), seqlens], vn)
    Q = oracle.from_bf16(q)
    ref = np.zeros((B, H, D))
    for b in range(B):
        L = seqlens[b] + 1
        for h in range(H):
            ref[b, h] = oracle.attention(Q[b, h][None], K[b, :L, h], Vv[b, :L, h])[0]
    assert_parity(host_f64(out), ref, f"decode attn D={D} append={append}")


@pytest.mark.parametrize("d", [768, 2056, 4096, 4104, 8192])
@pytest.mark.parametrize("M", [1, 3, 2048])
def test_norm_widths(fs, d, M):
    """RMSNorm and LayerNorm across the three launch shapes: one warp per
    row (d <= 2048), one 128-thread CTA per row (d <= 4096) and one
    256-thread CTA per row (up to 8192), with ragged vector counts."""
    if M == 2048 and d not in (4096, 8192):
        pytest.skip("many rows checked at the 7B width and the maximum")
    rng = synth.rng_for(4100 + d + M)
    x = synth.normal_bf16(rng, (M, d))
    g = synth.normal_bf16(rng, (d,), 0.1, 1.0)
    b = synth.normal_bf16(rng, (d,), 0.1)
    y = torch.empty((M, d), dtype=torch.bfloat16, device="cuda")
    X, G, Bb = oracle.from_bf16(x), oracle.from_bf16(g), oracle.from_bf16(b)
    fs.rmsnorm(dev_bf16(x), dev_bf16(g), y, M, d, 1e-5)
    torch.cuda.synchronize()
    assert_parity(host_f64(y), oracle.rmsnorm(X, G, 1e-5), f"rmsnorm d={d} M={M}")
    fs.layernorm(dev_bf16(x), dev_bf16(g), dev_bf16(b), y, M, d, 1e-12)
    torch.cuda.synchronize()
    assert_parity(host_f64(y), oracle.layernorm(X, G, Bb, 1e-12), f"layernorm d={d} M={M}")


def test_glue_kernels(fs):
    rng = synth.rng_for(4000)
    M, d = 5, 768
    x = synth.normal_bf16(rng, (M, d))
    g = synth.normal_bf16(rng, (d,), 0.1, 1.0)
    b = synth.normal_bf16(rng, (d,), 0.1)
    y = torch.empty((M, d), dtype=torch.bfloat16, device="cuda")
    fs.rmsnorm(dev_bf16(x), dev_bf16(g), y, M, d, 1e-5)
    torch.cuda.synchronize()
    assert_parity(host_f64(y), oracle.rmsnorm(oracle.from_bf16(x), oracle.from_bf16(g), 1e-5), "rmsnorm")
    fs.layernorm(dev_bf16(x), dev_bf16(g), dev_bf16(b), y, M, d, 1e-12)
    torch.cuda.synchronize()
    assert_parity(host_f64(y), oracle.layernorm(oracle.from_bf16(x), oracle.from_bf16(g),
                                                oracle.from_bf16(b), 1e-12), "layernorm")
    # rotary table
    S_max, D = 4096, 128
    c = torch.empty((S_max, D // 2), dtype=torch.float32, device="cuda")
    s = torch.empty_like(c)
    fs.rope_table(c, s, S_max, D, 10000.0)
    torch.cuda.synchronize()
    ang = np.arange(S_max)[:, None] * (10000.0 ** (-2.0 * np.arange(D // 2) / D))[None, :]
    assert np.max(np.abs(c.cpu().numpy() - np.cos(ang))) < 1e-6
    assert np.max(np.abs(s.cpu().numpy() - np.sin(ang))) < 1e-6
    # embedding gather, greedy pick, advance
    vocab = 1000
    emb = synth.normal_bf16(rng, (vocab, d))
    toks = np.array([3, 999, 0, 512], dtype=np.int32)
    xe = torch.empty((4, d), dtype=torch.bfloat16, device="cuda")
    fs.embed(torch.from_numpy(toks).cuda(), dev_bf16(emb), xe, 4, d, vocab)
    logits = rng.standard_normal((3, vocab)).astype(np.float32)
    logits[1, 10] = logits[1, 700] = 50.0  # tie -> lowest index
    nxt = torch.empty(3, dtype=torch.int32, device="cuda")
    fs.greedy(torch.from_numpy(logits).cuda(), nxt, 3, vocab)
    sl = torch.tensor([5, 7], dtype=torch.int32, device="cuda")
    fs.advance_seqlens(sl, 2)
    torch.cuda.synchronize()
    assert np.array_equal(host_bits(xe), emb[toks])
    assert list(nxt.cpu().numpy()) == list(oracle.greedy(logits))
    assert list(sl.cpu().numpy()) == [6, 8]


@pytest.mark.parametrize("vocab", [32000, 32003, 70001])
def test_greedy_large_vocab(fs, vocab):
    """Greedy pick over vocabularies that give every thread many entries:
    the maximum in the last entry, a tie between entries far apart (lowest
    index wins), a row of equal values, the maximum in the first entry, and
    a plain random row; against the oracle's argmax."""
    rng = synth.rng_for(4100 + vocab)
    logits = rng.standard_normal((5, vocab)).astype(np.float32)
    logits[0, vocab - 1] = 40.0
    logits[1, 7] = logits[1, vocab // 2 + 3] = logits[1, vocab - 2] = 40.0
    logits[2, :] = 1.5
    logits[3, 0] = 40.0
    nxt = torch.empty(5, dtype=torch.int32, device="cuda")
    fs.greedy(torch.from_numpy(logits).cuda(), nxt, 5, vocab)
    torch.cuda.synchronize()
    got = list(nxt.cpu().numpy())
    assert got == list(oracle.greedy(logits))
    assert got[:4] == [vocab - 1, 7, 0, 0]


def _layer_struct(fs, w, d, H, D, f, r, r_f, cos_t, sin_t, pack=True):
    """Layer descriptor over device copies of w; with pack, also the decode
    pack that the fused decode kernel streams (kept alive in dev)."""
    dev = {k: dev_bf16(v) for k, v in w.items() if isinstance(v, np.ndarray)}
    L = fs.Layer()
    L.kind = fs.DECODER
    L.d, L.H, L.D, L.f = d, H, D, f
    L.norm_eps = 1e-5
    L.norm1_g, L.norm2_g = dev["g1"].data_ptr(), dev["g2"].data_ptr()
    for name in ("q", "k", "v", "o"):
        F = getattr(L, name)
        F.U, F.V, F.bias, F.r = dev["U_" + name].data_ptr(), dev["V_" + name].data_ptr(), None, r
    L.U_gu, L.V_gu, L.r_f = dev["U_gu"].data_ptr(), dev["V_gu"].data_ptr(), r_f
    L.down.U, L.down.V, L.down.bias, L.down.r = dev["U_dn"].data_ptr(), dev["V_dn"].data_ptr(), None, r_f
    L.rope_cos, L.rope_sin = cos_t.data_ptr(), sin_t.data_ptr()
    if pack:
        dev["pack"] = torch.empty(fs.decode_pack_bytes(L), dtype=torch.uint8, device="cuda")
        fs.decode_pack(L, dev["pack"])
    return L, dev


def _expected_pack(w, d, H, D, f, r, r_f):
    """The decode pack written out from its definition in the header: per
    stage, per column tile, per 256-row chunk (kn rows), 16 regions of 4
    columns (region w: box w // 8, columns 4 (w % 8) .. + 3 of the box), each
    kn / 2 pieces of rows (2p, 2p + 1) x those 4 columns, row-major; zero
    beyond a factor's width."""
    def tiles(mats, K, cols_of_tile, ntiles, rows_of_box=None):
        out = []
        for M, T in zip(mats, ntiles):
            for t in range(T):
                for k0 in range(0, K, 256):
                    kn = min(256, K - k0)
                    boxes = []
                    for b in range(2):
                        c0 = cols_of_tile(t, b)
                        rs = rows_of_box(b) if rows_of_box else 0
                        blk = np.zeros((kn, 32), dtype=np.uint16)
                        src = M[rs + k0: rs + k0 + kn, c0: c0 + 32]
                        blk[:, :src.shape[1]] = src
                        boxes.append(blk)
                    for wr in range(16):
                        cols = boxes[wr // 8][:, 4 * (wr % 8): 4 * (wr % 8) + 4]  # [kn x 4]
                        out.append(cols.reshape(kn // 2, 2, 4).ravel())
        return out
    plain = lambda t, b: 64 * t + 32 * b
    def rope(t, b):
        tph = D // 64
        hh, j = divmod(t, tph)
        return hh * D + 32 * j + b * (D // 2)
    parts = []
    parts += tiles([w["U_q"], w["U_k"], w["U_v"]], d, plain, [-(-r // 64)] * 3)
    parts += tiles([w["V_q"], w["V_k"], w["V_v"]], r, rope, [d // 64] * 3)
    parts += tiles([w["U_o"]], d, plain, [-(-r // 64)])
    parts += tiles([w["V_o"]], r, plain, [d // 64])
    parts += tiles([w["U_gu"]], d, plain, [-(-2 * r_f // 64)])
    parts += tiles([w["V_gu"]], r_f, lambda t, b: 32 * t, [-(-f // 32)], lambda b: b * r_f)
    parts += tiles([w["U_dn"]], f, plain, [-(-r_f // 64)])
    parts += tiles([w["V_dn"]], r_f, plain, [d // 64])
    return np.concatenate(parts)


@pytest.mark.parametrize("shape", [(256, 4, 64, 688, 64, 64), (512, 4, 128, 1000, 200, 136)])
def test_decode_pack_layout(fs, shape):
    """The pack is a pure re-tiling: bit-exact against the layout written out
    on the host (ragged row chunks, partial column tiles, the RoPE and SwiGLU
    column maps)."""
    d, H, D, f, r, r_f = shape
    rng = synth.rng_for(3)
    w = synth.decoder_layer_weights(rng, d, f, r, r_f, gain_jitter=0.1)
    cos_t = torch.zeros((8, D // 2), dtype=torch.float32, device="cuda")
    L, dev = _layer_struct(fs, w, d, H, D, f, r, r_f, cos_t, cos_t)
    torch.cuda.synchronize()
    got = dev["pack"].cpu().numpy().view(np.uint16)
    exp = _expected_pack(w, d, H, D, f, r, r_f)
    # the factor blocks come first; the kernel's schedule records follow them
    assert got.size >= exp.size
    assert np.array_equal(got[:exp.size], exp)


@pytest.mark.parametrize("fused", [True, False])
@pytest.mark.parametrize("B", [1, 3])
def test_decoder_layer_decode_steps(fs, B, fused):
    """Tiny decoder layer (hidden 256, 4 heads of 64, SwiGLU 688, rank 64):
    16 decode steps after a 128-token history; each step is compared with
    the oracle's decode of the same layer over the GPU's cache contents
    (teacher forcing)."""
    d, H, D, f, r, steps, P = 256, 4, 64, 688, 64, 16, 128
    S_max = P + steps
    rng = synth.rng_for(0)
    w = synth.decoder_layer_weights(rng, d, f, r, r, gain_jitter=0.1)
    cos_t = torch.empty((S_max, D // 2), dtype=torch.float32, device="cuda")
    sin_t = torch.empty_like(cos_t)
    fs.rope_table(cos_t, sin_t, S_max, D, 10000.0)
    L, dev = _layer_struct(fs, w, d, H, D, f, r, r, cos_t, sin_t)
    kc = dev_bf16(synth.normal_bf16(rng, (B, S_max, H, D)))
    vc = dev_bf16(synth.normal_bf16(rng, (B, S_max, H, D)))
    seq = torch.full((B,), P, dtype=torch.int32, device="cuda")
    wf = oracle.widen_layer(w)
    fs.set_decode_path(fused)
    for t in range(steps):
        xt = synth.normal_bf16(rng, (B, d))
        hist_k, hist_v = host_f64(kc), host_f64(vc)
        x = dev_bf16(xt)
        fs.layer_forward(L, x, kc, vc, seq, B, 1, S_max, fs.DECODE)
        fs.advance_seqlens(seq, B)
        torch.cuda.synchronize()
        y, kn, vn = oracle.decoder_layer_decode(oracle.from_bf16(xt), wf, H, hist_k, hist_v,
                                                [P + t] * B)
        assert_parity(host_f64(x), y, f"layer decode step {t}")
        assert_parity(host_f64(kc)[:, P + t], kn, f"appended k step {t}")
        assert_parity(host_f64(vc)[:, P + t], vn, f"appended v step {t}")
    assert list(seq.cpu().numpy()) == [P + steps] * B
    fs.set_decode_path(True)


@pytest.mark.parametrize("B", [1, 4, 8])
def test_decoder_layer_decode_7b_shape(fs, B):
    """One Llama-2-7B-shaped low-rank layer (hidden 4096, 32 heads of 128,
    SwiGLU 11008, ranks 1216 / 1792) decoding at context 2048 on a random
    dense cache, fused and per-stage paths, against the oracle."""
    d, H, D, f, r, r_f, P = 4096, 32, 128, 11008, 1216, 1792, 2048
    S_max = P + 4
    rng = synth.rng_for(11)
    w = synth.decoder_layer_weights(rng, d, f, r, r_f, gain_jitter=0.1)
    cos_t = torch.empty((S_max, D // 2), dtype=torch.float32, device="cuda")
    sin_t = torch.empty_like(cos_t)
    fs.rope_table(cos_t, sin_t, S_max, D, 10000.0)
    L, dev = _layer_struct(fs, w, d, H, D, f, r, r_f, cos_t, sin_t)
    kc0 = synth.normal_bf16(rng, (B, S_max, H, D))
    vc0 = synth.normal_bf16(rng, (B, S_max, H, D))
    xt = synth.normal_bf16(rng, (B, d))
    wf = oracle.widen_layer(w)
    y, kn, vn = oracle.decoder_layer_decode(oracle.from_bf16(xt), wf, H, oracle.from_bf16(kc0),
                                            oracle.from_bf16(vc0), [P] * B)
    for fused in (True, False):
        fs.set_decode_path(fused)
        kc, vc = dev_bf16(kc0), dev_bf16(vc0)
        seq = torch.full((B,), P, dtype=torch.int32, device="cuda")
        x = dev_bf16(xt)
        fs.layer_forward(L, x, kc, vc, seq, B, 1, S_max, fs.DECODE)
        torch.cuda.synchronize()
        fs.check_device_status()
        assert_parity(host_f64(x), y, f"7B decode layer fused={fused}")
        assert_parity(host_f64(kc)[:, P], kn, f"7B appended k fused={fused}")
        assert_parity(host_f64(vc)[:, P], vn, f"7B appended v fused={fused}")
    fs.set_decode_path(True)


RAGGED_CASES = [
    # (d, H, D, f, r, positions of the batch rows)
    (256, 4, 64, 688, 64, [3999]),                 # few heads, long context
    (256, 4, 64, 688, 64, [0, 3999, 76]),          # an empty history among long rows
    (256, 4, 64, 688, 64, [7999, 0, 5, 0]),        # short rows beside a long one
    (2048, 32, 64, 1376, 128, [2999, 0, 0, 0]),    # 32 heads, three one-key rows
    (2048, 16, 128, 1376, 128, [16383]),           # the longest context, 16384 keys
]


@pytest.mark.parametrize("fused", [True, False])
@pytest.mark.parametrize("case", RAGGED_CASES, ids=lambda c: f"H{c[1]}D{c[2]}pos{'-'.join(map(str, c[5]))}")
def test_decoder_layer_decode_ragged_lengths(fs, case, fused):
    """One decode step of a layer whose batch rows sit at very different
    positions (long contexts, an empty history, few heads), fused and
    per-stage paths, against the oracle: the layer output and the k, v rows
    appended at each row's position."""
    d, H, D, f, r, pos = case
    B, S_max = len(pos), max(pos) + 1
    rng = synth.rng_for(12 + B * 131 + S_max)
    w = synth.decoder_layer_weights(rng, d, f, r, r, gain_jitter=0.1)
    cos_t = torch.empty((S_max, D // 2), dtype=torch.float32, device="cuda")
    sin_t = torch.empty_like(cos_t)
    fs.rope_table(cos_t, sin_t, S_max, D, 10000.0)
    L, dev = _layer_struct(fs, w, d, H, D, f, r, r, cos_t, sin_t)
    kc0 = synth.normal_bf16(rng, (B, S_max, H, D))
    vc0 = synth.normal_bf16(rng, (B, S_max, H, D))
    xt = synth.normal_bf16(rng, (B, d))
    y, kn, vn = oracle.decoder_layer_decode(oracle.from_bf16(xt), oracle.widen_layer(w), H,
                                            oracle.from_bf16(kc0), oracle.from_bf16(vc0), pos)
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
    assert_parity(host_f64(x), y, f"ragged decode fused={fused}")
    for b in range(B):
        assert_parity(host_f64(kc[b, pos[b]]), kn[b], f"appended k row {b} fused={fused}")
        assert_parity(host_f64(vc[b, pos[b]]), vn[b], f"appended v row {b} fused={fused}")


def test_decode_graph_replay_bitwise(fs):
    d, H, D, f, r, P, B = 256, 4, 64, 688, 64, 100, 2
    S_max = P + 8
    rng = synth.rng_for(5)
    w = synth.decoder_layer_weights(rng, d, f, r, r, gain_jitter=0.1)
    cos_t = torch.empty((S_max, D // 2), dtype=torch.float32, device="cuda")
    sin_t = torch.empty_like(cos_t)
    fs.rope_table(cos_t, sin_t, S_max, D, 10000.0)
    L, dev = _layer_struct(fs, w, d, H, D, f, r, r, cos_t, sin_t)
    kc0 = synth.normal_bf16(rng, (B, S_max, H, D))
    vc0 = synth.normal_bf16(rng, (B, S_max, H, D))
    xs = [synth.normal_bf16(rng, (B, d)) for _ in range(6)]

    def run(use_graph):
        kc, vc = dev_bf16(kc0), dev_bf16(vc0)
        seq = torch.full((B,), P, dtype=torch.int32, device="cuda")
        x = torch.empty((B, d), dtype=torch.bfloat16, device="cuda")
        stream = torch.cuda.Stream()
        outs = []
        with torch.cuda.stream(stream):
            g = fs.decode_graph_capture(L, x, kc, vc, seq, B, S_max, stream) if use_graph else None
            for xt in xs:
                x.copy_(dev_bf16(xt))
                if use_graph:
                    g.replay(stream)
                else:
                    fs.layer_forward(L, x, kc, vc, seq, B, 1, S_max, fs.DECODE, stream)
                fs.advance_seqlens(seq, B, stream)
                outs.append(x.clone())
        stream.synchronize()
        if g is not None:
            assert g.kernels >= 1
            g.destroy()
        return [host_bits(o) for o in outs], host_bits(kc)

    eager, kc_e = run(False)
    graph, kc_g = run(True)
    eager2, _ = run(False)
    for a, b, c in zip(eager, graph, eager2):
        assert np.array_equal(a, b)
        assert np.array_equal(a, c)
    assert np.array_equal(kc_e, kc_g)


def _torch_layer(fs, d, H, D, f, r, r_f, cos_t, sin_t, gen):
    """Random bf16 layer on the device (no oracle involved) with its pack."""
    def mat(rows, cols):
        return (torch.randn(rows, cols, device="cuda", generator=gen) * rows ** -0.5).to(torch.bfloat16)
    w = {}
    for n in ("q", "k", "v", "o"):
        w["U_" + n], w["V_" + n] = mat(d, r), mat(r, d)
    w["U_gu"], w["V_gu"] = mat(d, 2 * r_f), mat(2 * r_f, f)
    w["U_dn"], w["V_dn"] = mat(f, r_f), mat(r_f, d)
    w["g1"] = (1 + 0.1 * torch.randn(d, device="cuda", generator=gen)).to(torch.bfloat16)
    w["g2"] = (1 + 0.1 * torch.randn(d, device="cuda", generator=gen)).to(torch.bfloat16)
    L = fs.Layer()
    L.kind = fs.DECODER
    L.d, L.H, L.D, L.f = d, H, D, f
    L.norm_eps = 1e-5
    L.norm1_g, L.norm2_g = w["g1"].data_ptr(), w["g2"].data_ptr()
    for n in ("q", "k", "v", "o"):
        F = getattr(L, n)
        F.U, F.V, F.bias, F.r = w["U_" + n].data_ptr(), w["V_" + n].data_ptr(), None, r
    L.U_gu, L.V_gu, L.r_f = w["U_gu"].data_ptr(), w["V_gu"].data_ptr(), r_f
    L.down.U, L.down.V, L.down.bias, L.down.r = w["U_dn"].data_ptr(), w["V_dn"].data_ptr(), None, r_f
    L.rope_cos, L.rope_sin = cos_t.data_ptr(), sin_t.data_ptr()
    w["pack"] = torch.empty(fs.decode_pack_bytes(L), dtype=torch.uint8, device="cuda")
    fs.decode_pack(L, w["pack"])
    return L, w


@pytest.mark.parametrize("shape", ["tiny-mixed-ranks", "7b-2-layers"])
@pytest.mark.parametrize("B", [1, 4])
def test_decode_plan_matches_layer_calls(fs, shape, B):
    """A decode plan (all layers in one launch) gives bit-identical x and
    caches to one fused DECODE layer_forward call per layer: each layer's
    input is summed from the previous layer's partials in the same order
    the per-layer final pass uses."""
    if shape == "tiny-mixed-ranks":
        d, H, D, f, P = 256, 4, 64, 688, 100
        ranks = [(64, 64), (128, 96), (64, 128)]
    else:
        d, H, D, f, P = 4096, 32, 128, 11008, 2048
        ranks = [(1216, 1792), (832, 1216)]
    S_max = P + 4
    gen = torch.Generator(device="cuda")
    gen.manual_seed(7)
    cos_t = torch.empty((S_max, D // 2), dtype=torch.float32, device="cuda")
    sin_t = torch.empty_like(cos_t)
    fs.rope_table(cos_t, sin_t, S_max, D, 10000.0)
    layers = [_torch_layer(fs, d, H, D, f, r, rf, cos_t, sin_t, gen) for r, rf in ranks]
    kc0 = [torch.randn(B, S_max, H, D, device="cuda", generator=gen).to(torch.bfloat16) for _ in layers]
    vc0 = [torch.randn(B, S_max, H, D, device="cuda", generator=gen).to(torch.bfloat16) for _ in layers]
    x0 = torch.randn(B, d, device="cuda", generator=gen).to(torch.bfloat16)
    seq = torch.full((B,), P, dtype=torch.int32, device="cuda")

    x_a, kc_a, vc_a = x0.clone(), [k.clone() for k in kc0], [v.clone() for v in vc0]
    for (L, _), kc, vc in zip(layers, kc_a, vc_a):
        fs.layer_forward(L, x_a, kc, vc, seq, B, 1, S_max, fs.DECODE)
    x_b, kc_b, vc_b = x0.clone(), [k.clone() for k in kc0], [v.clone() for v in vc0]
    plan = fs.DecodePlan([L for L, _ in layers], kc_b, vc_b, B, S_max)
    plan.forward(x_b, seq)
    torch.cuda.synchronize()
    fs.check_device_status()
    plan.destroy()
    assert torch.equal(x_a.view(torch.int16), x_b.view(torch.int16))
    for a, b in zip(kc_a + vc_a, kc_b + vc_b):
        assert torch.equal(a.view(torch.int16), b.view(torch.int16))
    assert torch.isfinite(x_b.float()).all()
