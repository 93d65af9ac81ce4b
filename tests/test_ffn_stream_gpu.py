"""GPU parity of the streamed low-rank encoder FFN (flashsvd_lowrank_ffn)
against the CPU oracle, called through the C ABI:
    y = GELU((x U_up) V_up + b_up) U_dn V_dn + b_dn + resid
at the BERT-Base-shaped sizes (d 768, f 3072, rank 192), with a ragged last
row tile, f not a multiple of the 128-column chunk, unequal ranks, d not a
multiple of the 256-column output pass, and the residual aliasing the
output; then the encoder layer that uses it, with an FFN width above the
workspace's limit (possible only because the activation stays on chip)."""
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
    flashsvd.init(0, max_tokens=16384, max_rank=4096, max_hidden=4096, max_ffn=11008)
    return flashsvd


CASES = [
    # (M, d, r_up, f, r_dn, resid)
    (300, 768, 192, 3072, 192, "none"),
    (4096, 768, 192, 3072, 192, "separate"),
    (16384, 768, 192, 3072, 192, "alias"),
    (200, 768, 128, 3000, 256, "separate"),
    (130, 832, 64, 1000, 192, "alias"),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "M{}-d{}-r{}-f{}-r{}-{}".format(*c))
def test_lowrank_ffn(fs, case):
    M, d, r1, f, r2, resid = case
    rng = synth.rng_for(8100 + M + f)
    x = synth.normal_bf16(rng, (M, d))
    U1 = synth.normal_bf16(rng, (d, r1), d ** -0.5)
    V1 = synth.normal_bf16(rng, (r1, f), r1 ** -0.5)
    b1 = synth.normal_bf16(rng, (f,), 0.1)
    U2 = synth.normal_bf16(rng, (f, r2), f ** -0.5)
    V2 = synth.normal_bf16(rng, (r2, d), r2 ** -0.5)
    b2 = synth.normal_bf16(rng, (d,), 0.1)
    res = synth.normal_bf16(rng, (M, d))
    d_res = dev_bf16(res)
    y = d_res if resid == "alias" else torch.empty((M, d), dtype=torch.bfloat16, device="cuda")
    r_arg = None if resid == "none" else d_res
    for _ in range(2):   # a second call over the same scratch gives the same result
        if resid == "alias":
            y.copy_(dev_bf16(res))
        fs.lowrank_ffn(dev_bf16(x), dev_bf16(U1), dev_bf16(V1), dev_bf16(b1), dev_bf16(U2),
                       dev_bf16(V2), dev_bf16(b2), r_arg, y, M, d, r1, f, r2)
        torch.cuda.synchronize()
        fs.check_device_status()
        rows = np.arange(M) if M <= 4096 else np.unique(np.concatenate(
            [np.arange(0, 256), np.arange(M - 300, M), np.random.default_rng(3).integers(0, M, 200)]))
        ref = oracle.lowrank_gelu_ffn(oracle.from_bf16(x[rows]), oracle.from_bf16(U1),
                                      oracle.from_bf16(V1), oracle.from_bf16(b1), oracle.from_bf16(U2),
                                      oracle.from_bf16(V2), oracle.from_bf16(b2))
        if resid != "none":
            ref = ref + oracle.from_bf16(res[rows])
        assert_parity(host_f64(y)[rows], ref, f"streamed ffn {case}")


def test_lowrank_ffn_rejects_uncovered_ranks(fs):
    a = torch.empty(64, dtype=torch.bfloat16, device="cuda")
    p = a.data_ptr()
    L = fs.lib
    assert L.flashsvd_lowrank_ffn(p, p, p, None, p, p, None, None, p, 128, 768, 320, 3072, 192, None) == 3
    assert L.flashsvd_lowrank_ffn(p, p, p, None, p, p, None, None, p, 128, 768, 192, 3072, 96, None) == 3


def test_encoder_layer_streamed_ffn_beyond_workspace_width(fs):
    """An encoder layer whose FFN width exceeds the workspace's max_ffn runs
    only because the streamed FFN keeps the [M x f] activation on chip; a
    fresh context sized with max_ffn = 8 runs the BERT-shaped layer."""
    from tests.test_layers_gpu import _encoder_struct
    d, H, f, r, B, S = 768, 12, 3072, 192, 2, 256
    rng = synth.rng_for(8200)
    w = synth.bert_layer_weights(rng, d, f, r, bias_std=0.02, gain_jitter=0.1)
    L, dev = _encoder_struct(fs, w, d, H, f)
    xb = synth.normal_bf16(rng, (B, S, d))
    x = dev_bf16(xb.reshape(B * S, d))
    kb = torch.empty((B, S, H, d // H), dtype=torch.bfloat16, device="cuda")
    vb = torch.empty_like(kb)
    ctx = fs.Context(0, max_tokens=B * S, max_rank=r, max_hidden=d, max_ffn=8)
    try:
        with ctx:
            fs.layer_forward(L, x, kb, vb, None, B, S, S, fs.ENCODER_BIDIR)
            torch.cuda.synchronize()
            fs.check_device_status()
    finally:
        ctx.destroy()
    got = host_f64(x).reshape(B, S, d)
    wf = oracle.widen_layer(w)
    for b in range(B):
        assert_parity(got[b], oracle.bert_layer(oracle.from_bf16(xb[b]), wf, H), f"encoder b={b}")
