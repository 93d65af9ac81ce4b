"""Shared bases (FlashSVD v1.5 explainer, Methodology 1: Basis Sharing keeps
one physical copy of a basis that several layers use): decoder layers whose
input-side factors U_q, U_k, U_v, U_o, U_gu, U_dn are the same device
tensors.  A decode plan over them reads the shared factors' entries from the
first layer's decode pack; its output must equal, bit for bit, the same
layers run one fused launch each (every layer from its own pack), and each
of those layers must match the oracle."""
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


@pytest.mark.parametrize("B", [1, 2])
def test_shared_basis_plan(fs, B):
    from tests.test_decode_gpu import _layer_struct
    d, H, D, f, r, r_f, nl = 1024, 8, 128, 2752, 320, 448, 4
    pos = [700, 300][:B]
    S_max = 768
    rng = synth.rng_for(9700 + B)
    ws = [synth.decoder_layer_weights(rng, d, f, r, r_f, gain_jitter=0.1) for _ in range(nl)]
    shared = ("U_q", "U_k", "U_v", "U_o", "U_gu", "U_dn")
    for w in ws[1:]:
        for k in shared:
            w[k] = ws[0][k]                     # same host values ...
    cos_t = torch.empty((S_max, D // 2), dtype=torch.float32, device="cuda")
    sin_t = torch.empty_like(cos_t)
    fs.rope_table(cos_t, sin_t, S_max, D, 10000.0)
    Ls, devs = [], []
    for i, w in enumerate(ws):
        L, dev = _layer_struct(fs, w, d, H, D, f, r, r_f, cos_t, sin_t, pack=True)
        if i > 0:                               # ... and the same device tensors
            for k in shared:
                dev[k] = devs[0][k]
            L.q.U, L.k.U, L.v.U = dev["U_q"].data_ptr(), dev["U_k"].data_ptr(), dev["U_v"].data_ptr()
            L.o.U, L.U_gu, L.down.U = dev["U_o"].data_ptr(), dev["U_gu"].data_ptr(), dev["U_dn"].data_ptr()
        Ls.append(L)
        devs.append(dev)
    kc0 = [synth.normal_bf16(rng, (B, S_max, H, D)) for _ in range(nl)]
    vc0 = [synth.normal_bf16(rng, (B, S_max, H, D)) for _ in range(nl)]
    xt = synth.normal_bf16(rng, (B, d))
    seq = torch.tensor(pos, dtype=torch.int32, device="cuda")

    # one fused launch per layer, each from its own pack; oracle per layer
    kcs, vcs = [dev_bf16(k) for k in kc0], [dev_bf16(v) for v in vc0]
    x = dev_bf16(xt)
    for i in range(nl):
        x_in = host_f64(x)
        fs.layer_forward(Ls[i], x, kcs[i], vcs[i], seq, B, 1, S_max, fs.DECODE)
        torch.cuda.synchronize()
        y, _, _ = oracle.decoder_layer_decode(x_in, oracle.widen_layer(ws[i]), H,
                                              oracle.from_bf16(kc0[i]), oracle.from_bf16(vc0[i]), pos)
        assert_parity(host_f64(x), y, f"shared-basis layer {i}")
    per_layer = host_bits(x)

    # the plan: layers 1..3 read the shared factors from layer 0's pack
    kcp, vcp = [dev_bf16(k) for k in kc0], [dev_bf16(v) for v in vc0]
    plan = fs.DecodePlan(Ls, kcp, vcp, B, S_max)
    xp = dev_bf16(xt)
    plan.forward(xp, seq)
    torch.cuda.synchronize()
    fs.check_device_status()
    assert np.array_equal(host_bits(xp), per_layer), "plan over shared bases differs from per-layer launches"
    for i in range(nl):
        assert np.array_equal(host_bits(kcp[i]), host_bits(kcs[i]))
    plan.destroy()
