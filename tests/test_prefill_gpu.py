"""GPU parity of the prefill path (M > 32, tcgen05 tensor cores) against the
CPU oracle, called through the C ABI."""
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


def _factors(rng, d, r, n):
    return (synth.normal_bf16(rng, (d, r), d ** -0.5),
            synth.normal_bf16(rng, (r, n), r ** -0.5))


PREFILL_CASES = [
    (33, 256, 64, 688), (128, 256, 64, 256), (200, 688, 64, 256), (512, 768, 192, 3072),
    (513, 3072, 192, 768), (256, 4096, 512, 4096), (512, 4096, 1216, 4096),
    (384, 4096, 1792, 11008),
]


@pytest.mark.parametrize("M,d,r,n", PREFILL_CASES)
def test_lowrank_linear_prefill(fs, M, d, r, n):
    rng = synth.rng_for(5000 + M + d + r + n)
    U, V = _factors(rng, d, r, n)
    x = synth.normal_bf16(rng, (M, d))
    bias = synth.normal_bf16(rng, (n,), 0.02) if M % 2 else None
    y = torch.empty((M, n), dtype=torch.bfloat16, device="cuda")
    fs.lowrank_linear(dev_bf16(x), dev_bf16(U), dev_bf16(V),
                      dev_bf16(bias) if bias is not None else None, y, M, d, r, n)
    torch.cuda.synchronize()
    ref = oracle.lowrank_linear(oracle.from_bf16(x), oracle.from_bf16(U), oracle.from_bf16(V),
                                None if bias is None else oracle.from_bf16(bias))
    assert_parity(host_f64(y), ref, f"prefill lowrank M={M} d={d} r={r} n={n}")


def test_lowrank_linear_prefill_deterministic(fs):
    rng = synth.rng_for(5100)
    M, d, r, n = 300, 1024, 256, 1536
    U, V = _factors(rng, d, r, n)
    x = dev_bf16(synth.normal_bf16(rng, (M, d)))
    Ud, Vd = dev_bf16(U), dev_bf16(V)
    outs = []
    for _ in range(2):
        y = torch.empty((M, n), dtype=torch.bfloat16, device="cuda")
        fs.lowrank_linear(x, Ud, Vd, None, y, M, d, r, n)
        outs.append(y)
    torch.cuda.synchronize()
    assert torch.equal(outs[0], outs[1])


@pytest.mark.parametrize("M,d,r_f,f,r_dn", [(128, 256, 64, 688, 64), (300, 768, 128, 3072, 192),
                                           (512, 4096, 512, 11008, 1024)])
def test_packed_mlp_prefill(fs, M, d, r_f, f, r_dn):
    rng = synth.rng_for(5200 + M + r_f)
    U_gu = synth.normal_bf16(rng, (d, 2 * r_f), d ** -0.5)
    V_gu = synth.normal_bf16(rng, (2 * r_f, f), r_f ** -0.5)
    U_dn, V_dn = _factors(rng, f, r_dn, d)
    x = synth.normal_bf16(rng, (M, d))
    h = torch.empty((M, f), dtype=torch.bfloat16, device="cuda")
    y = torch.empty((M, d), dtype=torch.bfloat16, device="cuda")
    xs, ug, vg = dev_bf16(x), dev_bf16(U_gu), dev_bf16(V_gu)
    fs.gateup_swiglu(xs, ug, vg, h, M, d, r_f, f)
    fs.packed_gateup_mlp(xs, ug, vg, dev_bf16(U_dn), dev_bf16(V_dn), y, M, d, r_f, f, r_dn)
    torch.cuda.synchronize()
    X = oracle.from_bf16(x)
    w = [oracle.from_bf16(a) for a in (U_gu, V_gu, U_dn, V_dn)]
    assert_parity(host_f64(h), oracle.gateup_swiglu(X, w[0], w[1], r_f), "prefill gate|up h")
    assert_parity(host_f64(y), oracle.packed_gateup_mlp(X, *w, r_f), "prefill packed mlp")


@pytest.mark.parametrize("M,d,n", [(64, 256, 1000), (130, 512, 4096)])
def test_dense_linear_prefill(fs, M, d, n):
    rng = synth.rng_for(5300 + M)
    W = synth.normal_bf16(rng, (d, n), d ** -0.5)
    x = synth.normal_bf16(rng, (M, d))
    y = torch.empty((M, n), dtype=torch.float32, device="cuda")
    fs.dense_linear_f32(dev_bf16(x), dev_bf16(W), y, M, d, n)
    torch.cuda.synchronize()
    assert_parity(y.double().cpu().numpy(),
                  oracle.dense_linear(oracle.from_bf16(x), oracle.from_bf16(W)), "dense prefill")
