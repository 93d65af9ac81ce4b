"""GPU parity of the decode step's head with the final RMSNorm folded in
(flashsvd_head_logits: one split-K GEMV whose CTAs sum the squares of their
slice of x and whose tile reducers scale by rstd) against the CPU oracle,
called through the C ABI."""
import pytest

from oracle import flashsvd_oracle as oracle
from rank_transformer_b200 import synth
from tests.gpu_util import assert_parity, dev_bf16

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module")
def fs():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from rank_transformer_b200 import flashsvd
    flashsvd.init(0, max_tokens=4096, max_rank=4096, max_hidden=4096, max_ffn=11008)
    return flashsvd


@pytest.mark.parametrize("d,n", [(4096, 32000), (1000, 1000), (512, 64)])
@pytest.mark.parametrize("M", [1, 3, 8, 32])
@pytest.mark.parametrize("norm", [True, False])
def test_head_logits(fs, d, n, M, norm):
    if d * n > 4096 * 32000 // 4 and M not in (1, 8):
        pytest.skip("the full-size head is checked at M = 1 and 8")
    rng = synth.rng_for(9800 + M + d + norm)
    x = synth.normal_bf16(rng, (M, d))
    W = synth.normal_bf16(rng, (d, n), d ** -0.5)
    g = synth.normal_bf16(rng, (d,), 0.2, mean=1.0) if norm else None
    logits = torch.empty((M, n), dtype=torch.float32, device="cuda")
    fs.head_logits(dev_bf16(x), dev_bf16(g) if norm else None, 1e-5, dev_bf16(W), logits, M, d, n)
    torch.cuda.synchronize()
    fs.check_device_status()
    X, Wd = oracle.from_bf16(x), oracle.from_bf16(W)
    ref = oracle.lm_head(X, oracle.from_bf16(g), Wd, eps=1e-5) if norm else oracle.dense_linear(X, Wd)
    assert_parity(logits.double().cpu().numpy(), ref, f"head d={d} n={n} M={M} norm={norm}")


def test_head_rejects(fs):
    W = torch.zeros((64, 64), dtype=torch.bfloat16, device="cuda")
    x = torch.zeros((33, 64), dtype=torch.bfloat16, device="cuda")
    y = torch.empty((33, 64), dtype=torch.float32, device="cuda")
    with pytest.raises(fs.FlashSVDError) as e:
        fs.head_logits(x, None, 0.0, W, y, 33, 64, 64)
    assert e.value.status == 3   # more than 32 rows
    with pytest.raises(fs.FlashSVDError) as e:
        fs.head_logits(x, x[0], -1.0, W, y, 1, 64, 64)
    assert e.value.status == 1   # negative eps with a gain
