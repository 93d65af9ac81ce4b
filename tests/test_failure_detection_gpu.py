"""Failure detection of the fused decode kernel, without a GPU fault.

Its CTAs wait on one another at grid barriers, with bounded waits.  A
host-armed test hook (flashsvd_debug_drop_barrier_arrival) makes CTA 0 of
the next launch skip its first barrier arrival: the other CTAs' waits
expire, the launch completes, and the host reads FLASHSVD_ERR_TIMEOUT from
the device status word.  The next launch must then run normally and match
the oracle."""
import time

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


def test_dropped_barrier_arrival_times_out_then_recovers(fs):
    from tests.test_decode_gpu import _layer_struct
    d, H, D, f, r, P = 256, 4, 64, 688, 64, 40
    S_max = P + 8
    rng = synth.rng_for(9800)
    w = synth.decoder_layer_weights(rng, d, f, r, r, gain_jitter=0.1)
    cos_t = torch.empty((S_max, D // 2), dtype=torch.float32, device="cuda")
    sin_t = torch.empty_like(cos_t)
    fs.rope_table(cos_t, sin_t, S_max, D, 10000.0)
    L, dev = _layer_struct(fs, w, d, H, D, f, r, r, cos_t, sin_t)
    kc0 = synth.normal_bf16(rng, (1, S_max, H, D))
    vc0 = synth.normal_bf16(rng, (1, S_max, H, D))
    xt = synth.normal_bf16(rng, (1, d))
    seq = torch.full((1,), P, dtype=torch.int32, device="cuda")

    # the faulty launch: bounded waits expire, the status word says so
    fs.lib.flashsvd_debug_drop_barrier_arrival()
    x = dev_bf16(xt)
    t0 = time.time()
    fs.layer_forward(L, x, dev_bf16(kc0), dev_bf16(vc0), seq, 1, 1, S_max, fs.DECODE)
    torch.cuda.synchronize()
    elapsed = time.time() - t0
    with pytest.raises(fs.FlashSVDError) as err:
        fs.check_device_status()
    assert err.value.status == 7, err.value
    assert elapsed < 60.0, elapsed

    # the next launch is clean and correct
    x = dev_bf16(xt)
    kc, vc = dev_bf16(kc0), dev_bf16(vc0)
    fs.layer_forward(L, x, kc, vc, seq, 1, 1, S_max, fs.DECODE)
    torch.cuda.synchronize()
    fs.check_device_status()
    y, kn, vn = oracle.decoder_layer_decode(oracle.from_bf16(xt), oracle.widen_layer(w), H,
                                            oracle.from_bf16(kc0), oracle.from_bf16(vc0), [P])
    assert_parity(host_f64(x), y, "decode after a timed-out launch")
    assert_parity(host_f64(kc)[0, P], kn[0], "appended k after a timed-out launch")
