"""Two contexts (flashsvd_ctx_create) driven from two host threads on two
streams at the same time: each thread binds its own context, so the calls'
scratch (rank activations, split partial sums, tile counters, the bf16
prefill rank scratch and the per-layer buffers) is not shared, and every
result must match the CPU oracle."""
import threading

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
    return flashsvd


def _inputs(seed, M, d, r, n):
    rng = synth.rng_for(seed)
    return (synth.normal_bf16(rng, (M, d)), synth.normal_bf16(rng, (d, r), d ** -0.5),
            synth.normal_bf16(rng, (r, n), r ** -0.5))


def test_two_contexts_two_streams_concurrently(fs):
    reps = 6
    cases = {0: [(4, 4096, 1216, 4096), (512, 4096, 1216, 4096)],
             1: [(8, 4096, 1792, 11008), (384, 4096, 832, 4096)]}
    data = {}
    for t, shapes in cases.items():
        for j, (M, d, r, n) in enumerate(shapes):
            x, U, V = _inputs(8000 + 10 * t + j, M, d, r, n)
            data[t, j] = dict(shape=(M, d, r, n), x=x, U=U, V=V, dx=dev_bf16(x), dU=dev_bf16(U),
                              dV=dev_bf16(V),
                              ys=[torch.empty((M, n), dtype=torch.bfloat16, device="cuda")
                                  for _ in range(reps)])
    ctxs = [fs.Context(0, max_tokens=1024, max_rank=2048, max_hidden=4096, max_ffn=11008)
            for _ in range(2)]
    streams = [torch.cuda.Stream() for _ in range(2)]
    errors = []
    start = threading.Barrier(2)

    def worker(t):
        try:
            ctxs[t].bind()
            s = streams[t]
            start.wait()
            with torch.cuda.stream(s):
                for i in range(reps):
                    for j in range(2):
                        c = data[t, j]
                        M, d, r, n = c["shape"]
                        fs.lowrank_linear(c["dx"], c["dU"], c["dV"], None, c["ys"][i], M, d, r, n, s)
            s.synchronize()
            fs.check_device_status(s)
        except Exception as e:  # reported in the main thread
            errors.append(e)
        finally:
            fs.Context.unbind()

    th = [threading.Thread(target=worker, args=(t,)) for t in range(2)]
    for x in th:
        x.start()
    for x in th:
        x.join()
    for c in ctxs:
        c.destroy()
    assert not errors, errors
    for (t, j), c in data.items():
        ref = oracle.lowrank_linear(oracle.from_bf16(c["x"]), oracle.from_bf16(c["U"]),
                                    oracle.from_bf16(c["V"]))
        for i in range(reps):
            assert_parity(host_f64(c["ys"][i]), ref, f"context {t} case {j} rep {i}")
