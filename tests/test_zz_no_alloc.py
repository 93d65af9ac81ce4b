"""flashsvd_lowrank_linear_noalloc, called through the C ABI, against the
workspace-based flashsvd_lowrank_linear on the same inputs.

The no-allocation entry point serves callers that cannot allocate device
memory (flashsvd_init's workspace comes from cudaMalloc); it keeps its
scratch in a fixed device array instead.  Two calls in a row check that the
shared array, which keeps the previous call's contents, does not leak into
the next result.  This file is collected last on purpose.
"""
import ctypes as C

import numpy as np
import pytest

from rank_transformer_b200 import synth
from tests.gpu_util import assert_parity, dev_bf16, host_f64

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module")
def fs():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from rank_transformer_b200 import flashsvd
    flashsvd.init(0, max_tokens=64, max_rank=4096, max_hidden=4096, max_ffn=11008)
    return flashsvd


@pytest.mark.parametrize("M,d,r,n", [(1, 4096, 1216, 4096), (8, 4096, 1792, 11008),
                                     (3, 256, 64, 688)])
def test_noalloc_matches_workspace_entry(fs, M, d, r, n):
    for call in range(2):
        rng = synth.rng_for(9000 + 10 * call + M)
        U = dev_bf16(synth.normal_bf16(rng, (d, r), d ** -0.5))
        V = dev_bf16(synth.normal_bf16(rng, (r, n), r ** -0.5))
        x = dev_bf16(synth.normal_bf16(rng, (M, d)))
        bias = dev_bf16(synth.normal_bf16(rng, (n,), 0.02)) if call else None
        y_ref = torch.empty((M, n), dtype=torch.bfloat16, device="cuda")
        y_na = torch.empty((M, n), dtype=torch.bfloat16, device="cuda")
        fs.lowrank_linear(x, U, V, bias, y_ref, M, d, r, n)
        fs.lowrank_linear_noalloc(x, U, V, bias, y_na, M, d, r, n)
        torch.cuda.synchronize()
        assert_parity(host_f64(y_na), host_f64(y_ref), f"noalloc call {call} M={M}")


def test_noalloc_rejects_oversize(fs):
    a = torch.empty(16, dtype=torch.bfloat16, device="cuda")
    L = fs.lib
    p = a.data_ptr()
    assert L.flashsvd_lowrank_linear_noalloc(p, p, p, None, p, 9, 64, 64, 64, None) == 3
    assert L.flashsvd_lowrank_linear_noalloc(p, p, p, None, p, 1, 64, 8192, 64, None) == 3
    assert L.flashsvd_lowrank_linear_noalloc(p, p, p, None, p, 1, 64, 64, 20000, None) == 3
    assert L.flashsvd_lowrank_linear_noalloc(None, p, p, None, p, 1, 64, 64, 64, None) == 1
