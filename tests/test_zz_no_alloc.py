"""flashsvd_lowrank_linear_noalloc, called through the C ABI.

The no-allocation entry point serves callers that cannot allocate device
memory -- a plugin inside a framework whose allocator owns the GPU, or a
serving process that must not allocate after start-up -- since
flashsvd_init's workspace comes from cudaMalloc.  It keeps its scratch in a
fixed device array instead.  These tests check it against the CPU oracle and
bit for bit against the workspace-based flashsvd_lowrank_linear (same
kernels, same split), on two calls in a row so that the shared array, which
keeps the previous call's contents, cannot leak into the next result; one
test runs it in a fresh process that never calls flashsvd_init.  This file
is collected last on purpose.
"""
import os
import subprocess
import sys
import textwrap

import numpy as np
import pytest

from oracle import flashsvd_oracle as oracle
from rank_transformer_b200 import synth
from tests.gpu_util import assert_parity, dev_bf16, host_bits, host_f64

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def fs():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from rank_transformer_b200 import flashsvd
    flashsvd.init(0, max_tokens=64, max_rank=4096, max_hidden=4096, max_ffn=11008)
    return flashsvd


def _case(seed, M, d, r, n, bias):
    rng = synth.rng_for(seed)
    U = synth.normal_bf16(rng, (d, r), d ** -0.5)
    V = synth.normal_bf16(rng, (r, n), r ** -0.5)
    x = synth.normal_bf16(rng, (M, d))
    b = synth.normal_bf16(rng, (n,), 0.02) if bias else None
    return x, U, V, b


def _oracle(x, U, V, b):
    return oracle.lowrank_linear(oracle.from_bf16(x), oracle.from_bf16(U), oracle.from_bf16(V),
                                 None if b is None else oracle.from_bf16(b))


@pytest.mark.parametrize("M,d,r,n", [(1, 4096, 1216, 4096), (8, 4096, 1792, 11008),
                                     (3, 256, 64, 688), (5, 4096, 4096, 4096),
                                     (8, 8192, 2048, 8192)])
def test_noalloc_matches_oracle_and_workspace_entry(fs, M, d, r, n):
    for call in range(2):
        x, U, V, b = _case(9000 + 10 * call + M, M, d, r, n, bias=call == 1)
        dx, dU, dV = dev_bf16(x), dev_bf16(U), dev_bf16(V)
        db = None if b is None else dev_bf16(b)
        y_ref = torch.empty((M, n), dtype=torch.bfloat16, device="cuda")
        y_na = torch.empty((M, n), dtype=torch.bfloat16, device="cuda")
        fs.lowrank_linear(dx, dU, dV, db, y_ref, M, d, r, n)
        fs.lowrank_linear_noalloc(dx, dU, dV, db, y_na, M, d, r, n)
        torch.cuda.synchronize()
        assert_parity(host_f64(y_na), _oracle(x, U, V, b), f"noalloc call {call} M={M}")
        assert np.array_equal(host_bits(y_na), host_bits(y_ref)), \
            f"noalloc call {call} M={M}: differs from the workspace call"


def test_noalloc_acceptance_rule(fs):
    """The header's rule ceil(K/512) * ceil(N/64) * (64 m + 8) <= 2^19: with
    d = 16384 and r = 4096 the first product needs 32 * 64 splits x tiles,
    which fits at M = 1 (m = 1) but not at M = 8 (m = 8)."""
    M, d, r, n = 1, 16384, 4096, 1024
    x, U, V, _ = _case(9100, 8, d, r, n, bias=False)
    dx, dU, dV = dev_bf16(x), dev_bf16(U), dev_bf16(V)
    y = torch.empty((8, n), dtype=torch.bfloat16, device="cuda")
    L = fs.lib
    assert L.flashsvd_lowrank_linear_noalloc(dx.data_ptr(), dU.data_ptr(), dV.data_ptr(), None,
                                             y.data_ptr(), 8, d, r, n, None) == 3
    for _ in range(2):
        fs.lowrank_linear_noalloc(dx[:M], dU, dV, None, y[:M], M, d, r, n)
        torch.cuda.synchronize()
        assert_parity(host_f64(y[:M]), _oracle(x[:M], U, V, None), "noalloc d=16384 r=4096 M=1")


def test_noalloc_fresh_process_without_init(tmp_path):
    """A process that never calls flashsvd_init (and never runs the
    workspace path) calls only the no-allocation entry point, twice; its
    output is checked here against the oracle."""
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    out = tmp_path / "y.npy"
    child = textwrap.dedent(f"""
        import numpy as np, torch
        from rank_transformer_b200 import flashsvd as fs, synth
        from tests.gpu_util import dev_bf16, host_bits
        torch.cuda.set_device(0)
        ys = []
        for call in range(2):
            rng = synth.rng_for(9200 + call)
            U = synth.normal_bf16(rng, (4096, 1216), 4096 ** -0.5)
            V = synth.normal_bf16(rng, (1216, 4096), 1216 ** -0.5)
            x = synth.normal_bf16(rng, (4, 4096))
            y = torch.empty((4, 4096), dtype=torch.bfloat16, device="cuda")
            fs.lowrank_linear_noalloc(dev_bf16(x), dev_bf16(U), dev_bf16(V), None, y,
                                      4, 4096, 1216, 4096)
            torch.cuda.synchronize()
            ys.append(host_bits(y))
        np.save({str(out)!r}, np.stack(ys))
    """)
    env = dict(os.environ, PYTHONPATH=ROOT)
    res = subprocess.run([sys.executable, "-c", child], cwd=ROOT, env=env,
                         capture_output=True, text=True, timeout=600)
    assert res.returncode == 0, res.stderr[-2000:]
    ys = np.load(out)
    for call in range(2):
        x, U, V, _ = _case(9200 + call, 4, 4096, 1216, 4096, bias=False)
        assert_parity(oracle.from_bf16(ys[call]), _oracle(x, U, V, None),
                      f"fresh-process noalloc call {call}")


def test_noalloc_rejects_oversize(fs):
    a = torch.empty(16, dtype=torch.bfloat16, device="cuda")
    L = fs.lib
    p = a.data_ptr()
    assert L.flashsvd_lowrank_linear_noalloc(p, p, p, None, p, 9, 64, 64, 64, None) == 3
    assert L.flashsvd_lowrank_linear_noalloc(p, p, p, None, p, 1, 64, 8192, 64, None) == 3
    assert L.flashsvd_lowrank_linear_noalloc(p, p, p, None, p, 1, 64, 64, 20000, None) == 3
    assert L.flashsvd_lowrank_linear_noalloc(None, p, p, None, p, 1, 64, 64, 64, None) == 1
