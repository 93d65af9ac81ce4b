"""Host-only checks of the C ABI: the library builds and loads, exports every
function include/flashsvd.h declares, and rejects bad arguments with the
documented status before touching the GPU."""
import ctypes as C
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def fs():
    from rank_transformer_b200 import build
    build.build()
    from rank_transformer_b200 import flashsvd
    return flashsvd


def _declared():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            txt = open(os.path.join(ROOT, "include", fn)).read()
            names |= set(re.findall(r"FLASHSVD_API[^;(]*?\b(flashsvd_\w+)\s*\(", txt))
    return names


def test_header_declares_api():
    names = _declared()
    for n in ("flashsvd_lowrank_linear", "flashsvd_packed_gateup_mlp",
              "flashsvd_dense_kv_decode_attn", "flashsvd_layer_forward",
              "flashsvd_decode_graph_capture", "flashsvd_graph_replay"):
        assert n in names


def test_every_declared_symbol_is_exported(fs):
    for name in sorted(_declared()):
        assert hasattr(fs.lib, name), f"{name} not exported"
        assert name in fs.EXPORTED, f"{name} not bound in flashsvd.py"


def test_product_library_has_no_trace_code(fs):
    """The stage-timeline hooks exist only in the trace build
    (libflashsvd_trace.so); the product library exports none of them."""
    for name in ("flashsvd_trace_read", "flashsvd_trace_clear"):
        assert not hasattr(fs.lib, name), name


def test_status_strings(fs):
    assert fs.lib.flashsvd_status_string(0) == b"ok"
    for s in range(1, 9):
        assert fs.lib.flashsvd_status_string(s) not in (b"ok", b"unknown status")
    assert fs.lib.flashsvd_version() >= 100


def test_argument_errors_before_any_launch(fs):
    L = fs.lib
    aligned, misaligned = 0x10000, 0x10008
    # not initialised (nothing allocated on any device yet)
    if L.flashsvd_lowrank_linear(aligned, aligned, aligned, None, aligned, 1, 64, 64, 64, None) \
            != 4:
        pytest.skip("library already initialised in this process")
    assert L.flashsvd_layer_forward(None, aligned, aligned, aligned, None, 1, 1, 8, 1, None) == 4
    assert L.flashsvd_head_logits(aligned, None, 0.0, aligned, aligned, 1, 64, 64, None) == 4
    # null / misaligned / width not a multiple of 8 / negative sizes
    assert L.flashsvd_rmsnorm(None, aligned, aligned, 1, 64, 1e-5, None) == 1
    assert L.flashsvd_rmsnorm(misaligned, aligned, aligned, 1, 64, 1e-5, None) == 2
    assert L.flashsvd_rmsnorm(aligned, aligned, aligned, 1, 60, 1e-5, None) == 3
    assert L.flashsvd_rmsnorm(aligned, aligned, aligned, -1, 64, 1e-5, None) == 1
    assert L.flashsvd_layernorm(aligned, aligned, None, aligned, 1, 64, 1e-5, None) == 1
    assert L.flashsvd_embed(None, aligned, aligned, 1, 64, 10, None) == 1
    assert L.flashsvd_embed(aligned, aligned, aligned, 1, 64, 0, None) == 1
    assert L.flashsvd_greedy(None, aligned, 1, 10, None) == 1
    assert L.flashsvd_advance_seqlens(None, 1, None) == 1
    assert L.flashsvd_rope_table(aligned, aligned, 16, 7, 10000.0, None) == 1
    assert L.flashsvd_graph_replay(None, None) == 1
    assert L.flashsvd_graph_destroy(None) == 1
    assert L.flashsvd_graph_kernel_count(None) == -1
    assert L.flashsvd_capture_begin(None) == 1
    h = C.c_void_p()
    assert L.flashsvd_graph_compose(None, 0, C.byref(h)) == 1
    assert L.flashsvd_init(-1, 1, 1, 1, 1) == 1
    assert L.flashsvd_init(0, 0, 1, 1, 1) == 1
    # contexts: bad arguments rejected before any allocation
    assert L.flashsvd_ctx_create(-1, 1, 1, 1, 1, C.byref(h)) == 1
    assert L.flashsvd_ctx_create(0, 0, 1, 1, 1, C.byref(h)) == 1
    assert L.flashsvd_ctx_create(0, 1, 1, 1, 1, None) == 1
    assert L.flashsvd_ctx_destroy(None) == 1
    assert L.flashsvd_ctx_bind(None) == 0          # back to the default context


def test_binding_raises_on_error(fs):
    with pytest.raises(fs.FlashSVDError) as e:
        fs._call("flashsvd_rmsnorm", None, None, None, 1, 64, 1e-5, None)
    assert e.value.status == 1
