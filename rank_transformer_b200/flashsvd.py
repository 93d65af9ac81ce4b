"""ctypes binding of libflashsvd.so (argument marshalling only).

Every function here forwards to the C entry point of the same name in
``include/flashsvd.h``; tensors are passed as raw device pointers
(``tensor.data_ptr()``), streams as ``cudaStream_t`` handles.  All compute
runs in the library's CUDA kernels; there is no CPU fallback.  Importing this
module fails loudly if the library has not been built.
"""
from __future__ import annotations

import ctypes as C
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
# FLASHSVD_LIBRARY selects another build of the same library (the trace
# build, libflashsvd_trace.so); by default the in-tree product library.
LIB_PATH = os.environ.get("FLASHSVD_LIBRARY") or os.path.join(_HERE, "libflashsvd.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"{LIB_PATH} is missing: build it with `python -m rank_transformer_b200.build` "
        "(the CUDA library is required; there is no fallback path)")

lib = C.CDLL(LIB_PATH)

OK = 0
STATUS_NAMES = {
    0: "OK", 1: "ERR_INVALID_ARG", 2: "ERR_MISALIGNED", 3: "ERR_UNSUPPORTED_SHAPE",
    4: "ERR_NOT_INITIALIZED", 5: "ERR_CAPTURE_UNSAFE", 6: "ERR_CUDA",
    7: "ERR_TIMEOUT", 8: "ERR_NO_MEMORY",
}
DECODER, ENCODER = 0, 1
PREFILL_CAUSAL, DECODE, ENCODER_BIDIR = 0, 1, 2

_p = C.c_void_p
_i = C.c_int
_f = C.c_float


class FlashSVDError(RuntimeError):
    def __init__(self, fn, status):
        msg = lib.flashsvd_status_string(status).decode()
        if status == 6:
            msg += f" (cudaError {lib.flashsvd_last_cuda_error()})"
        super().__init__(f"{fn}: {STATUS_NAMES.get(status, status)}: {msg}")
        self.status = status


class Factor(C.Structure):
    _fields_ = [("U", _p), ("V", _p), ("bias", _p), ("r", _i)]


class Layer(C.Structure):
    _fields_ = [
        ("kind", _i), ("d", _i), ("H", _i), ("D", _i), ("f", _i),
        ("norm_eps", _f),
        ("norm1_g", _p), ("norm1_b", _p), ("norm2_g", _p), ("norm2_b", _p),
        ("q", Factor), ("k", Factor), ("v", Factor), ("o", Factor),
        ("U_gu", _p), ("V_gu", _p), ("r_f", _i),
        ("up", Factor), ("down", Factor),
        ("rope_cos", _p), ("rope_sin", _p),
        ("decode_pack", _p),
    ]


_SIGS = {
    "flashsvd_status_string": ([_i], C.c_char_p),
    "flashsvd_last_cuda_error": ([], _i),
    "flashsvd_version": ([], _i),
    "flashsvd_init": ([_i, _i, _i, _i, _i], _i),
    "flashsvd_shutdown": ([], _i),
    "flashsvd_check_device_status": ([_p], _i),
    "flashsvd_ctx_create": ([_i, _i, _i, _i, _i, C.POINTER(_p)], _i),
    "flashsvd_ctx_bind": ([_p], _i),
    "flashsvd_ctx_destroy": ([_p], _i),
    "flashsvd_launch_count": ([], C.c_int64),
    "flashsvd_set_decode_path": ([_i], _i),
    "flashsvd_set_prefill_attention": ([_i], _i),
    "flashsvd_set_l2_discard": ([_i], _i),
    "flashsvd_debug_drop_barrier_arrival": ([], _i),
    "flashsvd_decode_pack_bytes": ([_p, C.POINTER(C.c_size_t)], _i),
    "flashsvd_decode_pack": ([_p, _p, C.c_size_t, _p], _i),
    "flashsvd_decode_plan_create": ([_p, _i, _p, _p, _i, _i, _p], _i),
    "flashsvd_decode_plan_forward": ([_p, _p, _p, _p], _i),
    "flashsvd_decode_plan_destroy": ([_p], _i),
    "flashsvd_profile_enable": ([_i], _i),
    "flashsvd_profile_report": ([C.c_char_p, _i, _i], _i),
    "flashsvd_lowrank_linear": ([_p, _p, _p, _p, _p, _i, _i, _i, _i, _p], _i),
    "flashsvd_lowrank_linear_noalloc": ([_p, _p, _p, _p, _p, _i, _i, _i, _i, _p], _i),
    "flashsvd_dense_linear_f32": ([_p, _p, _p, _i, _i, _i, _p], _i),
    "flashsvd_head_logits": ([_p, _p, _f, _p, _p, _i, _i, _i, _p], _i),
    "flashsvd_packed_gateup_mlp": ([_p, _p, _p, _p, _p, _p, _i, _i, _i, _i, _i, _p], _i),
    "flashsvd_gateup_swiglu": ([_p, _p, _p, _p, _i, _i, _i, _i, _p], _i),
    "flashsvd_lowrank_ffn": ([_p, _p, _p, _p, _p, _p, _p, _p, _p, _i, _i, _i, _i, _i, _p], _i),
    "flashsvd_dense_kv_decode_attn": ([_p, _p, _p, _p, _p, _p, _p, _i, _i, _i, _i, _f, _p], _i),
    "flashsvd_prefill_attn": ([_p, _p, _p, _p, _i, _i, _i, _i, _i, _i, _f, _p], _i),
    "flashsvd_prefill_attn_factorized": ([_p, _p, _p, _p, _p, _p, _p, _i, _i, _i, _i, _i, _i, _i,
                                          _f, _p], _i),
    "flashsvd_rmsnorm": ([_p, _p, _p, _i, _i, _f, _p], _i),
    "flashsvd_layernorm": ([_p, _p, _p, _p, _i, _i, _f, _p], _i),
    "flashsvd_rope_table": ([_p, _p, _i, _i, _f, _p], _i),
    "flashsvd_embed": ([_p, _p, _p, _i, _i, _i, _p], _i),
    "flashsvd_greedy": ([_p, _p, _i, _i, _p], _i),
    "flashsvd_advance_seqlens": ([_p, _i, _p], _i),
    "flashsvd_layer_forward": ([C.POINTER(Layer), _p, _p, _p, _p, _i, _i, _i, _i, _p], _i),
    "flashsvd_decode_graph_capture": ([C.POINTER(Layer), _p, _p, _p, _p, _i, _i, _p,
                                       C.POINTER(_p)], _i),
    "flashsvd_capture_begin": ([_p], _i),
    "flashsvd_capture_end": ([_p, C.POINTER(_p)], _i),
    "flashsvd_graph_compose": ([C.POINTER(_p), _i, C.POINTER(_p)], _i),
    "flashsvd_graph_replay": ([_p, _p], _i),
    "flashsvd_graph_kernel_count": ([_p], _i),
    "flashsvd_graph_destroy": ([_p], _i),
}

for _name, (_args, _ret) in _SIGS.items():
    _fn = getattr(lib, _name)  # AttributeError here means the build is stale
    _fn.argtypes = _args
    _fn.restype = _ret

EXPORTED = tuple(_SIGS)


def check(fn_name: str, status: int) -> None:
    if status != OK:
        raise FlashSVDError(fn_name, status)


def ptr(t) -> int | None:
    """Device pointer of a tensor (None passes NULL)."""
    return None if t is None else t.data_ptr()


def stream_handle(stream=None) -> int | None:
    """cudaStream_t of a torch stream (default: torch's current stream)."""
    import torch
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


def _call(name, *args):
    check(name, getattr(lib, name)(*args))


# ---------------------------------------------------------------- setup --

def init(device: int = 0, max_tokens: int = 8192, max_rank: int = 4096,
         max_hidden: int = 4096, max_ffn: int = 11008) -> None:
    _call("flashsvd_init", device, max_tokens, max_rank, max_hidden, max_ffn)


def shutdown() -> None:
    _call("flashsvd_shutdown")


class Context:
    """A workspace of its own (flashsvd_ctx_create).  ``with ctx:`` binds it
    to the calling thread for the block (flashsvd_ctx_bind) and restores the
    default context afterwards."""

    def __init__(self, device: int = 0, max_tokens: int = 8192, max_rank: int = 4096,
                 max_hidden: int = 4096, max_ffn: int = 11008):
        h = _p()
        _call("flashsvd_ctx_create", device, max_tokens, max_rank, max_hidden, max_ffn,
              C.byref(h))
        self.handle = h.value

    def bind(self) -> None:
        _call("flashsvd_ctx_bind", self.handle)

    @staticmethod
    def unbind() -> None:
        _call("flashsvd_ctx_bind", None)

    def __enter__(self):
        self.bind()
        return self

    def __exit__(self, *exc):
        self.unbind()
        return False

    def destroy(self) -> None:
        if self.handle:
            _call("flashsvd_ctx_destroy", self.handle)
            self.handle = None


def check_device_status(stream=None) -> None:
    _call("flashsvd_check_device_status", stream_handle(stream))


def set_prefill_attention(mode: int) -> None:
    """1: query formed inside the attention kernel; 0: dense q projection
    (the default)."""
    _call("flashsvd_set_prefill_attention", mode)


def set_l2_discard(on: bool) -> None:
    _call("flashsvd_set_l2_discard", int(on))


def set_decode_path(fused: bool) -> None:
    _call("flashsvd_set_decode_path", int(fused))


def decode_pack_bytes(L: "Layer") -> int:
    n = C.c_size_t(0)
    _call("flashsvd_decode_pack_bytes", C.byref(L), C.byref(n))
    return int(n.value)


def decode_pack(L: "Layer", dst, stream=None) -> None:
    """Write L's decode pack into the device buffer dst (a torch tensor of
    at least decode_pack_bytes(L) bytes) and point L.decode_pack at it."""
    nbytes = dst.numel() * dst.element_size()
    _call("flashsvd_decode_pack", C.byref(L), ptr(dst), nbytes, stream_handle(stream))
    L.decode_pack = ptr(dst)


def launch_count() -> int:
    return int(lib.flashsvd_launch_count())


def profile_enable(on: bool = True) -> None:
    _call("flashsvd_profile_enable", int(on))


def profile_report(reset: bool = True) -> dict:
    """{name: dict(launches, ms, bytes, flops)} of eager launches since the
    last reset (synchronises the device)."""
    n = lib.flashsvd_profile_report(None, 0, 0)
    buf = C.create_string_buffer(max(n, 1) + 64)
    _call("flashsvd_profile_report", buf, len(buf), int(reset))
    out = {}
    for line in buf.value.decode().splitlines():
        name, cnt, ms, by, fl = line.split()
        out[name] = dict(launches=int(cnt), ms=float(ms), bytes=float(by), flops=float(fl))
    return out


# -------------------------------------------------------------- compute --

def lowrank_linear(x, U, V, bias, y, M, d, r, n, stream=None):
    _call("flashsvd_lowrank_linear", ptr(x), ptr(U), ptr(V), ptr(bias), ptr(y),
          M, d, r, n, stream_handle(stream))


def lowrank_linear_noalloc(x, U, V, bias, y, M, d, r, n, stream=None):
    """Decode-size factorized linear that allocates nothing (fixed device
    scratch; see include/flashsvd.h for its limits)."""
    _call("flashsvd_lowrank_linear_noalloc", ptr(x), ptr(U), ptr(V), ptr(bias), ptr(y),
          M, d, r, n, stream_handle(stream))


def dense_linear_f32(x, W, y, M, d, n, stream=None):
    _call("flashsvd_dense_linear_f32", ptr(x), ptr(W), ptr(y), M, d, n,
          stream_handle(stream))


def packed_gateup_mlp(x, U_gu, V_gu, U_dn, V_dn, y, M, d, r_f, f, r_dn, stream=None):
    _call("flashsvd_packed_gateup_mlp", ptr(x), ptr(U_gu), ptr(V_gu), ptr(U_dn),
          ptr(V_dn), ptr(y), M, d, r_f, f, r_dn, stream_handle(stream))


def gateup_swiglu(x, U_gu, V_gu, h, M, d, r_f, f, stream=None):
    _call("flashsvd_gateup_swiglu", ptr(x), ptr(U_gu), ptr(V_gu), ptr(h), M, d,
          r_f, f, stream_handle(stream))


def lowrank_ffn(x, U_up, V_up, b_up, U_dn, V_dn, b_dn, resid, y, M, d, r_up, f, r_dn,
                stream=None):
    _call("flashsvd_lowrank_ffn", ptr(x), ptr(U_up), ptr(V_up), ptr(b_up), ptr(U_dn), ptr(V_dn),
          ptr(b_dn), ptr(resid), ptr(y), M, d, r_up, f, r_dn, stream_handle(stream))


def dense_kv_decode_attn(q, k_new, v_new, k_cache, v_cache, cache_seqlens, out,
                         B, H, D, S_max, scale, stream=None):
    _call("flashsvd_dense_kv_decode_attn", ptr(q), ptr(k_new), ptr(v_new),
          ptr(k_cache), ptr(v_cache), ptr(cache_seqlens), ptr(out), B, H, D,
          S_max, scale, stream_handle(stream))


HEAD_MAX_ROWS = 32  # flashsvd_head_logits takes 1..32 rows


def head_logits(x, g, eps, W, logits, M, d, n, stream=None):
    _call("flashsvd_head_logits", ptr(x), ptr(g), eps, ptr(W), ptr(logits), M, d, n,
          stream_handle(stream))


def prefill_attn(q, k_cache, v_cache, out, B, S, H, D, S_max, causal, scale,
                 stream=None):
    _call("flashsvd_prefill_attn", ptr(q), ptr(k_cache), ptr(v_cache), ptr(out),
          B, S, H, D, S_max, int(causal), scale, stream_handle(stream))


def prefill_attn_factorized(z_q, V_q, rope_cos, rope_sin, k_cache, v_cache, out, B, S, H, D,
                            S_max, r, causal, scale, stream=None):
    _call("flashsvd_prefill_attn_factorized", ptr(z_q), ptr(V_q), ptr(rope_cos), ptr(rope_sin),
          ptr(k_cache), ptr(v_cache), ptr(out), B, S, H, D, S_max, r, int(causal), scale,
          stream_handle(stream))


def rmsnorm(x, g, y, M, d, eps, stream=None):
    _call("flashsvd_rmsnorm", ptr(x), ptr(g), ptr(y), M, d, eps, stream_handle(stream))


def layernorm(x, g, b, y, M, d, eps, stream=None):
    _call("flashsvd_layernorm", ptr(x), ptr(g), ptr(b), ptr(y), M, d, eps,
          stream_handle(stream))


def rope_table(cos_tab, sin_tab, S_max, D, base=10000.0, stream=None):
    _call("flashsvd_rope_table", ptr(cos_tab), ptr(sin_tab), S_max, D, base,
          stream_handle(stream))


def embed(tokens, emb, x, B, d, vocab, stream=None):
    _call("flashsvd_embed", ptr(tokens), ptr(emb), ptr(x), B, d, vocab,
          stream_handle(stream))


def greedy(logits, next_tokens, M, vocab, stream=None):
    _call("flashsvd_greedy", ptr(logits), ptr(next_tokens), M, vocab,
          stream_handle(stream))


def advance_seqlens(cache_seqlens, B, stream=None):
    _call("flashsvd_advance_seqlens", ptr(cache_seqlens), B, stream_handle(stream))


def layer_forward(layer: Layer, x, k_cache, v_cache, cache_seqlens, B, S, S_max,
                  mode, stream=None):
    _call("flashsvd_layer_forward", C.byref(layer), ptr(x), ptr(k_cache),
          ptr(v_cache), ptr(cache_seqlens), B, S, S_max, mode, stream_handle(stream))


# --------------------------------------------------------------- graphs --

class Graph:
    """Owner of a flashsvd_graph handle."""

    def __init__(self, handle: int):
        self.handle = handle

    @property
    def kernels(self) -> int:
        return int(lib.flashsvd_graph_kernel_count(self.handle))

    def replay(self, stream=None) -> None:
        _call("flashsvd_graph_replay", self.handle, stream_handle(stream))

    def destroy(self) -> None:
        if self.handle:
            _call("flashsvd_graph_destroy", self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.destroy()
        except Exception:
            pass


class DecodePlan:
    """Owner of a flashsvd_decode_plan: the decode step of several decoder
    layers (each with a decode pack) as one launch."""

    def __init__(self, layers, k_caches, v_caches, B: int, S_max: int):
        n = len(layers)
        arr = (Layer * n)(*layers)
        kc = (C.c_void_p * n)(*[ptr(t) for t in k_caches])
        vc = (C.c_void_p * n)(*[ptr(t) for t in v_caches])
        h = _p()
        _call("flashsvd_decode_plan_create", arr, n, kc, vc, B, S_max, C.byref(h))
        self.handle = h.value
        self._keep = (arr, kc, vc)

    def forward(self, x, cache_seqlens, stream=None) -> None:
        _call("flashsvd_decode_plan_forward", self.handle, ptr(x), ptr(cache_seqlens),
              stream_handle(stream))

    def destroy(self) -> None:
        if self.handle:
            _call("flashsvd_decode_plan_destroy", self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.destroy()
        except Exception:
            pass


def decode_graph_capture(layer: Layer, x, k_cache, v_cache, cache_seqlens, B,
                         S_max, stream) -> Graph:
    h = _p()
    _call("flashsvd_decode_graph_capture", C.byref(layer), ptr(x), ptr(k_cache),
          ptr(v_cache), ptr(cache_seqlens), B, S_max, stream_handle(stream), C.byref(h))
    return Graph(h.value)


def capture_begin(stream) -> None:
    _call("flashsvd_capture_begin", stream_handle(stream))


def capture_end(stream) -> Graph:
    h = _p()
    _call("flashsvd_capture_end", stream_handle(stream), C.byref(h))
    return Graph(h.value)


def graph_compose(parts) -> Graph:
    arr = (_p * len(parts))(*[g.handle for g in parts])
    h = _p()
    _call("flashsvd_graph_compose", arr, len(parts), C.byref(h))
    return Graph(h.value)
