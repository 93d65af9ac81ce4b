"""Whole-model drivers over libflashsvd.

PyTorch is used here only to own device memory and streams; every step of
the forward pass is a libflashsvd call.

``DecoderModel``: Llama-shaped pre-norm decoder whose seven per-layer
projections are rank-r factor pairs (q, k, v, o, packed gate|up, down), a
dense LM head and a contiguous bf16 KV cache per layer.  Each layer's
factors are also kept as a decode pack, and the decoder layers of a decode
step run as one fused launch (a decode plan); the step (embedding, layers,
head) is captured and replayed as a CUDA graph (FlashSVD v1.5 explainer,
Technical Summary, Methodology 4), with positions held in device memory.
Without packs, decode replays one graph per layer over the per-stage
kernels.

``EncoderModel``: BERT-shaped post-LN encoder with every linear factorized.
"""
from __future__ import annotations

import dataclasses
import math

import torch

from . import flashsvd as fs
from . import synth


@dataclasses.dataclass
class DecoderConfig:
    layers: int = 32
    d: int = 4096
    H: int = 32
    D: int = 128
    f: int = 11008
    vocab: int = 32000
    rho: tuple = (0.6,)          # per-layer retention ratios (one entry = all layers)
    eps: float = 1e-5
    rope_base: float = 10000.0

    def ranks(self, layer: int):
        rho = self.rho[layer % len(self.rho)] if len(self.rho) > 1 else self.rho[0]
        r_a = synth.rank_for_ratio(rho, self.d, self.d)
        r_f = synth.rank_for_ratio(rho, self.d, self.f)
        return r_a, r_f

    def layer_params(self, layer: int) -> int:
        """Factor parameters of one layer: q, k, v, o at rank r_a
        (r_a * 2d each), the packed gate|up pair U_gu [d x 2 r_f] and V_gu
        [2 r_f x f], and the down pair U_dn [f x r_f], V_dn [r_f x d]."""
        r_a, r_f = self.ranks(layer)
        return 4 * r_a * 2 * self.d + 2 * r_f * (self.d + self.f) + r_f * (self.f + self.d)


LLAMA7B = DecoderConfig()


def _bf16_normal(shape, std, gen, device):
    t = torch.randn(shape, generator=gen, device=device, dtype=torch.float32)
    return t.mul_(std).to(torch.bfloat16)


class DecoderModel:
    def __init__(self, cfg: DecoderConfig, B: int, S_max: int, seed: int = 0,
                 device: str = "cuda", weights=None, head=None, decode_pack: bool = True):
        """``weights``: optional list of per-layer dicts of device bf16
        tensors (U_q, V_q, ..., U_gu, V_gu, U_dn, V_dn, g1, g2); ``head``:
        optional dict with the device tensors emb [vocab x d], g_final [d]
        and W_lm [d x vocab].  Whatever is not given is random-initialised
        from ``seed``."""
        self.cfg, self.B, self.S_max, self.device = cfg, B, S_max, device
        gen = torch.Generator(device=device)
        gen.manual_seed(seed)
        d, f = cfg.d, cfg.f
        self.layers = []
        for i in range(cfg.layers):
            if weights is not None:
                w = weights[i]
            else:
                r_a, r_f = cfg.ranks(i)
                w = {}
                for n in ("q", "k", "v", "o"):
                    w["U_" + n] = _bf16_normal((d, r_a), d ** -0.5, gen, device)
                    w["V_" + n] = _bf16_normal((r_a, d), r_a ** -0.5, gen, device)
                w["U_gu"] = _bf16_normal((d, 2 * r_f), d ** -0.5, gen, device)
                w["V_gu"] = _bf16_normal((2 * r_f, f), r_f ** -0.5, gen, device)
                w["U_dn"] = _bf16_normal((f, r_f), f ** -0.5, gen, device)
                w["V_dn"] = _bf16_normal((r_f, d), r_f ** -0.5, gen, device)
                w["g1"] = torch.ones(d, dtype=torch.bfloat16, device=device)
                w["g2"] = torch.ones(d, dtype=torch.bfloat16, device=device)
            self.layers.append(w)
        if head is not None:
            self.emb, self.g_final, self.W_lm = head["emb"], head["g_final"], head["W_lm"]
        else:
            self.emb = _bf16_normal((cfg.vocab, d), 1.0, gen, device)
            self.g_final = torch.ones(d, dtype=torch.bfloat16, device=device)
            self.W_lm = _bf16_normal((d, cfg.vocab), d ** -0.5, gen, device)
        self.rope_cos = torch.empty((S_max, cfg.D // 2), dtype=torch.float32, device=device)
        self.rope_sin = torch.empty_like(self.rope_cos)
        fs.rope_table(self.rope_cos, self.rope_sin, S_max, cfg.D, cfg.rope_base)
        self.k_cache = [torch.zeros((B, S_max, cfg.H, cfg.D), dtype=torch.bfloat16, device=device)
                        for _ in range(cfg.layers)]
        self.v_cache = [torch.zeros_like(k) for k in self.k_cache]
        self.seqlens = torch.zeros(B, dtype=torch.int32, device=device)
        self.x = torch.zeros((B, d), dtype=torch.bfloat16, device=device)
        self.xn = torch.zeros((B, d), dtype=torch.bfloat16, device=device)
        self.tokens = torch.zeros(B, dtype=torch.int32, device=device)
        self.logits = torch.zeros((B, cfg.vocab), dtype=torch.float32, device=device)
        self.structs = [self._struct(w) for w in self.layers]
        # Decode packs: each layer's factors re-tiled for the fused decode
        # kernel (layers whose shapes it does not cover keep the per-stage
        # decode path).
        self.packs = []
        if decode_pack:
            for L in self.structs:
                try:
                    buf = torch.empty(fs.decode_pack_bytes(L), dtype=torch.uint8, device=device)
                    fs.decode_pack(L, buf)
                except fs.FlashSVDError:
                    L.decode_pack = None  # shapes the fused kernel does not cover
                    buf = None
                self.packs.append(buf)
        # With a pack on every layer, the decode step of all layers runs as
        # one launch of the fused kernel (a decode plan).
        self.plan = None
        if decode_pack and all(pk is not None for pk in self.packs):
            try:
                self.plan = fs.DecodePlan(self.structs, self.k_cache, self.v_cache, B, S_max)
            except fs.FlashSVDError:
                self.plan = None
        self.graphs = None
        self.step_graph = None

    # ------------------------------------------------------------ setup --
    def _struct(self, w) -> fs.Layer:
        cfg = self.cfg
        L = fs.Layer()
        L.kind = fs.DECODER
        L.d, L.H, L.D, L.f = cfg.d, cfg.H, cfg.D, cfg.f
        L.norm_eps = cfg.eps
        L.norm1_g, L.norm2_g = w["g1"].data_ptr(), w["g2"].data_ptr()
        for n in ("q", "k", "v", "o"):
            F = getattr(L, n)
            F.U, F.V, F.bias, F.r = w["U_" + n].data_ptr(), w["V_" + n].data_ptr(), None, \
                w["U_" + n].shape[1]
        L.U_gu, L.V_gu, L.r_f = w["U_gu"].data_ptr(), w["V_gu"].data_ptr(), w["U_gu"].shape[1] // 2
        L.down.U, L.down.V, L.down.bias, L.down.r = w["U_dn"].data_ptr(), w["V_dn"].data_ptr(), \
            None, w["U_dn"].shape[1]
        L.rope_cos, L.rope_sin = self.rope_cos.data_ptr(), self.rope_sin.data_ptr()
        return L

    def _unique_params(self) -> int:
        """Elements of the layers' weights, a tensor shared by several
        layers (shared bases) counted once."""
        seen, n = set(), 0
        for w in self.layers:
            for t in w.values():
                if t.data_ptr() not in seen:
                    seen.add(t.data_ptr())
                    n += t.numel()
        return n

    def weight_bytes(self) -> int:
        return 2 * (self._unique_params() + self.W_lm.numel())

    # ---------------------------------------------------------- prefill --
    def prefill(self, prompt, stream=None):
        """prompt: device int32 [B, S].  Runs every layer over the whole
        prompt (writing cache rows [0, S)), then the head on the last
        position; sets cache_seqlens = S and the next tokens."""
        B, S = prompt.shape
        cfg = self.cfg
        x = torch.empty((B * S, cfg.d), dtype=torch.bfloat16, device=self.device)
        fs.embed(prompt.reshape(-1), self.emb, x, B * S, cfg.d, cfg.vocab, stream)
        for i in range(cfg.layers):
            fs.layer_forward(self.structs[i], x, self.k_cache[i], self.v_cache[i], None, B, S,
                             self.S_max, fs.PREFILL_CAUSAL, stream)
        last = x.view(B, S, cfg.d)[:, S - 1]
        for b in range(B):
            fs.rmsnorm(last[b], self.g_final, self.xn[b], 1, cfg.d, cfg.eps, stream)
        if B <= fs.HEAD_MAX_ROWS:
            fs.head_logits(self.xn, None, 0.0, self.W_lm, self.logits, B, cfg.d, cfg.vocab, stream)
        else:
            fs.dense_linear_f32(self.xn, self.W_lm, self.logits, B, cfg.d, cfg.vocab, stream)
        fs.greedy(self.logits, self.tokens, B, cfg.vocab, stream)
        self.seqlens.fill_(S)
        return x

    # ----------------------------------------------------------- decode --
    def _head(self, stream):
        cfg = self.cfg
        if self.B <= fs.HEAD_MAX_ROWS:
            # final RMSNorm folded into the head GEMV
            fs.head_logits(self.x, self.g_final, cfg.eps, self.W_lm, self.logits, self.B, cfg.d,
                           cfg.vocab, stream)
        else:
            fs.rmsnorm(self.x, self.g_final, self.xn, self.B, cfg.d, cfg.eps, stream)
            fs.dense_linear_f32(self.xn, self.W_lm, self.logits, self.B, cfg.d, cfg.vocab, stream)
        fs.greedy(self.logits, self.tokens, self.B, cfg.vocab, stream)
        fs.advance_seqlens(self.seqlens, self.B, stream)

    def _layers_decode(self, stream):
        if self.plan is not None:
            self.plan.forward(self.x, self.seqlens, stream)
            return
        for i in range(self.cfg.layers):
            fs.layer_forward(self.structs[i], self.x, self.k_cache[i], self.v_cache[i],
                             self.seqlens, self.B, 1, self.S_max, fs.DECODE, stream)

    def decode_step_eager(self, stream=None):
        cfg = self.cfg
        fs.embed(self.tokens, self.emb, self.x, self.B, cfg.d, cfg.vocab, stream)
        self._layers_decode(stream)
        self._head(stream)

    def capture(self, stream, compose: bool = True):
        """Capture one graph per layer (plus the embedding and the head) and,
        with ``compose``, one graph for the whole step built from them."""
        cfg = self.cfg
        if self.plan is not None:
            # all layers are one launch: the step is one graph
            with torch.cuda.stream(stream):
                fs.capture_begin(stream)
                fs.embed(self.tokens, self.emb, self.x, self.B, cfg.d, cfg.vocab, stream)
                self.plan.forward(self.x, self.seqlens, stream)
                self._head(stream)
                g = fs.capture_end(stream)
            self.graphs = [g]
            self.step_graph = g
            return
        with torch.cuda.stream(stream):
            fs.capture_begin(stream)
            fs.embed(self.tokens, self.emb, self.x, self.B, cfg.d, cfg.vocab, stream)
            g_embed = fs.capture_end(stream)
            layers = [fs.decode_graph_capture(self.structs[i], self.x, self.k_cache[i],
                                              self.v_cache[i], self.seqlens, self.B,
                                              self.S_max, stream)
                      for i in range(cfg.layers)]
            fs.capture_begin(stream)
            self._head(stream)
            g_head = fs.capture_end(stream)
        self.graphs = [g_embed] + layers + [g_head]
        self.step_graph = fs.graph_compose(self.graphs) if compose else None

    def decode_step(self, stream=None):
        if self.step_graph is not None:
            self.step_graph.replay(stream)
        else:
            for g in self.graphs:
                g.replay(stream)

    def step_kernels(self) -> int:
        return sum(g.kernels for g in self.graphs)

    def release_graphs(self):
        for g in (self.graphs or []):
            g.destroy()
        if self.step_graph is not None:
            self.step_graph.destroy()
        self.graphs, self.step_graph = None, None

    # ---------------------------------------------------------- bytes ---
    def decode_step_bytes(self, context: int) -> int:
        """Algorithmic HBM bytes of one decode step at cache length
        ``context`` (before the step): every factor and the LM head once,
        the K/V history of every layer once, the new K/V rows, and the
        activations in and out (negligible)."""
        cfg = self.cfg
        kv = 2 * cfg.layers * (context + 1) * cfg.d * 2 * self.B
        act = self.B * cfg.d * 2 * 2 * cfg.layers
        return self.weight_bytes() + kv + act

    def layers_decode_bytes(self, context: int) -> int:
        """Algorithmic HBM bytes of the decoder layers of one decode step
        (the work of one decode-plan launch): every layer's factors and norm
        gains once, its K/V history at cache length ``context`` plus the new
        rows, and the activations in and out."""
        cfg = self.cfg
        n = self._unique_params()
        kv = 2 * cfg.layers * (context + 1) * cfg.d * 2 * self.B
        act = self.B * cfg.d * 2 * 2 * cfg.layers
        return 2 * n + kv + act

    def prefill_flops(self, S: int) -> float:
        """Algorithmic FLOPs of one prefill of B prompts of S tokens: every
        factorized linear over B*S rows (2 flops per multiply-add of both
        factors), causal attention (q.k and p.v over the S(S+1)/2 visible
        pairs of every head), and the head on the last position of each
        prompt."""
        cfg = self.cfg
        lin = 2.0 * self.B * S * sum(cfg.layer_params(i) for i in range(cfg.layers))
        attn = cfg.layers * 4.0 * self.B * cfg.H * cfg.D * S * (S + 1) / 2
        head = 2.0 * self.B * cfg.d * cfg.vocab
        return lin + attn + head

    # --------------------------------------------------------- generate --
    def generate(self, prompt_host, steps: int, stream=None):
        """End-to-end public call: host int32 prompt [B, S] (pinned or not)
        -> host int32 tokens [B, steps].  Copies the prompt in, prefills,
        decodes ``steps`` greedy tokens with the captured graphs and copies
        the generated tokens out."""
        B, S = prompt_host.shape
        prompt = prompt_host.to(self.device, non_blocking=True)
        gen = torch.empty((steps, B), dtype=torch.int32, device=self.device)
        self.prefill(prompt, stream)
        for t in range(steps):
            gen[t].copy_(self.tokens, non_blocking=True)
            self.decode_step(stream)
        out = torch.empty((B, steps), dtype=torch.int32, pin_memory=True)
        out.copy_(gen.t(), non_blocking=True)
        return out


class EncoderModel:
    """BERT-shaped post-LN encoder, every linear factorized at rank r with a
    bias."""

    def __init__(self, layers=12, d=768, H=12, f=3072, r=192, B=32, S=512, seed=0,
                 device="cuda", eps=1e-12, weights=None):
        self.d, self.H, self.D, self.f, self.r = d, H, d // H, f, r
        self.B, self.S, self.eps, self.device = B, S, eps, device
        gen = torch.Generator(device=device)
        gen.manual_seed(seed)
        self.layers = []
        shapes = {"q": (d, d), "k": (d, d), "v": (d, d), "o": (d, d), "up": (d, f), "dn": (f, d)}
        for i in range(layers):
            if weights is not None:
                w = weights[i]
            else:
                w = {}
                for n, (di, do) in shapes.items():
                    w["U_" + n] = _bf16_normal((di, r), di ** -0.5, gen, device)
                    w["V_" + n] = _bf16_normal((r, do), r ** -0.5, gen, device)
                    w["b_" + n] = torch.zeros(do, dtype=torch.bfloat16, device=device)
                for n in ("ln1", "ln2"):
                    w[n + "_g"] = torch.ones(d, dtype=torch.bfloat16, device=device)
                    w[n + "_b"] = torch.zeros(d, dtype=torch.bfloat16, device=device)
            self.layers.append(w)
        self.structs = [self._struct(w) for w in self.layers]
        self.k_buf = torch.empty((B, S, H, d // H), dtype=torch.bfloat16, device=device)
        self.v_buf = torch.empty_like(self.k_buf)

    def _struct(self, w) -> fs.Layer:
        L = fs.Layer()
        L.kind = fs.ENCODER
        L.d, L.H, L.D, L.f = self.d, self.H, self.D, self.f
        L.norm_eps = self.eps
        L.norm1_g, L.norm1_b = w["ln1_g"].data_ptr(), w["ln1_b"].data_ptr()
        L.norm2_g, L.norm2_b = w["ln2_g"].data_ptr(), w["ln2_b"].data_ptr()
        for n, field in (("q", "q"), ("k", "k"), ("v", "v"), ("o", "o"), ("up", "up"), ("dn", "down")):
            F = getattr(L, field)
            F.U, F.V, F.bias, F.r = w["U_" + n].data_ptr(), w["V_" + n].data_ptr(), \
                w["b_" + n].data_ptr(), w["U_" + n].shape[1]
        return L

    def forward(self, x, stream=None):
        """x: [B*S, d] bf16 on the device, updated in place."""
        for L in self.structs:
            fs.layer_forward(L, x, self.k_buf, self.v_buf, None, self.B, self.S, self.S,
                             fs.ENCODER_BIDIR, stream)
        return x

    def flops(self) -> float:
        M = self.B * self.S
        per_layer = 2 * M * self.r * (4 * 2 * self.d + 2 * (self.d + self.f))
        attn = 4 * self.B * self.H * self.S * self.S * self.D
        return len(self.layers) * (per_layer + attn)


def attention_scale(D: int) -> float:
    return 1.0 / math.sqrt(D)
