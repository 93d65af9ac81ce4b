"""Per-stage timeline of the fused decode kernel (trace build only).

    python -m rank_transformer_b200.build --trace
    FLASHSVD_LIBRARY=$PWD/rank_transformer_b200/libflashsvd_trace.so \\
        python -m rank_transformer_b200.decode_timeline [--batch B] [--layers L] [--context C]

Builds the Llama-2-7B-shaped decoder (random factors at rank ratio 0.6, every
layer in one decode plan), fills the K/V cache to `context` positions, runs
three decode steps, clears the trace, runs ONE more step and reads the
timeline the trace build records: per (layer, stage, CTA) four
%globaltimer stamps -- stage entry, previous stage complete on every CTA
(grid barrier passed), stage input built, stage body done.  It prints, per
stage, medians over CTAs and layers (the first layer excluded):

    wait     entry -> barrier passed (waiting for the slowest CTA of the
             previous stage, and the barrier's own latency)
    build    barrier passed -> input built (reading and summing the
             previous stage's partials, its epilogue)
    body     input built -> done (the stage's share of the factor or K/V
             stream and its multiply-accumulate)
    spread   last CTA done - first CTA done
    handoff  last CTA done -> median CTA past the next stage's barrier

The product library contains none of the trace code; this tool refuses to
run against it.
"""
from __future__ import annotations

import argparse
import ctypes as C
import dataclasses
import json
import os
import sys

import numpy as np

STAGES = ["qkv.U", "qkv.V", "attn", "o.U", "o.V", "gu.U", "gu.V", "dn.U", "dn.V"]


def main(argv=None) -> int:
    ap = argparse.ArgumentParser()
    ap.add_argument("--batch", type=int, default=1)
    ap.add_argument("--layers", type=int, default=32)
    ap.add_argument("--context", type=int, default=2048)
    ap.add_argument("--json", action="store_true", help="print one JSON line instead of the table")
    a = ap.parse_args(argv)
    if "trace" not in os.environ.get("FLASHSVD_LIBRARY", ""):
        print("point FLASHSVD_LIBRARY at libflashsvd_trace.so (python -m rank_transformer_b200.build --trace)",
              file=sys.stderr)
        return 2
    import torch
    from rank_transformer_b200 import flashsvd as fs
    from rank_transformer_b200.model import LLAMA7B, DecoderModel

    B, NL = a.batch, a.layers
    cfg = dataclasses.replace(LLAMA7B, layers=NL)
    fs.init(0, max_tokens=256, max_rank=2368, max_hidden=cfg.d, max_ffn=cfg.f)
    m = DecoderModel(cfg, B, a.context + 128, seed=1)
    if m.plan is None:
        print("the model did not build a decode plan", file=sys.stderr)
        return 1
    gen = torch.Generator(device="cuda")
    gen.manual_seed(0)
    for t in m.k_cache + m.v_cache:
        t.normal_(generator=gen)
    s = torch.cuda.Stream()
    m.seqlens.fill_(a.context)
    with torch.cuda.stream(s):
        for _ in range(3):
            m.decode_step_eager(s)
        s.synchronize()
        if fs.lib.flashsvd_trace_clear() != 0:
            raise RuntimeError("flashsvd_trace_clear failed")
        m.decode_step_eager(s)
        s.synchronize()
    fs.check_device_status(s)
    fs.lib.flashsvd_trace_read.argtypes = [C.c_void_p, C.c_size_t]
    buf = np.zeros((64, 9, 148, 2, 4), dtype=np.uint64)
    if fs.lib.flashsvd_trace_read(buf.ctypes.data, buf.nbytes) != 0:
        raise RuntimeError("flashsvd_trace_read failed")
    G = min(148, torch.cuda.get_device_properties(0).multi_processor_count)
    NLt = min(NL, 64)
    ns = buf[:NLt, :, :G, 0, :].astype(np.int64)   # [L, 9, G, 4]
    ns = ns - ns[ns > 0].min()
    span = ns[ns > 0].max() / 1e3
    Ls = slice(1, NLt) if NLt > 1 else slice(0, 1)
    rows = []
    for ph in range(9):
        x = ns[Ls, ph]
        wait = float(np.median(x[..., 1] - x[..., 0])) / 1e3
        build = float(np.median(x[..., 2] - x[..., 1])) / 1e3
        body = float(np.median(x[..., 3] - x[..., 2])) / 1e3
        spread = float(np.median(x[..., 3].max(axis=1) - x[..., 3].min(axis=1))) / 1e3
        nxt = ns[Ls, ph + 1, :, 1] if ph < 8 else (ns[1:NLt, 0, :, 1] if NLt > 1 else None)
        ho = float("nan")
        if nxt is not None and nxt.size:
            last_done = x[..., 3].max(axis=1)[: nxt.shape[0]]
            ho = float(np.median(np.median(nxt, axis=1) - last_done)) / 1e3
        rows.append({"stage": STAGES[ph], "wait_us": wait, "build_us": build, "body_us": body,
                     "done_spread_us": spread, "handoff_us": ho})
    if a.json:
        print(json.dumps({"batch": B, "layers": NL, "context": a.context, "ctas": G,
                          "step_us": span, "layer_us": span / NL, "stages": rows}))
        return 0
    print(f"B={B} layers={NL} context={a.context} CTAs={G}: step {span:.1f} us ({span / NL:.2f} us per layer)")
    print("stage     wait    build     body   spread  handoff   (us; medians over CTAs and layers 2..)")
    for r in rows:
        print(f"{r['stage']:7s} {r['wait_us']:7.2f} {r['build_us']:8.2f} {r['body_us']:8.2f} "
              f"{r['done_spread_us']:8.2f} {r['handoff_us']:8.2f}")
    tot = {k: sum(r[k] for r in rows) for k in ("wait_us", "build_us", "body_us")}
    print(f"sum     {tot['wait_us']:7.2f} {tot['build_us']:8.2f} {tot['body_us']:8.2f}")
    return 0


if __name__ == "__main__":
    sys.exit(main())
