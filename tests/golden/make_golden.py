"""Writes tiny_layer_seed0.json: oracle outputs for the tiny decoder layer.

The case is the small single-layer configuration (hidden 256, 4 heads of dim
64, SwiGLU 688, every linear at rank 64, one sequence of 128 tokens, then two
decode steps), drawn from the seeded input generator.  Only the oracle and
the generator are called here; nothing comes from the CUDA path.  The stored
values are a regression pin on the oracle itself.

Run:  python -m tests.golden.make_golden
"""
import json
import os

import numpy as np

from oracle import flashsvd_oracle as oracle
from rank_transformer_b200 import synth

D_MODEL, HEADS, FFN, RANK, SEQ = 256, 4, 688, 64, 128


def tiny_layer_case(seed=0):
    rng = synth.rng_for(seed)
    w = synth.decoder_layer_weights(rng, D_MODEL, FFN, RANK, RANK)
    x = synth.normal_bf16(rng, (SEQ, D_MODEL))
    x_dec = synth.normal_bf16(rng, (2, D_MODEL))
    wf = oracle.widen_layer(w)
    y, k, v = oracle.decoder_layer_prefill(oracle.from_bf16(x), wf, HEADS)
    kh, vh = k[None], v[None]
    dec = []
    for t in range(2):
        yt, kt, vt = oracle.decoder_layer_decode(
            oracle.from_bf16(x_dec[t:t + 1]), wf, HEADS, kh, vh, [SEQ + t])
        kh = np.concatenate([kh, kt[:, None]], axis=1)
        vh = np.concatenate([vh, vt[:, None]], axis=1)
        dec.append(yt[0])
    return {
        "prefill_row0_head": y[0, :8].tolist(),
        "prefill_row127_tail": y[SEQ - 1, -8:].tolist(),
        "prefill_row_sums": y.sum(axis=1)[::16].tolist(),
        "k_cache_t5_h2": k[5, 2, :8].tolist(),
        "v_cache_t100_h3": v[100, 3, -8:].tolist(),
        "decode_step0_head": dec[0][:8].tolist(),
        "decode_step1_sum": [float(dec[1].sum())],
    }


if __name__ == "__main__":
    out = {
        "what": "oracle outputs, tiny pre-norm low-rank decoder layer, seed 0",
        "writer": "tests/golden/make_golden.py (oracle + seeded generator only)",
        "values": tiny_layer_case(),
    }
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)),
                        "tiny_layer_seed0.json")
    with open(path, "w") as fh:
        json.dump(out, fh, indent=1)
    print("wrote", path)
