"""Writes llama3_8b_prefill_last_row.txt: what the fp64 oracle says the
Llama-3-8B-shaped prefill ends with on its last position.

    python tests/golden/make_llama3_8b_prefill_last_row.py [--layers N] [--out FILE]

The workload is the 8B prefill (batch 1 x 8192 uniform token ids, 32 blocks,
seeded N(0, 0.02) weights, norm weights 1.0), with every input drawn on the
host by ``inputs.stack_weights`` / ``inputs.token_ids`` (CPU generators), so
the GPU test regenerates exactly these inputs.  Only ``oracle/`` computes: the
exact pass and the bf16-storage pass (``rounding="bf16"``), block by block
over all 8192 tokens.  The file keeps, for the last position, both final
hidden rows (the LM head's logits follow from them and the output weights),
plus checksums of the inputs and the hashes of the oracle and input sources,
so that a test can tell when it no longer describes its inputs.  The whole
run takes tens of minutes of CPU.
"""
import argparse
import hashlib
import os
import sys
import time

import numpy as np
import torch

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(os.path.dirname(HERE))
sys.path.insert(0, ROOT)

from llama_decoder_only_rmsnorm_b200 import inputs as I  # noqa: E402
from oracle import llama3_oracle as O  # noqa: E402

NAME = "llama3_8b_prefill_last_row.txt"


def file_hash(rel):
    with open(os.path.join(ROOT, rel), "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()[:16]


def input_checksums(layers, outw, ids):
    """Cheap fingerprints of the drawn inputs: float64 sums of a few tensors."""
    f = lambda t: float(t.to(torch.float64).sum())
    return {"ids_sum": int(ids.to(torch.int64).sum()), "wqkv0_sum": f(layers[0]["wqkv"]),
            "w2_last_sum": f(layers[-1]["w2"]), "tok_embeddings_sum": f(outw["tok_embeddings"]),
            "output_sum": f(outw["output"])}


def f64(t):
    return t.to(torch.float32).numpy().astype(np.float64)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--layers", type=int, default=None)
    ap.add_argument("--out", default=os.path.join(HERE, NAME))
    a = ap.parse_args()
    w = I.WORKLOADS["llama3_8b_prefill"]
    if a.layers:
        w = w.replace(n_layers=a.layers)
    t0 = time.time()
    layers, outw = I.stack_weights(w, "cpu")
    ids = I.token_ids(w, "cpu")
    sums = input_checksums(layers, outw, ids)
    cfg = {k: v for k, v in w.cfg().items() if k not in ("vocab", "dtype")}
    table = outw["tok_embeddings"]
    x = f64(table[ids[0].long()])[None]                   # embedding rows of the prompt ([S1] §4)
    xs = {None: x, "bf16": x.copy()}
    for i, layer in enumerate(layers):
        ol = {k: f64(layer[k]) for k in ("attention_norm", "wq", "wk", "wv", "wo", "ffn_norm", "w1", "w2", "w3")}
        for rnd in xs:
            kc = np.zeros((1, w.seq, w.n_kv_heads, w.head_dim))
            vc = np.zeros_like(kc)
            xs[rnd] = O.decoder_block(xs[rnd], ol, cfg, kc, vc, 0, rounding=rnd)
        print(f"block {i} done, {time.time() - t0:.0f} s", flush=True)
    with open(a.out, "w") as f:
        f.write("# Final hidden state of the last position (8191) of the Llama-3-8B-shaped prefill\n")
        f.write("# (batch 1 x 8192 ids, seeded CPU draws of inputs.stack_weights / inputs.token_ids),\n")
        f.write("# from the fp64 oracle: exact, and with activations stored in bf16 between steps.\n")
        f.write(f"# written by tests/golden/make_llama3_8b_prefill_last_row.py in {time.time() - t0:.0f} s\n")
        f.write(f"workload {w.name} layers {w.n_layers} seq {w.seq} seed {w.seed}\n")
        f.write(f"oracle_sha {file_hash('oracle/llama3_oracle.py')}\n")
        f.write(f"inputs_sha {file_hash('llama_decoder_only_rmsnorm_b200/inputs.py')}\n")
        f.write(f"torch {torch.__version__.split('+')[0]}\n")
        for k, v in sums.items():
            f.write(f"{k} {v!r}\n")
        for tag, rnd in (("exact", None), ("bf16", "bf16")):
            f.write(f"hidden_{tag} " + " ".join(repr(float(v)) for v in xs[rnd][0, -1]) + "\n")
    print("wrote", a.out)


if __name__ == "__main__":
    main()
