"""The two 8B-shaped workloads end to end, in the launch configuration
bench.py times, against the fp64 oracle.

* Decode step: 32 sequences, each with 8192 cached positions (N(0,1) cache
  entries), one new token at position 8192: embedding, 32 blocks, final norm,
  the 128256 x 4096 LM head and argmax.  Every sequence's final hidden row,
  every block's new K/V rows, the logits and the ids are compared.
* Prefill: 1 x 8192 tokens through 32 blocks.  By causality the first 256
  positions of that run equal the oracle's 32-block pass over those 256
  tokens alone ("从0开发大模型—译llama3-from-scratch" §7: a position never
  sees a later one), so their final hidden rows, logits and ids are compared
  with an oracle run taking minutes instead of hours.  The last position is
  compared with the stored oracle result in tests/golden (written by the
  script beside it from the same seeded inputs).

Outputs 32 blocks deep are held to the full-size bound of helpers.py (the
GPU within 1.5x of the relative L2 error of the oracle's bf16-storage
variant; ids where the exact top-2 gap clears 6x that variant's logit
noise).  Weights are drawn by the host generators (inputs.stack_weights) so
that the stored golden describes the same model on every machine.
"""
import os

import numpy as np
import pytest
import torch

from conftest import GOLDEN
from helpers import (assert_argmax_beyond_noise, assert_within_bf16_noise, f64, oracle_cfg)
from llama_decoder_only_rmsnorm_b200 import binding as B
from llama_decoder_only_rmsnorm_b200 import inputs as I
from llama_decoder_only_rmsnorm_b200.model import Llama3Stack
from oracle import llama3_oracle as O

pytestmark = pytest.mark.gpu
DEV = "cuda"
PREFILL, DECODE = I.WORKLOADS["llama3_8b_prefill"], I.WORKLOADS["llama3_8b_decode"]
NAMES = ("attention_norm", "wq", "wk", "wv", "wo", "ffn_norm", "w1", "w2", "w3")
PREFIX = 256


@pytest.fixture(scope="module")
def model8b():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    layers_h, out_h = I.stack_weights(PREFILL, "cpu", threads=min(32, os.cpu_count() or 8))
    layers_d, out_d = [], {}
    for l in layers_h:
        d = {k: l[k].to(DEV) for k in ("attention_norm", "wqkv", "wo", "ffn_norm", "w1", "w2", "w3")}
        H, KV, hd = PREFILL.n_heads, PREFILL.n_kv_heads, PREFILL.head_dim
        d["wq"], d["wk"], d["wv"] = d["wqkv"][:H * hd], d["wqkv"][H * hd:(H + KV) * hd], d["wqkv"][(H + KV) * hd:]
        layers_d.append(d)
    out_d = {k: v.to(DEV) for k, v in out_h.items()}
    yield layers_h, out_h, layers_d, out_d
    del layers_d, out_d
    torch.cuda.empty_cache()


@pytest.fixture(autouse=True)
def _gpu_state():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    B.llama3_set_kernel_path(0)
    yield
    torch.cuda.synchronize()
    assert B.llama3_device_status() == 0, "device status word set"


def _host_layer(layer):
    return {k: f64(layer[k]) for k in NAMES}


def _embed_rows(ids_np, table):
    """Oracle embedding of a few ids without converting the whole table."""
    uniq, inv = np.unique(ids_np, return_inverse=True)
    return O.embed(inv.reshape(ids_np.shape), f64(table[torch.as_tensor(uniq).long()]))


def _lm_head_both(h_exact, h_bf16, out_h):
    nw, wo = f64(out_h["norm"]), f64(out_h["output"])
    lg_ex, _ = O.lm_head(h_exact, nw, wo, PREFILL.norm_eps)
    lg_bf, _ = O.lm_head(h_bf16, nw, wo, PREFILL.norm_eps, rounding="bf16")
    return lg_ex, lg_bf


def test_8b_decode_step_32_blocks_and_lm_head(model8b):
    layers_h, out_h, layers_d, out_d = model8b
    Bt, P, D = DECODE.batch, DECODE.cache_len, DECODE.dim
    caches = [I.kv_cache(DECODE, i, P + 1, DEV) for i in range(DECODE.n_layers)]
    st = Llama3Stack(PREFILL.cfg(), layers_d, out_d, Bt, P + 1, 1, lm_rows=Bt, caches=caches)
    ids = I.token_ids(DECODE, DEV)
    xd = torch.empty((Bt, 1, D), dtype=torch.bfloat16, device=DEV)
    st.embed(ids, xd)
    st.decode_layers(xd, P)
    logits = torch.empty((Bt, DECODE.vocab), dtype=torch.float32, device=DEV)
    got_ids = st.lm_head(xd, Bt, D, logits).clone()
    torch.cuda.synchronize()
    new_k = [f64(kc[:, P]) for kc, _ in caches]
    new_v = [f64(vc[:, P]) for _, vc in caches]
    del st, caches
    torch.cuda.empty_cache()

    cfg = oracle_cfg(PREFILL)
    x_ex = _embed_rows(ids.cpu().numpy(), out_h["tok_embeddings"])      # [32, 1, D]
    x_bf = x_ex.copy()
    for i, layer in enumerate(layers_h):
        ol = _host_layer(layer)
        kp, vp = I.kv_cache(DECODE, i, P + 1, DEV)     # the cache prefix is an input: same seeds, drawn again
        kp, vp = f64(kp), f64(vp)
        x_ex = O.decoder_block(x_ex, ol, cfg, kp, vp, P)
        k_ex, v_ex = kp[:, P].copy(), vp[:, P].copy()
        x_bf = O.decoder_block(x_bf, ol, cfg, kp, vp, P, rounding="bf16")
        assert_within_bf16_noise(new_k[i], k_ex, kp[:, P], f"block {i} new K rows")
        assert_within_bf16_noise(new_v[i], v_ex, vp[:, P], f"block {i} new V rows")
    info = assert_within_bf16_noise(xd, x_ex, x_bf, "final hidden rows")
    lg_ex, lg_bf = _lm_head_both(x_ex[:, 0], x_bf[:, 0], out_h)
    linfo = assert_within_bf16_noise(logits, lg_ex, lg_bf, "logits")
    n = assert_argmax_beyond_noise(got_ids, lg_ex, lg_bf, "next ids", need=4)
    print(f"decode 8B: hidden {info}; logits {linfo}; ids decided on {n} of {Bt} sequences")


def _golden_script():
    """The script that wrote the golden file, for its input fingerprint."""
    import importlib.util
    path = os.path.join(GOLDEN, "make_llama3_8b_prefill_last_row.py")
    spec = importlib.util.spec_from_file_location("make_llama3_8b_prefill_last_row", path)
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _golden_last_row():
    rec = {}
    with open(os.path.join(GOLDEN, "llama3_8b_prefill_last_row.txt")) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            key, _, rest = line.partition(" ")
            rec[key] = rest.strip()
    return rec


@pytest.fixture(scope="module")
def prefill_run(model8b):
    """The 8192-token prefill on the GPU, as bench.py runs it, plus the LM
    head on the last position and on the first PREFIX positions."""
    layers_h, out_h, layers_d, out_d = model8b
    S, D, V = PREFILL.seq, PREFILL.dim, PREFILL.vocab
    ids_h = I.token_ids(PREFILL, "cpu")
    st = Llama3Stack(PREFILL.cfg(), layers_d, out_d, 1, S, S, lm_rows=PREFIX)
    x = torch.empty((1, S, D), dtype=torch.bfloat16, device=DEV)
    st.embed(ids_h.to(DEV), x)
    st.forward_layers(x, S, 0)
    lg_last = torch.empty((1, V), dtype=torch.float32, device=DEV)
    id_last = st.lm_head(x[:, -1], 1, S * D, lg_last).clone()
    lg_pre = torch.empty((PREFIX, V), dtype=torch.float32, device=DEV)
    id_pre = st.lm_head(x[0, :PREFIX], PREFIX, D, lg_pre).clone()
    torch.cuda.synchronize()
    assert B.llama3_device_status() == 0
    out = dict(ids=ids_h, last=f64(x[0, -1]), prefix=f64(x[0, :PREFIX]), lg_last=f64(lg_last), id_last=id_last,
               lg_pre=f64(lg_pre), id_pre=id_pre)
    del st, x
    torch.cuda.empty_cache()
    return out


def test_8b_prefill_32_blocks_causal_prefix(model8b, prefill_run):
    layers_h, out_h, _, _ = model8b
    r = prefill_run
    cfg = oracle_cfg(PREFILL)
    x_ex = _embed_rows(r["ids"][:, :PREFIX].numpy(), out_h["tok_embeddings"])   # [1, PREFIX, D]
    x_bf = x_ex.copy()
    shape = (1, PREFIX, PREFILL.n_kv_heads, PREFILL.head_dim)
    for layer in layers_h:
        ol = _host_layer(layer)
        x_ex = O.decoder_block(x_ex, ol, cfg, np.zeros(shape), np.zeros(shape))
        x_bf = O.decoder_block(x_bf, ol, cfg, np.zeros(shape), np.zeros(shape), rounding="bf16")
    info = assert_within_bf16_noise(r["prefix"], x_ex[0], x_bf[0], f"final hidden rows 0..{PREFIX - 1}")
    lg_ex, lg_bf = _lm_head_both(x_ex[0], x_bf[0], out_h)
    linfo = assert_within_bf16_noise(r["lg_pre"], lg_ex, lg_bf, "prefix logits")
    n = assert_argmax_beyond_noise(r["id_pre"], lg_ex, lg_bf, "prefix ids", need=16)
    print(f"prefill 8B prefix: hidden {info}; logits {linfo}; ids decided on {n} of {PREFIX} rows")


def test_8b_prefill_32_blocks_last_position(model8b, prefill_run):
    layers_h, out_h, _, _ = model8b
    r = prefill_run
    gold = _golden_last_row()
    mk = _golden_script()
    assert gold["oracle_sha"] == mk.file_hash("oracle/llama3_oracle.py"), \
        "the oracle changed since the golden file was written: run the script beside it again"
    sums = mk.input_checksums(layers_h, out_h, r["ids"])
    assert int(gold["ids_sum"]) == sums["ids_sum"]
    for k, v in sums.items():
        assert abs(float(gold[k]) - v) <= 1e-9 * max(1.0, abs(v)), f"input {k} differs from the golden's"
    h_ex = np.array(gold["hidden_exact"].split(), dtype=np.float64)
    h_bf = np.array(gold["hidden_bf16"].split(), dtype=np.float64)
    info = assert_within_bf16_noise(r["last"], h_ex, h_bf, "last position hidden row")
    lg_ex, lg_bf = _lm_head_both(h_ex[None], h_bf[None], out_h)
    linfo = assert_within_bf16_noise(r["lg_last"], lg_ex, lg_bf, "last position logits")
    n = assert_argmax_beyond_noise(r["id_last"], lg_ex, lg_bf, "last position id", need=0)
    print(f"prefill 8B last position: hidden {info}; logits {linfo}; id decided: {bool(n)}")
