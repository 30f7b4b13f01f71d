"""Seeded synthetic inputs shared by the CUDA path's tests/bench and the oracle.

This module holds no arithmetic of the decoder itself: it only names the five
workloads and draws their weights, token ids, activations and KV-cache
contents from seeded generators.  Every tensor gets its own seed derived from
(workload seed, layer, tensor name), so one layer (or one cache slice) can be
regenerated on its own.

The weight roster and names follow the checkpoint keys printed in
"从0开发大模型—译llama3-from-scratch" §2 (tok_embeddings, layers.{i}.attention.
wq/wk/wv/wo, feed_forward.w1/w2/w3, attention_norm, ffn_norm, norm, output),
all Linear weights in [out, in] layout.

The q/k/v projection weights are drawn into one stacked buffer
``wqkv = [Wq; Wk; Wv]`` (rows) and ``wq``/``wk``/``wv`` are row views of it,
because the library's QKV call takes the stacked matrix.
"""
from __future__ import annotations

import dataclasses
import hashlib
from typing import Optional

import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    dim: int
    n_layers: int
    n_heads: int
    n_kv_heads: int
    ffn_hidden: int
    vocab: Optional[int]
    batch: int
    seq: int
    dtype: str                 # "bf16" or "f32"
    input_kind: str            # "ids" or "activations"
    cache_len: int = 0         # positions already in the cache (decode)
    lm_rows: str = "all"       # "all", "last" or "none"
    norm_eps: float = 1e-5
    rope_theta: float = 500000.0
    weight_std: float = 0.02
    seed: int = 0

    @property
    def head_dim(self):
        return self.dim // self.n_heads

    @property
    def torch_dtype(self):
        return torch.float32 if self.dtype == "f32" else torch.bfloat16

    def cfg(self):
        """Model hyper-parameters as a plain dict (oracle and binding)."""
        return dict(dim=self.dim, n_heads=self.n_heads, n_kv_heads=self.n_kv_heads,
                    head_dim=self.head_dim, ffn_hidden=self.ffn_hidden,
                    vocab=self.vocab or 0, norm_eps=self.norm_eps,
                    rope_theta=self.rope_theta, dtype=self.dtype)

    def replace(self, **kw):
        return dataclasses.replace(self, **kw)


# The five workloads, named by what they are.
WORKLOADS = {
    # Tiny fp32 block (shapes of the GPT-style hand-written LLM page: batch 4,
    # context 16, d_model 64, 4 heads, vocab 3771), 1 layer, activations in.
    "tiny_f32": Workload("tiny_f32", dim=64, n_layers=1, n_heads=4, n_kv_heads=2,
                         ffn_hidden=192, vocab=3771, batch=4, seq=16, dtype="f32",
                         input_kind="activations", lm_rows="all", seed=1000),
    # Char-level Llama-3 (ModelArgs defaults of the from-scratch page): ids in [0,68).
    "char_8l": Workload("char_8l", dim=512, n_layers=8, n_heads=8, n_kv_heads=4,
                        ffn_hidden=1536, vocab=68, batch=10, seq=256, dtype="bf16",
                        input_kind="ids", lm_rows="all", seed=2000),
    # GQA-heavy single layer (hidden 768, 8 heads, 2 KV heads, head_dim 96).
    "gqa_768": Workload("gqa_768", dim=768, n_layers=1, n_heads=8, n_kv_heads=2,
                        ffn_hidden=2048, vocab=None, batch=8, seq=2048, dtype="bf16",
                        input_kind="activations", lm_rows="none", seed=3000),
    # Llama-3-8B-shaped prefill, batch 1 x 8192 tokens, LM head on last position.
    "llama3_8b_prefill": Workload("llama3_8b_prefill", dim=4096, n_layers=32,
                                  n_heads=32, n_kv_heads=8, ffn_hidden=14336,
                                  vocab=128256, batch=1, seq=8192, dtype="bf16",
                                  input_kind="ids", lm_rows="last", seed=4000),
    # Llama-3-8B-shaped decode step: 32 sequences, 8192 cached positions each.
    "llama3_8b_decode": Workload("llama3_8b_decode", dim=4096, n_layers=32,
                                 n_heads=32, n_kv_heads=8, ffn_hidden=14336,
                                 vocab=128256, batch=32, seq=1, cache_len=8192,
                                 dtype="bf16", input_kind="ids", lm_rows="all",
                                 seed=4000),
}


def _seed(base: int, *parts) -> int:
    h = hashlib.sha256(repr((base,) + parts).encode()).digest()
    return int.from_bytes(h[:8], "little") & ((1 << 62) - 1)


def _gen(device, seed):
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def _normal_into(out: torch.Tensor, std: float, seed: int):
    """Fill ``out`` (any float dtype, contiguous) with N(0, std^2), rounded once."""
    g = _gen(out.device, seed)
    tmp = torch.randn(out.shape, generator=g, device=out.device, dtype=torch.float32)
    if std != 1.0:
        tmp.mul_(std)
    out.copy_(tmp)
    return out


def layer_weights(w: Workload, layer: int, device="cpu", norm_weight="ones"):
    """One decoder block's weights (page names, [out, in] layout).

    ``norm_weight``: "ones" (the pages' initialisation) or "random"
    (1 + N(0, 0.1^2), used by tests so that a dropped norm weight shows).
    """
    D, H, KV, hd, F = w.dim, w.n_heads, w.n_kv_heads, w.head_dim, w.ffn_hidden
    dt = w.torch_dtype
    s = lambda name: _seed(w.seed, "layer", layer, name)
    wqkv = torch.empty(((H + 2 * KV) * hd, D), dtype=dt, device=device)
    _normal_into(wqkv[:H * hd], w.weight_std, s("wq"))
    _normal_into(wqkv[H * hd:(H + KV) * hd], w.weight_std, s("wk"))
    _normal_into(wqkv[(H + KV) * hd:], w.weight_std, s("wv"))
    out = {
        "wqkv": wqkv,
        "wq": wqkv[:H * hd], "wk": wqkv[H * hd:(H + KV) * hd], "wv": wqkv[(H + KV) * hd:],
        "wo": _normal_into(torch.empty((D, H * hd), dtype=dt, device=device), w.weight_std, s("wo")),
        "w1": _normal_into(torch.empty((F, D), dtype=dt, device=device), w.weight_std, s("w1")),
        "w2": _normal_into(torch.empty((D, F), dtype=dt, device=device), w.weight_std, s("w2")),
        "w3": _normal_into(torch.empty((F, D), dtype=dt, device=device), w.weight_std, s("w3")),
    }
    for name in ("attention_norm", "ffn_norm"):
        out[name] = _norm_weight(w, device, norm_weight, s(name))
    return out


def stack_weights(w: Workload, device="cpu", norm_weight="ones", threads: int = 8):
    """All ``w.n_layers`` blocks' weights and the output weights, drawn on the
    host by the CPU generators (the same draws on every machine for a given
    torch build) in ``threads`` parallel threads, then moved to ``device``.
    Returns (layers, output_weights)."""
    from concurrent.futures import ThreadPoolExecutor
    with ThreadPoolExecutor(max(1, threads)) as ex:
        layers = list(ex.map(lambda i: layer_weights(w, i, "cpu", norm_weight), range(w.n_layers)))
    out = output_weights(w, "cpu", norm_weight)
    if str(device) != "cpu":
        def move(d):
            m = {k: v.to(device) for k, v in d.items() if k not in ("wq", "wk", "wv")}
            if "wqkv" in m:
                H, KV, hd = w.n_heads, w.n_kv_heads, w.head_dim
                m["wq"], m["wk"], m["wv"] = (m["wqkv"][:H * hd], m["wqkv"][H * hd:(H + KV) * hd],
                                             m["wqkv"][(H + KV) * hd:])
            return m
        layers = [move(l) for l in layers]
        out = move(out)
    return layers, out


def _norm_weight(w: Workload, device, kind, seed):
    t = torch.empty((w.dim,), dtype=w.torch_dtype, device=device)
    if kind == "ones":
        return t.fill_(1.0)
    g = _gen(device, seed)
    tmp = 1.0 + 0.1 * torch.randn((w.dim,), generator=g, device=device)
    return t.copy_(tmp)


def output_weights(w: Workload, device="cpu", norm_weight="ones"):
    """tok_embeddings [V, D], final norm [D], output [V, D]."""
    out = {"norm": _norm_weight(w, device, norm_weight, _seed(w.seed, "norm"))}
    if w.vocab:
        V, D, dt = w.vocab, w.dim, w.torch_dtype
        out["tok_embeddings"] = _normal_into(torch.empty((V, D), dtype=dt, device=device),
                                             w.weight_std, _seed(w.seed, "tok_embeddings"))
        out["output"] = _normal_into(torch.empty((V, D), dtype=dt, device=device),
                                     w.weight_std, _seed(w.seed, "output"))
    return out


def token_ids(w: Workload, device="cpu", step=0):
    """Uniform ids in [0, vocab), shape [batch, seq], int32."""
    g = _gen(device, _seed(w.seed, "ids", step))
    return torch.randint(0, w.vocab, (w.batch, w.seq), generator=g, device=device,
                         dtype=torch.int64).to(torch.int32)


def activations(w: Workload, device="cpu", step=0):
    """N(0,1) block input, shape [batch, seq, dim] in the workload dtype."""
    x = torch.empty((w.batch, w.seq, w.dim), dtype=w.torch_dtype, device=device)
    return _normal_into(x, 1.0, _seed(w.seed, "x", step))


def hidden_rows(w: Workload, rows: int, device="cpu", std=1.0, step=0):
    """Random [rows, dim] rows standing in for final hidden states."""
    x = torch.empty((rows, w.dim), dtype=w.torch_dtype, device=device)
    return _normal_into(x, std, _seed(w.seed, "hidden", rows, step))


def kv_cache(w: Workload, layer: int, capacity: int, device="cpu", first: int = 0, count: Optional[int] = None):
    """Per-layer caches [count, capacity, KV, hd] of sequences first ..
    first+count-1 (default: the whole batch); the first ``cache_len`` positions
    hold N(0,1) entries (already-rotated keys and values), the rest zeros.
    Each sequence has its own seed, so a shard of the batch draws exactly the
    rows the whole batch would hold."""
    count = w.batch - first if count is None else count
    shape = (count, capacity, w.n_kv_heads, w.head_dim)
    k = torch.zeros(shape, dtype=w.torch_dtype, device=device)
    v = torch.zeros(shape, dtype=w.torch_dtype, device=device)
    if w.cache_len:
        for name, t in (("k", k), ("v", v)):
            for i in range(count):
                _normal_into(t[i, :w.cache_len], 1.0, _seed(w.seed, "cache", layer, name, first + i))
    return k, v
