"""Plain, slow fp64 CPU oracle for the Llama-3 decoder forward pass.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path may import, call or
execute this module: only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline / reference legs of ``bench.py`` use it.  It shares no code, table
or constant with the CUDA library; both sides only receive the same seeded
inputs from ``llama_decoder_only_rmsnorm_b200.inputs``.

Every quantity is evaluated in float64 with NumPy.  The inputs (bf16- or
fp32-valued weights and activations) are upcast exactly, so a comparison with
the GPU measures only the GPU's own rounding.

Sources (the five web pages on the Llama-3 decoder; cited by title + section):
  [S1] "从0开发大模型—译llama3-from-scratch" (sunaigc.com), sections 1-12.
  [S2] "Build your own Llama 3 from scratch" (gitcode.csdn.net), sections
       二 (input block), 三 3.1-3.6 (decoder block), 四 (output block), 六 (inference).
  [S3] "llama3-from-scratch：输出层与预测" (agent.csdn.net), "预测流程的完整实现".
  [S4] "Llama3 architecture" blog (joto.ai), GQA and RoPE paragraphs.

Readings taken where the pages are silent or disagree:
  * RoPE pairs adjacent elements (2i, 2i+1) as one complex number, real part
    first ([S1] §6.6-6.9, [S2] §3.2); the exponent uses head_dim ([S2] §3.2,
    frequencies built for dim=head_dim); angles are evaluated exactly in fp64.
  * A query at position start_pos+t sees keys j <= start_pos+t (the training
    mask of [S2] §3.4 / [S1] §7.1, shifted by the cache offset).
  * Query head h reads KV head h // n_rep ([S2] §3.4 repeat_kv, [S1] §8 head//4).
  * RMSNorm is not rounded between normalising and weighting.
  * argmax breaks ties toward the lowest vocabulary index.

Precision variant (``rounding="bf16"``): the pages' own bf16 model holds
every activation passed between steps as a bf16 tensor (the RMSNorm output
cast back to the input type, [S2] §3.1; q, k, v and the attention
probabilities cast to the activation type, [S2] §3.4 and [S1] §7; the block
output and the residual stream in the model dtype).  With that option the
oracle rounds to bf16 (8 significant bits, ties to even) at exactly those
step boundaries -- normalised rows, rotated q/k and v, probabilities before
the P.V product, attention output, residual stream after each residual add,
SwiGLU product -- and keeps every sum, the softmax statistics and the RoPE
angles exact.  It measures how far bf16 storage alone takes a result from the
exact answer, which is what the full-size tests calibrate their bound with.

Parity status: every function below is pinned by ``tests/test_oracle_pins.py``
except ``forward_stack`` on real checkpoints (parity unpinned for real Meta
weights: the checkpoint and tokenizer are not available, so the worked
"42"/token-2983 example of [S1] §12 cannot be reproduced).
"""
from __future__ import annotations

import numpy as np

__all__ = [
    "bf16_round", "rms_norm", "ffn_hidden_dim", "rope_inverse_frequencies", "rope_angles",
    "apply_rope", "causal_mask", "gqa_attention", "silu", "swiglu_ffn",
    "decoder_block", "decoder_block_rows", "lm_head", "embed", "forward_stack",
    "generate_greedy", "philox4x64", "sampling_word", "top_p_sample",
]


def _f64(a):
    return np.asarray(a, dtype=np.float64)


# ---------------------------------------------------------------------------
# bf16 storage (the precision variant; see the module docstring)
# ---------------------------------------------------------------------------
def bf16_round(x):
    """Round to the nearest bfloat16 value (8 significant bits, ties to even),
    returned as float64.  Written out from the format: x = m * 2^e with
    m in [0.5, 1); keep m to 8 bits by rounding m * 2^8 to the nearest
    integer, ties to even.  (Values below 2^-126, where bf16 turns
    subnormal, never occur here and are not treated specially.)"""
    x = _f64(x)
    m, e = np.frexp(x)
    return np.ldexp(np.rint(m * 256.0), e - 8)


def _store(x, rounding):
    """An activation as the path stores it between steps."""
    if rounding is None:
        return x
    if rounding == "bf16":
        return bf16_round(x)
    raise ValueError(f"unknown rounding {rounding!r}")


# ---------------------------------------------------------------------------
# RMSNorm  ([S1] §5 rms_norm; [S2] §3.1 RMSNorm)
# ---------------------------------------------------------------------------
def rms_norm(x, weight, eps):
    """x / sqrt(mean(x^2 over the last axis) + eps) * weight, in fp64."""
    x = _f64(x)
    mean_sq = np.mean(x * x, axis=-1, keepdims=True)
    return x / np.sqrt(mean_sq + eps) * _f64(weight)


# ---------------------------------------------------------------------------
# FFN hidden size rule  ([S2] §3.5 FeedForward.__init__, §3.6 4*dim input)
# ---------------------------------------------------------------------------
def ffn_hidden_dim(dim, multiple_of, ffn_dim_multiplier=None):
    """The block is built with hidden = 4*dim; keep two thirds (truncated),
    optionally scale by the multiplier (truncated), then round up to a
    multiple of ``multiple_of``."""
    hidden = int(2 * (4 * dim) / 3)
    if ffn_dim_multiplier is not None:
        hidden = int(ffn_dim_multiplier * hidden)
    return multiple_of * ((hidden + multiple_of - 1) // multiple_of)


# ---------------------------------------------------------------------------
# RoPE  ([S1] §6.6-6.10; [S2] §3.2; [S4] RoPE paragraphs)
# ---------------------------------------------------------------------------
def rope_inverse_frequencies(head_dim, theta):
    """theta_i = theta ** (-(2i)/head_dim) for pair i in [0, head_dim/2)."""
    i = np.arange(head_dim // 2, dtype=np.float64)
    return np.power(np.float64(theta), -(2.0 * i) / head_dim)


def rope_angles(positions, head_dim, theta):
    """Angle m * theta_i for every position m and pair i -> [len(pos), hd/2]."""
    m = _f64(positions)
    return np.outer(m, rope_inverse_frequencies(head_dim, theta))


def apply_rope(x, positions, theta):
    """Rotate pairs (x[2i], x[2i+1]) of the last axis by e^{i*m*theta_i}.

    ``x`` has shape [..., S, n_heads, head_dim] and ``positions`` has length S
    (the token axis is the third from last).  Each pair is read as the complex
    number x[2i] + 1j*x[2i+1], multiplied by the unit phasor, and written back
    with the real part first -- the view_as_complex reading of [S2] §3.2.
    """
    x = _f64(x)
    hd = x.shape[-1]
    ang = rope_angles(positions, hd, theta)                 # [S, hd/2]
    phasor = np.exp(1j * ang)[:, None, :]                   # [S, 1, hd/2]
    z = x[..., 0::2] + 1j * x[..., 1::2]                    # [..., S, H, hd/2]
    zr = z * phasor
    out = np.empty_like(x)
    out[..., 0::2] = zr.real
    out[..., 1::2] = zr.imag
    return out


# ---------------------------------------------------------------------------
# Causal grouped-query attention  ([S1] §6.11-8; [S2] §3.4; [S4] GQA)
# ---------------------------------------------------------------------------
def causal_mask(n_queries, n_keys, start_pos=0, doc_start=None):
    """Additive mask: 0 where key j <= start_pos + t, -inf above ([S1] §7.1).

    With ``doc_start`` (one position per query: where that query's document
    begins) keys before it are masked too -- the document-level mask that
    keeps packed documents from attending to each other ([S2] 附 1).
    """
    t = np.arange(n_queries)[:, None] + start_pos
    j = np.arange(n_keys)[None, :]
    ok = j <= t
    if doc_start is not None:
        ok &= j >= np.asarray(doc_start)[:, None]
    return np.where(ok, 0.0, -np.inf)


def gqa_attention(q, k, v, start_pos=0, return_probs=False, doc_start=None, rounding=None):
    """softmax(q k^T / sqrt(hd) + mask) v for one sequence.

    q: [S, H, hd] (rotated); k, v: [T, KV, hd] with T = start_pos + S.
    Query head h reads KV head h // (H // KV).  Returns [S, H, hd]
    (and the [H, S, T] probabilities when ``return_probs``).
    rounding="bf16": the probabilities are stored in bf16 before the
    product with v (the softmax sum itself stays exact).
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    S, H, hd = q.shape
    T, KV, _ = k.shape
    assert H % KV == 0 and T == start_pos + S
    n_rep = H // KV
    mask = causal_mask(S, T, start_pos, doc_start)
    out = np.empty((S, H, hd))
    probs = np.empty((H, S, T)) if return_probs else None
    for h in range(H):
        g = h // n_rep
        scores = q[:, h, :] @ k[:, g, :].T / np.sqrt(hd) + mask
        scores = scores - scores.max(axis=1, keepdims=True)
        e = np.exp(scores)
        total = e.sum(axis=1, keepdims=True)
        p = e / total
        if rounding is None:
            out[:, h, :] = p @ v[:, g, :]
        else:
            out[:, h, :] = (_store(e, rounding) @ v[:, g, :]) / total
        if return_probs:
            probs[h] = p
    return (out, probs) if return_probs else out


# ---------------------------------------------------------------------------
# SwiGLU FFN  ([S1] §9.3; [S2] §3.5)
# ---------------------------------------------------------------------------
def silu(z):
    z = _f64(z)
    return z / (1.0 + np.exp(-z))


def swiglu_ffn(x, w1, w2, w3):
    """w2( silu(x w1^T) * (x w3^T) ) with Linear weights stored [out, in]."""
    x = _f64(x)
    return (silu(x @ _f64(w1).T) * (x @ _f64(w3).T)) @ _f64(w2).T


# ---------------------------------------------------------------------------
# One pre-norm decoder block  ([S2] §3.6 TransformerBlock; [S1] §6-10)
# ---------------------------------------------------------------------------
def decoder_block(x, layer, cfg, k_cache, v_cache, start_pos=0, doc_start=None, rounding=None):
    """h = x + Attn(RMSNorm(x)); out = h + FFN(RMSNorm(h)).

    x: [B, S, D].  ``layer`` maps the page's weight names (attention_norm, wq,
    wk, wv, wo, ffn_norm, w1, w2, w3) to arrays in [out, in] layout.
    k_cache / v_cache: fp64 arrays [B, cap, KV, hd]; positions
    [start_pos, start_pos+S) are overwritten with this call's rotated k and v
    ([S2] §3.3 / §3.4 inference branch).  ``doc_start`` [B, S] (optional):
    the position where each token's document begins (document mask).
    ``rounding``: None (exact) or "bf16" (activations stored in bf16 between
    steps; module docstring).  Returns out [B, S, D].
    """
    x = _f64(x)
    B, S, D = x.shape
    H, KV, hd = cfg["n_heads"], cfg["n_kv_heads"], cfg["head_dim"]
    eps, theta = cfg["norm_eps"], cfg["rope_theta"]
    pos = start_pos + np.arange(S)

    r = lambda a: _store(a, rounding)
    xn = r(rms_norm(x, layer["attention_norm"], eps))
    q = (xn @ _f64(layer["wq"]).T).reshape(B, S, H, hd)
    k = (xn @ _f64(layer["wk"]).T).reshape(B, S, KV, hd)
    v = r((xn @ _f64(layer["wv"]).T).reshape(B, S, KV, hd))
    q = r(apply_rope(q, pos, theta))
    k = r(apply_rope(k, pos, theta))
    k_cache[:B, start_pos:start_pos + S] = k
    v_cache[:B, start_pos:start_pos + S] = v

    o = np.empty((B, S, H, hd))
    for b in range(B):
        o[b] = gqa_attention(q[b], k_cache[b, :start_pos + S], v_cache[b, :start_pos + S], start_pos,
                             doc_start=None if doc_start is None else np.asarray(doc_start)[b],
                             rounding=rounding)
    h = r(x + r(o.reshape(B, S, H * hd)) @ _f64(layer["wo"]).T)
    hn = r(rms_norm(h, layer["ffn_norm"], eps))
    return r(h + _swiglu_rounded(hn, layer, rounding))


def _swiglu_rounded(hn, layer, rounding):
    """swiglu_ffn with the SwiGLU product stored as the path stores it."""
    if rounding is None:
        return swiglu_ffn(hn, layer["w1"], layer["w2"], layer["w3"])
    hn = _f64(hn)
    g = _store(silu(hn @ _f64(layer["w1"]).T) * (hn @ _f64(layer["w3"]).T), rounding)
    return g @ _f64(layer["w2"]).T


def decoder_block_rows(x, layer, cfg, rows, k_prefix=None, v_prefix=None, start_pos=0, rounding=None):
    """Selected output rows of ``decoder_block`` for ONE sequence.

    x: [S, D] (tokens at positions start_pos..start_pos+S-1); k_prefix /
    v_prefix: [start_pos, KV, hd] cached entries before them (or None when
    start_pos == 0).  Keys and values are projected for every token (each row
    attends to all earlier ones); queries, attention, wo, the FFN and both
    residuals only for the tokens in ``rows``.  Returns (out [len(rows), D],
    k [S, KV, hd], v [S, KV, hd]) with k rotated, i.e. what the cache receives.
    ``rounding`` as in ``decoder_block``.
    """
    x = _f64(x)
    S, D = x.shape
    H, KV, hd = cfg["n_heads"], cfg["n_kv_heads"], cfg["head_dim"]
    eps, theta = cfg["norm_eps"], cfg["rope_theta"]
    rows = list(rows)
    r = lambda a: _store(a, rounding)
    xn = r(rms_norm(x, layer["attention_norm"], eps))
    pos = start_pos + np.arange(S)
    k = r(apply_rope((xn @ _f64(layer["wk"]).T).reshape(S, KV, hd), pos, theta))
    v = r((xn @ _f64(layer["wv"]).T).reshape(S, KV, hd))
    if start_pos:
        k_all = np.concatenate([_f64(k_prefix), k], 0)
        v_all = np.concatenate([_f64(v_prefix), v], 0)
    else:
        k_all, v_all = k, v
    xr = x[rows]
    q = r(apply_rope((xn[rows] @ _f64(layer["wq"]).T).reshape(len(rows), H, hd),
                     start_pos + np.asarray(rows), theta))
    o = np.empty((len(rows), H, hd))
    for i, t in enumerate(rows):
        n_keys = start_pos + t + 1
        o[i] = gqa_attention(q[i:i + 1], k_all[:n_keys], v_all[:n_keys], n_keys - 1, rounding=rounding)[0]
    h = r(xr + r(o.reshape(len(rows), H * hd)) @ _f64(layer["wo"]).T)
    hn = r(rms_norm(h, layer["ffn_norm"], eps))
    return r(h + _swiglu_rounded(hn, layer, rounding)), k, v


# ---------------------------------------------------------------------------
# Output block  ([S1] §11-12; [S2] 四; [S3] 预测流程)
# ---------------------------------------------------------------------------
def lm_head(h_rows, norm_weight, w_out, eps, rounding=None):
    """RMSNorm the rows, project onto the vocabulary, take argmax.

    h_rows: [R, D].  Returns (logits [R, V], ids [R]); ids pick the lowest
    index among equal maxima.  rounding="bf16": the normalised rows are
    stored in bf16 before the projection.
    """
    hn = _store(rms_norm(h_rows, norm_weight, eps), rounding)
    logits = hn @ _f64(w_out).T
    return logits, np.argmax(logits, axis=-1).astype(np.int64)


def embed(ids, table):
    """Row gather x[t] = E[id[t]]  ([S1] §4; [S2] 四 tok_embeddings)."""
    return _f64(table)[np.asarray(ids)]


def forward_stack(x, layers, cfg, k_caches=None, v_caches=None, start_pos=0,
                  cache_len=None, doc_start=None, rounding=None):
    """Run x through every block in ``layers`` (the layer loop of [S2] 四).

    Creates fp64 caches of length ``cache_len`` (default start_pos+S) when none
    are given.  Returns (h, k_caches, v_caches).
    """
    x = _f64(x)
    B, S, _ = x.shape
    cap = cache_len or (start_pos + S)
    KV, hd = cfg["n_kv_heads"], cfg["head_dim"]
    if k_caches is None:
        k_caches = [np.zeros((B, cap, KV, hd)) for _ in layers]
        v_caches = [np.zeros((B, cap, KV, hd)) for _ in layers]
    for layer, kc, vc in zip(layers, k_caches, v_caches):
        x = decoder_block(x, layer, cfg, kc, vc, start_pos, doc_start, rounding)
    return x, k_caches, v_caches


# ---------------------------------------------------------------------------
# Greedy generation  ([S2] 六 generate with temperature 0: argmax of the last
# position's logits, fed back one token per step through the KV cache)
# ---------------------------------------------------------------------------
def generate_greedy(prompt_ids, table, layers, norm_weight, w_out, cfg, n_new, eos_id=None):
    """Greedy continuation of every prompt (all the same length).

    Prefills the prompts, then for each new token: embed it, run one cached
    decode step at the next position, take the argmax of the final-norm LM
    head.  Returns (tokens [B, n_new], gaps [B, n_new]) where gaps are the
    top-2 logit differences of each decision.  After a sequence emits eos_id
    its later tokens are eos_id as well (the page stops the loop there).
    """
    ids = np.asarray(prompt_ids)
    B, S = ids.shape
    cap = S + n_new
    h, kc, vc = forward_stack(embed(ids, table), layers, cfg, cache_len=cap)
    logits, nxt = lm_head(h[:, -1], norm_weight, w_out, cfg["norm_eps"])
    toks = np.zeros((B, n_new), dtype=np.int64)
    gaps = np.zeros((B, n_new))
    done = np.zeros(B, dtype=bool)
    for step in range(n_new):
        top2 = np.sort(logits, axis=1)[:, -2:]
        gaps[:, step] = top2[:, 1] - top2[:, 0]
        nxt = np.where(done, eos_id if eos_id is not None else nxt, nxt)
        toks[:, step] = nxt
        if eos_id is not None:
            done |= nxt == eos_id
        if step + 1 == n_new:
            break
        h, kc, vc = forward_stack(embed(nxt[:, None], table), layers, cfg, kc, vc, start_pos=S + step)
        logits, nxt = lm_head(h[:, -1], norm_weight, w_out, cfg["norm_eps"])
    return toks, gaps


# ---------------------------------------------------------------------------
# Temperature / top-p sampling  ([S2] 六 generate and sample_top_p; [S3]
# 预测流程 on temperature)
# ---------------------------------------------------------------------------
# The random numbers come from Philox-4x64-10, the counter-based generator of
# Salmon, Moraes, Dror and Shaw, "Parallel random numbers: as easy as 1, 2, 3"
# (SC 2011): ten rounds of two 64x64->128 multiplies with the constants below,
# the key bumped by two Weyl increments between rounds.
_MASK64 = (1 << 64) - 1
_PHILOX_MUL = (0xD2E7470EE14C6C93, 0xCA5A826395121157)
_PHILOX_WEYL = (0x9E3779B97F4A7C15, 0xBB67AE8584CAA73B)


def philox4x64(counter, key, rounds=10):
    """One Philox-4x64 block: 4 counter words and 2 key words -> 4 words."""
    c = [int(w) & _MASK64 for w in counter]
    k = [int(w) & _MASK64 for w in key]
    for _ in range(rounds):
        p0 = _PHILOX_MUL[0] * c[0]
        p1 = _PHILOX_MUL[1] * c[2]
        c = [(p1 >> 64) ^ c[1] ^ k[0], p1 & _MASK64, (p0 >> 64) ^ c[3] ^ k[1], p0 & _MASK64]
        k = [(k[0] + _PHILOX_WEYL[0]) & _MASK64, (k[1] + _PHILOX_WEYL[1]) & _MASK64]
    return c


def sampling_word(seed, offset, row):
    """The 64-bit random word of one draw: first output word of
    Philox-4x64-10 with key (seed, 0) and counter (offset, row, 0, 0)."""
    return philox4x64((offset, row, 0, 0), (seed, 0))[0]


def top_p_sample(logits, temperature, top_p, word):
    """Next token of one row as [S2] 六 generate draws it.

    temperature <= 0: argmax (lowest index on ties).  Otherwise
    p = softmax(logits / temperature); tokens are ranked by descending p
    (ties by ascending index, a stable sort); a token is kept iff the mass
    ranked before it is <= top_p (the page zeroes those whose cumulative sum
    minus their own probability exceeds top_p); the kept probabilities are
    renormalised and one token is drawn.  The draw maps u = word / 2^64 by the
    inverse CDF over the kept tokens in ascending index order: the first kept
    token whose running kept mass exceeds u * (kept mass).  (The page hands the
    draw to a multinomial routine; any fixed order gives the same law, and this
    one needs no sort.)

    Returns (token, margins) where margins = (cut, draw): the distance of
    top_p from the nearest kept/dropped decision, and of the draw target from
    the nearest boundary of the running kept mass, both as fractions of the
    row's total probability.
    """
    z = _f64(logits)
    if temperature <= 0:
        return int(np.argmax(z)), (np.inf, np.inf)
    z = z / float(temperature)
    e = np.exp(z - z.max())
    p = e / e.sum()
    order = np.argsort(-p, kind="stable")
    ranked = p[order]
    before = np.cumsum(ranked) - ranked
    keep_ranked = before <= top_p
    kept = np.zeros(p.shape, dtype=bool)
    kept[order[keep_ranked]] = True
    n_keep = int(keep_ranked.sum())
    # Decisions that rounding cannot flip are no boundary: the top token (mass
    # before it exactly 0) and, for top_p >= 1, every token (the mass before
    # any token is below 1).
    cut = np.inf
    if top_p < 1:
        if n_keep > 1:
            cut = top_p - before[n_keep - 1]
        if n_keep < len(ranked):
            cut = min(cut, before[n_keep] - top_p)
    idx = np.nonzero(kept)[0]
    run = np.cumsum(p[idx])
    target = (int(word) / 2.0 ** 64) * run[-1]
    i = int(np.searchsorted(run, target, side="right"))
    i = min(i, len(idx) - 1)
    draw = run[i] - target
    if i > 0:
        draw = min(draw, target - run[i - 1])
    return int(idx[i]), (float(cut), float(draw))
