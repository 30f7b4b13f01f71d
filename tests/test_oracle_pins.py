"""Pins for the fp64 oracle: each checks it against something other than itself.

Values printed on the pages (golden fixtures), closed forms, invariants the
pages state in prose, brute force on tiny inputs, and planted mistakes that a
pin must catch.  CPU only.
"""
import math
import types

import numpy as np
import pytest

from conftest import read_golden
from oracle import llama3_oracle as O

RNG = np.random.default_rng(12345)


def rand(*shape, scale=1.0):
    return RNG.standard_normal(shape) * scale


# ---------------------------------------------------------------- RMSNorm ---
def pin_rmsnorm(o):
    # Constant row c (length n): mean(x^2) = c^2, so the result is c/sqrt(c^2+eps)*w.
    for c in (3.0, -0.5, 1e-3):
        w = np.linspace(0.5, 2.0, 8)
        got = o.rms_norm(np.full((2, 8), c), w, 1e-5)
        np.testing.assert_allclose(got, np.broadcast_to(c / math.sqrt(c * c + 1e-5) * w, (2, 8)),
                                   rtol=1e-14, atol=0)
    # Hand example [3, 4]: mean square 12.5.
    got = o.rms_norm(np.array([3.0, 4.0]), np.ones(2), 0.0)
    np.testing.assert_allclose(got, [3 / math.sqrt(12.5), 4 / math.sqrt(12.5)], rtol=1e-15)
    # Each row is normalised over its own last axis, not over the batch.
    x = np.array([[1.0, 1.0], [10.0, 10.0]])
    np.testing.assert_allclose(o.rms_norm(x, np.ones(2), 0.0), np.ones((2, 2)), rtol=1e-15)


def test_rmsnorm_closed_forms():
    pin_rmsnorm(O)


def test_rmsnorm_scale_invariance_and_unit_rms():
    x = rand(5, 64)
    a = O.rms_norm(x, np.ones(64), 1e-12)
    b = O.rms_norm(7.5 * x, np.ones(64), 1e-12)
    np.testing.assert_allclose(a, b, rtol=1e-9)
    np.testing.assert_allclose(np.sqrt(np.mean(a * a, -1)), 1.0, rtol=1e-9)


# ------------------------------------------------------- FFN hidden rule ---
def test_ffn_hidden_rule_reproduces_printed_sizes():
    shapes = {l.split()[0]: l.split()[1] for l in read_golden("model_shapes.txt")}
    assert O.ffn_hidden_dim(int(shapes["dim"]), int(shapes["multiple_of"]),
                            float(shapes["ffn_dim_multiplier"])) == int(shapes["ffn_hidden_8b"])
    assert O.ffn_hidden_dim(int(shapes["char_dim"]), int(shapes["char_multiple_of"])) == 1536
    # GQA-heavy workload (hidden 768, multiple_of 256) gives its FFN hidden 2048.
    assert O.ffn_hidden_dim(768, 256) == 2048


# ------------------------------------------------------------------- RoPE ---
def test_rope_frequencies_match_printed_table():
    printed = np.array([float(v) for line in read_golden("rope_freqs_theta500000_hd128.txt")
                        for v in line.split()])
    assert printed.shape == (64,)
    got = O.rope_inverse_frequencies(128, 500000.0)
    # The page prints 5 significant figures.
    np.testing.assert_allclose(got, printed, rtol=6e-5)
    # Exponents are i/64 (the printed 0, 0.0156, ..., 0.9844 split of [0,1)).
    np.testing.assert_allclose(-np.log(got) / np.log(500000.0), np.arange(64) / 64, atol=1e-12)


def pin_rope_unit_vectors(o):
    # e_{2i} at position m rotates to cos(m t_i) e_{2i} + sin(m t_i) e_{2i+1};
    # e_{2i+1} rotates to -sin(m t_i) e_{2i} + cos(m t_i) e_{2i+1}.
    hd, theta = 16, 500000.0
    for m in (0, 1, 5, 8191):
        for i in (0, 3, 7):
            # i-th pair frequency written out from the definition theta^(-2i/hd)
            t = theta ** (-(2 * i) / hd)
            x = np.zeros((1, 1, hd)); x[0, 0, 2 * i] = 1.0
            y = o.apply_rope(x, [m], theta)[0, 0]
            want = np.zeros(hd); want[2 * i] = math.cos(m * t); want[2 * i + 1] = math.sin(m * t)
            np.testing.assert_allclose(y, want, atol=1e-12)
            x = np.zeros((1, 1, hd)); x[0, 0, 2 * i + 1] = 1.0
            y = o.apply_rope(x, [m], theta)[0, 0]
            want = np.zeros(hd); want[2 * i] = -math.sin(m * t); want[2 * i + 1] = math.cos(m * t)
            np.testing.assert_allclose(y, want, atol=1e-12)


def test_rope_unit_vectors_closed_form():
    pin_rope_unit_vectors(O)


def test_rope_identity_at_position_zero_and_norm_preserving():
    x = rand(3, 4, 32)
    np.testing.assert_array_equal(O.apply_rope(x, [0, 0, 0], 500000.0), x)
    y = O.apply_rope(x, [0, 17, 4000], 500000.0)
    pair_norm = lambda a: a[..., 0::2] ** 2 + a[..., 1::2] ** 2
    np.testing.assert_allclose(pair_norm(y), pair_norm(x), rtol=1e-12)


def test_rope_equals_explicit_rotation_matrix():
    # The joto.ai blog describes RoPE as a block-diagonal rotation matrix R.
    hd, theta, m = 8, 500000.0, 37
    x = rand(1, 1, hd)
    R = np.zeros((hd, hd))
    for i in range(hd // 2):
        a = m * theta ** (-(2 * i) / hd)
        R[2 * i:2 * i + 2, 2 * i:2 * i + 2] = [[math.cos(a), -math.sin(a)], [math.sin(a), math.cos(a)]]
    np.testing.assert_allclose(O.apply_rope(x, [m], theta)[0, 0], R @ x[0, 0], atol=1e-13)


def test_rope_relative_position_property():
    # <R_m q, R_n k> depends only on n - m.
    q, k = rand(1, 1, 64), rand(1, 1, 64)
    dots = []
    for shift in (0, 3, 1000, 7777):
        qm = O.apply_rope(q, [5 + shift], 500000.0)
        kn = O.apply_rope(k, [12 + shift], 500000.0)
        dots.append(float(np.sum(qm * kn)))
    np.testing.assert_allclose(dots, dots[0], rtol=1e-10)


# -------------------------------------------------------------- attention ---
def test_causal_mask_matches_printed_17x17():
    printed = np.array([[0.0 if tok == "0." else -np.inf for tok in line.split()]
                        for line in read_golden("causal_mask_17.txt")])
    np.testing.assert_array_equal(O.causal_mask(17, 17, 0), printed)
    # With a cache offset the same pattern is shifted right by start_pos.
    m = O.causal_mask(3, 8, 5)
    assert np.isneginf(m[0, 6]) and m[0, 5] == 0 and m[2, 7] == 0


def brute_force_attention(q, k, v, start_pos, n_rep):
    S, H, hd = q.shape
    out = np.zeros_like(q)
    for t in range(S):
        for h in range(H):
            g = h // n_rep
            s = [sum(q[t, h, d] * k[j, g, d] for d in range(hd)) / math.sqrt(hd)
                 for j in range(start_pos + t + 1)]
            mx = max(s)
            e = [math.exp(x - mx) for x in s]
            z = sum(e)
            for d in range(hd):
                out[t, h, d] = sum(e[j] * v[j, g, d] for j in range(len(e))) / z
    return out


def pin_attention_brute_force(o):
    for (S, H, KV, hd, P) in [(5, 4, 2, 4, 0), (3, 6, 3, 2, 4), (4, 2, 1, 8, 1)]:
        q, k, v = rand(S, H, hd), rand(P + S, KV, hd), rand(P + S, KV, hd)
        np.testing.assert_allclose(o.gqa_attention(q, k, v, P), brute_force_attention(q, k, v, P, H // KV),
                                   rtol=1e-11, atol=1e-12)


def test_attention_brute_force():
    pin_attention_brute_force(O)


def test_attention_first_row_is_v0_and_rows_sum_to_one():
    q, k, v = rand(6, 4, 8), rand(6, 2, 8), rand(6, 2, 8)
    out, p = O.gqa_attention(q, k, v, 0, return_probs=True)
    np.testing.assert_array_equal(out[0, 0], v[0, 0])
    np.testing.assert_array_equal(out[0, 3], v[0, 1])
    np.testing.assert_allclose(p.sum(-1), 1.0, rtol=1e-13)
    assert np.all(p[:, np.triu_indices(6, 1)[0], np.triu_indices(6, 1)[1]] == 0)


def test_attention_causality_under_perturbation():
    S, H, KV, hd = 9, 4, 2, 8
    q, k, v = rand(S, H, hd), rand(S, KV, hd), rand(S, KV, hd)
    base = O.gqa_attention(q, k, v)
    for t in (0, 4, 7):
        q2, k2, v2 = q.copy(), k.copy(), v.copy()
        q2[t + 1:] += 3.0; k2[t + 1:] -= 2.0; v2[t + 1:] *= -5.0
        np.testing.assert_array_equal(O.gqa_attention(q2, k2, v2)[:t + 1], base[:t + 1])


def test_gqa_reduces_to_mha_and_matches_repeat_kv():
    S, H, hd = 7, 4, 8
    q, k, v = rand(S, H, hd), rand(S, H, hd), rand(S, H, hd)
    # KV == H: every head has its own K/V (plain multi-head attention).
    mha = np.stack([O.gqa_attention(q[:, h:h + 1], k[:, h:h + 1], v[:, h:h + 1])[:, 0]
                    for h in range(H)], axis=1)
    np.testing.assert_allclose(O.gqa_attention(q, k, v), mha, rtol=1e-13)
    # KV < H: explicit repeat_kv expansion (each KV head repeated n_rep times
    # in place, as the from-scratch page's repeat_kv does), then plain MHA.
    KV = 2
    k2, v2 = rand(S, KV, hd), rand(S, KV, hd)
    rep = np.repeat(np.arange(KV), H // KV)            # [0,0,1,1]
    ke, ve = k2[:, rep], v2[:, rep]
    np.testing.assert_allclose(O.gqa_attention(q, k2, v2), O.gqa_attention(q, ke, ve), rtol=1e-13)


# -------------------------------------------------------------------- FFN ---
def test_silu_closed_forms():
    assert O.silu(0.0) == 0.0
    np.testing.assert_allclose(O.silu(1.0), 1.0 / (1.0 + math.exp(-1.0)), rtol=1e-15)
    np.testing.assert_allclose(O.silu(40.0), 40.0, rtol=1e-15)
    assert abs(O.silu(-40.0)) < 1e-15


def pin_swiglu_scalar(o):
    # One-dimensional block: x=[x0], w1=[[a]], w3=[[b]], w2=[[c]] gives c*silu(a x0)*(b x0).
    a, b, c, x0 = 0.7, -1.3, 2.5, 1.9
    got = o.swiglu_ffn(np.array([[x0]]), np.array([[a]]), np.array([[c]]), np.array([[b]]))
    want = c * (a * x0) / (1 + math.exp(-a * x0)) * (b * x0)
    np.testing.assert_allclose(got[0, 0], want, rtol=1e-14)


def test_swiglu_scalar():
    pin_swiglu_scalar(O)


# ------------------------------------------------------------------ block ---
def tiny_cfg(D=16, H=4, KV=2, F=24):
    return dict(dim=D, n_heads=H, n_kv_heads=KV, head_dim=D // H, ffn_hidden=F,
                norm_eps=1e-5, rope_theta=500000.0)


def tiny_layer(cfg, scale=0.2):
    D, H, KV, hd, F = cfg["dim"], cfg["n_heads"], cfg["n_kv_heads"], cfg["head_dim"], cfg["ffn_hidden"]
    return dict(attention_norm=1 + 0.1 * rand(D), ffn_norm=1 + 0.1 * rand(D),
                wq=rand(H * hd, D, scale=scale), wk=rand(KV * hd, D, scale=scale),
                wv=rand(KV * hd, D, scale=scale), wo=rand(D, H * hd, scale=scale),
                w1=rand(F, D, scale=scale), w2=rand(D, F, scale=scale), w3=rand(F, D, scale=scale))


def test_block_with_zero_projections_is_identity():
    cfg = tiny_cfg()
    layer = tiny_layer(cfg)
    layer["wo"] = np.zeros_like(layer["wo"]); layer["w2"] = np.zeros_like(layer["w2"])
    x = rand(2, 5, 16)
    kc = np.zeros((2, 5, 2, 4)); vc = np.zeros((2, 5, 2, 4))
    np.testing.assert_array_equal(O.decoder_block(x, layer, cfg, kc, vc), x)


def bf16_scalar(a):
    """One value rounded to bfloat16 (8 significant bits, ties to even), in
    plain Python: Python's round() of a float ties to even."""
    if a == 0.0:
        return 0.0
    m, e = math.frexp(a)
    return math.ldexp(round(m * 256.0), e - 8)


def brute_force_block(x, layer, cfg, start_pos, k_hist, v_hist, store=lambda a: a):
    """Scalar-loop restatement of one block for a single sequence [S, D].
    ``store`` is applied to every activation the bf16 variant holds in bf16
    (identity: the exact block)."""
    S, D = x.shape
    H, KV, hd = cfg["n_heads"], cfg["n_kv_heads"], cfg["head_dim"]
    eps, theta = cfg["norm_eps"], cfg["rope_theta"]

    def norm(row, w):
        r = math.sqrt(sum(a * a for a in row) / len(row) + eps)
        return [store(a / r * wi) for a, wi in zip(row, w)]

    def lin(row, W):
        return [sum(W[o_, i] * row[i] for i in range(len(row))) for o_ in range(W.shape[0])]

    def rot(vec, m):
        out = list(vec)
        for i in range(hd // 2):
            ang = m * theta ** (-(2 * i) / hd)
            a, b = vec[2 * i], vec[2 * i + 1]
            out[2 * i] = a * math.cos(ang) - b * math.sin(ang)
            out[2 * i + 1] = a * math.sin(ang) + b * math.cos(ang)
        return out

    ks = [list(r) for r in k_hist]; vs = [list(r) for r in v_hist]   # each [KV*hd]
    qs = []
    for t in range(S):
        xn = norm(x[t], layer["attention_norm"])
        q, k, v = lin(xn, layer["wq"]), lin(xn, layer["wk"]), [store(a) for a in lin(xn, layer["wv"])]
        m = start_pos + t
        q = [store(a) for a in sum((rot(q[h * hd:(h + 1) * hd], m) for h in range(H)), [])]
        k = [store(a) for a in sum((rot(k[g * hd:(g + 1) * hd], m) for g in range(KV)), [])]
        qs.append(q); ks.append(k); vs.append(v)
    out = np.zeros((S, D))
    for t in range(S):
        att = []
        for h in range(H):
            g = h // (H // KV)
            sc = [sum(qs[t][h * hd + d] * ks[j][g * hd + d] for d in range(hd)) / math.sqrt(hd)
                  for j in range(start_pos + t + 1)]
            mx = max(sc); e = [math.exp(s - mx) for s in sc]; z = sum(e)
            e = [store(a) for a in e]      # probabilities stored; their sum stays exact
            att += [store(sum(e[j] * vs[j][g * hd + d] for j in range(len(e))) / z) for d in range(hd)]
        hrow = [store(a + b) for a, b in zip(x[t], lin(att, layer["wo"]))]
        hn = norm(hrow, layer["ffn_norm"])
        g1, g3 = lin(hn, layer["w1"]), lin(hn, layer["w3"])
        gate = [store(a / (1 + math.exp(-a)) * b) for a, b in zip(g1, g3)]
        out[t] = [store(a + b) for a, b in zip(hrow, lin(gate, layer["w2"]))]
    return out, ks, vs


def test_block_brute_force_with_cache_offset():
    cfg = tiny_cfg()
    layer = tiny_layer(cfg)
    P, S = 3, 4
    k_hist, v_hist = rand(P, 8), rand(P, 8)
    x = rand(1, S, 16)
    kc = np.zeros((1, P + S, 2, 4)); vc = np.zeros((1, P + S, 2, 4))
    kc[0, :P] = k_hist.reshape(P, 2, 4); vc[0, :P] = v_hist.reshape(P, 2, 4)
    got = O.decoder_block(x, layer, cfg, kc, vc, start_pos=P)
    want, ks, vs = brute_force_block(x[0], layer, cfg, P, k_hist, v_hist)
    np.testing.assert_allclose(got[0], want, rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(kc[0].reshape(P + S, 8), np.array(ks), rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(vc[0].reshape(P + S, 8), np.array(vs), rtol=1e-12, atol=1e-13)


def test_bf16_round_hand_values_and_library_conversion():
    # ties go to the even neighbour; 1/3 = 1.0101010|101..b x 2^-2 rounds up
    cases = {1 + 2 ** -8: 1.0, 1 + 3 * 2 ** -8: 1 + 2 ** -6, -(1 + 2 ** -8): -1.0, 0.0: 0.0,
             1 + 2 ** -7: 1 + 2 ** -7, 3.140625: 3.140625, 1 / 3: 0.333984375, 255.5: 256.0, 254.5: 254.0}
    for a, want in cases.items():
        assert O.bf16_round(np.array([a]))[0] == want, a
        assert bf16_scalar(a) == want, a
    # float32 inputs against torch's float32 -> bfloat16 conversion (round to nearest even)
    import torch
    g = torch.Generator().manual_seed(3)
    x = torch.randn(200_000, generator=g) * torch.exp(torch.randn(200_000, generator=g) * 6)
    want = x.to(torch.bfloat16).to(torch.float64).numpy()
    np.testing.assert_array_equal(O.bf16_round(x.to(torch.float64).numpy()), want)


def test_bf16_storage_variant_matches_brute_force():
    """The bf16 precision variant rounds at exactly the step boundaries the
    scalar restatement rounds at (a skipped or extra rounding shows as a
    2^-9-sized difference)."""
    cfg = tiny_cfg()
    layer = tiny_layer(cfg)
    P, S = 3, 4
    k_hist = O.bf16_round(rand(P, 8)); v_hist = O.bf16_round(rand(P, 8))
    x = O.bf16_round(rand(1, S, 16))
    kc = np.zeros((1, P + S, 2, 4)); vc = np.zeros((1, P + S, 2, 4))
    kc[0, :P] = k_hist.reshape(P, 2, 4); vc[0, :P] = v_hist.reshape(P, 2, 4)
    got = O.decoder_block(x, layer, cfg, kc, vc, start_pos=P, rounding="bf16")
    want, ks, vs = brute_force_block(x[0], layer, cfg, P, k_hist, v_hist, store=bf16_scalar)
    np.testing.assert_allclose(got[0], want, rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(kc[0].reshape(P + S, 8), np.array(ks), rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(vc[0].reshape(P + S, 8), np.array(vs), rtol=1e-12, atol=1e-14)
    assert np.array_equal(O.bf16_round(got), got)            # the block output is stored in bf16
    exact = O.decoder_block(x, layer, cfg, kc.copy(), vc.copy(), start_pos=P)
    rel = np.abs(got - exact).max() / np.abs(exact).max()
    assert 1e-4 < rel < 2e-2                                  # rounding noise, not a different function
    rows, k, v = O.decoder_block_rows(x[0], layer, cfg, [0, 2, 3], k_hist.reshape(P, 2, 4),
                                      v_hist.reshape(P, 2, 4), P, rounding="bf16")
    np.testing.assert_allclose(rows, want[[0, 2, 3]], rtol=1e-12, atol=1e-14)
    # the LM head of the variant stores the normalised rows
    w_out = rand(11, 16)
    lg, _ = O.lm_head(got[0], np.ones(16), w_out, 1e-5, rounding="bf16")
    np.testing.assert_allclose(lg, O.bf16_round(O.rms_norm(got[0], np.ones(16), 1e-5)) @ w_out.T, rtol=1e-13)


def test_block_rows_matches_brute_force_block():
    cfg = tiny_cfg()
    layer = tiny_layer(cfg)
    P, S = 2, 6
    k_hist, v_hist = rand(P, 8), rand(P, 8)
    x = rand(S, 16)
    want, ks, vs = brute_force_block(x, layer, cfg, P, k_hist, v_hist)
    rows = [0, 3, 5]
    got, k, v = O.decoder_block_rows(x, layer, cfg, rows, k_hist.reshape(P, 2, 4), v_hist.reshape(P, 2, 4), P)
    np.testing.assert_allclose(got, want[rows], rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(k.reshape(S, 8), np.array(ks[P:]), rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(v.reshape(S, 8), np.array(vs[P:]), rtol=1e-12, atol=1e-13)


def test_prefill_equals_chunked_prefill_equals_token_by_token_decode():
    # The KV-cache argument of "Build your own Llama 3 from scratch" §3.3: the
    # cached path must give the same result as the full causal pass.
    cfg = tiny_cfg()
    layers = [tiny_layer(cfg) for _ in range(2)]
    B, S = 2, 7
    x = rand(B, S, 16)
    full, _, _ = O.forward_stack(x, layers, cfg)
    kcs = [np.zeros((B, S, 2, 4)) for _ in layers]; vcs = [np.zeros((B, S, 2, 4)) for _ in layers]
    a, _, _ = O.forward_stack(x[:, :4], layers, cfg, kcs, vcs, start_pos=0)
    b, _, _ = O.forward_stack(x[:, 4:], layers, cfg, kcs, vcs, start_pos=4)
    np.testing.assert_allclose(np.concatenate([a, b], 1), full, rtol=1e-11, atol=1e-12)
    kcs = [np.zeros((B, S, 2, 4)) for _ in layers]; vcs = [np.zeros((B, S, 2, 4)) for _ in layers]
    steps = [O.forward_stack(x[:, t:t + 1], layers, cfg, kcs, vcs, start_pos=t)[0] for t in range(S)]
    np.testing.assert_allclose(np.concatenate(steps, 1), full, rtol=1e-11, atol=1e-12)


# ---------------------------------------------------------------- LM head ---
def test_lm_head_one_hot_and_planted_max_and_ties():
    D, V = 8, 11
    W = rand(V, D)
    h = np.zeros((1, D)); h[0, 3] = 2.0
    logits, ids = O.lm_head(h, np.ones(D), W, 0.0)
    # RMSNorm of 2*e_3 is sqrt(D)*e_3, so the logits are sqrt(D) * column 3 of W.
    np.testing.assert_allclose(logits[0], math.sqrt(D) * W[:, 3], rtol=1e-14)
    W2 = W.copy(); W2[7] = 50.0
    assert O.lm_head(rand(3, D) ** 2 + 0.1, np.ones(D), W2, 1e-5)[1].tolist() == [7, 7, 7]
    W3 = np.zeros((V, D)); W3[[2, 5, 9]] = 1.0
    assert O.lm_head(np.ones((1, D)), np.ones(D), W3, 1e-5)[1][0] == 2


def test_embed_gathers_rows():
    table = rand(10, 4)
    np.testing.assert_array_equal(O.embed([[3, 0, 9]], table)[0], table[[3, 0, 9]])


# ----------------------------------------------- planted mistakes are caught ---
def mutated(**overrides):
    ns = types.SimpleNamespace(**{k: getattr(O, k) for k in O.__all__})
    for k, v in overrides.items():
        setattr(ns, k, v)
    return ns


def test_pins_catch_planted_mistakes():
    def rope_split_half(x, positions, theta):
        x = np.asarray(x, float); hd = x.shape[-1]
        ang = O.rope_angles(positions, hd, theta)[:, None, :]
        a, b = x[..., :hd // 2], x[..., hd // 2:]
        return np.concatenate([a * np.cos(ang) - b * np.sin(ang), a * np.sin(ang) + b * np.cos(ang)], -1)

    def rope_wrong_sign(x, positions, theta):
        return O.apply_rope(x, -np.asarray(positions, float), theta)

    def attention_mod_mapping(q, k, v, start_pos=0, return_probs=False):
        H, KV = q.shape[1], k.shape[1]
        perm = np.array([h % KV for h in range(H)])
        out = np.stack([O.gqa_attention(q[:, h:h + 1], k[:, perm[h]:perm[h] + 1],
                                        v[:, perm[h]:perm[h] + 1], start_pos)[:, 0] for h in range(H)], 1)
        return out

    def attention_wrong_scale(q, k, v, start_pos=0, return_probs=False):
        return O.gqa_attention(np.asarray(q) / math.sqrt(q.shape[-1]), k, v, start_pos)

    def attention_strict_mask(q, k, v, start_pos=0, return_probs=False):
        # excludes the diagonal (a position does not see itself)
        S = q.shape[0]
        out = O.gqa_attention(q, k, v, start_pos)
        out[0] = 0.0
        return out

    def rmsnorm_no_eps(x, w, eps):
        return O.rms_norm(x, w, 0.0)

    def swiglu_swapped(x, w1, w2, w3):
        return O.swiglu_ffn(x, w3, w2, w1)

    cases = [
        (pin_rope_unit_vectors, dict(apply_rope=rope_split_half)),
        (pin_rope_unit_vectors, dict(apply_rope=rope_wrong_sign)),
        (pin_attention_brute_force, dict(gqa_attention=attention_mod_mapping)),
        (pin_attention_brute_force, dict(gqa_attention=attention_wrong_scale)),
        (pin_attention_brute_force, dict(gqa_attention=attention_strict_mask)),
        (pin_rmsnorm, dict(rms_norm=rmsnorm_no_eps)),
        (pin_swiglu_scalar, dict(swiglu_ffn=swiglu_swapped)),
    ]
    for pin, override in cases:
        with pytest.raises(AssertionError):
            pin(mutated(**override))


def test_greedy_generation_with_cache_equals_recomputing_the_whole_sequence():
    # The KV-cache path of the inference section must pick the same tokens as
    # re-running the full causal model on the growing sequence every step.
    cfg = tiny_cfg()
    layers = [tiny_layer(cfg, scale=0.4) for _ in range(2)]
    V, D = 23, 16
    table, w_out, nw = rand(V, D), rand(V, D), 1 + 0.1 * rand(D)
    prompt = RNG.integers(0, V, (2, 5))
    toks, gaps = O.generate_greedy(prompt, table, layers, nw, w_out, cfg, 6)
    seq = prompt.copy()
    for step in range(6):
        h, _, _ = O.forward_stack(O.embed(seq, table), layers, cfg)
        logits, nxt = O.lm_head(h[:, -1], nw, w_out, cfg["norm_eps"])
        np.testing.assert_array_equal(toks[:, step], nxt)
        seq = np.concatenate([seq, nxt[:, None]], 1)
    assert np.all(gaps >= 0)


def test_greedy_generation_holds_eos():
    cfg = tiny_cfg()
    layers = [tiny_layer(cfg)]
    V, D = 7, 16
    table, w_out = rand(V, D), np.zeros((V, D))
    # all logits tie at 0, so the lowest index (0) wins every step; with 0 as
    # the end token every sequence ends at once and stays ended
    toks, _ = O.generate_greedy(RNG.integers(0, V, (2, 3)), table, layers, np.ones(D), w_out, cfg, 4, eos_id=0)
    assert np.all(toks == 0)


# ----------------------------------------------------------- document mask ---
def test_document_mask_single_document_is_plain_causal():
    q, k, v = rand(9, 4, 8), rand(9, 2, 8), rand(9, 2, 8)
    np.testing.assert_array_equal(O.gqa_attention(q, k, v, doc_start=np.zeros(9, int)), O.gqa_attention(q, k, v))


def test_document_mask_brute_force():
    S, H, KV, hd = 8, 4, 2, 4
    q, k, v = rand(S, H, hd), rand(S, KV, hd), rand(S, KV, hd)
    ds = np.array([0, 0, 0, 3, 3, 5, 5, 5])
    got = O.gqa_attention(q, k, v, doc_start=ds)
    for t in range(S):
        for h in range(H):
            g = h // (H // KV)
            keys = range(ds[t], t + 1)
            sc = [sum(q[t, h, d] * k[j, g, d] for d in range(hd)) / math.sqrt(hd) for j in keys]
            mx = max(sc); e = [math.exp(x - mx) for x in sc]; z = sum(e)
            want = [sum(e[i] * v[j, g, d] for i, j in enumerate(keys)) / z for d in range(hd)]
            np.testing.assert_allclose(got[t, h], want, rtol=1e-11, atol=1e-12)


def test_packed_documents_equal_separate_documents():
    # Two documents packed into one sequence, positions running on: each
    # document's block outputs equal running it alone from position 0 (the
    # attention sees only its own document, and RoPE scores depend only on
    # relative positions).
    cfg = tiny_cfg()
    layers = [tiny_layer(cfg) for _ in range(2)]
    a, b = rand(1, 5, 16), rand(1, 7, 16)
    packed = np.concatenate([a, b], 1)
    ds = np.array([[0] * 5 + [5] * 7])
    out, _, _ = O.forward_stack(packed, layers, cfg, doc_start=ds)
    alone_a, _, _ = O.forward_stack(a, layers, cfg)
    alone_b, _, _ = O.forward_stack(b, layers, cfg)
    np.testing.assert_allclose(out[:, :5], alone_a, rtol=1e-10, atol=1e-11)
    np.testing.assert_allclose(out[:, 5:], alone_b, rtol=1e-10, atol=1e-11)


# ------------------------------------------------------ top-p sampling ---
def _word(u):
    """The 64-bit word whose draw fraction is u (0 <= u < 1)."""
    return int(u * 2.0 ** 64)


def pin_philox(o):
    # Philox-4x64-10 is also numpy's Philox bit generator, which advances its
    # counter before each block: block for counter c = random_raw after
    # starting from c - 1.
    for key, ctr in [((0, 0), (1, 0, 0, 0)), ((7, 0), (5, 3, 0, 0)),
                     ((0x0123456789ABCDEF, 0xFEDCBA9876543210), (2 ** 63 + 11, 17, 2 ** 40, 9))]:
        k = key[0] | (key[1] << 64)
        start = ((ctr[0] - 1) | (ctr[1] << 64) | (ctr[2] << 128) | (ctr[3] << 192))
        bg = np.random.Philox(key=k, counter=start)
        want = [int(w) for w in bg.random_raw(4)]
        assert o.philox4x64(ctr, key) == want
    # the published known-answer vector for zero counter and key
    assert o.philox4x64((0, 0, 0, 0), (0, 0)) == [0x16554D9ECA36314C, 0xDB20FE9D672D0FDC,
                                                  0xD7E772CEE186176B, 0x7E68B68AEC7BA23B]


def pin_top_p_hand_example(o):
    # p = (0.05, 0.5, 0.15, 0.3): ranked 1, 3, 2, 0 with mass before 0, .5, .8, .95.
    # top_p = 0.6 keeps tokens 1 and 3 (kept mass 0.8, running 0.5, 0.8 by index).
    lg = np.log([0.05, 0.5, 0.15, 0.3])
    for u, want in [(0.0, 1), (0.3, 1), (0.62, 1), (0.63, 3), (0.9, 3), (0.999, 3)]:
        assert o.top_p_sample(lg, 1.0, 0.6, _word(u))[0] == want, u
    # p = (.25, .5, .25), top_p = 0.5: token 0 is kept (the mass ranked before
    # it is exactly 0.5), its tie token 2 is ranked after it and dropped
    tie = np.log([0.25, 0.5, 0.25])
    assert o.top_p_sample(tie, 1.0, 0.5, _word(0.2))[0] == 0
    assert o.top_p_sample(tie, 1.0, 0.5, _word(0.9))[0] == 1
    # top_p = 0.49 keeps only the top token
    assert o.top_p_sample(lg, 1.0, 0.49, _word(0.999))[0] == 1


def pin_top_p_ties(o):
    # eight equal logits: ranked by index, the mass before token k is k/8
    # (exact in binary), so top_p = 0.5 keeps tokens 0..4 (draw floor(5u))
    # and top_p = 0.45 keeps 0..3
    lg = np.zeros(8)
    for k in range(5):
        assert o.top_p_sample(lg, 0.7, 0.5, _word((k + 0.5) / 5))[0] == k
    for k in range(4):
        assert o.top_p_sample(lg, 1.3, 0.45, _word((k + 0.5) / 4))[0] == k


def pin_top_p_limits(o):
    rng = np.random.default_rng(4)
    for _ in range(20):
        lg = rng.standard_normal(50) * 3
        w = int(rng.integers(0, 2 ** 63)) * 2 + 1
        # a vanishing top_p keeps only the most probable token; temperature 0 is argmax
        assert o.top_p_sample(lg, 0.8, 1e-12, w)[0] == int(np.argmax(lg))
        assert o.top_p_sample(lg, 0.0, 0.9, w)[0] == int(np.argmax(lg))
        # dividing by T is the same as scaling the logits by 1/T (exact for T = 2)
        assert o.top_p_sample(lg * 2, 2.0, 0.9, w)[0] == o.top_p_sample(lg, 1.0, 0.9, w)[0]


def pin_top_p_frequencies(o):
    # The law of the draw: frequencies over many independent words equal the
    # renormalised kept probabilities (here p = (.4, .25, .2, .1, .05), top_p
    # 0.7 keeps the three largest: .4/.85, .25/.85, .2/.85).
    p = np.array([0.1, 0.4, 0.05, 0.25, 0.2])
    lg = np.log(p)
    n = 20000
    counts = np.zeros(5)
    for i in range(n):
        counts[o.top_p_sample(lg, 1.0, 0.7, o.sampling_word(99, i, 3))[0]] += 1
    want = np.array([0, 0.4, 0, 0.25, 0.2]) / 0.85
    sigma = np.sqrt(want * (1 - want) / n) + 1e-12
    assert np.all(np.abs(counts / n - want) <= 5 * sigma + 1e-12), counts / n


def test_philox_matches_numpy_and_known_answer():
    pin_philox(O)


def test_top_p_hand_example():
    pin_top_p_hand_example(O)


def test_top_p_ties_follow_index_order():
    pin_top_p_ties(O)


def test_top_p_limits_and_temperature():
    pin_top_p_limits(O)


def test_top_p_draw_frequencies():
    pin_top_p_frequencies(O)


def test_sampling_pins_catch_planted_mistakes():
    def philox_swapped_constants(counter, key, rounds=10):
        return O.philox4x64(counter, (key[1], key[0]), rounds)

    def keep_by_inclusive_sum(logits, temperature, top_p, word):
        # drops a token once the mass up to and INCLUDING it exceeds top_p
        z = np.asarray(logits, float) / temperature
        p = np.exp(z - z.max()); p /= p.sum()
        order = np.argsort(-p, kind="stable")
        keep = np.zeros(p.shape, bool)
        keep[order[np.cumsum(p[order]) <= top_p]] = True
        keep[order[0]] = True
        idx = np.nonzero(keep)[0]
        run = np.cumsum(p[idx])
        return int(idx[min(np.searchsorted(run, word / 2.0 ** 64 * run[-1], "right"), len(idx) - 1)]), (0, 0)

    def no_renormalisation(logits, temperature, top_p, word):
        # draws u against the full mass instead of the kept mass
        tok, m = O.top_p_sample(logits, temperature, top_p, word)
        z = np.asarray(logits, float) / temperature
        p = np.exp(z - z.max()); p /= p.sum()
        u = word / 2.0 ** 64
        order = np.argsort(-p, kind="stable")
        before = np.cumsum(p[order]) - p[order]
        idx = np.sort(order[before <= top_p])
        run = np.cumsum(p[idx])
        return int(idx[min(np.searchsorted(run, u, "right"), len(idx) - 1)]), m

    def temperature_multiplies(logits, temperature, top_p, word):
        return O.top_p_sample(np.asarray(logits, float) * temperature * temperature, temperature, top_p, word)

    cases = [
        (pin_philox, dict(philox4x64=philox_swapped_constants)),
        (pin_top_p_hand_example, dict(top_p_sample=keep_by_inclusive_sum)),
        (pin_top_p_frequencies, dict(top_p_sample=no_renormalisation)),
        (pin_top_p_limits, dict(top_p_sample=temperature_multiplies)),
    ]
    for pin, override in cases:
        with pytest.raises(AssertionError):
            pin(mutated(**override))
