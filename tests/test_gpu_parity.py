"""GPU parity: every step of the decoder, through the C ABI, against the fp64
oracle on the same seeded inputs.  Tolerance |gpu - oracle| <= 2e-2 +
2e-2*|oracle| per element for bf16 paths, 1e-4 + 1e-4*|oracle| for fp32;
argmax ids must match wherever the oracle's top-2 logit gap exceeds 1e-2."""
import numpy as np
import pytest
import torch

from helpers import GuardArena, assert_argmax, assert_close, f64, oracle_cfg, oracle_layer
from llama_decoder_only_rmsnorm_b200 import binding as B
from llama_decoder_only_rmsnorm_b200 import inputs as I
from llama_decoder_only_rmsnorm_b200.model import Llama3Stack
from oracle import llama3_oracle as O

pytestmark = pytest.mark.gpu
DEV = "cuda"


G = None   # the running test's guard arena: every output / cache / workspace sits between guard bands


@pytest.fixture(autouse=True)
def _gpu_state():
    global G
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    B.llama3_set_kernel_path(0)
    G = GuardArena(DEV)
    yield
    B.llama3_set_kernel_path(0)
    torch.cuda.synchronize()
    assert B.llama3_device_status() == 0, "device status word set"
    G.check()


def Stack(*a, **k):
    """Llama3Stack whose buffers all come from the guard arena."""
    return Llama3Stack(*a, alloc=G.alloc, **k)


def wl(name, **kw):
    return I.WORKLOADS[name].replace(**kw)


def small_bf16(**kw):
    d = dict(name="small", dim=512, n_layers=2, n_heads=8, n_kv_heads=2, ffn_hidden=1024, vocab=1000,
             batch=3, seq=70, dtype="bf16", input_kind="activations", seed=77)
    d.update(kw)
    return I.Workload(**d)


# ------------------------------------------------------------------ RMSNorm
@pytest.mark.parametrize("dtype,D,H,rows", [("bf16", 4096, 32, 37), ("bf16", 576, 9, 37), ("f32", 64, 4, 37),
                                            ("bf16", 4096, 32, 600), ("bf16", 8192, 64, 3), ("bf16", 960, 10, 513), ("bf16", 960, 10, 5)])
def test_rmsnorm(dtype, D, H, rows):
    tdt = torch.float32 if dtype == "f32" else torch.bfloat16
    g = torch.Generator(device="cpu").manual_seed(5)
    stride = D + 64
    x = (torch.randn((rows, stride), generator=g) * 3).to(tdt).to(DEV)
    nw = (1 + 0.1 * torch.randn((D,), generator=g)).to(tdt).to(DEV)
    y = G.empty((rows, D), dtype=tdt, device=DEV)
    cfg = B.make_config(D, H, 1, 8 * D, dtype=dtype)
    B.llama3_rmsnorm(cfg, x, stride, nw, y, rows)
    want = O.rms_norm(f64(x)[:, :D], f64(nw), 1e-5)
    assert_close(y, want, dtype, "rmsnorm")


# ------------------------------------------------------------------ Linear
@pytest.mark.parametrize("m,n,k", [(128, 256, 64), (300, 264, 200), (1000, 1536, 512), (77, 4096, 4096),
                                   (2048, 6144, 4096)])
@pytest.mark.parametrize("residual", [False, True])
@pytest.mark.parametrize("path", [0, 1])
def test_linear(m, n, k, residual, path):
    if path == 1 and m * n > 2_000_000:
        pytest.skip("SIMT cross-check only on the smaller shapes")
    B.llama3_set_kernel_path(path)
    g = torch.Generator(device="cpu").manual_seed(m * 7 + n + k)
    x = torch.randn((m, k), generator=g).to(torch.bfloat16).to(DEV)
    w = (torch.randn((n, k), generator=g) * 0.05).to(torch.bfloat16).to(DEV)
    r = torch.randn((m, n), generator=g).to(torch.bfloat16).to(DEV) if residual else None
    y = G.empty((m, n), dtype=torch.bfloat16, device=DEV)
    cfg = B.make_config(512, 8, 8, 1024)
    ws = G.empty((m * n * 4,), dtype=torch.uint8, device=DEV)
    B.llama3_linear(cfg, x, w, r, y, m, n, k, ws, ws.numel())
    want = f64(x) @ f64(w).T + (f64(r) if residual else 0.0)
    assert_close(y, want, "bf16", f"linear {m}x{n}x{k}")


def test_linear_in_place_residual():
    m, n, k = 256, 512, 512
    g = torch.Generator(device="cpu").manual_seed(3)
    x = torch.randn((m, k), generator=g).to(torch.bfloat16).to(DEV)
    w = (torch.randn((n, k), generator=g) * 0.05).to(torch.bfloat16).to(DEV)
    y = torch.randn((m, n), generator=g).to(torch.bfloat16).to(DEV)
    want = f64(x) @ f64(w).T + f64(y)
    B.llama3_linear(B.make_config(512, 8, 8, 1024), x, w, y, y, m, n, k)
    assert_close(y, want, "bf16", "in-place residual")


@pytest.mark.parametrize("n,k,residual", [(768, 512, False), (4096, 4096, True), (264, 200, True)])
def test_linear_cta_pairs_match_single_cta_bit_for_bit(n, k, residual):
    """From 256 rows on, the prefill GEMMs run on CTA pairs (256-row tiles,
    half of each weight tile per CTA); below, on single CTAs.  Both reduce
    every output element over k in the same order, so the first 255 rows of
    a 512-row product equal, bit for bit, the same rows computed alone."""
    g = torch.Generator(device="cpu").manual_seed(n + k)
    x = torch.randn((512, k), generator=g).to(torch.bfloat16).to(DEV)
    w = (torch.randn((n, k), generator=g) * 0.05).to(torch.bfloat16).to(DEV)
    r = torch.randn((512, n), generator=g).to(torch.bfloat16).to(DEV) if residual else None
    cfg = B.make_config(512, 8, 8, 1024)
    y_pair = G.empty((512, n), dtype=torch.bfloat16, device=DEV)
    B.llama3_linear(cfg, x, w, r, y_pair, 512, n, k)
    y_single = G.empty((255, n), dtype=torch.bfloat16, device=DEV)
    B.llama3_linear(cfg, x[:255].contiguous(), w, r[:255].contiguous() if residual else None, y_single, 255, n, k)
    torch.cuda.synchronize()
    assert torch.equal(y_pair[:255], y_single)
    want = f64(x) @ f64(w).T + (f64(r) if residual else 0.0)
    assert_close(y_pair, want, "bf16", f"CTA-pair linear {n}x{k}")


# --------------------------------------------------------------- attention
def _attn_case(Bn, S, P, H, KV, hd, seed):
    g = torch.Generator(device="cpu").manual_seed(seed)
    cap = P + S + 5
    q = torch.randn((Bn, S, H, hd), generator=g).to(torch.bfloat16)
    kc = torch.randn((Bn, cap, KV, hd), generator=g).to(torch.bfloat16)
    vc = torch.randn((Bn, cap, KV, hd), generator=g).to(torch.bfloat16)
    return q, kc, vc, cap


@pytest.mark.parametrize("Bn,S,P,H,KV,hd", [
    (2, 200, 0, 8, 2, 64), (2, 129, 37, 8, 2, 96), (1, 300, 0, 32, 8, 128), (3, 64, 500, 4, 4, 128),
    (1, 1, 0, 8, 2, 128), (4, 1, 1, 8, 1, 64), (3, 1, 1000, 32, 8, 128), (2, 1, 300, 8, 2, 96),
    (2, 1, 777, 16, 16, 64), (2, 1, 500, 12, 4, 64), (1, 150, 20, 12, 4, 64), (2, 1, 130, 16, 1, 128),
    (1, 1, 8192, 32, 8, 128), (2, 300, 0, 6, 2, 96), (1, 200, 10, 12, 4, 128), (2, 129, 0, 16, 2, 128)])
def test_attention(Bn, S, P, H, KV, hd):
    q, kc, vc, cap = _attn_case(Bn, S, P, H, KV, hd, Bn * 1000 + S + P + hd)
    cfg = B.make_config(H * hd, H, KV, 1024)
    ws_bytes = B.llama3_workspace_size(cfg, Bn, S, 1)
    ws = G.empty((ws_bytes,), dtype=torch.uint8, device=DEV)
    out = G.empty((Bn, S, H * hd), dtype=torch.bfloat16, device=DEV)
    B.llama3_attention(cfg, q.to(DEV), kc.to(DEV), vc.to(DEV), cap, Bn, S, P, out, ws, ws_bytes)
    for b in range(Bn):
        want = O.gqa_attention(f64(q[b]), f64(kc[b, :P + S]), f64(vc[b, :P + S]), P)
        assert_close(out[b], want.reshape(S, H * hd), "bf16", f"attention b={b}")


# ------------------------------------------------------- whole workloads
def _run_layers_vs_oracle(w, norm_weight="random", path=0):
    B.llama3_set_kernel_path(path)
    layers = [I.layer_weights(w, i, DEV, norm_weight) for i in range(w.n_layers)]
    outw = I.output_weights(w, DEV, norm_weight)
    cfg = w.cfg()
    rows = w.batch * w.seq if w.lm_rows == "all" else w.batch
    st = Stack(cfg, layers, outw, w.batch, w.seq, w.seq, lm_rows=rows if w.vocab else 0)
    if w.input_kind == "ids":
        ids = I.token_ids(w, DEV)
        x = G.empty((w.batch, w.seq, w.dim), dtype=w.torch_dtype, device=DEV)
        st.embed(ids, x)
        x0 = O.embed(ids.cpu().numpy(), f64(outw["tok_embeddings"]))
    else:
        x = G.to(I.activations(w, DEV))
        x0 = f64(x)
    st.forward_layers(x, w.seq)
    torch.cuda.synchronize()
    oc = oracle_cfg(w)
    h, kcs, vcs = O.forward_stack(x0, [oracle_layer(l) for l in layers], oc)
    assert_close(x, h, w.dtype, f"{w.name} hidden")
    for i, (kc, vc) in enumerate(st.caches):
        assert_close(kc, kcs[i], w.dtype, f"{w.name} k cache layer {i}")
        assert_close(vc, vcs[i], w.dtype, f"{w.name} v cache layer {i}")
    if w.vocab:
        logits = G.empty((rows, w.vocab), dtype=torch.float32, device=DEV)
        ids_out = st.lm_head(x, rows, w.dim, logits)
        want_logits, _ = O.lm_head(h.reshape(rows, w.dim), f64(outw["norm"]), f64(outw["output"]), w.norm_eps)
        assert_close(logits, want_logits, w.dtype, f"{w.name} logits")
        assert_argmax(ids_out, want_logits, f"{w.name} ids")


def test_tiny_f32_block_and_lm_head():
    _run_layers_vs_oracle(wl("tiny_f32"))


def test_tiny_f32_pages_init():
    _run_layers_vs_oracle(wl("tiny_f32"), norm_weight="ones")


@pytest.mark.parametrize("path", [0, 1])
def test_char_8l_stack_and_lm_head(path):
    _run_layers_vs_oracle(wl("char_8l"), path=path)


def test_gqa_768_layer():
    _run_layers_vs_oracle(wl("gqa_768"))


@pytest.mark.parametrize("hd,H,KV", [(16, 8, 2), (32, 8, 4)])
def test_bf16_small_head_dims_prefill_decode_lm_head(hd, H, KV):
    """bf16 models with head_dim 16 or 32 (the SIMT kernels): a 2-block
    prefill with the LM head on every row, then two decode steps."""
    w = small_bf16(dim=H * hd, n_heads=H, n_kv_heads=KV, ffn_hidden=4 * H * hd, batch=2, seq=40, vocab=500,
                   seed=hd)
    _run_layers_vs_oracle(w)
    layers = [I.layer_weights(w, i, DEV, "random") for i in range(w.n_layers)]
    st = Stack(w.cfg(), layers, I.output_weights(w, DEV), w.batch, 48, 40)
    g = torch.Generator(device="cpu").manual_seed(hd)
    xs = torch.randn((w.batch, 42, w.dim), generator=g).to(torch.bfloat16)
    a = G.to(xs[:, :40].contiguous())
    st.forward_layers(a, 40, 0)
    outs = [a]
    for t in (40, 41):
        d = G.to(xs[:, t:t + 1].contiguous())
        st.decode_layers(d, t)
        outs.append(d)
    want, _, _ = O.forward_stack(f64(xs), [oracle_layer(l) for l in layers], oracle_cfg(w))
    assert_close(torch.cat([o.cpu() for o in outs], 1), want, "bf16", f"bf16 head_dim {hd}")


def test_chunked_prefill_then_decode_steps():
    """Prefill 70 tokens, prefill a second chunk of 50 at start_pos 70, then
    three one-token decode steps -- against the oracle's full causal pass."""
    w = small_bf16()
    layers = [I.layer_weights(w, i, DEV, "random") for i in range(w.n_layers)]
    cap, total = 200, 70 + 50 + 3
    st = Stack(w.cfg(), layers, I.output_weights(w, DEV), w.batch, cap, 70)
    g = torch.Generator(device="cpu").manual_seed(9)
    xs = torch.randn((w.batch, total, w.dim), generator=g).to(torch.bfloat16)
    outs = []
    a = G.to(xs[:, :70].contiguous()); st.forward_layers(a, 70, 0); outs.append(a)
    b = G.to(xs[:, 70:120].contiguous()); st.forward_layers(b, 50, 70); outs.append(b)
    for t in range(120, total):
        d = G.to(xs[:, t:t + 1].contiguous())
        st.decode_layers(d, t)
        outs.append(d)
    got = torch.cat([o.cpu() for o in outs], 1)
    want, kcs, vcs = O.forward_stack(f64(xs), [oracle_layer(l) for l in layers], oracle_cfg(w))
    assert_close(got, want, "bf16", "chunked + decode")
    for i, (kc, vc) in enumerate(st.caches):
        assert_close(kc[:, :total], kcs[i], "bf16", f"k cache {i}")
        assert_close(vc[:, :total], vcs[i], "bf16", f"v cache {i}")


def test_decode_step_matches_prefill_path_for_large_batch():
    """batch > 256 decode routes to the prefill GEMMs; same answer as the oracle."""
    w = small_bf16(batch=300, n_layers=1, dim=256, n_heads=4, n_kv_heads=2, ffn_hidden=512)
    layers = [I.layer_weights(w, 0, DEV, "random")]
    st = Stack(w.cfg(), layers, I.output_weights(w, DEV), w.batch, 8, 3)
    g = torch.Generator(device="cpu").manual_seed(11)
    xs = torch.randn((w.batch, 4, w.dim), generator=g).to(torch.bfloat16)
    a = G.to(xs[:, :3].contiguous())
    st.forward_layers(a, 3, 0)
    d = G.to(xs[:, 3:4].contiguous())
    st.decode_layers(d, 3)
    want, _, _ = O.forward_stack(f64(xs), [oracle_layer(l) for l in layers], oracle_cfg(w))
    assert_close(torch.cat([a.cpu(), d.cpu()], 1), want, "bf16", "batch-300 decode")


def test_decode_stream_k_gemm_with_garbage_workspace():
    """dim 512, FFN 5632, 32 sequences: the w1|w3 decode GEMM takes the
    stream-K schedule (3 partial slabs, some tiles written by fewer CTAs, whose
    unused slabs the tile's last CTA zeroes).  The workspace starts as NaN, so a
    slab left unwritten poisons the block output."""
    w = small_bf16(batch=32, n_layers=1, dim=512, n_heads=8, n_kv_heads=2, ffn_hidden=5632)
    layers = [I.layer_weights(w, 0, DEV, "random")]
    st = Stack(w.cfg(), layers, I.output_weights(w, DEV), w.batch, 48, 40)
    st.ws.view(torch.float32).fill_(float("nan"))
    g = torch.Generator(device="cpu").manual_seed(17)
    xs = torch.randn((w.batch, 42, w.dim), generator=g).to(torch.bfloat16)
    a = G.to(xs[:, :40].contiguous())
    st.forward_layers(a, 40, 0)
    outs = [a]
    for t in (40, 41):
        d = G.to(xs[:, t:t + 1].contiguous())
        st.decode_layers(d, t)
        outs.append(d)
    want, _, _ = O.forward_stack(f64(xs), [oracle_layer(l) for l in layers], oracle_cfg(w))
    assert_close(torch.cat([o.cpu() for o in outs], 1), want, "bf16", "stream-K decode")


# -------------------------------------------------------------- LM head
@pytest.mark.parametrize("rows", [1, 5, 32, 300])
def test_lm_head_8b_vocab(rows):
    w = wl("llama3_8b_prefill")
    outw = I.output_weights(w, DEV, "random")
    h = I.hidden_rows(w, rows, DEV, std=2.0)
    cfg = B.make_config(w.dim, w.n_heads, w.n_kv_heads, w.ffn_hidden, w.vocab)
    ws_bytes = B.llama3_workspace_size(cfg, 1, 1, rows)
    ws = G.empty((ws_bytes,), dtype=torch.uint8, device=DEV)
    ids = G.empty((rows,), dtype=torch.int32, device=DEV)
    logits = G.empty((rows, w.vocab), dtype=torch.float32, device=DEV)
    B.llama3_lm_head_argmax(cfg, outw["norm"], outw["output"], h, rows, w.dim, ids, logits, ws, ws_bytes)
    ids2 = G.empty_like(ids)
    B.llama3_lm_head_argmax(cfg, outw["norm"], outw["output"], h, rows, w.dim, ids2, None, ws, ws_bytes)
    want, _ = O.lm_head(f64(h), f64(outw["norm"]), f64(outw["output"]), w.norm_eps)
    assert_close(logits, want, "bf16", "8b logits")
    assert_argmax(ids, want, "8b ids")
    assert torch.equal(ids, ids2)


def test_lm_head_row_stride_selects_last_positions():
    w = small_bf16()
    outw = I.output_weights(w, DEV, "random")
    x = G.to(I.activations(w, DEV))  # [3, 70, 512]
    cfg = B.make_config(w.dim, w.n_heads, w.n_kv_heads, w.ffn_hidden, w.vocab)
    ws_bytes = B.llama3_workspace_size(cfg, 1, 1, w.batch)
    ws = G.empty((ws_bytes,), dtype=torch.uint8, device=DEV)
    ids = G.empty((w.batch,), dtype=torch.int32, device=DEV)
    logits = G.empty((w.batch, w.vocab), dtype=torch.float32, device=DEV)
    B.llama3_lm_head_argmax(cfg, outw["norm"], outw["output"], x[:, -1], w.batch, w.seq * w.dim, ids, logits,
                            ws, ws_bytes)
    want, _ = O.lm_head(f64(x)[:, -1], f64(outw["norm"]), f64(outw["output"]), w.norm_eps)
    assert_close(logits, want, "bf16", "last-position logits")
    assert_argmax(ids, want, "last-position ids")


def test_lm_head_ties_pick_lowest_index():
    V, D = 300, 512
    cfg = B.make_config(D, 8, 2, 1024, V)
    wout = G.zeros((V, D), dtype=torch.bfloat16, device=DEV)
    wout[[17, 40, 299]] = 1.0
    h = torch.ones((2, D), dtype=torch.bfloat16, device=DEV)
    nw = torch.ones((D,), dtype=torch.bfloat16, device=DEV)
    ws_bytes = B.llama3_workspace_size(cfg, 1, 1, 2)
    ws = G.empty((ws_bytes,), dtype=torch.uint8, device=DEV)
    ids = G.empty((2,), dtype=torch.int32, device=DEV)
    for path in (0, 1):
        B.llama3_set_kernel_path(path)
        B.llama3_lm_head_argmax(cfg, nw, wout, h, 2, D, ids, None, ws, ws_bytes)
        assert ids.tolist() == [17, 17]


def test_embed_out_of_range_id_is_reported():
    w = small_bf16()
    outw = I.output_weights(w, DEV)
    cfg = B.make_config(w.dim, w.n_heads, w.n_kv_heads, w.ffn_hidden, w.vocab)
    ids = torch.tensor([0, 5, w.vocab + 3], dtype=torch.int32, device=DEV)
    x = G.empty((3, w.dim), dtype=torch.bfloat16, device=DEV)
    B.llama3_embed(cfg, ids, outw["tok_embeddings"], x, 3)
    assert B.llama3_device_status() == 6
    assert torch.equal(x[1], outw["tok_embeddings"][5])
    assert torch.count_nonzero(x[2]) == 0


def test_greedy_generation_matches_oracle():
    """Prefill + greedy decode loop on the device vs the oracle's greedy
    generation; tokens must agree at every step whose oracle top-2 gap exceeds
    1e-2 (after an undecided step a sequence may legitimately diverge)."""
    w = small_bf16(batch=3, seq=20, vocab=1000)
    layers = [I.layer_weights(w, i, DEV, "random") for i in range(w.n_layers)]
    outw = I.output_weights(w, DEV, "random")
    n_new = 12
    st = Stack(w.cfg(), layers, outw, w.batch, w.seq + n_new, w.seq, lm_rows=w.batch)
    prompt = I.token_ids(w, DEV)
    got = st.generate(prompt, n_new)
    st2 = Stack(w.cfg(), layers, outw, w.batch, w.seq + n_new, w.seq, lm_rows=w.batch)
    np.testing.assert_array_equal(st2.generate(prompt, n_new, cuda_graph=True), got)   # graph replay, same tokens
    toks, gaps = O.generate_greedy(prompt.cpu().numpy(), f64(outw["tok_embeddings"]),
                                   [oracle_layer(l) for l in layers], f64(outw["norm"]), f64(outw["output"]),
                                   oracle_cfg(w), n_new)
    compared = 0
    for b in range(w.batch):
        for t in range(n_new):
            if gaps[b, t] <= 1e-2:
                break
            assert got[b, t] == toks[b, t], (b, t, got[b], toks[b])
            compared += 1
    assert compared >= n_new  # the check covered a real stretch of tokens


def test_greedy_generation_with_prompts_of_different_lengths():
    """Prompts of lengths 20, 7 and 13 padded to 20: each sequence's tokens
    equal the oracle's greedy generation from its own prompt alone (at every
    step whose top-2 gap exceeds 1e-2), with and without the CUDA graph."""
    w = small_bf16(batch=3, seq=20, vocab=1000)
    layers = [I.layer_weights(w, i, DEV, "random") for i in range(w.n_layers)]
    outw = I.output_weights(w, DEV, "random")
    n_new, lens = 10, [20, 7, 13]
    st = Stack(w.cfg(), layers, outw, w.batch, w.seq + n_new, w.seq, lm_rows=w.batch)
    prompt = I.token_ids(w, DEV)
    got = st.generate(prompt, n_new, prompt_lens=lens)
    st2 = Stack(w.cfg(), layers, outw, w.batch, w.seq + n_new, w.seq, lm_rows=w.batch)
    np.testing.assert_array_equal(st2.generate(prompt, n_new, prompt_lens=lens, cuda_graph=True), got)
    host = prompt.cpu().numpy()
    compared = 0
    for b, L in enumerate(lens):
        toks, gaps = O.generate_greedy(host[b:b + 1, :L], f64(outw["tok_embeddings"]),
                                       [oracle_layer(l) for l in layers], f64(outw["norm"]), f64(outw["output"]),
                                       oracle_cfg(w), n_new)
        for t in range(n_new):
            if gaps[0, t] <= 1e-2:
                break
            assert got[b, t] == toks[0, t], (b, t, got[b], toks[0])
            compared += 1
    assert compared >= n_new


def _first_decided_new_token(toks, gaps, b, lo=2):
    """A step t >= lo of sequence b whose token has not appeared before in
    the row and whose steps 0..t all have a decided (top-2 gap > 1e-2)
    argmax, or None."""
    for t in range(len(toks[b])):
        if gaps[b, t] <= 1e-2:
            return None
        if t >= lo and toks[b, t] not in toks[b, :t]:
            return t
    return None


def test_greedy_generation_stops_at_end_token():
    """The end token is one the oracle's greedy run emits with a decided gap
    (sequence 1 at some step t >= 2); with it as eos_id every sequence must
    match the oracle's generate_greedy(eos_id=...) at each decided step, and
    sequence 1 must hold the end token from step t on, eager and in the graph."""
    w = small_bf16(batch=3, seq=20, vocab=1000)
    layers = [I.layer_weights(w, i, DEV, "random") for i in range(w.n_layers)]
    outw = I.output_weights(w, DEV, "random")
    n_new = 12
    prompt = I.token_ids(w, DEV)
    args = (prompt.cpu().numpy(), f64(outw["tok_embeddings"]), [oracle_layer(l) for l in layers],
            f64(outw["norm"]), f64(outw["output"]), oracle_cfg(w), n_new)
    toks, gaps = O.generate_greedy(*args)
    t_end = _first_decided_new_token(toks, gaps, 1)
    assert t_end is not None, "no decided step to plant the end token at"
    eos = int(toks[1, t_end])
    want, wgaps = O.generate_greedy(*args, eos_id=eos)
    assert np.all(want[1, t_end:] == eos)
    for graph in (False, True):
        st = Stack(w.cfg(), layers, outw, w.batch, w.seq + n_new, w.seq, lm_rows=w.batch)
        got = st.generate(prompt, n_new, eos_id=eos, cuda_graph=graph)
        assert np.all(got[1, t_end:] == eos), (graph, got[1])
        for b in range(w.batch):
            for t in range(n_new):
                forced = eos in want[b, :t]     # after the end token the row is held at it
                if not forced and wgaps[b, t] <= 1e-2:
                    break
                assert got[b, t] == want[b, t], (graph, b, t, got[b], want[b])


def test_generation_ends_when_every_sequence_is_done():
    """One sequence whose greedy run emits the end token at step t: the
    device loop stops right there (t + 1 steps run, not n_new) and the rest
    of the row is the end token, eager and in the graph."""
    w = small_bf16(batch=1, seq=16, vocab=1000, seed=91)
    layers = [I.layer_weights(w, i, DEV, "random") for i in range(w.n_layers)]
    outw = I.output_weights(w, DEV, "random")
    n_new = 12
    prompt = I.token_ids(w, DEV)
    toks, gaps = O.generate_greedy(prompt.cpu().numpy(), f64(outw["tok_embeddings"]),
                                   [oracle_layer(l) for l in layers], f64(outw["norm"]), f64(outw["output"]),
                                   oracle_cfg(w), n_new)
    t_end = _first_decided_new_token(toks, gaps, 0)
    assert t_end is not None and t_end + 1 < n_new
    eos = int(toks[0, t_end])
    for graph in (False, True):
        st = Stack(w.cfg(), layers, outw, w.batch, w.seq + n_new, w.seq, lm_rows=w.batch)
        got = st.generate(prompt, n_new, eos_id=eos, cuda_graph=graph)
        np.testing.assert_array_equal(got[0, :t_end + 1], toks[0, :t_end + 1])
        assert np.all(got[0, t_end:] == eos)
        assert st.steps_run == t_end + 1, (graph, st.steps_run, t_end)


@pytest.mark.parametrize("order", [[0, 2, 1], [1, 2, 0]])
def test_decode_blocks_in_any_order(order):
    """Blocks run in a caller-chosen order: the normalised input is handed on
    only between consecutive blocks (1 -> 2 in the second order), never
    across a jump, so the result equals the oracle running the blocks in
    that order (norm weights random, so a wrong hand-off shows)."""
    w = small_bf16(n_layers=3, batch=4, seq=30)
    layers = [I.layer_weights(w, i, DEV, "random") for i in range(w.n_layers)]
    st = Stack(w.cfg(), layers, I.output_weights(w, DEV), w.batch, 40, 30)
    g = torch.Generator(device="cpu").manual_seed(23)
    xs = torch.randn((w.batch, 32, w.dim), generator=g).to(torch.bfloat16)
    a = G.to(xs[:, :30].contiguous())
    st.forward_layers(a, 30, 0, layers=order)
    outs = [a]
    for t in (30, 31):
        d = G.to(xs[:, t:t + 1].contiguous())
        st.decode_layers(d, t, layers=order)
        outs.append(d)
    want, kcs, vcs = O.forward_stack(f64(xs), [oracle_layer(layers[i]) for i in order], oracle_cfg(w))
    assert_close(torch.cat([o.cpu() for o in outs], 1), want, "bf16", f"blocks in order {order}")
    for n, i in enumerate(order):
        assert_close(st.caches[i][0][:, :32], kcs[n], "bf16", f"k cache of block {i}")


# ------------------------------------------------------------ document mask
def _doc_starts(Bn, S, P, seed):
    """Per-token document start positions: random document lengths packed
    after `P` already-cached positions of one document starting at 0."""
    rng = np.random.default_rng(seed)
    ds = np.zeros((Bn, S), dtype=np.int32)
    for b in range(Bn):
        start, t = 0, 0
        while t < S:
            n = int(rng.integers(1, max(2, S // 2)))
            if t > 0 or P == 0:
                start = P + t if t > 0 else 0
            ds[b, t:t + n] = start
            t += n
    return ds


@pytest.mark.parametrize("Bn,S,P,H,KV,hd,path", [
    (2, 300, 0, 8, 2, 128, 0), (2, 200, 37, 8, 2, 64, 0), (1, 257, 0, 12, 4, 96, 0), (2, 130, 5, 8, 2, 64, 1)])
def test_attention_document_mask(Bn, S, P, H, KV, hd, path):
    B.llama3_set_kernel_path(path)
    q, kc, vc, cap = _attn_case(Bn, S, P, H, KV, hd, 77 + S + P)
    ds = _doc_starts(Bn, S, P, S + hd)
    cfg = B.make_config(H * hd, H, KV, 1024)
    ws_bytes = B.llama3_workspace_size(cfg, Bn, S, 1)
    ws = G.empty((ws_bytes,), dtype=torch.uint8, device=DEV)
    out = G.empty((Bn, S, H * hd), dtype=torch.bfloat16, device=DEV)
    B.llama3_attention_docs(cfg, q.to(DEV), kc.to(DEV), vc.to(DEV), cap, Bn, S, P, torch.from_numpy(ds).to(DEV), out,
                            ws, ws_bytes)
    for b in range(Bn):
        want = O.gqa_attention(f64(q[b]), f64(kc[b, :P + S]), f64(vc[b, :P + S]), P, doc_start=ds[b])
        assert_close(out[b], want.reshape(S, H * hd), "bf16", f"doc attention b={b}")


def test_layer_forward_packed_documents():
    w = small_bf16(n_layers=2, seq=150)
    layers = [I.layer_weights(w, i, DEV, "random") for i in range(w.n_layers)]
    st = Stack(w.cfg(), layers, I.output_weights(w, DEV), w.batch, w.seq, w.seq)
    ds = _doc_starts(w.batch, w.seq, 0, 11)
    dsd = torch.from_numpy(ds).to(DEV)
    x = G.to(I.activations(w, DEV))
    x0 = f64(x)
    for i in range(w.n_layers):
        kc, vc = st.caches[i]
        B.llama3_layer_forward_docs(st.cfg, st.wstructs[i], st.rope, st.rope_len, x, kc, vc, st.cache_cap,
                                    w.batch, w.seq, 0, dsd, st.ws, st.ws_bytes)
    want, _, _ = O.forward_stack(x0, [oracle_layer(l) for l in layers], oracle_cfg(w), doc_start=ds)
    assert_close(x, want, "bf16", "packed documents")


# ------------------------------------------------------------ ragged decode
@pytest.mark.parametrize("dtype,path", [("bf16", 0), ("bf16", 1), ("f32", 0)])
def test_ragged_decode_step_matches_per_sequence_oracle(dtype, path):
    """One decode step where every sequence's token sits at its own position
    (empty prefix, tile boundaries, the maximum): each sequence equals the
    oracle's block run alone at that position; new K/V land at their rows."""
    B.llama3_set_kernel_path(path)
    if dtype == "f32":
        w = I.Workload(name="tiny", dim=64, n_layers=1, n_heads=4, n_kv_heads=2, ffn_hidden=192, vocab=100,
                       batch=5, seq=1, dtype="f32", input_kind="activations", seed=13)
    else:
        w = small_bf16(batch=5, n_layers=1)
    layer = I.layer_weights(w, 0, DEV, "random")
    cap = 200
    positions = np.array([0, 37, 128, 129, 150], dtype=np.int32)
    st = Stack(w.cfg(), [layer], I.output_weights(w, DEV), w.batch, cap, 1)
    kc, vc = st.caches[0]
    g = torch.Generator(device="cpu").manual_seed(21)
    k0 = torch.randn(kc.shape, generator=g).to(kc.dtype)
    v0 = torch.randn(vc.shape, generator=g).to(vc.dtype)
    kc.copy_(k0.to(DEV)); vc.copy_(v0.to(DEV))
    x = torch.randn((w.batch, 1, w.dim), generator=g).to(kc.dtype)
    xd = x.to(DEV)
    st.decode_layers_ragged(xd, torch.from_numpy(positions).to(DEV), int(positions.max()))
    torch.cuda.synchronize()
    lo, oc = oracle_layer(layer), oracle_cfg(w)
    for b, p in enumerate(positions):
        kb, vb = f64(k0[b:b + 1]), f64(v0[b:b + 1])
        want = O.decoder_block(f64(x[b:b + 1]), lo, oc, kb, vb, start_pos=int(p))
        assert_close(xd[b:b + 1], want, dtype, f"ragged decode b={b} pos={p}")
        assert_close(kc[b, p], kb[0, p], dtype, f"k row b={b}")
        assert_close(vc[b, p], vb[0, p], dtype, f"v row b={b}")
        # the rest of the cache is untouched
        np.testing.assert_array_equal(f64(kc[b, :p]), f64(k0[b, :p]))
