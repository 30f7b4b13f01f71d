"""GPU parity of the temperature / top-p draw against the fp64 oracle.

Floating point decides an integer here (which tokens are kept, which one the
draw lands on), so ids are compared where the oracle's decision margins --
the distance of top_p from the nearest keep/drop boundary and of the draw
target from the nearest boundary of the running kept mass, as fractions of
the row's probability -- both exceed MARGIN (the device's fp32
probabilities and 2^-40 integer masses are off by well under 1e-6 of the
total).  Cases whose arithmetic is exact on both sides (ties of equal
logits, argmax) are compared without that filter."""
import numpy as np
import pytest
import torch

from helpers import GuardArena, assert_close, f64, oracle_cfg, oracle_layer
from llama_decoder_only_rmsnorm_b200 import binding as B
from llama_decoder_only_rmsnorm_b200 import inputs as I
from llama_decoder_only_rmsnorm_b200.model import Llama3Stack
from oracle import llama3_oracle as O

pytestmark = pytest.mark.gpu
DEV = "cuda"
MARGIN = 1e-5


G = None   # the running test's guard arena: outputs, caches and workspaces sit between guard bands


@pytest.fixture(autouse=True)
def _gpu_state():
    global G
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    G = GuardArena(DEV)
    yield
    torch.cuda.synchronize()
    assert B.llama3_device_status() == 0, "device status word set"
    G.check()


def Stack(*a, **k):
    """Llama3Stack whose buffers all come from the guard arena."""
    return Llama3Stack(*a, alloc=G.alloc, **k)


def _sample(lg, T, top_p, seed, offset, ld=None):
    R, V = lg.shape
    ld = ld or V
    buf = torch.zeros((R, ld), dtype=torch.float32)
    buf[:, :V] = torch.from_numpy(lg)
    d = buf.to(DEV)
    ids = G.full((R,), -1, dtype=torch.int32, device=DEV)
    B.llama3_sample_top_p(d, R, ld, V, T, top_p, seed, offset, ids)
    return ids.cpu().numpy()


@pytest.mark.parametrize("R,V,T,top_p,scale,ld", [
    (7, 5, 1.0, 0.6, 2.0, None), (32, 1000, 0.7, 0.9, 3.0, 1004), (5, 32000, 0.6, 0.9, 4.0, None),
    (3, 128256, 0.6, 0.9, 5.0, None), (4, 128256, 1.0, 1.0, 6.0, None), (6, 777, 1.5, 0.3, 2.0, None),
    (8, 4096, 0.8, 0.0, 2.0, None), (2, 68, 0.9, 0.95, 1.0, None)])
def test_sample_matches_oracle(R, V, T, top_p, scale, ld):
    rng = np.random.default_rng(R * 7919 + V)
    lg = (rng.standard_normal((R, V)) * scale).astype(np.float32)
    T32, p32 = float(np.float32(T)), float(np.float32(top_p))
    seed = 0x5EED0000 + V
    decided = total = 0
    for offset in range(6):
        got = _sample(lg, T, top_p, seed, offset, ld)
        for r in range(R):
            tok, (cut, draw) = O.top_p_sample(lg[r].astype(np.float64), T32, p32, O.sampling_word(seed, offset, r))
            total += 1
            if cut > MARGIN and draw > MARGIN:
                assert got[r] == tok, (offset, r, got[r], tok, cut, draw)
                decided += 1
            else:
                assert 0 <= got[r] < V
    assert decided >= 0.8 * total, (decided, total)


def test_sample_equal_logits_follow_index_order():
    # 8 equal logits: masses are exact on both sides; top_p 0.5 keeps tokens 0..4
    lg = np.zeros((16, 8), dtype=np.float32)
    got = _sample(lg, 0.7, 0.5, 1234, 9)
    for r in range(16):
        want, _ = O.top_p_sample(lg[r].astype(np.float64), 0.7, 0.5, O.sampling_word(1234, 9, r))
        word = O.sampling_word(1234, 9, r)
        exact = (word * 5) >> 64          # floor(5 u) computed exactly
        assert got[r] == exact
        if abs(word * 5 / 2.0 ** 64 - round(word * 5 / 2.0 ** 64)) > 1e-9:
            assert got[r] == want


def test_sample_temperature_zero_is_argmax_with_lowest_index_ties():
    rng = np.random.default_rng(5)
    lg = rng.standard_normal((9, 3000)).astype(np.float32)
    lg[1, [10, 2000]] = 50.0          # tie: the lower index wins
    lg[2, -1] = 60.0                  # maximum at the last index
    got = _sample(lg, 0.0, 0.9, 1, 0)
    np.testing.assert_array_equal(got, np.argmax(lg, axis=1))
    assert got[1] == 10


def test_sample_is_deterministic_and_varies_with_offset():
    rng = np.random.default_rng(6)
    lg = (rng.standard_normal((32, 5000)) * 2).astype(np.float32)
    a = _sample(lg, 1.0, 0.95, 77, 3)
    b = _sample(lg, 1.0, 0.95, 77, 3)
    c = _sample(lg, 1.0, 0.95, 77, 4)
    np.testing.assert_array_equal(a, b)
    assert (a != c).sum() >= 16       # a fresh draw per step


def test_sample_frequencies_follow_the_kept_law():
    # one row, many offsets: empirical frequencies against the renormalised
    # kept probabilities of the oracle (p_keep for top_p 0.8 over 6 tokens)
    p = np.array([0.05, 0.3, 0.1, 0.25, 0.2, 0.1])
    lg = np.log(p).astype(np.float32)[None, :].repeat(512, 0)
    n = 0
    counts = np.zeros(6)
    for off in range(8):
        got = _sample(lg, 1.0, 0.8, 4242, off)
        np.add.at(counts, got, 1)
        n += len(got)
    # ranked 1 (.3), 3 (.25), 4 (.2), 2 (.1), 5 (.1), 0: before = 0, .3, .55, .75, .85 -> keep 1, 3, 4, 2
    want = np.array([0, 0.3, 0.1, 0.25, 0.2, 0]) / 0.85
    sigma = np.sqrt(want * (1 - want) / n)
    assert np.all(np.abs(counts / n - want) <= 5 * sigma + 1e-12), counts / n


def test_sampled_generation_draws_from_the_models_logits():
    """Prefill + decode loop with temperature 0.8 / top_p 0.9: each step's
    token is the oracle's draw from that step's device logits (where the
    margins are clear), and those logits match the oracle model run on the
    generated sequence (teacher forcing, bf16 tolerance)."""
    w = I.Workload(name="small", dim=512, n_layers=2, n_heads=8, n_kv_heads=2, ffn_hidden=1024, vocab=1000,
                   batch=3, seq=20, dtype="bf16", input_kind="ids", seed=91)
    layers = [I.layer_weights(w, i, DEV, "random") for i in range(w.n_layers)]
    outw = I.output_weights(w, DEV, "random")
    n_new, T, top_p, seed = 10, 0.8, 0.9, 2024
    st = Stack(w.cfg(), layers, outw, w.batch, w.seq + n_new, w.seq, lm_rows=w.batch)
    prompt = I.token_ids(w, DEV)
    toks, logits = st.generate(prompt, n_new, temperature=T, top_p=top_p, seed=seed, return_logits=True)
    T32, p32 = float(np.float32(T)), float(np.float32(top_p))
    decided = 0
    for step in range(n_new):
        for b in range(w.batch):
            want, (cut, draw) = O.top_p_sample(logits[step, b].astype(np.float64), T32, p32,
                                               O.sampling_word(seed, w.seq - 1 + step, b))
            if cut > MARGIN and draw > MARGIN:
                assert toks[b, step] == want, (step, b)
                decided += 1
    assert decided >= 0.8 * n_new * w.batch
    # teacher-forced oracle logits on prompt + generated tokens
    seq = np.concatenate([prompt.cpu().numpy(), toks[:, :-1]], axis=1)
    h, _, _ = O.forward_stack(O.embed(seq, f64(outw["tok_embeddings"])), [oracle_layer(l) for l in layers],
                              oracle_cfg(w))
    rows = h[:, w.seq - 1:].reshape(-1, w.dim)
    want_logits, _ = O.lm_head(rows, f64(outw["norm"]), f64(outw["output"]), w.norm_eps)
    got = logits.transpose(1, 0, 2).reshape(-1, w.vocab)
    assert_close(got, want_logits, "bf16", "generation logits")
    # the same loop captured once in a CUDA graph and replayed draws the same tokens
    st2 = Stack(w.cfg(), layers, outw, w.batch, w.seq + n_new, w.seq, lm_rows=w.batch)
    toks_graph = st2.generate(prompt, n_new, temperature=T, top_p=top_p, seed=seed, cuda_graph=True)
    np.testing.assert_array_equal(toks_graph, toks)
