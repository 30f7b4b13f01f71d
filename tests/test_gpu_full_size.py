"""Parity of single blocks at the full Llama-3-8B sizes the benchmark runs, and
of layers wider than 8B, against the fp64 oracle: one block of the
8192-token prefill (64 output rows spread over the sequence, plus every K/V
row the block writes) and one block of the 32-sequence decode step at 8192
cached positions (all 32 sequences and their new cache rows).  Same kernels
and launch configuration as bench.py.

Block outputs at these widths are held to the full-size bound of helpers.py
(the GPU within 1.5x of the relative L2 error that bf16 storage alone gives,
measured on the same inputs by the oracle's bf16 variant); the K/V rows,
one projection deep, keep the per-element bound 2e-2 + 2e-2|oracle|."""
import numpy as np
import pytest
import torch

from helpers import GuardArena, assert_close, assert_within_bf16_noise, f64, oracle_cfg, oracle_layer
from llama_decoder_only_rmsnorm_b200 import binding as B
from llama_decoder_only_rmsnorm_b200 import inputs as I
from llama_decoder_only_rmsnorm_b200.model import Llama3Stack
from oracle import llama3_oracle as O

pytestmark = pytest.mark.gpu
DEV = "cuda"


G = None   # the running test's guard arena: outputs, caches and workspaces sit between guard bands


@pytest.fixture(autouse=True)
def _gpu_state():
    global G
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    B.llama3_set_kernel_path(0)
    G = GuardArena(DEV)
    yield
    torch.cuda.synchronize()
    assert B.llama3_device_status() == 0, "device status word set"
    G.check()


def Stack(*a, **k):
    """Llama3Stack whose buffers all come from the guard arena."""
    return Llama3Stack(*a, alloc=G.alloc, **k)


def _spread_rows(S, n, seed):
    """Tile edges and ends of the sequence plus random rows, sorted."""
    fixed = {0, 1, 127, 128, 129, 255, 256, S // 2, S - 129, S - 128, S - 2, S - 1}
    rng = np.random.default_rng(seed)
    extra = rng.choice(S, size=n - len(fixed), replace=False)
    return sorted(fixed | {int(r) for r in extra})[:n]


def test_8b_prefill_block_full_sequence():
    w = I.WORKLOADS["llama3_8b_prefill"].replace(input_kind="activations")
    layer = I.layer_weights(w, 0, DEV)
    S = w.seq
    st = Stack(w.cfg(), [layer], I.output_weights(w, DEV), 1, S, S, lm_rows=1)
    x = G.to(I.activations(w, DEV))
    x0 = f64(x)[0]
    st.forward_layers(x, S, 0)
    torch.cuda.synchronize()
    rows = _spread_rows(S, 64, 1)
    lo, oc = oracle_layer(layer), oracle_cfg(w)
    want, k, v = O.decoder_block_rows(x0, lo, oc, rows)
    want_bf, _, _ = O.decoder_block_rows(x0, lo, oc, rows, rounding="bf16")
    assert_within_bf16_noise(x[0, rows], want, want_bf, "8B prefill block rows")
    kc, vc = st.caches[0]
    assert_close(kc[0, :S], k, "bf16", "8B prefill K cache (all positions)")
    assert_close(vc[0, :S], v, "bf16", "8B prefill V cache (all positions)")


def test_8b_decode_block_all_sequences():
    wd = I.WORKLOADS["llama3_8b_decode"]
    w8 = I.WORKLOADS["llama3_8b_prefill"]
    layer = I.layer_weights(w8, 0, DEV)
    P = wd.cache_len
    kc, vc = (G.to(t) for t in I.kv_cache(wd, 0, P + 1, DEV))
    st = Stack(w8.cfg(), [layer], I.output_weights(w8, DEV), wd.batch, P + 1, 1, lm_rows=wd.batch,
               caches=[(kc, vc)])
    g = torch.Generator(device="cpu").manual_seed(31)
    x = torch.randn((wd.batch, 1, wd.dim), generator=g).to(torch.bfloat16)
    xd = G.to(x)
    st.decode_layers(xd, P)
    torch.cuda.synchronize()
    # the cache prefix is an input: draw it again (same seeds) for the oracle
    kp, vp = I.kv_cache(wd, 0, P, DEV)
    kp, vp = f64(kp), f64(vp)
    lo, oc = oracle_layer(layer), oracle_cfg(w8)
    got, want, want_bf = [], [], []
    for b in range(wd.batch):
        o_ex, k_new, v_new = O.decoder_block_rows(f64(x[b]), lo, oc, [0], kp[b], vp[b], start_pos=P)
        o_bf, _, _ = O.decoder_block_rows(f64(x[b]), lo, oc, [0], kp[b], vp[b], start_pos=P, rounding="bf16")
        got.append(f64(xd[b])); want.append(o_ex); want_bf.append(o_bf)
        assert_close(kc[b, P], k_new[0], "bf16", f"8B decode new K seq {b}")
        assert_close(vc[b, P], v_new[0], "bf16", f"8B decode new V seq {b}")
    assert_within_bf16_noise(np.stack(got), np.stack(want), np.stack(want_bf), "8B decode block")


@pytest.mark.parametrize("dim,H,KV,F", [(8192, 64, 8, 22016), (8448, 66, 6, 22528)])
def test_wide_prefill_layer(dim, H, KV, F):
    """Layers wider than 8B (dim 8192, and 8448 = 33 tiles of 256): all 640
    output rows of a one-layer prefill.  At these widths the per-element bound
    is missed by the oracle's own bf16 variant as well."""
    w = I.Workload("wide", dim=dim, n_layers=1, n_heads=H, n_kv_heads=KV, ffn_hidden=F, vocab=None, batch=1,
                   seq=640, dtype="bf16", input_kind="activations", seed=dim)
    layer = I.layer_weights(w, 0, DEV, "random")
    st = Stack(w.cfg(), [layer], {}, 1, w.seq, w.seq)
    x = G.to(I.activations(w, DEV))
    x0 = f64(x)
    st.forward_layers(x, w.seq, 0)
    torch.cuda.synchronize()
    lo, oc = oracle_layer(layer), oracle_cfg(w)
    kc0 = np.zeros((1, w.seq, KV, dim // H)); vc0 = np.zeros_like(kc0)
    want = O.decoder_block(x0, lo, oc, kc0, vc0)
    want_bf = O.decoder_block(x0, lo, oc, np.zeros_like(kc0), np.zeros_like(vc0), rounding="bf16")
    assert_within_bf16_noise(x, want, want_bf, f"dim-{dim} prefill layer")
    assert_close(st.caches[0][0], kc0, "bf16", f"dim-{dim} K cache")
    assert_close(st.caches[0][1], vc0, "bf16", f"dim-{dim} V cache")


def test_wide_decode_layer_uses_separate_reductions():
    """dim 16896 (> 16384): the decode step's residual sums and the RMSNorm
    after them run as separate kernels instead of the fused one."""
    w = I.Workload("wide_decode", dim=16896, n_layers=1, n_heads=132, n_kv_heads=12, ffn_hidden=4096, vocab=None,
                   batch=4, seq=1, dtype="bf16", input_kind="activations", seed=16896, cache_len=300)
    layer = I.layer_weights(w, 0, DEV, "random")
    P = w.cache_len
    kc, vc = (G.to(t) for t in I.kv_cache(w, 0, P + 1, DEV))
    st = Stack(w.cfg(), [layer], {}, w.batch, P + 1, 1, caches=[(kc, vc)])
    x = G.to(I.activations(w, DEV))
    x0 = f64(x)
    st.decode_layers(x, P)
    torch.cuda.synchronize()
    kp, vp = I.kv_cache(w, 0, P, DEV)
    kp, vp = f64(kp), f64(vp)
    lo, oc = oracle_layer(layer), oracle_cfg(w)
    want = np.stack([O.decoder_block_rows(x0[b], lo, oc, [0], kp[b], vp[b], start_pos=P)[0]
                     for b in range(w.batch)])
    want_bf = np.stack([O.decoder_block_rows(x0[b], lo, oc, [0], kp[b], vp[b], start_pos=P, rounding="bf16")[0]
                        for b in range(w.batch)])
    assert_within_bf16_noise(x, want, want_bf, "dim-16896 decode layer")
