"""Parity at the full Llama-3-8B sizes the benchmark runs, on outputs the fp64
oracle can compute one by one: one decoder block of the 8192-token prefill
(sampled output rows, plus every K/V row the block writes to the cache) and
one block of the 32-sequence decode step at 8192 cached positions (sampled
sequences, plus their new cache rows).  Same kernels and launch configuration
as bench.py (tcgen05 GEMMs, the default prefill attention design, split-KV
decode attention)."""
import numpy as np
import pytest
import torch

from helpers import assert_close, f64, oracle_cfg, oracle_layer
from llama_decoder_only_rmsnorm_b200 import binding as B
from llama_decoder_only_rmsnorm_b200 import inputs as I
from llama_decoder_only_rmsnorm_b200.model import Llama3Stack
from oracle import llama3_oracle as O

pytestmark = pytest.mark.gpu
DEV = "cuda"

# One full-size bf16 block carries rounding noise from its bf16 intermediates
# (normalised rows, SwiGLU product, residual stream), each rounded to a
# relative 2^-9/sqrt(3) ~ 1.1e-3.  With the seeded N(0, 0.02) weights the w2
# output (K = 14336) has a standard deviation near 1.9, and the rounding of its
# inputs alone reaches the block output with a standard deviation near 5e-3.
# Measured, the fp64 arithmetic with bf16 rounding at the GPU's rounding points
# differs from the exact oracle by a standard deviation of 1.2e-2, as much as
# the GPU does, so the per-element bound 2e-2 + 2e-2|o| of the smaller
# workloads is missed on a fraction of a percent of near-zero elements.  At these sizes the tests require the bound on at
# least 99 % of the elements, 4x the bound on every element, and a relative
# L2 error below 1e-2; the K/V rows keep the plain bound.
BULK, SLACK, REL_L2 = 0.99, 4.0, 1e-2


def assert_close_bulk(gpu, oracle, what):
    g = f64(gpu) if isinstance(gpu, torch.Tensor) else np.asarray(gpu, float)
    o = np.asarray(oracle, float)
    assert g.shape == o.shape, (what, g.shape, o.shape)
    err = np.abs(g - o)
    bound = 2e-2 + 2e-2 * np.abs(o)
    within = float(np.mean(err <= bound))
    worst = float(np.max(err / bound))
    rel = float(np.linalg.norm(g - o) / np.linalg.norm(o))
    assert np.all(np.isfinite(g)), what
    assert within >= BULK and worst <= SLACK and rel <= REL_L2, (what, within, worst, rel)


@pytest.fixture(autouse=True)
def _gpu_state():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    B.llama3_set_kernel_path(0)
    yield
    torch.cuda.synchronize()
    assert B.llama3_device_status() == 0, "device status word set"


def test_8b_prefill_block_full_sequence_sampled_rows():
    w = I.WORKLOADS["llama3_8b_prefill"].replace(input_kind="activations")
    layer = I.layer_weights(w, 0, DEV)
    S = w.seq
    st = Llama3Stack(w.cfg(), [layer], I.output_weights(w, DEV), 1, S, S, lm_rows=1)
    x = I.activations(w, DEV)
    x0 = f64(x)[0]
    st.forward_layers(x, S, 0)
    torch.cuda.synchronize()
    rows = [0, 1, 127, 128, 129, 2047, 4096, 6000, 8190, 8191]
    want, k, v = O.decoder_block_rows(x0, oracle_layer(layer), oracle_cfg(w), rows)
    assert_close_bulk(x[0, rows], want, "8B prefill rows")
    kc, vc = st.caches[0]
    assert_close(kc[0, :S], k, "bf16", "8B prefill K cache (all positions)")
    assert_close(vc[0, :S], v, "bf16", "8B prefill V cache (all positions)")


def test_8b_decode_step_sampled_sequences():
    wd = I.WORKLOADS["llama3_8b_decode"]
    w8 = I.WORKLOADS["llama3_8b_prefill"]
    layer = I.layer_weights(w8, 0, DEV)
    P = wd.cache_len
    kc, vc = I.kv_cache(wd, 0, P + 1, DEV)
    st = Llama3Stack(w8.cfg(), [layer], I.output_weights(w8, DEV), wd.batch, P + 1, 1, lm_rows=wd.batch,
                     caches=[(kc, vc)])
    g = torch.Generator(device="cpu").manual_seed(31)
    x = torch.randn((wd.batch, 1, wd.dim), generator=g).to(torch.bfloat16)
    k_prefix = {b: (f64(kc[b, :P]), f64(vc[b, :P])) for b in (0, 17, 31)}
    xd = x.to(DEV)
    st.decode_layers(xd, P)
    torch.cuda.synchronize()
    lo, oc = oracle_layer(layer), oracle_cfg(w8)
    for b, (kp, vp) in k_prefix.items():
        want, k_new, v_new = O.decoder_block_rows(f64(x[b]), lo, oc, [0], kp, vp, start_pos=P)
        assert_close_bulk(xd[b], want, f"8B decode seq {b}")
        assert_close(kc[b, P], k_new[0], "bf16", f"8B decode new K seq {b}")
        assert_close(vc[b, P], v_new[0], "bf16", f"8B decode new V seq {b}")
