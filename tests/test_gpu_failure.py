"""Failure detection on the device, without a GPU fault.

Every wait of one kernel role for another is bounded.  The test hook
llama3_set_test_withheld_arrival makes one such wait run out on purpose (one
arrival that nothing else provides): the kernel must record LLAMA3_ERR_TIMEOUT
in the status word, let its copies land, free its tensor memory and return,
and the next call on the same context must give the oracle's answer.  The
wait limit is lowered to 5 ms for these calls."""
import numpy as np
import pytest
import torch

from helpers import GuardArena, assert_close, f64
from llama_decoder_only_rmsnorm_b200 import binding as B
from oracle import llama3_oracle as O

pytestmark = pytest.mark.gpu
DEV = "cuda"
TIMEOUT = 5  # LLAMA3_ERR_TIMEOUT
G = None     # guard arena of the running test


@pytest.fixture(autouse=True)
def _hook_off():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    B.llama3_set_kernel_path(0)
    assert B.llama3_device_status() == 0
    old = B.llama3_set_wait_limit_ms(5)
    global G
    G = GuardArena(DEV)
    yield
    B.llama3_set_test_withheld_arrival(0)
    B.llama3_set_wait_limit_ms(old)
    torch.cuda.synchronize()
    G.check()   # an abandoned call still writes nothing outside its buffers


def test_gemm_accumulator_wait_gives_up_then_next_call_is_exact():
    # 10 x 23 tiles of 256 x 256 on at most 74 CTA pairs: at least three tiles
    # per pair, so the withheld release of the first accumulator is waited for
    m, n, k = 2560, 5888, 64
    g = torch.Generator(device="cpu").manual_seed(41)
    x = torch.randn((m, k), generator=g).to(torch.bfloat16).to(DEV)
    w = (torch.randn((n, k), generator=g) * 0.1).to(torch.bfloat16).to(DEV)
    y = G.empty((m, n), dtype=torch.bfloat16, device=DEV)
    cfg = B.make_config(512, 8, 8, 1024)
    B.llama3_set_test_withheld_arrival(1)
    B.llama3_linear(cfg, x, w, None, y, m, n, k)
    assert B.llama3_device_status() == TIMEOUT
    B.llama3_set_test_withheld_arrival(0)
    B.llama3_linear(cfg, x, w, None, y, m, n, k)
    assert B.llama3_device_status() == 0
    assert_close(y, f64(x) @ f64(w).T, "bf16", "GEMM after a timed-out call")


def test_attention_wait_for_p_gives_up_then_next_call_is_exact():
    Bn, S, H, KV, hd = 1, 256, 8, 2, 128
    g = torch.Generator(device="cpu").manual_seed(43)
    q = torch.randn((Bn, S, H, hd), generator=g).to(torch.bfloat16)
    kc = torch.randn((Bn, S, KV, hd), generator=g).to(torch.bfloat16)
    vc = torch.randn((Bn, S, KV, hd), generator=g).to(torch.bfloat16)
    cfg = B.make_config(H * hd, H, KV, 1024)
    ws_bytes = B.llama3_workspace_size(cfg, Bn, S, 1)
    ws = G.empty((ws_bytes,), dtype=torch.uint8, device=DEV)
    out = G.empty((Bn, S, H * hd), dtype=torch.bfloat16, device=DEV)
    qd, kd, vd = q.to(DEV), kc.to(DEV), vc.to(DEV)
    B.llama3_set_test_withheld_arrival(2)
    B.llama3_attention(cfg, qd, kd, vd, S, Bn, S, 0, out, ws, ws_bytes)
    assert B.llama3_device_status() == TIMEOUT
    B.llama3_set_test_withheld_arrival(0)
    B.llama3_attention(cfg, qd, kd, vd, S, Bn, S, 0, out, ws, ws_bytes)
    assert B.llama3_device_status() == 0
    want = O.gqa_attention(f64(q[0]), f64(kc[0]), f64(vc[0]), 0)
    assert_close(out[0], want.reshape(S, H * hd), "bf16", "attention after a timed-out call")
