"""The workspace-free LM-head entry point.

Some hosts cannot give the library device memory for a workspace (their
device memory is owned by another allocator, or their footprint is fixed
after start-up).  llama3_lm_head_argmax_noalloc serves them from a fixed
4 MiB scratch array inside the library; it must produce exactly what
llama3_lm_head_argmax (with a caller workspace) produces, call after call,
even though every call reuses the same scratch."""
import ctypes

import pytest
import torch

from helpers import assert_close, f64
from llama_decoder_only_rmsnorm_b200 import binding as B
from llama_decoder_only_rmsnorm_b200 import inputs as I

DEV = "cuda"


@pytest.mark.gpu
@pytest.mark.parametrize("workload,row_counts", [
    ("llama3_8b_prefill", (32, 7)),     # tcgen05 path, few rows
    ("llama3_8b_prefill", (511, 300)),  # the most rows the scratch holds at dim 4096 bf16, two n-tiles of hn
    ("tiny_f32", (64, 5)),              # fp32: the SIMT LM head reading its rows from the scratch
])
def test_noalloc_lm_head_matches_workspace_entry_point_on_consecutive_calls(workload, row_counts):
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    B.llama3_set_kernel_path(0)
    w = I.WORKLOADS[workload]
    outw = I.output_weights(w, DEV, "random")
    cfg = B.make_config(w.dim, w.n_heads, w.n_kv_heads, w.ffn_hidden, w.vocab, dtype=w.dtype)
    ws_bytes = B.llama3_workspace_size(cfg, 1, 1, max(row_counts))
    ws = torch.empty((ws_bytes,), dtype=torch.uint8, device=DEV)
    # two calls in a row; the second has fewer rows and new inputs, so any
    # maximum left in the shared scratch by the first call would show
    for call, rows in enumerate(row_counts):
        h = I.hidden_rows(w, rows, DEV, std=2.0, step=100 + call)
        ref_ids = torch.empty((rows,), dtype=torch.int32, device=DEV)
        ref_logits = torch.empty((rows, w.vocab), dtype=torch.float32, device=DEV)
        B.llama3_lm_head_argmax(cfg, outw["norm"], outw["output"], h, rows, w.dim, ref_ids, ref_logits, ws,
                                ws_bytes)
        ids = torch.full((rows,), -1, dtype=torch.int32, device=DEV)
        logits = torch.empty((rows, w.vocab), dtype=torch.float32, device=DEV)
        B.llama3_lm_head_argmax_noalloc(cfg, outw["norm"], outw["output"], h, rows, w.dim, ids, logits)
        torch.cuda.synchronize()
        assert torch.equal(ids, ref_ids), f"call {call}: ids differ"
        assert_close(logits, f64(ref_logits), w.dtype, f"call {call} logits")
    assert B.llama3_device_status() == 0


def test_noalloc_lm_head_rejects_rows_beyond_its_scratch():
    # dim 4096 bf16: roundup(rows*8, 256) + rows*8192 <= 4 MiB allows 511 rows
    cfg = B.make_config(4096, 32, 8, 14336, 128256)
    fake = ctypes.c_void_p(1 << 20)
    lib = B.lib()
    st = lib.llama3_lm_head_argmax_noalloc(ctypes.byref(cfg), fake, fake, fake, 512, 4096, fake, None, None)
    assert st == 3  # LLAMA3_ERR_WORKSPACE, before anything touches the device
    assert lib.llama3_lm_head_argmax_noalloc(ctypes.byref(cfg), fake, fake, fake, 0, 4096, fake, None, None) == 1
