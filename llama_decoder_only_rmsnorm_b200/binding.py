"""ctypes binding of libllama3.so: the C ABI of include/llama3.h under the same
names.  Argument marshalling only -- every step of the decoder runs in the
library's CUDA kernels.  Tensors are passed as device pointers
(``tensor.data_ptr()``); the stream defaults to torch's current stream.

The library must have been built (``python -m llama_decoder_only_rmsnorm_b200.build``);
importing a missing library raises instead of falling back to anything else.
"""
from __future__ import annotations

import ctypes
import os
import re

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libllama3.so")
HEADER_PATH = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "llama3.h")

DTYPE_BF16, DTYPE_F32 = 0, 1
STATUS = {0: "LLAMA3_OK", 1: "LLAMA3_ERR_ARG", 2: "LLAMA3_ERR_ALIGN", 3: "LLAMA3_ERR_WORKSPACE",
          4: "LLAMA3_ERR_CUDA", 5: "LLAMA3_ERR_TIMEOUT", 6: "LLAMA3_ERR_TOKEN", 7: "LLAMA3_ERR_UNSUPPORTED"}


class llama3_config(ctypes.Structure):
    _fields_ = [("dim", ctypes.c_int), ("n_heads", ctypes.c_int), ("n_kv_heads", ctypes.c_int),
                ("head_dim", ctypes.c_int), ("ffn_hidden", ctypes.c_int), ("vocab", ctypes.c_int),
                ("norm_eps", ctypes.c_float), ("rope_theta", ctypes.c_double), ("dtype", ctypes.c_int)]


class llama3_layer_weights(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in
                ("attention_norm", "wqkv", "wo", "ffn_norm", "w1", "w2", "w3")]


class Llama3Error(RuntimeError):
    def __init__(self, name, status, cuda_error=0):
        self.status = status
        self.cuda_error = cuda_error
        msg = f"{name} -> {STATUS.get(status, status)}"
        if cuda_error:
            msg += f" (cuda error {cuda_error})"
        super().__init__(msg)


_lib = None
_i, _ll, _sz, _p, _d = ctypes.c_int, ctypes.c_longlong, ctypes.c_size_t, ctypes.c_void_p, ctypes.c_double
_cfgp, _wp = ctypes.POINTER(llama3_config), ctypes.POINTER(llama3_layer_weights)

_SIGNATURES = {
    "llama3_init_rope_table": [_p, _i, _i, _d, _p],
    "llama3_workspace_size": [_cfgp, _i, _i, _i, ctypes.POINTER(_sz)],
    "llama3_embed": [_cfgp, _p, _p, _p, _i, _p],
    "llama3_layer_forward": [_cfgp, _wp, _p, _i, _p, _p, _p, _i, _i, _i, _i, _p, _sz, _p],
    "llama3_layer_decode": [_cfgp, _wp, _p, _i, _p, _p, _p, _i, _i, _i, _p, _sz, _p],
    "llama3_layer_decode_ragged": [_cfgp, _wp, _p, _i, _p, _p, _p, _i, _i, _p, _i, _p, _sz, _p],
    "llama3_layer_decode_chained": [_cfgp, _wp, _p, _i, _p, _p, _p, _i, _i, _i, _p, _p, _i, _p, _sz, _p],
    "llama3_decode_step": [_cfgp, _wp, _i, _p, _i, _p, _p, _p, _i, _i, _i, _p, _p, _sz, _p],
    "llama3_layer_forward_docs": [_cfgp, _wp, _p, _i, _p, _p, _p, _i, _i, _i, _i, _p, _p, _sz, _p],
    "llama3_attention_docs": [_cfgp, _p, _p, _p, _i, _i, _i, _i, _p, _p, _p, _sz, _p],
    "llama3_lm_head_argmax": [_cfgp, _p, _p, _p, _i, _ll, _p, _p, _p, _sz, _p],
    "llama3_lm_head_argmax_noalloc": [_cfgp, _p, _p, _p, _i, _ll, _p, _p, _p],
    "llama3_rmsnorm": [_cfgp, _p, _ll, _p, _p, _i, _p],
    "llama3_linear": [_cfgp, _p, _p, _p, _p, _i, _i, _i, _p, _sz, _p],
    "llama3_attention": [_cfgp, _p, _p, _p, _i, _i, _i, _i, _p, _p, _sz, _p],
    "llama3_status_string": [_i],
    "llama3_device_status": [ctypes.POINTER(_i)],
    "llama3_last_cuda_error": [],
    "llama3_set_kernel_path": [_i],
    "llama3_set_wait_limit_ms": [_i],
    "llama3_set_test_withheld_arrival": [_i],
    "llama3_set_programmatic_launch": [_i],
    "llama3_sample_top_p": [_p, _i, _ll, _i, ctypes.c_float, ctypes.c_float, ctypes.c_ulonglong, ctypes.c_ulonglong, _p, _p, _p],
    "llama3_generation_advance": [_p, _p, _p, _p, _p, _i, _i, _i, _ll, _p],
    "llama3_gather_rows": [_cfgp, _p, _ll, _i, _p, _i, _p, _p],
    "llama3_set_launch_timer": [_i, _p, _p, _i],
    "llama3_launch_timer_used": [],
    "llama3_launch_count": [],
}


def lib():
    """Load libllama3.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -m llama_decoder_only_rmsnorm_b200.build`")
        l = ctypes.CDLL(LIB_PATH)
        for name, args in _SIGNATURES.items():
            f = getattr(l, name)
            f.argtypes = args
            f.restype = {"llama3_status_string": ctypes.c_char_p,
                         "llama3_launch_count": ctypes.c_ulonglong}.get(name, ctypes.c_int)
        _lib = l
    return _lib


def header_functions():
    """Names of the functions include/llama3.h declares."""
    text = open(HEADER_PATH).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:[\w*]+\s+)+\**(llama3_\w+)\s*\(", text, flags=re.M)))


# ---------------------------------------------------------------- helpers ---
def _ptr(t):
    if t is None:
        return None
    if isinstance(t, int):
        return ctypes.c_void_p(t)
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        import torch
        return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    if isinstance(stream, int):
        return ctypes.c_void_p(stream)
    return ctypes.c_void_p(stream.cuda_stream)


def _check(name, status):
    if status != 0:
        raise Llama3Error(name, status, lib().llama3_last_cuda_error() if status == 4 else 0)


def make_config(dim, n_heads, n_kv_heads, ffn_hidden, vocab=0, norm_eps=1e-5, rope_theta=500000.0,
                dtype="bf16", head_dim=None):
    return llama3_config(dim, n_heads, n_kv_heads, head_dim or dim // n_heads, ffn_hidden, vocab or 0,
                         norm_eps, rope_theta, DTYPE_F32 if dtype == "f32" else DTYPE_BF16)


def make_layer_weights(layer):
    """Struct of device pointers from a dict with the page's weight names
    (attention_norm, wqkv, wo, ffn_norm, w1, w2, w3).  The caller keeps the
    tensors alive."""
    return llama3_layer_weights(*[layer[n].data_ptr() for n in
                                  ("attention_norm", "wqkv", "wo", "ffn_norm", "w1", "w2", "w3")])


# ------------------------------------------------------------ the C ABI ---
def llama3_init_rope_table(cos_sin, head_dim, max_pos, theta, stream=None):
    _check("llama3_init_rope_table",
           lib().llama3_init_rope_table(_ptr(cos_sin), head_dim, max_pos, theta, _stream(stream)))


def llama3_workspace_size(cfg, batch, seq, lm_rows=0):
    n = ctypes.c_size_t(0)
    _check("llama3_workspace_size", lib().llama3_workspace_size(ctypes.byref(cfg), batch, seq, lm_rows,
                                                                ctypes.byref(n)))
    return n.value


def llama3_embed(cfg, ids, table, x, n_tokens, stream=None):
    _check("llama3_embed", lib().llama3_embed(ctypes.byref(cfg), _ptr(ids), _ptr(table), _ptr(x), n_tokens,
                                              _stream(stream)))


def llama3_layer_forward(cfg, w, rope, rope_len, x, k_cache, v_cache, cache_cap, batch, seq, start_pos, ws,
                         ws_bytes, stream=None):
    _check("llama3_layer_forward", lib().llama3_layer_forward(
        ctypes.byref(cfg), ctypes.byref(w), _ptr(rope), rope_len, _ptr(x), _ptr(k_cache), _ptr(v_cache),
        cache_cap, batch, seq, start_pos, _ptr(ws), ws_bytes, _stream(stream)))


def llama3_layer_forward_docs(cfg, w, rope, rope_len, x, k_cache, v_cache, cache_cap, batch, seq, start_pos,
                              doc_start, ws, ws_bytes, stream=None):
    _check("llama3_layer_forward_docs", lib().llama3_layer_forward_docs(
        ctypes.byref(cfg), ctypes.byref(w), _ptr(rope), rope_len, _ptr(x), _ptr(k_cache), _ptr(v_cache),
        cache_cap, batch, seq, start_pos, _ptr(doc_start), _ptr(ws), ws_bytes, _stream(stream)))


def llama3_attention_docs(cfg, q, k_cache, v_cache, cache_cap, batch, seq, start_pos, doc_start, out, ws,
                          ws_bytes, stream=None):
    _check("llama3_attention_docs", lib().llama3_attention_docs(
        ctypes.byref(cfg), _ptr(q), _ptr(k_cache), _ptr(v_cache), cache_cap, batch, seq, start_pos,
        _ptr(doc_start), _ptr(out), _ptr(ws), ws_bytes, _stream(stream)))


def llama3_layer_decode(cfg, w, rope, rope_len, x, k_cache, v_cache, cache_cap, batch, start_pos, ws, ws_bytes,
                        stream=None):
    _check("llama3_layer_decode", lib().llama3_layer_decode(
        ctypes.byref(cfg), ctypes.byref(w), _ptr(rope), rope_len, _ptr(x), _ptr(k_cache), _ptr(v_cache),
        cache_cap, batch, start_pos, _ptr(ws), ws_bytes, _stream(stream)))


def llama3_layer_decode_ragged(cfg, w, rope, rope_len, x, k_cache, v_cache, cache_cap, batch, positions,
                               max_position, ws, ws_bytes, stream=None):
    """One decode step with every sequence at its own position (int32 device tensor [batch])."""
    _check("llama3_layer_decode_ragged", lib().llama3_layer_decode_ragged(
        ctypes.byref(cfg), ctypes.byref(w), _ptr(rope), rope_len, _ptr(x), _ptr(k_cache), _ptr(v_cache),
        cache_cap, batch, _ptr(positions), max_position, _ptr(ws), ws_bytes, _stream(stream)))


def llama3_layer_decode_chained(cfg, w, rope, rope_len, x, k_cache, v_cache, cache_cap, batch, start_pos, positions,
                                next_attention_norm, input_normalised, ws, ws_bytes, stream=None):
    """One decode step of one block that can take its normalised input from the
    previous block's call and leave the next block's in the workspace."""
    _check("llama3_layer_decode_chained", lib().llama3_layer_decode_chained(
        ctypes.byref(cfg), ctypes.byref(w), _ptr(rope), rope_len, _ptr(x), _ptr(k_cache), _ptr(v_cache),
        cache_cap, batch, start_pos, _ptr(positions), _ptr(next_attention_norm), 1 if input_normalised else 0,
        _ptr(ws), ws_bytes, _stream(stream)))


def llama3_decode_step(cfg, weights, rope, rope_len, x, k_caches, v_caches, cache_cap, batch, start_pos, positions,
                       ws, ws_bytes, stream=None):
    """One decode step through every block of the stack, in order: ``weights``
    is a sequence of llama3_layer_weights structs, ``k_caches``/``v_caches``
    the blocks' cache tensors."""
    n = len(weights)
    arr = (llama3_layer_weights * n)(*weights)
    kp = (ctypes.c_void_p * n)(*[t.data_ptr() for t in k_caches])
    vp = (ctypes.c_void_p * n)(*[t.data_ptr() for t in v_caches])
    _check("llama3_decode_step", lib().llama3_decode_step(
        ctypes.byref(cfg), arr, n, _ptr(rope), rope_len, _ptr(x), ctypes.cast(kp, ctypes.c_void_p),
        ctypes.cast(vp, ctypes.c_void_p), cache_cap, batch, start_pos, _ptr(positions), _ptr(ws), ws_bytes,
        _stream(stream)))


def llama3_lm_head_argmax(cfg, norm_w, w_out, h, rows, row_stride, ids_out, logits_out, ws, ws_bytes,
                          stream=None):
    _check("llama3_lm_head_argmax", lib().llama3_lm_head_argmax(
        ctypes.byref(cfg), _ptr(norm_w), _ptr(w_out), _ptr(h), rows, row_stride, _ptr(ids_out),
        _ptr(logits_out), _ptr(ws), ws_bytes, _stream(stream)))


def llama3_sample_top_p(logits, rows, ld, vocab, temperature, top_p, seed, offset, ids_out, stream=None,
                        positions=None):
    """Temperature / top-p draw of one token per row of fp32 logits (the
    draw counter of row r is offset, plus positions[r] when given)."""
    _check("llama3_sample_top_p", lib().llama3_sample_top_p(
        _ptr(logits), rows, ld, vocab, float(temperature), float(top_p), int(seed) & (2 ** 64 - 1),
        int(offset) & (2 ** 64 - 1), _ptr(positions), _ptr(ids_out), _stream(stream)))


def llama3_gather_rows(cfg, x, row_stride, n_rows, row_index, rows, out, stream=None):
    """out[r] = x[row_index[r]] (dim elements per row)."""
    _check("llama3_gather_rows", lib().llama3_gather_rows(
        ctypes.byref(cfg), _ptr(x), row_stride, n_rows, _ptr(row_index), rows, _ptr(out), _stream(stream)))


def llama3_generation_advance(positions, ids, history, step, batch, history_rows, history_stride, stream=None,
                              done=None, eos_id=-1):
    """history[step] = ids, positions += 1, step += 1, all on the device; with
    eos_id >= 0 and done (int32 [batch + 1]), sequences stop at the end token."""
    _check("llama3_generation_advance", lib().llama3_generation_advance(
        _ptr(positions), _ptr(ids), _ptr(history), _ptr(step), _ptr(done), int(eos_id), batch, history_rows,
        history_stride, _stream(stream)))


NOALLOC_SCRATCH_BYTES = 4 << 20


def llama3_lm_head_argmax_noalloc(cfg, norm_w, w_out, h, rows, row_stride, ids_out, logits_out, stream=None):
    """LM head + argmax for callers that cannot pass a workspace: the library
    uses its own fixed 4 MiB device scratch (shared by all calls)."""
    _check("llama3_lm_head_argmax_noalloc", lib().llama3_lm_head_argmax_noalloc(
        ctypes.byref(cfg), _ptr(norm_w), _ptr(w_out), _ptr(h), rows, row_stride, _ptr(ids_out),
        _ptr(logits_out), _stream(stream)))


def llama3_rmsnorm(cfg, x, row_stride, w, y, rows, stream=None):
    _check("llama3_rmsnorm", lib().llama3_rmsnorm(ctypes.byref(cfg), _ptr(x), row_stride, _ptr(w), _ptr(y), rows,
                                                  _stream(stream)))


def llama3_linear(cfg, x, w, residual, y, m, n, k, ws=None, ws_bytes=0, stream=None):
    _check("llama3_linear", lib().llama3_linear(ctypes.byref(cfg), _ptr(x), _ptr(w), _ptr(residual), _ptr(y), m, n,
                                                k, _ptr(ws), ws_bytes, _stream(stream)))


def llama3_attention(cfg, q, k_cache, v_cache, cache_cap, batch, seq, start_pos, out, ws, ws_bytes, stream=None):
    _check("llama3_attention", lib().llama3_attention(
        ctypes.byref(cfg), _ptr(q), _ptr(k_cache), _ptr(v_cache), cache_cap, batch, seq, start_pos, _ptr(out),
        _ptr(ws), ws_bytes, _stream(stream)))


def llama3_status_string(status):
    return lib().llama3_status_string(status).decode()


def llama3_device_status():
    v = ctypes.c_int(0)
    _check("llama3_device_status", lib().llama3_device_status(ctypes.byref(v)))
    return v.value


def llama3_last_cuda_error():
    return lib().llama3_last_cuda_error()


def llama3_set_kernel_path(path):
    return lib().llama3_set_kernel_path(path)


def llama3_set_wait_limit_ms(ms):
    return lib().llama3_set_wait_limit_ms(ms)


def llama3_set_test_withheld_arrival(which):
    """Failure-detection test hook (0 = off): 1 makes the GEMMs' accumulator
    wait give up, 2 the prefill attention's wait for P."""
    return lib().llama3_set_test_withheld_arrival(int(which))


def llama3_set_programmatic_launch(on):
    return lib().llama3_set_programmatic_launch(1 if on else 0)


KERNEL_KINDS = {"gemm_qkv": 1, "gemm_wo": 2, "gemm_w13": 3, "gemm_w2": 4, "attention": 5, "decode_gemm": 6,
                "decode_attention": 7, "lm_head": 8, "norm": 9, "elementwise": 10, "sample": 11}


def llama3_set_launch_timer(kind, start_events, stop_events):
    """Time the next len(start_events) launches of a kernel family with the
    given torch.cuda.Event pairs (created with enable_timing=True)."""
    n = len(start_events)
    arr = (ctypes.c_void_p * max(n, 1))
    s = arr(*[e.cuda_event for e in start_events])
    t = arr(*[e.cuda_event for e in stop_events])
    k = KERNEL_KINDS.get(kind, kind)
    _check("llama3_set_launch_timer", lib().llama3_set_launch_timer(k, s, t, n))


def llama3_launch_timer_used():
    return lib().llama3_launch_timer_used()


def llama3_launch_count():
    return lib().llama3_launch_count()
