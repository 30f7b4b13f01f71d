"""The C-ABI library without a GPU: it loads, exports every symbol the header
declares, and rejects bad arguments on the host before launching anything.
No compute call reaches the device here."""
import ctypes
import subprocess

import pytest

from llama_decoder_only_rmsnorm_b200 import binding as B


def test_library_loads_and_exports_every_header_symbol():
    lib = B.lib()
    declared = B.header_functions()
    assert len(declared) >= 14
    for name in declared:
        assert hasattr(lib, name), name
    out = subprocess.run(["nm", "-D", "--defined-only", B.LIB_PATH], capture_output=True, text=True).stdout
    exported = {l.split()[-1] for l in out.splitlines() if " T " in l}
    assert set(declared) <= exported
    assert set(B._SIGNATURES) == set(declared)


def test_status_strings():
    for code in range(8):
        assert B.llama3_status_string(code)
    assert B.llama3_status_string(0) == "ok"
    assert "unknown" in B.llama3_status_string(99)


def cfg8b(**kw):
    d = dict(dim=4096, n_heads=32, n_kv_heads=8, ffn_hidden=14336, vocab=128256)
    d.update(kw)
    return B.make_config(**d)


def test_workspace_size_and_config_validation():
    n = B.llama3_workspace_size(cfg8b(), 1, 8192, 1)
    # xn, q, o: 3 x 8192 x 4096 bf16; g: 8192 x 14336 bf16
    assert n >= (3 * 8192 * 4096 + 8192 * 14336) * 2
    assert B.llama3_workspace_size(cfg8b(), 32, 1, 32) < n
    bad = [cfg8b(dim=4000), cfg8b(n_kv_heads=7), cfg8b(dim=4096 + 32, n_heads=33),
           B.make_config(48 * 8, 8, 2, 1024, 10),           # head_dim 48: not a supported size
           cfg8b(ffn_hidden=14337), cfg8b(norm_eps=0.0), cfg8b(rope_theta=1.0)]
    for c in bad:
        with pytest.raises(B.Llama3Error) as e:
            B.llama3_workspace_size(c, 1, 16, 1)
        assert e.value.status == 1
    # head_dim 16 and 32 are valid in fp32 and bf16 (SIMT kernels)
    assert B.llama3_workspace_size(B.make_config(64, 4, 2, 192, 3771, dtype="f32"), 4, 16, 64) > 0
    assert B.llama3_workspace_size(B.make_config(64, 4, 2, 192, 10, dtype="bf16"), 4, 16, 1) > 0
    assert B.llama3_workspace_size(B.make_config(1024, 32, 8, 4096, 10), 2, 16, 1) > 0
    with pytest.raises(B.Llama3Error):
        B.llama3_workspace_size(cfg8b(), 0, 16, 1)


FAKE = 1 << 20  # an aligned, never-dereferenced address: these calls must fail first


def _weights(ptr=FAKE):
    return B.llama3_layer_weights(*([ptr] * 7))


def test_layer_calls_reject_bad_arguments_before_launch():
    c = cfg8b()
    lib = B.lib()
    w = _weights()
    ws_bytes = B.llama3_workspace_size(c, 2, 16, 1)
    call = lambda **k: lib.llama3_layer_forward(
        ctypes.byref(c), ctypes.byref(k.get("w", w)), k.get("rope", FAKE), k.get("rope_len", 64),
        k.get("x", FAKE), FAKE, FAKE, k.get("cap", 64), k.get("batch", 2), k.get("seq", 16),
        k.get("start", 0), k.get("ws", FAKE), k.get("ws_bytes", ws_bytes), None)
    assert call(start=60) == 1            # start_pos + seq > cache_cap
    assert call(rope_len=8) == 1          # RoPE table too short
    assert call(batch=0) == 1
    assert call(x=None) == 1
    assert call(x=FAKE + 8) == 2          # misaligned
    assert call(w=_weights(FAKE + 2)) == 2
    assert call(ws=None) == 3
    assert call(ws_bytes=ws_bytes - 1) == 3
    dec = lib.llama3_layer_decode(ctypes.byref(c), ctypes.byref(w), FAKE, 64, FAKE, FAKE, FAKE, 64, 2, 64,
                                  FAKE, ws_bytes, None)
    assert dec == 1                       # position 64 does not fit a 64-entry cache
    chained = lambda **k: lib.llama3_layer_decode_chained(
        ctypes.byref(c), ctypes.byref(w), FAKE, 64, FAKE, FAKE, FAKE, 64, 2, k.get("start", 10),
        k.get("positions", None), k.get("next_norm", None), 1, FAKE, ws_bytes, None)
    assert chained(start=64) == 1         # max position 64 does not fit a 64-entry cache
    assert chained(next_norm=FAKE + 2) == 2
    assert chained(positions=FAKE + 2) == 2


def test_lm_head_and_helpers_reject_bad_arguments():
    c = cfg8b()
    lib = B.lib()
    ws_bytes = B.llama3_workspace_size(c, 1, 1, 32)
    lm = lambda **k: lib.llama3_lm_head_argmax(ctypes.byref(c), FAKE, FAKE, FAKE, k.get("rows", 32),
                                               k.get("stride", 4096), FAKE, None, k.get("ws", FAKE),
                                               k.get("ws_bytes", ws_bytes), None)
    assert lm(rows=0) == 1
    assert lm(stride=100) == 1
    assert lm(stride=4100) == 2           # row stride not a multiple of 16 bytes
    assert lm(ws_bytes=16) == 3
    assert lib.llama3_rmsnorm(ctypes.byref(c), FAKE, 4095, FAKE, FAKE, 4, None) == 1
    assert lib.llama3_embed(ctypes.byref(cfg8b(vocab=0)), FAKE, FAKE, FAKE, 4, None) == 1
    assert lib.llama3_init_rope_table(FAKE, 127, 16, 500000.0, None) == 1
    assert lib.llama3_init_rope_table(FAKE, 128, 16, 1.0, None) == 1
    assert lib.llama3_attention(ctypes.byref(c), FAKE, FAKE, FAKE, 8, 1, 9, 0, FAKE, FAKE, 1 << 30, None) == 1


def test_decode_step_rejects_bad_arguments_before_launch():
    lib = B.lib()
    c = cfg8b()
    ws = (B.llama3_layer_weights * 2)(_weights(), _weights())
    caches = (ctypes.c_void_p * 2)(FAKE, FAKE)
    cp = ctypes.cast(caches, ctypes.c_void_p)
    step = lambda **k: lib.llama3_decode_step(ctypes.byref(c), k.get("w", ws), k.get("n", 2), FAKE, 9000, FAKE,
                                              k.get("kc", cp), cp, k.get("cap", 8193), k.get("batch", 32),
                                              k.get("pos", 8192), k.get("positions", None), FAKE,
                                              k.get("ws_bytes", 1 << 40), None)
    assert step(n=0) == 1
    assert step(w=None) == 1
    assert step(kc=None) == 1
    assert step(pos=8193) == 1                        # start_pos + 1 > cache capacity
    assert step(batch=0) == 1
    assert step(positions=ctypes.c_void_p(FAKE + 2)) == 2
    assert step(ws_bytes=16) == 3
    bad = (ctypes.c_void_p * 2)(FAKE, FAKE + 8)       # second block's cache not 16-byte aligned
    assert step(kc=ctypes.cast(bad, ctypes.c_void_p)) == 2


def test_kernel_path_and_wait_limit_switches():
    assert B.llama3_set_kernel_path(1) == 0
    assert B.llama3_set_kernel_path(0) == 1
    assert B.llama3_set_kernel_path(2) == 0        # anything but 1 selects the tcgen05 kernels
    assert B.llama3_set_kernel_path(0) == 0
    old = B.llama3_set_wait_limit_ms(500)
    assert B.llama3_set_wait_limit_ms(old) == 500
    assert B.llama3_set_test_withheld_arrival(1) == 0      # test hook, off by default
    assert B.llama3_set_test_withheld_arrival(7) == 1      # unknown values switch it off
    assert B.llama3_set_test_withheld_arrival(0) == 0


def test_sample_top_p_rejects_bad_arguments_before_launch():
    lib = B.lib()
    f = ctypes.c_float
    s = lambda **k: lib.llama3_sample_top_p(k.get("logits", FAKE), k.get("rows", 4), k.get("ld", 100),
                                            k.get("vocab", 100), f(k.get("t", 0.7)), f(k.get("p", 0.9)),
                                            1, 0, k.get("pos", None), k.get("ids", FAKE), None)
    assert s(rows=0) == 1
    assert s(vocab=0) == 1
    assert s(ld=99) == 1
    assert s(p=-0.1) == 1
    assert s(p=float("nan")) == 1
    assert s(t=float("nan")) == 1
    assert s(logits=None) == 1
    assert s(ids=ctypes.c_void_p(18)) == 2   # ids not 4-byte aligned
    assert s(pos=ctypes.c_void_p(FAKE + 2)) == 2
    c = cfg8b()
    gat = lambda **k: lib.llama3_gather_rows(ctypes.byref(c), FAKE, k.get("stride", 4096), k.get("n", 8), FAKE,
                                             k.get("rows", 2), FAKE, None)
    assert gat(rows=0) == 1
    assert gat(n=0) == 1
    assert gat(stride=100) == 1
    assert gat(stride=4100) == 2
    adv = lambda **k: lib.llama3_generation_advance(k.get("pos", FAKE), FAKE, FAKE, FAKE, k.get("done", None),
                                                    k.get("eos", -1), k.get("batch", 4), k.get("rows", 8),
                                                    k.get("stride", 4), None)
    assert adv(eos=7) == 1                          # an end token needs the done flags
    assert adv(eos=7, done=ctypes.c_void_p(FAKE + 2)) == 2
    assert adv(batch=0) == 1
    assert adv(rows=0) == 1
    assert adv(stride=3) == 1
    assert adv(pos=None) == 1
    assert adv(pos=ctypes.c_void_p(FAKE + 1)) == 2
    assert B.KERNEL_KINDS["sample"] == 11
