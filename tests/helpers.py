"""Shared test glue: tolerance checks, host copies, oracle-side weight dicts."""
import numpy as np
import torch

# Tolerances per element: |gpu - oracle| <= atol + rtol * |oracle|
TOL = {"bf16": (2e-2, 2e-2), "f32": (1e-4, 1e-4)}
ARGMAX_GAP = 1e-2


def f64(t):
    """Exact host copy of a bf16/fp32 tensor as float64."""
    return t.detach().to(torch.float32).cpu().numpy().astype(np.float64)


def assert_close(gpu, oracle, dtype, what=""):
    g = f64(gpu) if isinstance(gpu, torch.Tensor) else np.asarray(gpu, dtype=np.float64)
    o = np.asarray(oracle, dtype=np.float64)
    assert g.shape == o.shape, (what, g.shape, o.shape)
    atol, rtol = TOL[dtype]
    err = np.abs(g - o)
    bound = atol + rtol * np.abs(o)
    bad = ~(err <= bound)   # a NaN on either side counts as out of tolerance
    if bad.any():
        i = np.unravel_index(np.argmax(err - bound), err.shape)
        raise AssertionError(f"{what}: {bad.sum()} of {bad.size} elements out of tolerance; worst at {i}: "
                             f"gpu={g[i]!r} oracle={o[i]!r} (max |err|={err.max():.3g})")


def assert_argmax(gpu_ids, oracle_logits, what=""):
    """ids must equal the oracle's argmax wherever its top-2 gap exceeds 1e-2."""
    ids = gpu_ids.detach().cpu().numpy().astype(np.int64).reshape(-1)
    lg = np.asarray(oracle_logits).reshape(len(ids), -1)
    top2 = np.sort(lg, axis=1)[:, -2:]
    decided = (top2[:, 1] - top2[:, 0]) > ARGMAX_GAP
    want = np.argmax(lg, axis=1)
    assert decided.any(), f"{what}: no row has a decided argmax"
    mism = decided & (ids != want)
    assert not mism.any(), f"{what}: ids differ at rows {np.nonzero(mism)[0][:10]}"
    assert np.all((ids >= 0) & (ids < lg.shape[1]))


def oracle_layer(layer):
    """Host fp64 copies of one layer's weights under the page's names."""
    return {k: f64(layer[k]) for k in ("attention_norm", "wq", "wk", "wv", "wo", "ffn_norm", "w1", "w2", "w3")}


def oracle_cfg(w):
    c = w.cfg()
    return dict(dim=c["dim"], n_heads=c["n_heads"], n_kv_heads=c["n_kv_heads"], head_dim=c["head_dim"],
                ffn_hidden=c["ffn_hidden"], norm_eps=c["norm_eps"], rope_theta=c["rope_theta"])
