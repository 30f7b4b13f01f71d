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


# ---------------------------------------------------------------------------
# Full-size bound.  At the 8B sizes (and any layer of comparable width) the
# per-element bound above is out of reach for a path that stores its
# activations in bf16: the fp64 oracle with bf16 storage at the same step
# boundaries (oracle rounding="bf16") already misses it on a few percent of
# a block's outputs, and on most elements after 32 blocks.  There the GPU is
# held to that variant instead: its relative L2 distance from the exact
# oracle may be at most NOISE_FACTOR times the variant's own distance, and
# argmax ids must match wherever the exact top-2 gap exceeds ARGMAX_NOISE_K
# times the variant's logit error (and 1e-2).
NOISE_FACTOR = 1.5
ARGMAX_NOISE_K = 6.0


def rel_l2(a, b):
    a, b = np.asarray(a, np.float64), np.asarray(b, np.float64)
    return float(np.linalg.norm(a - b) / np.linalg.norm(b))


def within_bound_fraction(got, want, dtype="bf16"):
    atol, rtol = TOL[dtype]
    got, want = np.asarray(got, np.float64), np.asarray(want, np.float64)
    return float(np.mean(np.abs(got - want) <= atol + rtol * np.abs(want)))


def assert_within_bf16_noise(gpu, exact, bf16_variant, what, factor=NOISE_FACTOR):
    """rel_l2(gpu, exact) <= factor * rel_l2(bf16 variant, exact); returns both
    (and the fraction of elements each keeps inside the per-element bound)."""
    g = f64(gpu) if isinstance(gpu, torch.Tensor) else np.asarray(gpu, dtype=np.float64)
    e = np.asarray(exact, np.float64)
    r = np.asarray(bf16_variant, np.float64)
    assert g.shape == e.shape == r.shape, (what, g.shape, e.shape, r.shape)
    assert np.all(np.isfinite(g)), f"{what}: non-finite values"
    rg, rr = rel_l2(g, e), rel_l2(r, e)
    info = dict(rel_gpu=rg, rel_bf16=rr, in_bound_gpu=within_bound_fraction(g, e),
                in_bound_bf16=within_bound_fraction(r, e))
    assert rg <= factor * rr, f"{what}: {info}"
    return info


def assert_argmax_beyond_noise(gpu_ids, exact_logits, bf16_logits, what, k=ARGMAX_NOISE_K, need=1):
    """ids equal the exact argmax on every row whose exact top-2 gap exceeds
    max(1e-2, k * std(bf16 variant logits - exact logits) of that row); at
    least `need` rows must be decided that way.  Returns the decided count."""
    ids = gpu_ids.detach().cpu().numpy().astype(np.int64).reshape(-1)
    lg = np.asarray(exact_logits, np.float64).reshape(len(ids), -1)
    lr = np.asarray(bf16_logits, np.float64).reshape(len(ids), -1)
    noise = np.std(lr - lg, axis=1)
    top2 = np.sort(lg, axis=1)[:, -2:]
    decided = (top2[:, 1] - top2[:, 0]) > np.maximum(ARGMAX_GAP, k * noise)
    want = np.argmax(lg, axis=1)
    assert decided.sum() >= need, f"{what}: only {decided.sum()} decided rows (noise {noise.mean():.3g})"
    mism = decided & (ids != want)
    assert not mism.any(), f"{what}: ids differ at rows {np.nonzero(mism)[0][:10]}"
    assert np.all((ids >= 0) & (ids < lg.shape[1]))
    return int(decided.sum())


# ---------------------------------------------------------------------------
# Guard bands: the cheap stand-in for a memory checker.  Every output, cache,
# workspace and state buffer a GPU test hands the library sits between two
# bands of a fixed byte pattern; after the test every band must be intact, so
# a kernel writing past either end of a buffer fails the test that ran it.
# ---------------------------------------------------------------------------
class GuardArena:
    BAND = 4096          # bytes on each side (keeps the payload 256-byte aligned)
    PATTERN = 0xA5

    def __init__(self, device="cuda"):
        self.device = device
        self.bufs = []

    def empty(self, shape, dtype=torch.float32, device=None):
        shape = tuple(shape) if isinstance(shape, (tuple, list)) else (int(shape),)
        n = 1
        for s in shape:
            n *= int(s)
        nbytes = n * torch.tensor([], dtype=dtype).element_size()
        raw = torch.empty((2 * self.BAND + nbytes,), dtype=torch.uint8, device=device or self.device)
        raw[:self.BAND].fill_(self.PATTERN)
        raw[self.BAND + nbytes:].fill_(self.PATTERN)
        self.bufs.append((raw, nbytes))
        return raw[self.BAND:self.BAND + nbytes].view(dtype).view(shape)

    def zeros(self, shape, dtype=torch.float32, device=None):
        return self.empty(shape, dtype, device).zero_()

    def full(self, shape, value, dtype=torch.float32, device=None):
        return self.empty(shape, dtype, device).fill_(value)

    def empty_like(self, t):
        return self.empty(t.shape, t.dtype, t.device)

    def to(self, t):
        """A guarded device copy of host tensor t (for buffers a call updates in place)."""
        return self.empty(t.shape, t.dtype).copy_(t)

    def alloc(self, shape, dtype, device):
        return self.empty(shape, dtype, device)

    def check(self):
        bad = []
        for i, (raw, nbytes) in enumerate(self.bufs):
            head = raw[:self.BAND]
            tail = raw[self.BAND + nbytes:]
            if not (bool(torch.all(head == self.PATTERN)) and bool(torch.all(tail == self.PATTERN))):
                bad.append((i, nbytes))
        self.bufs.clear()
        assert not bad, f"guard band overwritten around buffers (index, bytes): {bad}"
