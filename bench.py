#!/usr/bin/env python
"""Throughput of the Llama-3-8B-shaped decoder on B200 through the C ABI.

One JSON line (rank 0).  `value` is prefill tokens/s for batch 1 x 8192 tokens
through embedding, 32 decoder blocks, final norm and LM-head argmax on the
last position; the `decode` object is the same for one decode step of 32
sequences against 8192 cached positions each (new token at position 8192).
Weights are seeded random-init N(0, 0.02) bf16 of the 8B architecture, token
ids uniform; everything is resident in HBM before the timed region, and the
16 GB of weights streamed per step are far larger than L2.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Under torchrun (N > 1) every rank runs its own replica of the prefill (no
collective on the data path; `scaling: weak`), and the decode step's 32
sequences are split over the ranks (each holds the model and its own
sequences' caches; the next-token ids are gathered on the host); times are the
max over ranks.
"""
import argparse
import datetime
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

from llama_decoder_only_rmsnorm_b200 import binding as B  # noqa: E402
from llama_decoder_only_rmsnorm_b200 import inputs as I  # noqa: E402
from llama_decoder_only_rmsnorm_b200.model import Llama3Stack  # noqa: E402
from llama_decoder_only_rmsnorm_b200.sharding import gather_ids, shard  # noqa: E402

METRIC = "prefill & decode tokens/s on 1 B200; % of bf16 tensor / HBM roofline"
PREFILL, DECODE = I.WORKLOADS["llama3_8b_prefill"], I.WORKLOADS["llama3_8b_decode"]
PEAKS_PATH = os.path.join(ROOT, "MEASURED_PEAKS.json")
TRAFFIC_PATH = os.path.join(ROOT, "profiles", "traffic.json")
# Used only when MEASURED_PEAKS.json is absent: the pool's earlier measurement
# of a plain copy (HBM) and of a cuBLAS bf16 GEMM burst.  No sustained figure
# exists for the fallback, so a kernel inside a long step is compared with the
# burst one (reported as such).
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0}


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=10)
    p.add_argument("--warmup", type=int, default=3)
    p.add_argument("--impl", default="ours", choices=["ours", "reference"])
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-decode", action="store_true")
    p.add_argument("--layers", type=int, default=None, help=argparse.SUPPRESS)  # profiling captures only
    p.add_argument("--no-pdl", action="store_true", help=argparse.SUPPRESS)   # A/B of programmatic launch
    return p.parse_args()


# --------------------------------------------------------------- plumbing ---
def dist_setup():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    if world > 1:
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                             device_id=torch.device("cuda", local))
    return world, rank, local


def barrier(world):
    if world > 1:
        torch.distributed.barrier()


def max_over_ranks(v, world, device="cuda"):
    """Largest value over all ranks (timings: the slowest rank defines the step)."""
    if world == 1:
        return v
    t = torch.tensor([v], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def load_peaks():
    try:
        with open(PEAKS_PATH) as f:
            return json.load(f), "measured"
    except OSError:
        return FALLBACK_PEAKS, "fallback"


def source_hash(files):
    h = hashlib.sha256()
    for f in files:
        with open(os.path.join(ROOT, f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def recorded_traffic(kind, files):
    """Per-launch DRAM bytes from a committed ncu capture, if the kernel's
    sources are unchanged since it was taken; else None."""
    try:
        with open(TRAFFIC_PATH) as f:
            rec = json.load(f).get(kind)
    except (OSError, ValueError):
        return None
    if not rec or rec.get("source_sha") != source_hash(files):
        return None
    return rec.get("traffic_bytes_per_launch")


class ClockSampler:
    """nvidia-smi clock/throttle samples every 200 ms while the timed region runs."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def __enter__(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                                          "-i", str(self.gpu), "-lms", "200"], stdout=open(self.path, "w"),
                                         stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *a):
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        rows = []
        try:
            for line in open(self.path):
                parts = [x.strip() for x in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        except OSError:
            pass
        finally:
            if self.path and os.path.exists(self.path):
                os.remove(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        smax = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        power = [float(r[3]) for r in rows if r[3].replace(".", "").isdigit()]
        loaded = [s for s, p in zip(sm, power) if p > 300.0] or sm
        reasons = set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            for n, v in zip(names, r[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(loaded) if loaded else None, "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(rows)}


def event_pairs(n):
    """n (start, stop) event pairs, each recorded once so that its CUDA event
    exists before its handle goes to the library (torch creates them lazily)."""
    pairs = ([torch.cuda.Event(enable_timing=True) for _ in range(n)],
             [torch.cuda.Event(enable_timing=True) for _ in range(n)])
    for e in pairs[0] + pairs[1]:
        e.record()
    return pairs


# ------------------------------------------------------------------ model ---
def build(dev, n_layers):
    w = PREFILL
    layers = [I.layer_weights(w, i, dev) for i in range(n_layers)]
    outw = I.output_weights(w, dev)
    return layers, outw


def time_steps(fn, steps, warmup, world, name="timed"):
    """W untimed warm-up steps, then K steps between CUDA events on the
    current stream, bracketed by a barrier and a synchronize on both sides.
    Returns (max over ranks of ms per step, library launches in the region)."""
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    if B.llama3_device_status() != 0:
        raise RuntimeError("device status word set during warm-up")
    barrier(world)
    torch.cuda.synchronize()
    l0 = B.llama3_launch_count()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.nvtx.range_push(name)
    t0.record()
    for _ in range(steps):
        fn()
    t1.record()
    torch.cuda.nvtx.range_pop()
    torch.cuda.synchronize()
    launches = B.llama3_launch_count() - l0
    if B.llama3_device_status() != 0:
        raise RuntimeError("device status word set during the timed region")
    barrier(world)
    ms = t0.elapsed_time(t1) / steps
    return max_over_ranks(ms, world), launches


def kernel_times(fn, kind, n_pairs, steps=1):
    """Per-launch times (ms) of the first n_pairs launches of kernel family
    `kind` during `steps` eager calls of fn, from CUDA events the library
    records on the launching stream.  Run apart from the timed region: an
    event between two kernels ends their programmatic overlap."""
    starts, stops = event_pairs(n_pairs)
    B.llama3_set_launch_timer(kind, starts, stops)
    try:
        for _ in range(steps):
            fn()
        torch.cuda.synchronize()
        used = B.llama3_launch_timer_used()
    finally:
        B.llama3_set_launch_timer(kind, [], [])
    return [s.elapsed_time(e) for s, e in zip(starts[:used], stops[:used])]


def graph_kernel_times(step, kind, n_pairs, replays=3):
    """As kernel_times, for a step captured in its own CUDA graph: the events
    become graph nodes and every replay re-records them; the last replay's
    times are returned."""
    starts, stops = event_pairs(n_pairs)
    B.llama3_set_launch_timer(kind, starts, stops)
    g = torch.cuda.CUDAGraph()
    try:
        with torch.cuda.graph(g):
            step()
        used = B.llama3_launch_timer_used()
    finally:
        B.llama3_set_launch_timer(kind, [], [])
    for _ in range(replays):
        g.replay()
    torch.cuda.synchronize()
    out = [s.elapsed_time(e) for s, e in zip(starts[:used], stops[:used])]
    del g
    return out


# ------------------------------------------------------- oracle baseline ---
def oracle_sample(layers, outw, caches, prefix, decode_seq=True):
    """Time the fp64 oracle (as it stands) on a bounded sample of both
    workloads: the first `prefix` tokens of the prefill through all blocks +
    final norm + LM head, and one sequence's decode step at position 8192.
    Weight conversion to fp64 is outside the timed region."""
    from oracle import llama3_oracle as O
    import threadpoolctl
    cfg = {k: v for k, v in PREFILL.cfg().items() if k not in ("vocab", "dtype")}
    f64 = lambda t: t.detach().to(torch.float32).cpu().numpy().astype(np.float64)
    ids = I.token_ids(PREFILL, "cuda")[:, :prefix].cpu().numpy()
    dids = I.token_ids(DECODE, "cuda")[:1].cpu().numpy()
    table = outw["tok_embeddings"]

    def embed(id_arr):
        # the oracle's gather over the rows this sample uses (a small table)
        uniq, inv = np.unique(id_arr, return_inverse=True)
        sub = f64(table[torch.as_tensor(uniq, device=table.device).long()])
        return O.embed(inv.reshape(id_arr.shape), sub)

    x = embed(ids)
    xd = embed(dids)
    t_pre = t_dec = 0.0
    P = DECODE.cache_len
    for i, layer in enumerate(layers):
        ol = {k: f64(layer[k]) for k in ("attention_norm", "wq", "wk", "wv", "wo", "ffn_norm", "w1", "w2", "w3")}
        kc = np.zeros((1, prefix, cfg["n_kv_heads"], cfg["head_dim"]))
        vc = np.zeros_like(kc)
        t = time.perf_counter()
        x = O.decoder_block(x, ol, cfg, kc, vc, 0)
        t_pre += time.perf_counter() - t
        if decode_seq:
            kd = np.zeros((1, P + 1, cfg["n_kv_heads"], cfg["head_dim"]))
            vd = np.zeros_like(kd)
            kd[0, :P] = f64(caches[i][0][0, :P])
            vd[0, :P] = f64(caches[i][1][0, :P])
            t = time.perf_counter()
            xd = O.decoder_block(xd, ol, cfg, kd, vd, P)
            t_dec += time.perf_counter() - t
        del ol
    nw, wout = f64(outw["norm"]), f64(outw["output"])
    t = time.perf_counter()
    O.lm_head(x[:, -1], nw, wout, PREFILL.norm_eps)
    t_pre += time.perf_counter() - t
    if decode_seq:
        t = time.perf_counter()
        O.lm_head(xd[:, -1], nw, wout, PREFILL.norm_eps)
        t_dec += time.perf_counter() - t
    info = threadpoolctl.threadpool_info()
    cores = max([d.get("num_threads", 1) for d in info] or [os.cpu_count()])
    return t_pre, t_dec, cores


# ------------------------------------------------------------- our arm ---
DECODE_GEMMS = (("wqkv", 6144 * 4096 * 2), ("wo", 4096 * 4096 * 2), ("w1|w3", 2 * 14336 * 4096 * 2),
                ("w2", 4096 * 14336 * 2))   # weight bytes each decode GEMM streams (8B shapes)


def attention_alone(cfg, dev, peaks, peak_kind, a_flop, warmup=3, reps=20):
    """The prefill attention kernel timed alone: one launch per pair of CUDA
    events, with a 256 MB buffer (more than L2) written before each launch.
    Seeded N(0, 1) bf16 q, k and v of the 8B prefill shape.  A kernel timed
    alone is compared with the burst GEMM peak."""
    S, H, KV, hd = PREFILL.seq, PREFILL.n_heads, PREFILL.n_kv_heads, PREFILL.head_dim
    g = torch.Generator(device=dev).manual_seed(8192)
    q = torch.randn((1, S, H, hd), generator=g, device=dev).to(torch.bfloat16)
    kc = torch.randn((1, S, KV, hd), generator=g, device=dev).to(torch.bfloat16)
    vc = torch.randn((1, S, KV, hd), generator=g, device=dev).to(torch.bfloat16)
    out = torch.empty((1, S, H * hd), dtype=torch.bfloat16, device=dev)
    ws = torch.empty(B.llama3_workspace_size(cfg, 1, S), dtype=torch.uint8, device=dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    times = []
    for i in range(warmup + reps):
        flush.zero_()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        B.llama3_attention(cfg, q, kc, vc, S, 1, S, 0, out, ws, ws.numel())
        e1.record()
        torch.cuda.synchronize()
        if i >= warmup:
            times.append(e0.elapsed_time(e1))
    ms = sum(times) / len(times)
    tf = a_flop / (ms / 1e3) / 1e12
    peak = peaks["bf16_tflops"]
    return {"kernel_ms": ms, "launches": reps, "tflops": tf, "peak": peak,
            "peak_source": f"{peak_kind} bf16_tflops (burst: the kernel runs alone)", "frac_of_peak": tf / peak,
            "l2": "256 MB written between launches"}


def run_ours(args):
    world, rank, local = dist_setup()
    dev = f"cuda:{local}"
    if args.no_pdl:
        B.llama3_set_programmatic_launch(False)
    B.llama3_set_kernel_path(0)
    peaks, peak_kind = load_peaks()
    n_layers = args.layers or PREFILL.n_layers
    layers, outw = build(dev, n_layers)
    cfg = PREFILL.cfg()
    S, D = PREFILL.seq, PREFILL.dim
    if "bf16_tflops_sustained" in peaks:
        peak, peak_src = peaks["bf16_tflops_sustained"], f"{peak_kind} bf16_tflops_sustained"
    else:
        peak, peak_src = peaks["bf16_tflops"], f"{peak_kind} bf16_tflops (burst; no sustained figure)"

    # ---------------- prefill (every rank a full replica)
    pst = Llama3Stack(cfg, layers, outw, batch=1, cache_cap=S, max_seq=S, lm_rows=DECODE.batch, device=dev)
    ids = I.token_ids(PREFILL, dev)
    x = torch.empty((1, S, D), dtype=torch.bfloat16, device=dev)

    def prefill_step():
        pst.embed(ids, x)
        pst.forward_layers(x, S, 0)
        return pst.lm_head(x[:, -1], 1, S * D)

    # attention alone first, before the long power-capped prefill passes
    with ClockSampler(torch.cuda.current_device()) as aclk:
        alone = attention_alone(pst.cfg, dev, peaks, peak_kind,
                                PREFILL.n_heads * 2.0 * 2.0 * (S * (S + 1) / 2) * PREFILL.head_dim)
    alone["clocks"] = aclk.summary()

    with ClockSampler(torch.cuda.current_device()) as clk:
        ms, launches = time_steps(prefill_step, args.steps, args.warmup, world, name="prefill_timed")
    clocks = clk.summary()
    value = world * S / (ms / 1e3)
    # Kernel times in separate passes with the launch timer on (never inside
    # the timed region above).  Algorithmic flops: the w1|w3 GEMM's 2*M*N*K;
    # attention's QK^T and PV over the visible (causal) keys only.
    k_steps = max(1, min(3, args.steps))
    w13 = kernel_times(prefill_step, "gemm_w13", k_steps * n_layers, k_steps)
    k_ms = sum(w13) / len(w13) if w13 else None
    F = PREFILL.ffn_hidden
    w13_flop = 2.0 * S * (2 * F) * D
    achieved = w13_flop / (k_ms / 1e3) / 1e12 if k_ms else None
    roofline = {"bound": "tensor", "kernel": "tc_gemm_pair w1|w3 + SwiGLU (M=8192, N=2x14336, K=4096; CTA pairs)",
                "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                "frac": (achieved / peak) if achieved else None, "peak_source": peak_src,
                "traffic": recorded_traffic("gemm_w13", ["llama_decoder_only_rmsnorm_b200/csrc/tc_gemm.cuh",
                                                         "llama_decoder_only_rmsnorm_b200/csrc/tc_gemm_pair.cuh",
                                                         "llama_decoder_only_rmsnorm_b200/csrc/llama3.cu"]),
                "kernel_ms": k_ms, "timed_launches": len(w13)}
    total_flop = n_layers * (2.0 * S * 6.979e9 / 32) + 2.0 * D * PREFILL.vocab  # linear layers + LM head row
    attn_flop = n_layers * PREFILL.n_heads * 2.0 * S * (S + 1) * PREFILL.head_dim
    whole = {"flop_per_step": total_flop + attn_flop,
             "tflops": (total_flop + attn_flop) / (ms / 1e3) / 1e12}
    whole["frac_of_peak"] = whole["tflops"] / peak
    at = kernel_times(prefill_step, "attention", k_steps * n_layers, k_steps)
    a_ms = sum(at) / len(at) if at else None
    a_flop = PREFILL.n_heads * 2.0 * 2.0 * (S * (S + 1) / 2) * PREFILL.head_dim
    attention = {"kernel": "causal GQA flash attention (S=8192, 32 q heads, 8 kv heads, hd 128)",
                 "kernel_ms": a_ms, "flop_per_launch": a_flop,
                 "tflops": a_flop / (a_ms / 1e3) / 1e12 if a_ms else None}
    if attention["tflops"]:
        attention["frac_of_peak"] = attention["tflops"] / peak
        attention["peak_source"] = peak_src
    attention["alone"] = alone

    # e2e through the public API with host buffers: ids in, next id out, read
    # on the host every step
    ids_h = ids.cpu().pin_memory()
    out_h = torch.empty((1,), dtype=torch.int32).pin_memory()

    def prefill_e2e():
        ids.copy_(ids_h, non_blocking=True)
        out_h.copy_(prefill_step(), non_blocking=True)
        torch.cuda.current_stream().synchronize()

    e2e_ms, _ = time_steps(prefill_e2e, args.steps, 1, world, name="prefill_e2e")
    e2e = {"value": world * S / (e2e_ms / 1e3), "unit": "tokens/s", "h2d_bytes_per_step": ids_h.numel() * 4,
           "d2h_bytes_per_step": 4}
    del pst, x
    torch.cuda.empty_cache()

    # ---------------- decode (the batch of 32 sequences split over the ranks)
    decode = None
    caches = None
    if not args.no_decode:
        Bt, P = DECODE.batch, DECODE.cache_len
        first, Bd = shard(Bt, world, rank)
        caches = [I.kv_cache(DECODE, i, P + 1, dev, first, Bd) for i in range(n_layers)]
        dst = Llama3Stack(cfg, layers, outw, batch=Bd, cache_cap=P + 1, max_seq=1, lm_rows=Bd, device=dev,
                          caches=caches)
        dids = I.token_ids(DECODE, dev)[first:first + Bd].contiguous()
        xd = torch.empty((Bd, 1, D), dtype=torch.bfloat16, device=dev)

        def decode_step():
            dst.embed(dids, xd)
            dst.decode_layers(xd, P)
            return dst.lm_head(xd, Bd, D)

        # The decode step (about a dozen launches per block) is captured once
        # in a CUDA graph after eager warm-up and replayed.
        for _ in range(args.warmup):
            decode_step()
        torch.cuda.synchronize()
        graph = torch.cuda.CUDAGraph()
        l0 = B.llama3_launch_count()
        with torch.cuda.graph(graph):
            nxt_dev = decode_step()
        per_step_launches = B.llama3_launch_count() - l0
        with ClockSampler(torch.cuda.current_device()) as clk2:
            dms, _ = time_steps(graph.replay, args.steps, args.warmup, world, name="decode_timed")
        # kernel times from separately captured graphs: the first 4 blocks'
        # attention launches, and their 4 weight-streaming GEMMs each
        nb = min(4, n_layers)
        att = graph_kernel_times(decode_step, "decode_attention", nb)
        gem = graph_kernel_times(decode_step, "decode_gemm", 4 * nb)
        dk_ms = sum(att) / len(att) if att else None
        kv_bytes = Bd * (P + 1) * DECODE.n_kv_heads * DECODE.head_dim * 2 * 2
        dach = kv_bytes / (dk_ms / 1e3) / 1e9 if dk_ms else None
        hbm = peaks.get("hbm_gbs")
        gemms = {}
        for j, (name, wbytes) in enumerate(DECODE_GEMMS):
            t = [gem[i] for i in range(j, len(gem), 4)]
            if t:
                tm = sum(t) / len(t)
                gemms[name] = {"kernel_ms": tm, "weight_bytes": wbytes, "gbs": wbytes / (tm / 1e3) / 1e9,
                               "frac_of_hbm": wbytes / (tm / 1e3) / 1e9 / hbm}
        step_bytes = n_layers * (kv_bytes + 2 * 6.979e9 / 32) + 2.0 * DECODE.vocab * D
        dids_h = dids.cpu().pin_memory()
        dout_h = torch.empty((Bd,), dtype=torch.int32).pin_memory()
        gloo = torch.distributed.new_group(backend="gloo") if world > 1 else None

        def decode_e2e():
            dids.copy_(dids_h, non_blocking=True)
            graph.replay()
            dout_h.copy_(nxt_dev, non_blocking=True)
            torch.cuda.current_stream().synchronize()
            gather_ids(dout_h, Bt, world, rank, gloo)   # the 32 next ids on rank 0's host

        de2e_ms, _ = time_steps(decode_e2e, args.steps, 1, world, name="decode_e2e")
        decode = {"metric": "decode tokens/s", "value": Bt / (dms / 1e3), "unit": "tokens/s",
                  "ms_per_step": dms, "steps": args.steps, "warmup": args.warmup,
                  "scaling": "strong" if world > 1 else "weak",
                  "config": {"workload": "llama3_8b_decode", "batch": Bt, "cached_positions": P,
                             "new_token_position": P,
                             "parallelism": f"batch split over {world} ranks ({Bd} sequences on rank {rank}); "
                                            "ids gathered on the host"},
                  "roofline": {"bound": "hbm", "kernel": "split-KV decode attention (K/V of this rank's "
                                                          f"{Bd} sequences per launch)",
                               "achieved": dach, "peak": hbm, "unit": "GB/s",
                               "frac": (dach / hbm) if dach else None, "peak_source": f"{peak_kind} hbm_gbs",
                               "traffic": recorded_traffic("decode_attention", [
                                   "llama_decoder_only_rmsnorm_b200/csrc/decode_attention.cuh"])
                               if Bd == Bt else None,
                               "kernel_ms": dk_ms},
                  "decode_gemms": gemms,
                  "whole_step": {"bytes_per_step": step_bytes, "gbs": step_bytes / (dms / 1e3) / 1e9,
                                 "frac_of_hbm": step_bytes / (dms / 1e3) / 1e9 / hbm},
                  "e2e": {"value": Bt / (de2e_ms / 1e3), "unit": "tokens/s",
                          "h2d_bytes_per_step": Bd * 4, "d2h_bytes_per_step": Bd * 4},
                  "gpu_launches": per_step_launches * args.steps, "cuda_graph": True, "clocks": clk2.summary()}
        del graph
        if gloo is not None:
            torch.distributed.destroy_process_group(gloo)

    # ---------------- oracle on the host cores
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        prefix = 64
        t_pre, t_dec, cores = oracle_sample(layers, outw, caches, prefix, decode_seq=caches is not None)
        # per-token work of the 64-token prefix against the whole 8192-token
        # prefill (linear layers per token, plus causal attention over ~t keys)
        lin = 2.0 * 6.979e9 * n_layers / 32
        att_tok = lambda n: n_layers * PREFILL.n_heads * 2.0 * (n + 1) * PREFILL.head_dim
        ratio = (lin + att_tok(prefix)) / (lin + att_tok(S))
        cpu = {"value": prefix / t_pre, "unit": "tokens/s", "cores": cores, "kind": "oracle",
               "sample": f"fp64 oracle, first {prefix} tokens of the prefill through all {n_layers} blocks + "
                         "final norm + LM head on the last position (weight fp64 conversion not timed); the "
                         "whole 8192-token prefill does more attention work per token, so at the same rate "
                         f"of work the oracle would reach about {ratio:.2f} of this value there",
               "full_sequence_estimate": prefix / t_pre * ratio}
        if decode is not None and t_dec > 0:
            decode["cpu_baseline"] = {"value": 1.0 / t_dec, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                                      "sample": "fp64 oracle, one sequence's decode step at position 8192 "
                                                f"through all {n_layers} blocks + LM head"}

    if rank == 0:
        line = {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
                "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
                "vs_baseline": None, "dtype": "bf16",
                "data": "synthetic: seeded random-init N(0,0.02) weights of the Llama-3-8B shape, uniform token ids",
                "config": {"workload": "llama3_8b_prefill", "batch": 1, "seq_len": S, "layers": n_layers,
                           "lm_head_rows": "last position", "parallelism": f"replicas x{world}",
                           "l2": "inputs larger than L2 (16 GB of weights streamed per step)"},
                "roofline": roofline, "whole_step": whole, "attention": attention, "cpu_baseline": cpu, "e2e": e2e,
                "gpu_launches": launches, "clocks": clocks, "decode": decode}
        print(json.dumps(line), flush=True)
    if world > 1:
        torch.distributed.destroy_process_group()


# ------------------------------------------------------- reference arm ---
def run_reference(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    dev = f"cuda:{int(os.environ.get('LOCAL_RANK', '0'))}"
    torch.cuda.set_device(dev)
    layers, outw = build(dev, PREFILL.n_layers)
    prefix = 16
    times = []
    for _ in range(args.warmup + args.steps):
        t_pre, _, cores = oracle_sample(layers, outw, None, prefix, decode_seq=False)
        times.append(t_pre)
    ts = times[args.warmup:]
    ms = 1e3 * sum(ts) / len(ts)
    v = prefix / (ms / 1e3)
    sample = (f"fp64 oracle, first {prefix} tokens of the 8B-shaped prefill through all 32 blocks + final norm "
              "+ LM head on the last position, per step (weight fp64 conversion not timed)")
    line = {"impl": "reference", "metric": METRIC, "value": v, "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic (same seeds as ours)",
            "config": {"workload": "llama3_8b_prefill", "batch": 1, "seq_len": PREFILL.seq,
                       "sampled_tokens": prefix},
            "cpu_baseline": {"value": v, "unit": "tokens/s", "cores": cores, "kind": "oracle", "sample": sample},
            "e2e": {"value": v, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


if __name__ == "__main__":
    a = parse()
    if a.impl == "reference":
        run_reference(a)
    else:
        run_ours(a)
