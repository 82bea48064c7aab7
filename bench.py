"""Benchmark of the TurboQuant KV-vector hot path on B200.

Workload (default, "c4_batched_decode"): a batched decode step of a serving engine with a
TurboQuant key cache, shaped like Llama-3.1-8B attention (8 kv-heads, head_dim 128, GQA 4):
  * cache: 64 sequences x 8 kv-heads x 8192 tokens, keys at b = 3 (2-bit Lloyd-Max + 1-bit
    QJL, m = 128), 52 B per key (218 MB packed);
  * one step = tq_quantize of a 64 x 512-token append (262,144 bf16 vectors) followed by
    tq_logits of 64 x 32 query heads (bf16) over the whole cache (4,194,304 keys).
Synthetic data with the pages' laws: key norms 4-182x value norms, 4 outlier channels per
kv-head scaled x20, queries N(0, 1); generated on the device from a seeded generator.

One JSON line on rank 0. `value` = cache keys scanned per second by whole steps (the
quantize of the append included); per-kernel times, the logits roofline and the quantize
throughput are reported beside it. `--impl reference` times the fp64 CPU oracle on a
bounded sample of the same step instead.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import socket
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "tq_logits keys/s & HBM GB/s (% of ~8 TB/s); tq_quantize vectors/s"
N_SEQ, N_KV, N_TOK, G, D = 64, 8, 8192, 4, 128
N_APPEND = 512
MSE_BITS = 2  # b = 3 keys


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            pk = json.load(f)
        return pk, "measured"
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "sm_max_mhz": 1965.0}, \
        "fallback"


# ----------------------------------------------------------------------------- distributed plumbing
def dist_init(backend="nccl"):
    """One process per GPU (torchrun env). The short timeout ends ranks that wait for a peer
    that is gone; the CPU tests use backend="gloo"."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime

        import torch
        import torch.distributed as dist
        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(world, v):
    if world == 1:
        return v
    import torch
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([v], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ----------------------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons while the timed loop runs. Sampling
    starts (first line received) before the caller's timed region; only samples stamped inside
    [mark_start, mark_end] (plus one sampling period on each side) are summarised."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    PERIOD_MS = 50

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []
        self.t0 = self.t1 = None

    def _read(self):
        for ln in self.proc.stdout:
            if ln.strip():
                self.lines.append((time.time(), ln))

    def __enter__(self):
        import threading
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", str(self.PERIOD_MS)], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
            return self
        self.reader = threading.Thread(target=self._read, daemon=True)
        self.reader.start()
        deadline = time.time() + 5.0
        while not self.lines and time.time() < deadline:
            time.sleep(0.01)
        return self

    def mark_start(self):
        self.t0 = time.time()

    def mark_end(self):
        self.t1 = time.time()
        # at least two periods of samples after the work ends
        time.sleep(2 * self.PERIOD_MS / 1000.0)

    def __exit__(self, *a):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            self.reader.join(timeout=5)

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        pad = self.PERIOD_MS / 1000.0
        for ts, ln in self.lines:
            if self.t0 is not None and not (self.t0 - pad <= ts <= (self.t1 or ts) + pad):
                continue
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx = float(parts[2])
            except ValueError:
                continue
            for nm, val in zip(names, parts[5:9]):
                if val.lower().startswith("active"):
                    reasons.add(nm)
        return {"sm_mhz": float(np.median(sm)) if sm else None, "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# ----------------------------------------------------------------------------- device workload
def make_keys_device(torch, gen, n_streams, n_tok, heads_per_seq, d=D):
    """Keys with the decode law on the device, bf16 [n_streams, n_tok, d]; stream = seq*8 + head."""
    import tq_inputs as ti
    out = torch.empty((n_streams, n_tok, d), dtype=torch.bfloat16, device="cuda")
    mult = torch.ones((heads_per_seq, d), device="cuda")
    for h in range(heads_per_seq):
        mult[h, torch.as_tensor(ti.outlier_channels(4, h, d), device="cuda")] = 20.0
    chunk = 64
    lo, hi = math.log(4.0), math.log(182.0)
    for s0 in range(0, n_streams, chunk):
        s1 = min(n_streams, s0 + chunk)
        heads = torch.arange(s0, s1, device="cuda") % heads_per_seq
        g = torch.randn((s1 - s0, n_tok, d), generator=gen, device="cuda") * mult[heads][:, None, :]
        v = torch.randn((s1 - s0, n_tok, d), generator=gen, device="cuda")
        rho = torch.exp(lo + (hi - lo) * torch.rand((s1 - s0, n_tok, 1), generator=gen, device="cuda"))
        k = g / g.norm(dim=-1, keepdim=True) * rho * v.norm(dim=-1, keepdim=True)
        out[s0:s1] = k.to(torch.bfloat16)
        del g, v, k
    return out


def run_gpu(args, world, rank, local):
    import torch

    import kv_cache_vector_03_b200 as tq
    import tq_inputs as ti

    peaks, peak_kind = load_peaks()
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    gen = torch.Generator(device="cuda")
    gen.manual_seed(20260000 + rank)
    cfg = ti.C4
    pi = torch.from_numpy(cfg.pi().astype(np.float32))
    s = torch.from_numpy(cfg.s().astype(np.float32))
    codec = tq.Codec(D, D, MSE_BITS, True, pi, s)
    n_streams = N_SEQ * N_KV

    # resident cache (quantized once, outside the timed region)
    keys = make_keys_device(torch, gen, n_streams, N_TOK, N_KV)
    cache = torch.empty(codec.packed_bytes(n_streams, N_TOK), dtype=torch.uint8, device="cuda")
    wsq = tq.workspace(codec.workspace_bytes(tq.TQ_OP_QUANTIZE))
    tq.tq_quantize(codec, keys, n_streams, N_TOK, N_TOK * D, cache, wsq)
    del keys
    append = make_keys_device(torch, gen, n_streams, N_APPEND, N_KV)
    append_packed = torch.empty(codec.packed_bytes(n_streams, N_APPEND), dtype=torch.uint8, device="cuda")
    q = torch.randn((N_SEQ, N_KV * G, D), generator=gen, device="cuda").to(torch.bfloat16)
    out = torch.empty((N_SEQ, N_KV * G, N_TOK), dtype=torch.float32, device="cuda")
    wsl = tq.workspace(codec.workspace_bytes(tq.TQ_OP_LOGITS, N_SEQ, N_KV, G))
    scale = 1.0 / math.sqrt(D)
    stream = torch.cuda.current_stream()
    torch.cuda.synchronize()
    assert tq.tq_get_status(wsq) == tq.TQ_OK

    def step(ev=None):
        if ev is not None:
            ev[0].record(stream)
        tq.tq_quantize(codec, append, n_streams, N_APPEND, N_APPEND * D, append_packed, wsq, stream)
        if ev is not None:
            ev[1].record(stream)
        tq.tq_logits(codec, cache, N_SEQ, N_KV, N_TOK, q, G, None, 0, scale, out, wsl, stream)
        if ev is not None:
            ev[2].record(stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clk:
        barrier(world)
        torch.cuda.synchronize()
        clk.mark_start()
        start.record(stream)
        for i in range(args.steps):
            step(evs[i])
        stop.record(stream)
        torch.cuda.synchronize()
        clk.mark_end()
        barrier(world)
    total_ms = start.elapsed_time(stop)
    t_quant = float(np.mean([e[0].elapsed_time(e[1]) for e in evs]))
    t_logit = float(np.mean([e[1].elapsed_time(e[2]) for e in evs]))
    ms_step = max_over_ranks(world, total_ms / args.steps)
    t_quant = max_over_ranks(world, t_quant)
    t_logit = max_over_ranks(world, t_logit)
    clocks = clk.summary()

    keys_per_step = n_streams * N_TOK
    vec_per_step = n_streams * N_APPEND
    rec = codec.record_bytes()
    logit_bytes = keys_per_step * rec + N_SEQ * N_KV * G * N_TOK * 4 + N_SEQ * N_KV * G * D * 2
    quant_bytes = vec_per_step * (D * 2 + rec)
    logit_gbs = logit_bytes / (t_logit * 1e-3) / 1e9
    quant_flops = vec_per_step * 2 * (2 * D * D)  # two d x d contractions per vector
    quant_tf = quant_flops / (t_quant * 1e-3) / 1e12

    # end to end through the public API: append + queries from pinned host memory in, logits
    # out, pipelined over two buffer slots as a serving loop would run it: step i's inputs are
    # copied in on one copy stream while step i - 1 computes, and step i's logits are copied
    # back on another while step i + 1 computes (the copy engines move both directions at once)
    h_append = torch.empty(append.shape, dtype=torch.bfloat16, pin_memory=True)
    h_append.copy_(append.cpu())
    h_q = torch.empty(q.shape, dtype=torch.bfloat16, pin_memory=True)
    h_q.copy_(q.cpu())
    h_out = [torch.empty(out.shape, dtype=torch.float32, pin_memory=True) for _ in range(2)]
    d_app, d_q, d_out = [append, torch.empty_like(append)], [q, torch.empty_like(q)], [out, torch.empty_like(out)]
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
    ev_in, ev_done, ev_out = ([torch.cuda.Event() for _ in range(2)] for _ in range(3))
    used = [False, False]

    def e2e_step(i):
        b = i % 2
        with torch.cuda.stream(s_in):
            if used[b]:
                s_in.wait_event(ev_done[b])      # step i - 2 has consumed this slot's inputs
            d_app[b].copy_(h_append, non_blocking=True)
            d_q[b].copy_(h_q, non_blocking=True)
            ev_in[b].record(s_in)
        stream.wait_event(ev_in[b])
        if used[b]:
            stream.wait_event(ev_out[b])         # step i - 2's logits have left this slot
        tq.tq_quantize(codec, d_app[b], n_streams, N_APPEND, N_APPEND * D, append_packed, wsq, stream)
        tq.tq_logits(codec, cache, N_SEQ, N_KV, N_TOK, d_q[b], G, None, 0, scale, d_out[b], wsl, stream)
        ev_done[b].record(stream)
        with torch.cuda.stream(s_out):
            s_out.wait_event(ev_done[b])
            h_out[b].copy_(d_out[b], non_blocking=True)
            ev_out[b].record(s_out)
        used[b] = True

    for i in range(2):
        e2e_step(i)
    torch.cuda.synchronize()
    e_steps = max(3, min(args.steps, 20))
    barrier(world)
    torch.cuda.synchronize()
    start.record(s_in)
    for i in range(e_steps):
        e2e_step(2 + i)
    stop.record(s_out)
    torch.cuda.synchronize()
    barrier(world)
    e2e_ms = max_over_ranks(world, start.elapsed_time(stop) / e_steps)
    h_out = h_out[0]
    h2d = h_append.numel() * 2 + h_q.numel() * 2
    d2h = h_out.numel() * 4

    # kernels launched per step: quantize 1, logits 2 (prologue + stream)
    launches_per_step = 3
    dominant = "tq_logits" if t_logit >= t_quant else "tq_quantize"
    read_gbs = read_stream_gbs(torch)
    logits_roof = {"kernel": "tq_logits (prologue + int8-MMA stream)", "bound": "hbm", "achieved": round(logit_gbs, 1),
                   "peak": peaks["hbm_gbs"], "unit": "GB/s", "frac": round(logit_gbs / peaks["hbm_gbs"], 4),
                   "traffic": ncu_traffic("tq_logits"), "peak_kind": peak_kind,
                   "algorithmic_bytes_per_launch": logit_bytes,
                   "read_stream_gbs": round(read_gbs, 1), "frac_of_read_stream": round(logit_gbs / read_gbs, 4)}
    # quantize: the roofline time is the larger of its algorithmic bytes at the HBM peak and its
    # algorithmic flops (two d x d contractions per vector, one pass each) at the dense bf16
    # peak; the kernel runs the contractions as split passes for fp32-equivalent precision
    # (three bf16 passes for Pi x, three fp16 passes for M r), reported beside it
    tpeak = peaks["bf16_tflops"]
    t_hbm = quant_bytes / (peaks["hbm_gbs"] * 1e9)
    t_tc = quant_flops / (tpeak * 1e12)
    passes = 3.0
    q_bound = "hbm" if t_hbm >= t_tc else "tensor"
    quant_roof = {"kernel": "tq_quantize (warp-specialized tcgen05: TMA rows, split-precision MMAs, TMEM epilogue)",
                  "bound": q_bound,
                  "achieved": round(quant_bytes / (t_quant * 1e-3) / 1e9, 1) if q_bound == "hbm" else round(quant_tf, 2),
                  "peak": peaks["hbm_gbs"] if q_bound == "hbm" else tpeak,
                  "unit": "GB/s" if q_bound == "hbm" else "TFLOP/s",
                  "frac": round(max(t_hbm, t_tc) / (t_quant * 1e-3), 4),
                  "traffic": ncu_traffic("tq_quantize"), "algorithmic_bytes_per_launch": quant_bytes,
                  "algorithmic_flops_per_launch": quant_flops, "tensor_TFLOP_per_s": round(quant_tf, 2),
                  "tensor_frac": round(quant_tf / tpeak, 4), "split_passes": passes,
                  "tensor_frac_with_split_passes": round(passes * quant_tf / tpeak, 4),
                  "peak_kind": peak_kind + (" (HBM copy)" if q_bound == "hbm" else " (bf16 burst)")}
    also = {} if args.no_extras else extra_workloads(torch, tq, ti, gen, peaks)
    if not args.no_extras:
        # the same append with a randomized Walsh-Hadamard rotation H D / sqrt(d): the rotation
        # is an exact +-1 operand, one tensor-core pass instead of three
        hcodec = tq.Codec(D, D, MSE_BITS, True, torch.from_numpy(ti.hadamard_rotation(D, 1004).astype(np.float32)), s)
        hms = time_calls(torch, lambda i: tq.tq_quantize(hcodec, append, n_streams, N_APPEND, N_APPEND * D,
                                                          append_packed, wsq, stream), 20, 3)
        also["c4_append_quantize_hadamard_rotation"] = {
            "ms": hms, "vectors_per_s": vec_per_step / (hms * 1e-3), "dense_rotation_ms": t_quant,
            "GB_per_s": quant_bytes / (hms * 1e-3) / 1e9}
        # the query prologue (query rotation, sketch and operand fragments of the 2048 heads)
        # followed by one 32-key block per stream, with the dense rotation and with the
        # Hadamard one, whose query rotation runs as a fast Walsh-Hadamard transform; then the
        # whole c4 logits call under the Hadamard codec (same records)
        pro_ms = time_graph(torch, lambda i: tq.tq_logits(codec, cache, N_SEQ, N_KV, 32, q, G, None, 0, scale, out,
                                                           wsl), 20)
        hpro_ms = time_graph(torch, lambda i: tq.tq_logits(hcodec, cache, N_SEQ, N_KV, 32, q, G, None, 0, scale, out,
                                                            wsl), 20)
        hlog_ms = time_calls(torch, lambda i: tq.tq_logits(hcodec, cache, N_SEQ, N_KV, N_TOK, q, G, None, 0, scale,
                                                            out, wsl, stream), 20, 3)
        also["c4_query_prologue_plus_one_block"] = {"dense_rotation_ms": pro_ms, "walsh_hadamard_ms": hpro_ms,
                                                    "q_heads": N_SEQ * N_KV * G, "keys_per_stream": 32,
                                                    "timing": "CUDA graph of 20 calls, median of 7 runs of 20 replays, inputs in L2"}
        also["c4_logits_hadamard_rotation"] = {"ms": hlog_ms, "keys_per_s": keys_per_step / (hlog_ms * 1e-3),
                                               "dense_rotation_ms": t_logit}
        # the same c4 logits with the MSE-only estimator (no sign-plane MMAs; same records read)
        mms = time_calls(torch, lambda i: tq.tq_logits(codec, cache, N_SEQ, N_KV, N_TOK, q, G, None, 0, scale, out, wsl,
                                                        stream, estimator=tq.TQ_EST_MSE), 20, 3)
        also["c4_logits_mse_only_estimator"] = {
            "ms": mms, "keys_per_s": keys_per_step / (mms * 1e-3), "GB_per_s": logit_bytes / (mms * 1e-3) / 1e9,
            "frac_of_measured_hbm": logit_bytes / (mms * 1e-3) / 1e9 / peaks["hbm_gbs"], "qjl_estimator_ms": t_logit}
    line = {
        "metric": METRIC, "value": keys_per_step * world / (ms_step * 1e-3), "unit": "keys/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "u8 codes, int8/fp32 arithmetic",
        "data": "synthetic (device-generated, pages' key law)",
        "config": {"workload": "c4_batched_decode: 64 seq x 8 kv-heads x 8192 tok, d=128, b=3 keys; "
                               "step = quantize 64x512x8 append + logits 64x32 q-heads",
                   "seq_len": N_TOK, "n_seq_per_gpu": N_SEQ, "kv_heads": N_KV, "q_heads": N_KV * G, "head_dim": D,
                   "key_bits": MSE_BITS + 1, "record_bytes": rec, "parallelism": f"replicas x{world}",
                   "l2": "inputs larger than L2 (packed cache 218 MB + 67 MB logits); no flush"},
        "kernels": {
            "tq_logits": {"ms": t_logit, "keys_per_s": keys_per_step / (t_logit * 1e-3), "GB_per_s": logit_gbs,
                          "frac_of_8TBps": logit_gbs / 8000.0, "frac_of_measured_hbm": logit_gbs / peaks["hbm_gbs"]},
            "tq_quantize": {"ms": t_quant, "vectors_per_s": vec_per_step / (t_quant * 1e-3),
                            "GB_per_s": quant_bytes / (t_quant * 1e-3) / 1e9, "TFLOP_per_s": quant_tf}},
        "roofline": logits_roof if dominant == "tq_logits" else quant_roof,
        "roofline_other": quant_roof if dominant == "tq_logits" else logits_roof,
        "e2e": {"value": keys_per_step * world / (e2e_ms * 1e-3), "unit": "keys/s", "ms_per_step": e2e_ms,
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "pipelining": "two buffer slots: a step's copies overlap the neighbouring steps' kernels"},
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clocks,
        "also": also,
    }
    return line


# DRAM bytes (read + write) per launch of the step's kernels on the c4 workload, each from one
# ncu capture (profiles/), valid only while the kernel sources it was taken on are unchanged:
# name -> (bytes, {source file: sha256 prefix at capture time})
NCU_TRAFFIC = {
    "tq_logits": (0.69e6 + 220.83e6 + 41.23e6, {"k_logits.cu": "cbd75199fb8bcf87"}),
    "tq_quantize": (67.34e6 + 2.42e6, {"k_quantize_ws.cu": "62ed39abb5c6c030", "tq_tc.cuh": "5fd2f8a68cb68dcc"}),
}


def _src_sha(name):
    import hashlib
    path = os.path.join(ROOT, "kv_cache_vector_03_b200", "csrc", name)
    with open(path, "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()[:16]


def ncu_traffic(kernel):
    """The captured DRAM traffic of a kernel, or None once its source has changed since."""
    byts, srcs = NCU_TRAFFIC[kernel]
    if byts is None:
        return None
    for name, sha in srcs.items():
        if sha is None or _src_sha(name) != sha:
            return None
    return byts


def read_stream_gbs(torch):
    """A read-only streaming reference measured in this run: torch's sum over a 2 GiB fp32
    buffer (device time per pass with CUDA events, best of 5), for context beside the
    measured copy peak."""
    x = torch.ones(1 << 29, dtype=torch.float32, device="cuda")
    x.sum()
    torch.cuda.synchronize()
    best = float("inf")
    for _ in range(5):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        x.sum()
        b.record()
        torch.cuda.synchronize()
        best = min(best, a.elapsed_time(b))
    del x
    return (1 << 31) / (best * 1e-3) / 1e9


def time_calls(torch, fn, n_iter, n_warm=3):
    """Mean device time of fn(i) over n_iter calls (CUDA events on the current stream)."""
    for i in range(n_warm):
        fn(i)
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for i in range(n_iter):
        fn(i)
    b.record()
    torch.cuda.synchronize()
    return a.elapsed_time(b) / n_iter


def time_graph(torch, fn, n_calls, n_replays=20, n_runs=7):
    """Device time per call of fn(0) .. fn(n_calls - 1) captured once in a CUDA graph: the
    median over n_runs runs of n_replays back-to-back replays each (host launch overhead
    amortised, as in a captured decode loop)."""
    for i in range(n_calls):   # first calls (one-time launch setup) outside the capture
        fn(i)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        for i in range(n_calls):
            fn(i)
    graph.replay()
    torch.cuda.synchronize()
    runs = []
    for _ in range(n_runs):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        for _ in range(n_replays):
            graph.replay()
        b.record()
        torch.cuda.synchronize()
        runs.append(a.elapsed_time(b) / (n_replays * n_calls))
    del graph
    return float(np.median(runs))


def extra_workloads(torch, tq, ti, gen, peaks):
    """The other workloads of the hot path, each timed on its own (device time per call).
    Inputs that fit in L2 are rotated over enough copies to exceed it."""
    out = {}
    d = 128
    # c2: Llama-3.1-8B-shaped decode, 8 kv-heads x 32768 tokens (32640 packed + 128 bf16), 32 q-heads
    n_kv, n_all, n_tail = 8, 32768, 128
    n_tok = n_all - n_tail
    for b in (4, 3):
        cfg = ti.C2
        codec = tq.Codec(d, d, b - 1, True, torch.from_numpy(cfg.pi().astype(np.float32)),
                         torch.from_numpy(cfg.s().astype(np.float32)))
        keys = make_keys_device(torch, gen, n_kv, n_all, n_kv)
        copies = 12
        packs = []
        for _ in range(copies):
            pk = torch.empty(codec.packed_bytes(n_kv, n_tok), dtype=torch.uint8, device="cuda")
            tq.tq_quantize(codec, keys, n_kv, n_tok, n_all * d, pk, tq.workspace(256))
            packs.append(pk)
        tail = keys[:, n_tok:].contiguous()
        q = torch.randn((1, n_kv * 4, d), generator=gen, device="cuda").to(torch.bfloat16)
        lo = torch.empty((1, n_kv * 4, n_all), dtype=torch.float32, device="cuda")
        ws = tq.workspace(codec.workspace_bytes(tq.TQ_OP_LOGITS, 1, n_kv, 4))
        ms = time_graph(torch, lambda i: tq.tq_logits(codec, packs[i % copies], 1, n_kv, n_tok, q, 4, tail, n_tail,
                                                      1.0 / math.sqrt(d), lo, ws), copies)
        byts = n_kv * n_tok * codec.record_bytes() + n_kv * n_tail * d * 2 + lo.numel() * 4
        out[f"c2_llama8b_decode_logits_b{b}"] = {
            "ms": ms, "keys_per_s": n_kv * n_all / (ms * 1e-3), "GB_per_s": byts / (ms * 1e-3) / 1e9,
            "frac_of_measured_hbm": byts / (ms * 1e-3) / 1e9 / peaks["hbm_gbs"],
            "l2": f"{copies} rotating copies of the packed cache", "timing": "CUDA graph of 12 calls, median of 7 runs of 20 replays"}
        # the same decode step fused: logits -> online softmax -> P.V over packed keys and values
        # (value cache at b bits, MSE only), the 128 recent keys and values in bf16
        vcodec = tq.Codec(d, 0, b, False, torch.from_numpy(ti.C3.pi().astype(np.float32)), None)
        vals = torch.randn((n_kv, n_all, d), generator=gen, device="cuda").to(torch.bfloat16)
        vpacks = []
        for _ in range(copies):
            pv_ = torch.empty(vcodec.packed_bytes(n_kv, n_tok), dtype=torch.uint8, device="cuda")
            tq.tq_quantize(vcodec, vals, n_kv, n_tok, n_all * d, pv_, tq.workspace(256))
            vpacks.append(pv_)
        tail_v = vals[:, n_tok:].contiguous()
        ao = torch.empty((1, n_kv * 4, d), dtype=torch.float32, device="cuda")
        aws = tq.workspace(tq.tq_attention_workspace_bytes(codec, vcodec, 1, n_kv, n_tok, 4, n_tail))
        ms = time_graph(torch, lambda i: tq.tq_attention(codec, vcodec, packs[i % copies], vpacks[i % copies], 1, n_kv,
                                                         n_tok, q, 4, tail, tail_v, n_tail, 1.0 / math.sqrt(d), ao,
                                                         aws), copies)
        byts = n_kv * n_tok * (codec.record_bytes() + vcodec.record_bytes()) + 2 * n_kv * n_tail * d * 2 + ao.numel() * 4
        out[f"c2_llama8b_decode_attention_k{b}v{b}"] = {
            "ms": ms, "tokens_per_s": n_kv * n_all / (ms * 1e-3), "GB_per_s": byts / (ms * 1e-3) / 1e9,
            "frac_of_measured_hbm": byts / (ms * 1e-3) / 1e9 / peaks["hbm_gbs"],
            "l2": f"{copies} rotating copies of the packed keys and values", "timing": "CUDA graph of 12 calls, median of 7 runs of 20 replays"}
        # sparse values: blocks whose weights are all below 1e-4 of the running maximum skip
        # their values (the bytes still stream: the value block shares the key block's stage)
        ms = time_graph(torch, lambda i: tq.tq_attention(codec, vcodec, packs[i % copies], vpacks[i % copies], 1, n_kv,
                                                         n_tok, q, 4, tail, tail_v, n_tail, 1.0 / math.sqrt(d), ao,
                                                         aws, v_skip=1e-4), copies)
        out[f"c2_llama8b_decode_attention_k{b}v{b}_sparse_v1e-4"] = {
            "ms": ms, "tokens_per_s": n_kv * n_all / (ms * 1e-3), "GB_per_s": byts / (ms * 1e-3) / 1e9,
            "frac_of_measured_hbm": byts / (ms * 1e-3) / 1e9 / peaks["hbm_gbs"],
            "timing": "CUDA graph of 12 calls, median of 7 runs of 20 replays"}
        del keys, packs, vals, vpacks
    # the key side of the asymmetric configuration at c2: 8-bit keys (q8_0-style), same queries and tail
    keys = make_keys_device(torch, gen, n_kv, n_all, n_kv)
    copies = 12
    q8s = []
    for _ in range(copies):
        pk = torch.empty(tq.tq_q8_packed_bytes(d, n_kv, n_tok), dtype=torch.uint8, device="cuda")
        tq.tq_q8_quantize(keys, d, n_kv, n_tok, n_all * d, pk, tq.workspace(256))
        q8s.append(pk)
    tail = keys[:, n_tok:].contiguous()
    q = torch.randn((1, n_kv * 4, d), generator=gen, device="cuda").to(torch.bfloat16)
    lo = torch.empty((1, n_kv * 4, n_all), dtype=torch.float32, device="cuda")
    ms = time_graph(torch, lambda i: tq.tq_q8_logits(q8s[i % copies], d, 1, n_kv, n_tok, q, 4, tail, n_tail,
                                                     1.0 / math.sqrt(d), lo), copies)
    byts = n_kv * n_tok * 136 + n_kv * n_tail * d * 2 + lo.numel() * 4
    out["c2_llama8b_decode_logits_q8_keys"] = {
        "ms": ms, "keys_per_s": n_kv * n_all / (ms * 1e-3), "GB_per_s": byts / (ms * 1e-3) / 1e9,
        "frac_of_measured_hbm": byts / (ms * 1e-3) / 1e9 / peaks["hbm_gbs"],
        "l2": f"{copies} rotating copies of the packed cache", "timing": "CUDA graph of 12 calls, median of 7 runs of 20 replays"}
    # the asymmetric decode step fused: 8-bit keys, 4-bit TurboQuant values, 128 bf16 tail tokens
    vcodec = tq.Codec(d, 0, 4, False, torch.from_numpy(ti.C3.pi().astype(np.float32)), None)
    vals = torch.randn((n_kv, n_all, d), generator=gen, device="cuda").to(torch.bfloat16)
    vpacks = []
    for _ in range(copies):
        pv_ = torch.empty(vcodec.packed_bytes(n_kv, n_tok), dtype=torch.uint8, device="cuda")
        tq.tq_quantize(vcodec, vals, n_kv, n_tok, n_all * d, pv_, tq.workspace(256))
        vpacks.append(pv_)
    tail_v = vals[:, n_tok:].contiguous()
    ao = torch.empty((1, n_kv * 4, d), dtype=torch.float32, device="cuda")
    aws = tq.workspace(tq.tq_attention_q8_workspace_bytes(vcodec, 1, n_kv, n_tok, 4, n_tail))
    ms = time_graph(torch, lambda i: tq.tq_attention_q8(vcodec, q8s[i % copies], vpacks[i % copies], 1, n_kv, n_tok, q,
                                                        4, tail, tail_v, n_tail, 1.0 / math.sqrt(d), ao, aws), copies)
    byts = n_kv * n_tok * (136 + vcodec.record_bytes()) + 2 * n_kv * n_tail * d * 2 + ao.numel() * 4
    out["c2_llama8b_decode_attention_q8_keys_v4"] = {
        "ms": ms, "tokens_per_s": n_kv * n_all / (ms * 1e-3), "GB_per_s": byts / (ms * 1e-3) / 1e9,
        "frac_of_measured_hbm": byts / (ms * 1e-3) / 1e9 / peaks["hbm_gbs"],
        "l2": f"{copies} rotating copies of the packed keys and values", "timing": "CUDA graph of 12 calls, median of 7 runs of 20 replays"}
    del keys, q8s, vals, vpacks
    # c3: values at 128K, 8 kv-heads x 131072 tokens, 32 q-heads, P ~ N(0, 4)
    n_kv, n_tok, g = 8, 131072, 4
    vals = torch.randn((n_kv, n_tok, d), generator=gen, device="cuda").to(torch.bfloat16)
    P = [2.0 * torch.randn((1, n_kv * g, n_tok), generator=gen, device="cuda") for _ in range(2)]
    for B in (3, 4):
        codec = tq.Codec(d, 0, B, False, torch.from_numpy(ti.C3.pi().astype(np.float32)), None)
        copies = 4
        packs = []
        for _ in range(copies):
            pk = torch.empty(codec.packed_bytes(n_kv, n_tok), dtype=torch.uint8, device="cuda")
            tq.tq_quantize(codec, vals, n_kv, n_tok, n_tok * d, pk, tq.workspace(256))
            packs.append(pk)
        o = torch.empty((1, n_kv * g, d), dtype=torch.float32, device="cuda")
        ws = tq.workspace(codec.workspace_bytes(tq.TQ_OP_PV, n_kv, n_tok, g))
        ms = time_graph(torch, lambda i: tq.tq_pv(codec, packs[i % copies], 1, n_kv, n_tok, P[i % 2], g, o, ws), copies)
        byts = n_kv * n_tok * codec.record_bytes() + P[0].numel() * 4
        out[f"c3_values_128k_pv_{B}bit"] = {
            "ms": ms, "tokens_per_s": n_kv * n_tok / (ms * 1e-3), "GB_per_s": byts / (ms * 1e-3) / 1e9,
            "frac_of_measured_hbm": byts / (ms * 1e-3) / 1e9 / peaks["hbm_gbs"],
            "l2": f"{copies} rotating copies of the packed values, 2 of P", "timing": "CUDA graph of 4 calls, median of 7 runs of 20 replays"}
        del packs
    del vals, P
    # c5: vector search, 1M x d=200 database (anisotropic, unit rows), 10,000 queries, top-10
    dd, n_db, n_q = 200, 1_000_000, 10_000
    sig = torch.from_numpy(ti.c5_scales(dd).astype(np.float32)).cuda()
    for b in (2, 4):
        codec = tq.Codec(dd, dd, b - 1, True, torch.from_numpy(ti.C5.pi().astype(np.float32)),
                         torch.from_numpy(ti.C5.s().astype(np.float32)))
        db = torch.randn((n_db, dd), generator=gen, device="cuda") * sig
        db /= db.norm(dim=1, keepdim=True)
        qs = torch.randn((n_q, dd), generator=gen, device="cuda") * sig
        qs /= qs.norm(dim=1, keepdim=True)
        pk = torch.empty(codec.packed_bytes(1, n_db), dtype=torch.uint8, device="cuda")
        wq = tq.workspace(256)
        tq_ms = time_calls(torch, lambda i: tq.tq_quantize(codec, db, 1, n_db, n_db * dd, pk, wq), 3, 1)
        idx = torch.empty((n_q, 10), dtype=torch.int64, device="cuda")
        sc = torch.empty((n_q, 10), dtype=torch.float32, device="cuda")
        ws = tq.workspace(codec.workspace_bytes(tq.TQ_OP_TOPK, n_q, n_db, 10))
        ms = time_calls(torch, lambda i: tq.tq_topk(codec, pk, n_db, qs, n_q, 10, idx, sc, ws), 3, 1)
        # the MSE-only ranking on the same records (no sign K-blocks)
        mms = time_calls(torch, lambda i: tq.tq_topk(codec, pk, n_db, qs, n_q, 10, idx, sc, ws,
                                                     estimator=tq.TQ_EST_MSE), 3, 1)
        out[f"c5_vector_search_b{b}"] = {
            "topk_ms": ms, "queries_per_s": n_q / (ms * 1e-3), "pairs_per_s": n_q * n_db / (ms * 1e-3),
            "topk_mse_only_ms": mms, "quantize_ms": tq_ms, "quantize_vectors_per_s": n_db / (tq_ms * 1e-3)}
        del db, qs, pk
    torch.cuda.empty_cache()
    return out


# ----------------------------------------------------------------------------- oracle (CPU)
def oracle_sample():
    """One sequence of the step (8 kv-heads x 8192 cached keys, 8 x 512 appended vectors,
    32 query heads) with the cache already quantized by the oracle."""
    import oracle
    import tq_inputs as ti
    cfg = ti.C4
    pi, s = cfg.pi(), cfg.s()
    c, t, _, _ = oracle.codebook(D, MSE_BITS)
    n_tok = N_TOK
    keys = [ti.bf16_to_f64(ti.key_stream(4, 0, h, n_tok)) for h in range(N_KV)]
    cache = [oracle.quantize(k, pi, s, c, t, MSE_BITS, qjl=True, keep_yz=False) for k in keys]
    app = [ti.bf16_to_f64(ti.key_stream(4, 1000, h, N_APPEND)) for h in range(N_KV)]
    q = ti.bf16_to_f64(ti.decode_queries(4, 1, N_KV * G))[0]
    return dict(oracle=oracle, pi=pi, s=s, c=c, t=t, cache=cache, app=app, q=q)


def oracle_step(smp):
    o = smp["oracle"]
    for h in range(N_KV):
        o.quantize(smp["app"][h], smp["pi"], smp["s"], smp["c"], smp["t"], MSE_BITS, qjl=True, keep_yz=False)
        ch = smp["cache"][h]
        o.logits(ch.idx, ch.sbit, ch.nhat, ch.ghat, smp["pi"], smp["s"], smp["c"], smp["q"][h * G:(h + 1) * G],
                 qjl=True, scale=1.0 / math.sqrt(D))


SAMPLE_DESC = ("1 of 64 sequences: oracle quantize of 8 x 512 appended vectors + oracle logits of 32 q-heads "
               "over 8 x 8192 cached keys (cache quantized beforehand)")


def cpu_baseline(min_seconds=10.0):
    import oracle
    smp = oracle_sample()
    oracle_step(smp)
    t0 = time.perf_counter()
    n = 0
    while n < 1 or time.perf_counter() - t0 < min_seconds:
        oracle_step(smp)
        n += 1
    dt = (time.perf_counter() - t0) / n
    return {"value": N_KV * N_TOK / dt, "unit": "keys/s", "cores": oracle.threads(), "kind": "oracle",
            "sample": SAMPLE_DESC, "s_per_sample_step": dt}


def run_reference(args, world, rank):
    if rank != 0:
        return None
    import oracle
    smp = oracle_sample()
    for _ in range(args.warmup):
        oracle_step(smp)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle_step(smp)
    dt = (time.perf_counter() - t0) / args.steps
    v = N_KV * N_TOK / dt
    return {"impl": "reference", "metric": METRIC, "value": v, "unit": "keys/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic (numpy, pages' key law)",
            "config": {"workload": "c4_batched_decode (sampled: 1 of 64 sequences per step)", "seq_len": N_TOK,
                       "kv_heads": N_KV, "q_heads": N_KV * G, "head_dim": D, "key_bits": MSE_BITS + 1},
            "cpu_baseline": {"value": v, "unit": "keys/s", "cores": oracle.threads(), "kind": "oracle",
                             "sample": SAMPLE_DESC},
            "e2e": {"value": v, "unit": "keys/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def relaunch(argv, n_ranks):
    """`--gpus N` run without a torchrun environment: start N ranks on this node, one process
    per GPU, through torch.distributed.run (loopback rendezvous), and return its exit code."""
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        port = sk.getsockname()[1]
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", f"--nproc-per-node={n_ranks}",
           "--master-addr", "127.0.0.1", f"--master-port={port}", os.path.abspath(__file__), *argv]
    return subprocess.call(cmd)


def run_plumbing(args, world, rank):
    """The N-rank plumbing alone (process group, barrier, max over ranks), no GPU work: each
    rank times a fixed host wait; rank 0 reports the slowest rank's time and the world size."""
    barrier(world)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        time.sleep(0.001 * (rank + 1))
    ms = max_over_ranks(world, (time.perf_counter() - t0) * 1e3 / args.steps)
    barrier(world)
    if rank != 0:
        return None
    return {"plumbing_only": True, "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "scaling": "weak"}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="tq", choices=["tq", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extras", action="store_true", help="skip the c2/c3/c5 side measurements")
    ap.add_argument("--plumbing-only", action="store_true",
                    help="run only the multi-rank plumbing over gloo (no GPU work); for tests")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    env_world = os.environ.get("WORLD_SIZE")
    if env_world is None and args.gpus > 1:
        sys.exit(relaunch(sys.argv[1:], args.gpus))
    if env_world is not None and int(env_world) != args.gpus:
        sys.exit(f"bench.py: --gpus {args.gpus} but WORLD_SIZE={env_world}: launch one rank per GPU")
    if args.plumbing_only:
        world, rank, _ = dist_init(backend="gloo")
        line = run_plumbing(args, world, rank)
        if line is not None:
            print(json.dumps(line), flush=True)
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
        return
    world, rank, local = dist_init() if args.impl == "tq" else (int(os.environ.get("WORLD_SIZE", "1")),
                                                                 int(os.environ.get("RANK", "0")), 0)
    if args.impl == "reference":
        line = run_reference(args, world, rank)
        if line is not None:
            print(json.dumps(line), flush=True)
        return
    line = run_gpu(args, world, rank, local)
    if rank == 0:
        if world == 1 and not args.no_cpu_baseline:
            line["cpu_baseline"] = cpu_baseline()
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
