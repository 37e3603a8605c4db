#!/usr/bin/env python
"""Benchmark of the TurboQuant-style KV-cache hot path (compress + decode attention).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl tq|reference]
                    [--workload batched] [--bits 4] [--rotation haar|hadamard]

One step = the whole hot path over one batch: tq_compress of the batch's
prefill (K and V of every token and kv head) and tq_decode_attention of one
decode query per sequence over the cache the previous step compressed (two
caches alternate, so the decode reads pages that 700 MB of compress traffic
has since pushed out of L2).  Inputs are resident in HBM before the timed
region.

`value` is the headline metric: decode-attention KV GB/s = the decode's
algorithmic bytes (packed K+V pages of every attended token, q in, out, block
table) / the decode's device time, summed over ranks.  Compress Mtokens/s and
both kernels' fractions of the measured HBM bandwidth sit beside it.  Under
torchrun every rank runs its own batch (weak scaling, no collective on the data
path); times are the max over ranks.

--impl reference times the CPU oracle (the plain fp64 restatement of the
method) on a bounded sample of the same workload, in the same unit.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import platform
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "TQ4 decode-attention KV GB/s (% of HBM peak); compress Mtokens/s"
PAGE = 16
D = 128
FALLBACK_HBM_GBS = 6650.0


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="tq", choices=["tq", "reference"])
    ap.add_argument("--workload", default="batched")
    ap.add_argument("--bits", type=int, default=4)
    ap.add_argument("--rotation", default="haar", choices=["haar", "hadamard"])
    ap.add_argument("--e2e-steps", type=int, default=20)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--prefill", action="store_true",
                    help="time the causal prefill attention of one sequence of the workload instead (1 GPU)")
    return ap.parse_args()


# ---------------------------------------------------------------- byte accounting
def chunk_bytes(bits: int, kind: int) -> int:
    """Packed bytes of one 16-token page chunk (same layout the library exports)."""
    w = lambda b: 4 if b >= 3 else (2 if b == 2 else 1)  # noqa: E731
    if kind == 1:
        return PAGE * (D * w(bits) // 8 + 4)
    return PAGE * (D * w(bits - 1) // 8 + D // 8 + 8)


def step_bytes(w):
    """Algorithmic bytes of one step: (compress bytes, decode bytes)."""
    vec = w.B * w.T * w.layers * w.Hkv
    packed = (chunk_bytes(w.bits, 0) + chunk_bytes(w.bits, 1)) // PAGE
    compress = vec * (2 * D * 2 + packed)
    ctx_tokens = w.B * w.T * w.Hkv
    decode = ctx_tokens * packed + 2 * w.B * w.Hq * D * 2 + w.B * w.max_blocks * 4 + w.B * 4
    return compress, decode


def measured_peak():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            j = json.load(f)
        return float(j["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def traffic_record(kernel: str):
    """ncu DRAM bytes per launch recorded under profiles/, if the kernel source
    is unchanged since the capture (else None)."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(p) as f:
            rec = json.load(f)[kernel]
    except Exception:
        return None
    h = hashlib.sha256()
    for src in rec["sources"]:
        with open(os.path.join(ROOT, src), "rb") as f:
            h.update(f.read())
    if h.hexdigest() != rec["sha256"]:
        return None
    return rec


# ---------------------------------------------------------------- clocks
class ClockSampler:
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.path = os.path.join("/tmp", "tq_clocks_%d_%d.csv" % (os.getpid(), index))

    def start(self):
        try:
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.index), "--query-gpu=" + self.Q,
                                          "--format=csv,noheader,nounits", "-lms", "100"], stdout=self.f,
                                         stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.f.close()
        rows = []
        with open(self.path) as f:
            for line in f:
                p = [x.strip() for x in line.split(",")]
                if len(p) >= 9:
                    rows.append(p)
        try:
            os.remove(self.path)
        except OSError:
            pass
        if not rows:
            return None
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(rows)}


# ---------------------------------------------------------------- distributed
def dist_setup(backend: str = "nccl"):
    """One process per GPU (torchrun env).  Returns (world_size, rank, local_rank)."""
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if ws > 1:
        import datetime

        import torch
        import torch.distributed as dist
        kw = {}
        if backend == "nccl":
            torch.cuda.set_device(local)
            kw["device_id"] = torch.device("cuda", local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120), **kw)
    return ws, rank, local


def barrier(ws):
    if ws > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(ws, x: float, device: str = "cuda") -> float:
    """Largest x over all ranks (every rank gets it)."""
    if ws == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def rank_data_seed(rank: int) -> int:
    """Each replica compresses and attends over its own seeded batch."""
    return 1 + 1000003 * rank


def whole_job_gbs(ws: int, bytes_per_rank_step: float, ms_step_max: float) -> float:
    """Weak scaling: every rank moves the same bytes per step; the step time is
    the slowest rank's."""
    return ws * bytes_per_rank_step / (ms_step_max * 1e-3) / 1e9


# ---------------------------------------------------------------- oracle (CPU) leg
def cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return platform.processor() or "unknown"


def oracle_sample(w, target_s: float = 10.0, threads: int = 0, min_seqs: int = 1, max_seqs: int | None = None):
    """The CPU oracle on whole sequences of the workload: compress K and V of the
    sequence (timed separately), then decode all its query heads (timed), until
    about target_s seconds of decode time have passed.  threads = 0: every core.
    Returns dict(decode_s, decode_bytes, compress_s, compress_bytes, seqs, threads)."""
    import numpy as np

    import oracle
    from kv_cache_vector_02_b200 import workloads as W
    nth = threads if threads > 0 else oracle.max_threads()
    o = oracle.Oracle(D, w.bits, w.param_seed, rot=w.rotation, key_mode=w.key_mode, nthreads=nth)
    one = w.with_(B=1, layers=1, decode_steps=0)
    bt = np.arange(one.max_blocks, dtype=np.int32)[None]
    slots = W.prefill_slots(one, bt)
    cb, db = step_bytes(one)
    r = {"decode_s": 0.0, "decode_bytes": 0.0, "compress_s": 0.0, "compress_bytes": 0.0, "seqs": 0, "threads": nth}
    cap = max_seqs if max_seqs is not None else w.B * w.layers
    while True:
        n = r["seqs"]
        wi = one.with_(data_seed=w.data_seed + 1000 + n)
        k, v = W.gen_kv(wi, 0).numpy(), W.gen_kv(wi, 1).numpy()
        q = W.gen_q(wi).numpy().astype(np.float64)
        ts = time.perf_counter()
        kc, vc = o.new_cache(0, one.num_blocks, one.Hkv), o.new_cache(1, one.num_blocks, one.Hkv)
        o.compress_paged(0, k, slots, kc)
        o.compress_paged(1, v, slots, vc)
        r["compress_s"] += time.perf_counter() - ts
        r["compress_bytes"] += cb
        ts = time.perf_counter()
        o.decode(q, kc, vc, bt, np.array([one.T], np.int32), one.Hkv)
        r["decode_s"] += time.perf_counter() - ts
        r["decode_bytes"] += db
        r["seqs"] = n + 1
        if (r["seqs"] >= min_seqs and r["decode_s"] >= target_s) or r["seqs"] >= cap:
            break
    return r


def run_reference(args):
    """Reference arm: the oracle as it stands, timed on the host cores, on the same
    metric (decode-attention KV GB/s) over bounded samples of the workload."""
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    from kv_cache_vector_02_b200 import workloads as W
    w = W.WORKLOADS[args.workload].with_(bits=args.bits, rotation=1 if args.rotation == "hadamard" else 0)
    per_step = max(1.0, 90.0 / max(1, args.steps + args.warmup))
    for _ in range(args.warmup):
        oracle_sample(w, target_s=0.0)
    dec_s = dec_b = comp_s = comp_b = 0.0
    seqs = 0
    threads = 1
    for _ in range(args.steps):
        r = oracle_sample(w, target_s=per_step)
        dec_s += r["decode_s"]
        dec_b += r["decode_bytes"]
        comp_s += r["compress_s"]
        comp_b += r["compress_bytes"]
        seqs += r["seqs"]
        threads = r["threads"]
    gbs = dec_b / dec_s / 1e9
    line = {
        "impl": "reference", "metric": METRIC, "value": gbs, "unit": "GB/s", "n_gpus": ws, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": 1e3 * (dec_s + comp_s) / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(w),
        "compress": {"mtokens_per_s": seqs * w.T / comp_s / 1e6, "gbs": comp_b / comp_s / 1e9},
        "cpu_baseline": {"value": gbs, "unit": "GB/s", "cores": threads, "kind": "oracle", "cpu": cpu_model(),
                         "sample": "%d whole sequences (%d tokens x %d kv heads): compress K+V untimed for the "
                                   "metric, decode of %d query heads timed" % (seqs, w.T, w.Hkv, w.Hq)},
        "e2e": {"value": gbs, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line))
    return 0


def workload_config(w):
    rot = "hadamard" if w.rotation == 1 else "haar"
    desc = {"batched": "32 sequences x 4096 tokens, 8 kv / 32 q heads (Llama-3-8B layout), d=128",
            "long70b": "1 sequence x 131072 tokens, 8 kv / 64 q heads (70B layer), d=128",
            "llama8b": "1 sequence x 4096 tokens, 8 kv / 32 q heads, d=128",
            "tiny": "1 sequence x 1024 tokens, 1 kv / 1 q head, d=128",
            "prefill80": "80 layers x 8 kv heads x 32768 tokens, d=128"}.get(w.name, w.name)
    return {"workload": "%s: %s; TQ%d (values %d-bit MSE, keys %d-bit + 1-bit QJL), %s rotation, "
                        "16-token pages, shuffled block table" % (w.name, desc, w.bits, w.bits, w.bits - 1, rot),
            "global_batch": w.B, "seq_len": w.T, "kv_heads": w.Hkv, "q_heads": w.Hq, "bits": w.bits,
            "rotation": rot, "parallelism": "replicas (weak)",
            "l2": "inputs larger than L2: compress reads 537 MB of fp16 K/V per step; decode reads the 164 MB "
                  "cache written one step earlier, evicted by the 700 MB of compress traffic in between"}


def bench_slots(w):
    """Prefill slot mapping and decode block table.  Several layers flatten into the
    token axis (page-aligned, shuffled blocks); the decode then attends the first
    layer's pages."""
    import numpy as np

    from kv_cache_vector_02_b200 import workloads as W
    if w.layers == 1:
        bt = W.block_table(w)
        return W.prefill_slots(w, bt), bt
    assert w.B == 1, "layered workloads hold one sequence per layer"
    slots = W.flat_slots(w.tokens, perm_seed=w.data_seed)
    bt = (slots[: w.T : PAGE] // PAGE).astype(np.int32)[None]
    return slots, bt


# ---------------------------------------------------------------- GPU arm
def run_prefill(args):
    """Causal prefill attention of the workload's first sequence (all T tokens as one
    chunk) over its compressed cache: one JSON line, attended (query head, token) pairs
    per second, and the tensor-pipe roofline of its contractions."""
    import numpy as np
    import torch
    from kv_cache_vector_02_b200 import tq, workloads as W
    dev = torch.device("cuda")
    rot = 1 if args.rotation == "hadamard" else 0
    w = W.WORKLOADS[args.workload].with_(bits=args.bits, rotation=rot, decode_steps=0, B=1)
    ctx = tq.tq_init(D, w.bits, w.param_seed, w.rotation, w.key_mode)
    slots_np, bt_np = bench_slots(w)
    slots = torch.as_tensor(slots_np, device=dev)
    ck, cv = tq.tq_chunk_bytes(ctx, tq.KIND_KEY), tq.tq_chunk_bytes(ctx, tq.KIND_VALUE)
    kc = torch.zeros((w.num_blocks, w.Hkv, ck), dtype=torch.uint8, device=dev)
    vc = torch.zeros((w.num_blocks, w.Hkv, cv), dtype=torch.uint8, device=dev)
    tq.tq_compress(ctx, W.gen_kv(w, 0, device=dev), W.gen_kv(w, 1, device=dev), slots, kc, vc)
    Tq = w.T
    q = (torch.randn((Tq, w.Hq, D), device=dev, generator=torch.Generator(device=dev).manual_seed(5)) /
         math.sqrt(D)).to(torch.float16)
    bt = torch.as_tensor(np.asarray(bt_np)[0], device=dev)
    out = torch.empty((Tq, w.Hq, D), dtype=torch.float16, device=dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    for _ in range(max(args.warmup, 3)):
        tq.tq_prefill_attention(ctx, q, kc, vc, bt, 0, out)
    torch.cuda.synchronize()
    steps = min(args.steps, 50)
    ts = []
    for i in range(steps):
        flush.fill_(i & 0xff)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        tq.tq_prefill_attention(ctx, q, kc, vc, bt, 0, out)
        e1.record()
        torch.cuda.synchronize()
        ts.append(e0.elapsed_time(e1))
    if tq.tq_get_device_error(ctx) != 0:
        raise RuntimeError("device error word set during the prefill")
    ms = statistics.median(ts)
    pairs = w.Hq * Tq * (Tq + 1) / 2  # attended (query head, token) pairs, causal
    per_pair = (6 if w.key_mode == 0 else 4) * D  # QK^T (+ the QJL sign term) and PV, 2 flops per MAC
    tflops = pairs * per_pair / (ms * 1e-3) / 1e12
    peak = None
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            peak = float(json.load(f)["bf16_tflops"])
    except Exception:
        peak = None
    line = {"metric": "prefill attention (query head, token) pairs/s over the compressed cache", "impl": "tq",
            "value": pairs / (ms * 1e-3), "unit": "pairs/s", "ms": ms, "higher_is_better": True, "n_gpus": 1,
            "steps": steps, "dtype": "f16 operands, f32 accumulate", "data": "synthetic",
            "config": {"workload": "%s: one sequence of %d tokens as one causal chunk, %d kv / %d q heads, TQ%d, %s"
                       % (w.name, Tq, w.Hkv, w.Hq, w.bits, args.rotation), "l2": "flushed (256 MB write) before each call"},
            "roofline": {"bound": "tensor", "achieved": tflops, "peak": peak, "unit": "TFLOP/s",
                         "frac": (tflops / peak) if peak else None,
                         "flops": "%d per attended pair (QK^T, QJL sign term, PV)" % per_pair}}
    print(json.dumps(line))


def main():
    args = parse()
    if args.impl == "reference":
        return run_reference(args)
    if args.prefill:
        return run_prefill(args)
    ws, rank, local = dist_setup("nccl")
    import numpy as np
    import torch

    from kv_cache_vector_02_b200 import tq, workloads as W
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    rot = 1 if args.rotation == "hadamard" else 0
    w = W.WORKLOADS[args.workload].with_(bits=args.bits, rotation=rot, decode_steps=0,
                                         data_seed=rank_data_seed(rank))
    ctx = tq.tq_init(D, w.bits, w.param_seed, w.rotation, w.key_mode)
    slots_np, bt_np = bench_slots(w)
    k = W.gen_kv(w, 0, device=dev)
    v = W.gen_kv(w, 1, device=dev)
    q = W.gen_q(w, 0, device=dev)
    slots = torch.as_tensor(slots_np, device=dev)
    bt = torch.as_tensor(bt_np, device=dev)
    seq = torch.full((w.B,), w.T, dtype=torch.int32, device=dev)
    ck, cv = tq.tq_chunk_bytes(ctx, tq.KIND_KEY), tq.tq_chunk_bytes(ctx, tq.KIND_VALUE)
    caches = [(torch.zeros((w.num_blocks, w.Hkv, ck), dtype=torch.uint8, device=dev),
               torch.zeros((w.num_blocks, w.Hkv, cv), dtype=torch.uint8, device=dev)) for _ in range(2)]
    out = torch.empty((w.B, w.Hq, D), dtype=torch.float16, device=dev)
    wsb = tq.tq_decode_workspace_bytes(ctx, w.B, w.Hq, w.Hkv, w.T)
    workspace = torch.zeros(wsb, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()

    ev = []

    def step(i, record):
        kc, vc = caches[i % 2]
        pk, pv = caches[(i + 1) % 2]
        if record:
            e0, e1, e2 = (torch.cuda.Event(enable_timing=True) for _ in range(3))
            e0.record(stream)
        tq.tq_compress(ctx, k, v, slots, kc, vc, stream=stream)
        if record:
            e1.record(stream)
        tq.tq_decode_attention(ctx, q, pk, pv, bt, seq, w.T, out, workspace, stream=stream)
        if record:
            e2.record(stream)
            ev.append((e0, e1, e2))

    for i in range(max(args.warmup, 3)):
        step(i, False)
    torch.cuda.synchronize()
    if tq.tq_get_device_error(ctx) != 0:
        raise RuntimeError("device error word set during warm-up")

    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.3)
    launches0 = tq.tq_launch_count()
    barrier(ws)
    torch.cuda.synchronize()
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    t_start.record(stream)
    for i in range(args.steps):
        step(args.warmup + i, True)
    t_end.record(stream)
    torch.cuda.synchronize()
    barrier(ws)
    launches = tq.tq_launch_count() - launches0
    clk = clocks.stop()
    ms_total = max_over_ranks(ws, t_start.elapsed_time(t_end))
    comp_ms = [a.elapsed_time(b) for a, b, _ in ev]
    dec_ms = [b.elapsed_time(c) for _, b, c in ev]
    if tq.tq_get_device_error(ctx) != 0:
        raise RuntimeError("device error word set during the timed steps")

    cbytes, dbytes = step_bytes(w)
    ms_step = ms_total / args.steps
    peak, peak_kind = measured_peak()
    comp_avg = max_over_ranks(ws, sum(comp_ms) / len(comp_ms))
    dec_avg = max_over_ranks(ws, sum(dec_ms) / len(dec_ms))
    comp_gbs = cbytes / (comp_avg * 1e-3) / 1e9
    dec_gbs = dbytes / (dec_avg * 1e-3) / 1e9
    value = whole_job_gbs(ws, dbytes, dec_avg)  # the headline: decode-attention KV GB/s
    tokens = w.B * w.T * w.layers

    def roofline(kind):
        rec = traffic_record(kind)
        r = {"kernel": "tq_compress (K and V launches)" if kind == "compress" else
             "tq_decode_attention (one kernel launch)",
             "bound": "hbm", "achieved": comp_gbs if kind == "compress" else dec_gbs,
             "peak": peak, "peak_kind": peak_kind, "unit": "GB/s",
             "traffic": (rec["bytes_per_call"] if rec else None)}
        r["frac"] = r["achieved"] / peak
        if rec and rec.get("tensor_pipe_pct") is not None:
            r["tensor_pipe_pct"] = rec["tensor_pipe_pct"]
        return r
    dominant = "compress" if comp_avg >= dec_avg else "decode"

    # ---- end to end through the C ABI with host buffers (pinned), copies inside the timed region:
    # decode (the metric's call): q host -> device, tq_decode_attention over the resident cache,
    # out device -> host; compress: K, V and the slot mapping host -> device, tq_compress.
    hk = k.cpu().pin_memory()
    hv = v.cpu().pin_memory()
    hq = q.cpu().pin_memory()
    hslots = slots.cpu().pin_memory()
    hout = torch.empty_like(out, device="cpu").pin_memory()
    dk, dv, dq, dsl = torch.empty_like(k), torch.empty_like(v), torch.empty_like(q), torch.empty_like(slots)
    h2d_dec = hq.numel() * 2
    d2h_dec = hout.numel() * 2
    h2d_comp = hk.numel() * 2 + hv.numel() * 2 + hslots.numel() * 4

    def e2e_decode(i):
        kc, vc = caches[i % 2]
        dq.copy_(hq, non_blocking=True)
        tq.tq_decode_attention(ctx, dq, kc, vc, bt, seq, w.T, out, workspace, stream=stream)
        hout.copy_(out, non_blocking=True)

    def e2e_compress(i):
        kc, vc = caches[i % 2]
        dk.copy_(hk, non_blocking=True)
        dv.copy_(hv, non_blocking=True)
        dsl.copy_(hslots, non_blocking=True)
        tq.tq_compress(ctx, dk, dv, dsl, kc, vc, stream=stream)

    def e2e_time(fn, n):
        fn(0)
        torch.cuda.synchronize()
        barrier(ws)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for i in range(n):
            fn(i)
        b.record(stream)
        torch.cuda.synchronize()
        barrier(ws)
        return max_over_ranks(ws, a.elapsed_time(b)) / n

    e2e_dec_ms = e2e_time(e2e_decode, max(1, args.e2e_steps))
    e2e_comp_ms = e2e_time(e2e_compress, max(1, args.e2e_steps // 4))
    if tq.tq_get_device_error(ctx) != 0:
        raise RuntimeError("device error word set during the end-to-end steps")

    cpu = None
    if rank == 0 and ws == 1 and not args.no_cpu_baseline:
        ra = oracle_sample(w, target_s=8.0)   # every core first: the single-thread run lowers OpenMP's default
        r1 = oracle_sample(w, target_s=3.0, threads=1, max_seqs=1)
        cpu = {"value": ra["decode_bytes"] / ra["decode_s"] / 1e9, "unit": "GB/s", "cores": ra["threads"],
               "kind": "oracle", "cpu": cpu_model(),
               "single_thread": {"value": r1["decode_bytes"] / r1["decode_s"] / 1e9, "unit": "GB/s", "cores": 1},
               "compress_mtokens_per_s": ra["seqs"] * w.T / ra["compress_s"] / 1e6,
               "sample": "%d whole sequences of the workload (%d tokens x %d kv heads) compressed, then decode of "
                         "their %d query heads timed: %.1f s on %d threads; single thread: %d sequence, %.1f s"
                         % (ra["seqs"], w.T, w.Hkv, w.Hq, ra["decode_s"], ra["threads"], r1["seqs"],
                            r1["decode_s"])}

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": ws, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f16 operands, f32 accumulate", "data": "synthetic",
            "config": workload_config(w),
            "decode": {"gbs": dec_gbs, "ms": dec_avg, "frac_hbm": dec_gbs / peak, "bytes": dbytes},
            "compress": {"mtokens_per_s": ws * tokens / (comp_avg * 1e-3) / 1e6, "gbs": comp_gbs,
                         "ms": comp_avg, "frac_hbm": comp_gbs / peak, "bytes": cbytes},
            "roofline": roofline(dominant),
            "roofline_decode": roofline("decode"),
            "cpu_baseline": cpu,
            "e2e": {"value": whole_job_gbs(ws, dbytes, e2e_dec_ms), "unit": "GB/s", "h2d_bytes_per_step": h2d_dec,
                    "d2h_bytes_per_step": d2h_dec, "ms_per_step": e2e_dec_ms,
                    "compress": {"mtokens_per_s": ws * tokens / (e2e_comp_ms * 1e-3) / 1e6,
                                 "h2d_bytes_per_step": h2d_comp, "ms_per_step": e2e_comp_ms}},
            "gpu_launches": int(launches),
            "clocks": clk,
        }
        print(json.dumps(line))
    tq.tq_destroy(ctx)
    if ws > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
