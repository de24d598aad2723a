"""Benchmark: non-causal long-sequence attention on B200, one JSON line.

Default workload: S=32768, 32 heads x 128, Q ~ N(0, 4^2), K,V ~ N(0,1), fp16.
One step = the whole hot path over that input: monolithic attention
(attn_fwd) plus the ring-attention emulation (the 8 key-chunk partials with
attn_fwd_partials, then attn_merge).  Both passes do 4*S^2*d*H flops, so the
step's work is 2 * 4*S^2*d*H.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                  [--workload NAME]

N > 1 runs under torchrun as N independent replicas (one per GPU, nothing
exchanged on the data path); the timing is the max over ranks.  The
``reference`` arm times the FP64 CPU oracle on a bounded sample of the same
workload on this host's cores.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads as W  # noqa: E402

METRIC = "attention TFLOP/s (4·S²·d·H, FP16) and % of B200 dense FP16 peak; ms/call"
UNIT = "TFLOP/s"
L2_BYTES = 126 * 2 ** 20


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=25)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default=W.SEQ32K.name,
                    choices=sorted(W.ATTN_WORKLOADS) + sorted(W.STACK_WORKLOADS))
    ap.add_argument("--chunks", type=int, default=None,
                    help="override the workload's number of KV chunks P")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-configs", action="store_true",
                    help="skip the per-configuration side measurements")
    ap.add_argument("--attn-kernel", default="auto", choices=["auto", "single", "pair"],
                    help="head-dim-128 attention kernel (default: chosen by key count)")
    return ap.parse_args()


ATTN_KERNEL_CHOICE = {"auto": 0, "single": 1, "pair": 2}


# ------------------------------------------------------------ distributed --

def dist_setup(n_gpus):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local))
    return rank, world, local


def reduce_max(x: float, world: int) -> float:
    """Max of ``x`` over ranks (the timing rule: the slowest rank sets the time)."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(world: int, units_per_rank: float, max_ms: float) -> float:
    """Whole-job rate: every rank's units over the slowest rank's time (units/s)."""
    return world * units_per_rank / (max_ms * 1e-3)


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


# ----------------------------------------------------------------- clocks --

CLOCK_FIELDS = ("pci.bus_id,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
                "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
                "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
REASONS = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")


class ClockSampler:
    def __init__(self, bus_id: str | None):
        self.bus_id = bus_id
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={CLOCK_FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "200"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        return self

    def __exit__(self, *exc):
        self.rows = []
        if self.proc is None:
            return False
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=10)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        for line in out.splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) != 9:
                continue
            self.rows.append(parts)
        return False

    def summary(self):
        rows = getattr(self, "rows", [])
        if self.bus_id:
            mine = [r for r in rows if r[0].lower().endswith(self.bus_id.lower()[-12:])]
            rows = mine or rows
        buses = {r[0] for r in rows}
        if len(buses) > 1:
            rows = [r for r in rows if r[0] == sorted(buses)[0]]
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        sm = [float(r[1]) for r in rows if r[1].replace(".", "", 1).isdigit()]
        smax = [float(r[2]) for r in rows if r[2].replace(".", "", 1).isdigit()]
        reasons = sorted({name for r in rows for name, v in zip(REASONS, r[5:9]) if v == "Active"})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None, "reasons": reasons,
                "samples": len(rows)}


def bus_id_of(device_index: int):
    try:
        import torch
        p = torch.cuda.get_device_properties(device_index)
        return "%08X:%02X:%02X.0" % (p.pci_domain_id, p.pci_bus_id, p.pci_device_id)
    except Exception:
        return None


# ------------------------------------------------------------------ peaks --

def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            m = json.load(f)
        return {"hbm_gbs": m["hbm_gbs"], "tc_burst": m["bf16_tflops"],
                "tc_sustained": m.get("bf16_tflops_sustained", m["bf16_tflops"]),
                "source": "measured (MEASURED_PEAKS.json; fp16 dense rate = bf16 rate)"}
    return {"hbm_gbs": 6650.0, "tc_burst": 1590.0, "tc_sustained": 1400.0,
            "source": "fallback (profiling recipe figures)"}


def attn_kernel_name(b2a, d: int, Skv: int, mode: int = 0) -> str:
    """The attention kernel the library launches for these sizes (mode 0:
    monolithic, 1: partial, 2: accumulate)."""
    if b2a.attn_kernel_for(d, Skv) == b2a.ATTN_KERNEL_PAIR:
        return f"attn_pair_kernel<{mode}>"
    return f"attn_fwd_kernel<{d}, {mode}, 0>"


def merge_kernel_name(d: int, P: int, partial_type: str) -> str:
    """The merge kernel the library launches: the pipelined persistent form
    up to 16 chunks, else the one-group-per-block form."""
    if P <= 16:
        return f"attn_merge_pipe_kernel<{d}, {partial_type}>"
    return f"attn_merge_kernel<{d}, {partial_type}>"


def committed_traffic(kernel: str, workload: str):
    """DRAM bytes per launch from a committed ncu summary, if it matches the source."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        table = json.load(f)
    ent = table.get(kernel, {}).get(workload)
    if not ent:
        return None
    # the counters hold only while every source the kernel compiles from is unchanged
    h = hashlib.sha256()
    for name in ent["sources"]:
        with open(os.path.join(ROOT, "long_context_bidirectional_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    if h.hexdigest()[:16] != ent["sources_sha256_16"]:
        return None
    return ent["bytes_per_launch"]


# ---------------------------------------------------------- CPU baseline --

def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:
        return 1


def oracle_sample(w, rows_per_head: int):
    """Time the FP64 oracle on ``rows_per_head`` query rows of every head."""
    from oracle import attention as OA
    q, k, v = W.workload_qkv(w)
    rows = [W.sample_rows(w.S, 1, h, seed=w.seed, n=rows_per_head) for h in range(w.H)]
    t0 = time.perf_counter()
    OA.attention(q, k, v, w.scale, rows=rows)
    dt = time.perf_counter() - t0
    flops = 4.0 * rows_per_head * w.S * w.d * w.H
    return flops, dt


def cpu_baseline(w, budget_s: float = 10.0):
    rows = 8
    flops, dt = oracle_sample(w, rows)
    while dt < budget_s / 4 and rows < 1024:
        rows *= 2
        flops, dt = oracle_sample(w, rows)
    return {"value": flops / dt / 1e12, "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
            "sample": f"FP64 numpy oracle, monolithic attention of {rows} query rows per head x "
                      f"{w.H} heads against all {w.S} keys ({flops / 1e9:.1f} GFLOP in {dt:.2f} s); "
                      f"host has {os.cpu_count()} logical cores"}


# --------------------------------------------------------------- our arm --

def measure_batched(b2a, S, B, H, d, dev, stream, world, pk, n=5):
    """attn_fwd_batched on the (S, B, hidden) layout, one launch over every
    (row block, head, batch); inputs seeded like the attention workloads."""
    import torch
    q, k, v = W.qkv(S, B * H, d, seed=0)
    qd, kd, vd = (torch.from_numpy(x).to(dev).view(S, B, H, d) for x in (q, k, v))
    out = torch.empty_like(qd)
    lse = torch.empty((B, H, S), dtype=torch.float32, device=dev)
    fn = lambda: b2a.attn_fwd_batched(qd, kd, vd, out=out, lse=lse, scale=1 / math.sqrt(d), stream=stream)
    for _ in range(2):
        fn()
    torch.cuda.synchronize()
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(n):
        fn()
    b.record(stream)
    torch.cuda.synchronize()
    b2a.check_status(stream)
    ms = reduce_max(a.elapsed_time(b) / n, world)
    tfl = 4.0 * S * S * d * H * B / (ms * 1e-3) / 1e12
    return {"S": S, "B": B, "H": H, "d": d, "attn_fwd_batched_ms": ms, "attn_fwd_batched_tflops": tfl,
            "attn_fwd_batched_frac": tfl / pk["tc_burst"], "launches": 1}


def measure_attn_config(b2a, w, dev, stream, world, pk, n=5):
    """One attention workload, CUDA-event timed: monolithic attn_fwd and, for
    workloads with P > 1 key chunks, the partials launch and the merge."""
    import torch
    q, k, v = W.workload_qkv(w)
    qd, kd, vd = (torch.from_numpy(x).to(dev) for x in (q, k, v))
    S, H, d = w.S, w.H, w.d
    out = torch.empty((S, H, d), dtype=torch.float16, device=dev)
    lse = torch.empty((H, S), dtype=torch.float32, device=dev)

    def timed(fn, reps):
        for _ in range(2):
            fn()
        torch.cuda.synchronize()
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(reps):
            fn()
        b.record(stream)
        torch.cuda.synchronize()
        b2a.check_status(stream)
        return reduce_max(a.elapsed_time(b) / reps, world)

    mono_ms = timed(lambda: b2a.attn_fwd(qd, kd, vd, out=out, lse=lse, scale=w.scale, stream=stream), n)
    tfl = w.flops / (mono_ms * 1e-3) / 1e12
    res = {"S": S, "H": H, "d": d, "q_sigma": w.q_sigma, "attn_kernel": attn_kernel_name(b2a, d, S),
           "attn_fwd_ms": mono_ms, "attn_fwd_tflops": tfl, "attn_fwd_frac": tfl / pk["tc_burst"]}
    if w.P > 1:
        P = w.P
        o_parts = torch.empty((P, S, H, d), dtype=torch.float32, device=dev)
        lse_parts = torch.empty((P, H, S), dtype=torch.float32, device=dev)
        part_ms = timed(lambda: b2a.attn_fwd_partials(qd, kd, vd, P, o_parts, lse_parts, scale=w.scale,
                                                      stream=stream), n)
        out_c = torch.empty_like(out)
        lse_c = torch.empty_like(lse)
        merge_ms = timed(lambda: b2a.attn_merge(o_parts, lse_parts, out=out_c, lse_out=lse_c, stream=stream),
                         4 * n)
        merge_bytes = P * S * H * d * 4 + P * H * S * 4 + S * H * d * 2 + H * S * 4
        ptf = w.flops / (part_ms * 1e-3) / 1e12
        gbs = merge_bytes / (merge_ms * 1e-3) / 1e9
        res.update({"P": P, "partials_ms": part_ms, "partials_tflops": ptf, "partials_frac": ptf / pk["tc_burst"],
                    "partials_kernel": attn_kernel_name(b2a, d, (S + P - 1) // P, 1),
                    "merge_ms": merge_ms, "merge_gbs": gbs, "merge_hbm_frac": gbs / pk["hbm_gbs"],
                    "step_ms": mono_ms + part_ms + merge_ms,
                    "step_tflops": 2 * w.flops / ((mono_ms + part_ms + merge_ms) * 1e-3) / 1e12})
    res["peaks"] = "tensor-bound kernels against the burst bf16 figure, the merge against the copy bandwidth"
    return res



def run_ours(args, rank, world, local):
    import torch
    import long_context_bidirectional_b200 as b2a

    w = W.ATTN_WORKLOADS[args.workload]
    b2a.set_attn_kernel(ATTN_KERNEL_CHOICE[args.attn_kernel])
    P = max(args.chunks or w.P, 1)
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    q, k, v = W.workload_qkv(w)
    qd, kd, vd = (torch.from_numpy(x).to(dev) for x in (q, k, v))
    S, H, d = w.S, w.H, w.d
    out = torch.empty((S, H, d), dtype=torch.float16, device=dev)
    lse = torch.empty((H, S), dtype=torch.float32, device=dev)
    out_c = torch.empty_like(out)
    lse_c = torch.empty_like(lse)
    o_parts = torch.empty((P, S, H, d), dtype=torch.float32, device=dev)
    lse_parts = torch.empty((P, H, S), dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)
    bounds = b2a.chunk_bounds(S, P)

    ev = {name: [] for name in ("mono", "partials", "merge")}

    def step(record):
        def mark():
            e = torch.cuda.Event(enable_timing=True)
            e.record(stream)
            return e
        e0 = mark() if record else None
        b2a.attn_fwd(qd, kd, vd, out=out, lse=lse, scale=w.scale, stream=stream)
        e1 = mark() if record else None
        b2a.attn_fwd_partials(qd, kd, vd, P, o_parts, lse_parts, scale=w.scale, stream=stream)
        e2 = mark() if record else None
        b2a.attn_merge(o_parts, lse_parts, out=out_c, lse_out=lse_c, stream=stream)
        e3 = mark() if record else None
        if record:
            ev["mono"].append((e0, e1))
            ev["partials"].append((e1, e2))
            ev["merge"].append((e2, e3))

    for _ in range(args.warmup):
        step(False)
    b2a.check_status(stream)
    barrier(world)
    torch.cuda.synchronize()

    with ClockSampler(bus_id_of(local)) as clk:
        t0 = torch.cuda.Event(enable_timing=True)
        t1 = torch.cuda.Event(enable_timing=True)
        t0.record(stream)
        for _ in range(args.steps):
            step(True)
        t1.record(stream)
        torch.cuda.synchronize()
    barrier(world)
    b2a.check_status(stream)
    local_ms = t0.elapsed_time(t1) / args.steps
    ms = reduce_max(local_ms, world)

    def avg(name):
        return sum(a.elapsed_time(b) for a, b in ev[name]) / len(ev[name])

    mono_ms = reduce_max(avg("mono"), world)
    part_ms = reduce_max(avg("partials"), world)
    merge_ms = reduce_max(avg("merge"), world)

    step_flops = 2.0 * w.flops
    value = job_throughput(world, step_flops, ms) / 1e12
    pk = peaks()
    mono_tflops = w.flops / (mono_ms * 1e-3) / 1e12
    part_tflops = w.flops / (part_ms * 1e-3) / 1e12
    merge_bytes = P * S * H * d * 4 + P * H * S * 4 + S * H * d * 2 + H * S * 4
    merge_gbs = merge_bytes / (merge_ms * 1e-3) / 1e9

    # Roofline of each kernel of the step (per-launch averages from the CUDA
    # events above); the line's ``roofline`` is the one with the largest share.
    chunk_keys = max(hi_ - lo_ for lo_, hi_ in bounds)
    # attn_fwd_partials: one launch of the single-CTA kernel over every chunk
    # when the chunks are short enough for it (and none is empty)
    part_kernel = attn_kernel_name(b2a, d, chunk_keys, 1)
    one_launch = S >= P and part_kernel.startswith("attn_fwd_kernel")
    part_launches = 1 if one_launch else P
    rl = [
        {"bound": "tensor", "kernel": attn_kernel_name(b2a, d, S, 0), "role": "attn_fwd (monolithic)",
         "launches_per_step": 1, "ms_per_launch": mono_ms, "achieved": mono_tflops, "unit": "TFLOP/s",
         "peak": pk["tc_burst"], "algorithmic": "4*S^2*d*H flops per launch"},
        {"bound": "tensor", "kernel": part_kernel, "role": f"attn_fwd_partials ({P} chunks)",
         "launches_per_step": part_launches, "ms_per_launch": part_ms / part_launches, "achieved": part_tflops,
         "unit": "TFLOP/s", "peak": pk["tc_burst"],
         "algorithmic": ("4*S^2*d*H flops per launch (all chunks)" if one_launch
                         else "4*S*(S/P)*d*H flops per launch (one chunk)")},
        {"bound": "hbm", "kernel": merge_kernel_name(d, P, "float"), "role": "attn_merge",
         "launches_per_step": 1, "ms_per_launch": merge_ms, "achieved": merge_gbs, "unit": "GB/s",
         "peak": pk["hbm_gbs"],
         "algorithmic": "P*S*H*d*4 + P*H*S*4 + S*H*d*2 + H*S*4 bytes per launch (o_parts, lse_parts, out, lse)"},
    ]
    step_kernel_ms = sum(e["launches_per_step"] * e["ms_per_launch"] for e in rl)
    for e in rl:
        e["frac"] = e["achieved"] / e["peak"]
        e["share_of_step"] = e["launches_per_step"] * e["ms_per_launch"] / step_kernel_ms
        e["traffic"] = committed_traffic(e["kernel"], w.name)
        if e["bound"] == "tensor":
            e["frac_of_sustained_peak"] = e["achieved"] / pk["tc_sustained"]
    dominant = max(rl, key=lambda e: e["share_of_step"])

    # The ring-step form (attn_fwd_accumulate): the same P chunks folded into
    # one running fp32 output in place, the last step writing fp16.  Timed
    # separately from the step; not part of ``value``.
    o_acc = torch.empty((S, H, d), dtype=torch.float32, device=dev)
    lse_acc = torch.empty((H, S), dtype=torch.float32, device=dev)
    out_r = torch.empty_like(out)

    def ring_pass():
        lse_acc.fill_(float("-inf"))
        for c, (lo, hi) in enumerate(bounds):
            b2a.attn_fwd_accumulate(qd, kd[lo:hi], vd[lo:hi], o_acc, lse_acc,
                                    out_r if c == P - 1 else None, scale=w.scale, stream=stream)

    for _ in range(2):
        ring_pass()
    b2a.check_status(stream)
    barrier(world)
    torch.cuda.synchronize()
    ra = torch.cuda.Event(enable_timing=True)
    rb = torch.cuda.Event(enable_timing=True)
    n_ring = 5
    ra.record(stream)
    for _ in range(n_ring):
        ring_pass()
    rb.record(stream)
    torch.cuda.synchronize()
    b2a.check_status(stream)
    ring_ms = reduce_max(ra.elapsed_time(rb) / n_ring, world)
    del o_acc, lse_acc, out_r

    # Per-rank shapes of the context-parallel variants (8 ranks), on this GPU:
    # AllGather-KV rank 3 (its 1/8 of the query rows against every key) and
    # Ulysses rank 3 (every row for 1/8 of the heads).  Not part of ``value``.
    def time_calls(fn, n=5):
        for _ in range(2):
            fn()
        torch.cuda.synchronize()
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(n):
            fn()
        b.record(stream)
        torch.cuda.synchronize()
        b2a.check_status(stream)
        return reduce_max(a.elapsed_time(b) / n, world)

    lo, hi = b2a.chunk_bounds(S, 8)[3]
    cp_out = torch.empty((hi - lo, H, d), dtype=torch.float16, device=dev)
    ag_ms = time_calls(lambda: b2a.attn_fwd_gathered_kv(qd[lo:hi], kd, vd, out=cp_out, return_lse=False,
                                                        scale=w.scale, stream=stream))
    hs = slice(3 * (H // 8), 4 * (H // 8)) if H >= 8 else slice(0, H)
    nh = hs.stop - hs.start
    uly_ms = time_calls(lambda: b2a.attn_fwd(qd[:, hs], kd[:, hs], vd[:, hs], out=out[:, hs], return_lse=False,
                                             scale=w.scale, stream=stream))
    del cp_out

    # The same partials as one attn_fwd_partial call per chunk (what a ring
    # rank does as each K/V block arrives).  Not part of ``value``.
    def per_chunk_pass():
        for c, (c_lo, c_hi) in enumerate(bounds):
            b2a.attn_fwd_partial(qd, kd[c_lo:c_hi], vd[c_lo:c_hi], o_parts[c], lse_parts[c], scale=w.scale,
                                 stream=stream)

    pcc_ms = time_calls(per_chunk_pass, n=3)

    # The FP16 split-reduction: the same P partials stored in fp16, and the
    # merge reading them (half the partial bytes).  Not part of ``value``.
    o16_parts = torch.empty((P, S, H, d), dtype=torch.float16, device=dev)

    def part16_pass():
        b2a.attn_fwd_partials(qd, kd, vd, P, o16_parts, lse_parts, scale=w.scale, stream=stream,
                              partial_dtype=torch.float16)

    p16_ms = time_calls(part16_pass, n=3)
    m16_ms = time_calls(lambda: b2a.attn_merge_f16(o16_parts, lse_parts, out=out_c, lse_out=lse_c,
                                                   stream=stream))
    merge16_bytes = P * S * H * d * 2 + P * H * S * 4 + S * H * d * 2 + H * S * 4
    merge16_gbs = merge16_bytes / (m16_ms * 1e-3) / 1e9

    # The other configurations of the pages' validation tables, each timed
    # with CUDA events on its own inputs (not part of ``value``): S=8192 at
    # hidden 4096 (monolithic + 2 key chunks + merge), S=65536 at hidden
    # 4096, S=8192 at hidden 8192 (64 heads), and the 6-block stack at
    # S=32768 with its attention and projection GEMMs reported separately.
    configs = {}
    if not args.no_configs:
        del o16_parts
        for cw in (W.SEQ8K, W.SEQ64K, W.SEQ8K_H64):
            configs[cw.name] = measure_attn_config(b2a, cw, dev, stream, world, pk)
            torch.cuda.empty_cache()
        configs[W.STACK6.name] = measure_stack(b2a, W.STACK6, dev, stream, steps=3, warmup=2, world=world)
        torch.cuda.empty_cache()
        configs["batched_s8192_b4_h32_d128"] = measure_batched(b2a, 8192, 4, 32, 128, dev, stream, world, pk)
        torch.cuda.empty_cache()
    else:
        del o16_parts

    # end to end from pinned host memory through the C-ABI host entry point
    e2e = None
    if not args.no_e2e:
        qh, kh, vh = (torch.from_numpy(x).pin_memory() for x in (q, k, v))
        oh = torch.empty((S, H, d), dtype=torch.float16).pin_memory()
        lh = torch.empty((H, S), dtype=torch.float32).pin_memory()
        oh2 = torch.empty_like(oh).pin_memory()
        lh2 = torch.empty_like(lh).pin_memory()
        del o_parts, lse_parts
        # The step's two calls are independent: each goes on its own stream
        # with its own workspace, so one call's host<->device copies run
        # under the other's kernels (each call still copies its own inputs
        # in and its results out every step).
        stream2 = torch.cuda.Stream(dev)
        ws = torch.empty(b2a.host_workspace_bytes(S, H, d, 1), dtype=torch.uint8, device=dev)
        ws2 = torch.empty(b2a.host_workspace_bytes(S, H, d, P), dtype=torch.uint8, device=dev)

        def e2e_step():
            b2a.attn_fwd_host(qh, kh, vh, oh, lh, ws, P=1, scale=w.scale, stream=stream)
            b2a.attn_fwd_host(qh, kh, vh, oh2, lh2, ws2, P=P, scale=w.scale, stream=stream2)

        for _ in range(max(1, min(args.warmup, 2))):
            e2e_step()
        torch.cuda.synchronize()
        b2a.check_status(stream)
        barrier(world)
        torch.cuda.synchronize()
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record(stream)
        stream2.wait_event(a)
        for _ in range(args.steps):
            e2e_step()
        j = torch.cuda.Event()
        j.record(stream2)
        stream.wait_event(j)
        b.record(stream)
        torch.cuda.synchronize()
        e2e_ms = reduce_max(a.elapsed_time(b) / args.steps, world)
        b2a.check_status(stream)
        n16 = S * H * d * 2
        e2e = {"value": job_throughput(world, step_flops, e2e_ms) / 1e12, "unit": UNIT,
               "ms_per_step": e2e_ms,
               "h2d_bytes_per_step": 2 * 3 * n16, "d2h_bytes_per_step": 2 * (n16 + H * S * 4),
               "path": ("attn_fwd_host(P=1) and attn_fwd_host(P=%d) from pinned host buffers, on two "
                        "streams with a workspace each" % P)}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(w)

    clocks = clk.summary()
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f16", "data": "synthetic",
        "config": {"workload": w.name, "S": S, "H": H, "d": d, "P": P, "batch": 1,
                   "q_sigma": w.q_sigma, "kv_sigma": w.kv_sigma,
                   "step": f"attn_fwd + attn_fwd_partials ({P} chunks) + attn_merge",
                   "step_flops": step_flops, "attn_kernel": args.attn_kernel,
                   "l2": f"inputs larger than L2 (Q,K,V {3 * S * H * d * 2 / 2**20:.0f} MiB, "
                         f"partials {P * S * H * d * 4 / 2**20:.0f} MiB per step)",
                   "parallelism": f"replicas x{world}"},
        "roofline": dict(dominant, peak_source=pk["source"] + "; burst figure for the tensor-bound kernels "
                         "(each launch is well under a second and the SM clock stays near its maximum)",
                         all_kernels=[{k: v for k, v in e.items() if k != "algorithmic"} for e in rl]),
        "kernels": {"attn_fwd_ms": mono_ms, "attn_fwd_tflops": mono_tflops,
                    "partial_pass_ms": part_ms,
                    "partial_pass_tflops": part_tflops,
                    "partial_pass": f"attn_fwd_partials, {P} chunks, {part_launches} launch(es) of {part_kernel}",
                    "partial_per_chunk_calls_ms": pcc_ms,
                    "partial_per_chunk_calls_tflops": w.flops / (pcc_ms * 1e-3) / 1e12,
                    "merge_ms": merge_ms, "merge_gbs": merge_gbs,
                    "ring_pass_ms": ring_ms,
                    "ring_pass_tflops": w.flops / (ring_ms * 1e-3) / 1e12,
                    "ring_pass": f"{P} x attn_fwd_accumulate in place (not in value)",
                    "cp_gather_kv_rank_ms": ag_ms,
                    "cp_gather_kv_rank_tflops": 4.0 * (hi - lo) * S * d * H / (ag_ms * 1e-3) / 1e12,
                    "cp_ulysses_rank_ms": uly_ms,
                    "cp_ulysses_rank_tflops": 4.0 * S * S * d * nh / (uly_ms * 1e-3) / 1e12,
                    "cp_ranks": f"8-way: AllGather-KV rank 3 ({hi - lo} rows x {S} keys), Ulysses rank 3 "
                                f"({nh} of {H} heads); not in value",
                    "merge_hbm_frac": merge_gbs / pk["hbm_gbs"], "merge_bytes": merge_bytes,
                    "fp16_partial_pass_ms": p16_ms,
                    "fp16_partial_pass_tflops": w.flops / (p16_ms * 1e-3) / 1e12,
                    "merge_f16_ms": m16_ms, "merge_f16_gbs": merge16_gbs,
                    "merge_f16_hbm_frac": merge16_gbs / pk["hbm_gbs"], "merge_f16_bytes": merge16_bytes,
                    "fp16_split_reduction": "attn_fwd_partials_f16 + attn_merge_f16 (not in value)"},
        "configs": configs,
        "cpu_baseline": cpu,
        "e2e": e2e,
        "gpu_launches": args.steps * (part_launches + 2),
        "clocks": clocks,
    }
    if rank == 0:
        print(json.dumps(line), flush=True)


# ------------------------------------------------------- stack workload --

def measure_stack(b2a, w, dev, stream, steps, warmup, world, sample_clocks=False):
    """Time ``w.blocks`` stacked blocks (fused QKV GEMM, attention on strided
    views of its output, output GEMM + residual) on x [S, H*d]: the whole
    step from CUDA events around it, and each kernel's share from events
    around every launch.  Returns the figures as a dict."""
    import torch
    S, H, d, h = w.S, w.H, w.d, w.hidden
    x0 = torch.from_numpy(W.stack_x(w)).to(dev)
    weights = [tuple(torch.from_numpy(t).to(dev) for t in W.stack_weights(w, i)) for i in range(w.blocks)]
    x = torch.empty_like(x0)
    qkv_ws = torch.empty((S, 3 * h), dtype=torch.float16, device=dev)
    attn_ws = torch.empty((S, h), dtype=torch.float16, device=dev)
    ev = []

    def step(record):
        x.copy_(x0)
        for w_qkv, w_o in weights:
            if record:
                e = [torch.cuda.Event(enable_timing=True) for _ in range(4)]
                e[0].record(stream)
            b2a.qkv_proj(x, w_qkv, out=qkv_ws, stream=stream)
            if record:
                e[1].record(stream)
            b2a.attn_fwd(qkv_ws[:, 0:h].view(S, H, d), qkv_ws[:, h:2 * h].view(S, H, d),
                         qkv_ws[:, 2 * h:].view(S, H, d), out=attn_ws.view(S, H, d), scale=w.scale,
                         return_lse=False, stream=stream)
            if record:
                e[2].record(stream)
            b2a.out_proj(attn_ws, w_o, residual=x, out=x, stream=stream)
            if record:
                e[3].record(stream)
                ev.append(e)

    for _ in range(warmup):
        step(False)
    b2a.check_status(stream)
    barrier(world)
    torch.cuda.synchronize()
    clk = ClockSampler(bus_id_of(dev.index)) if sample_clocks else None
    if clk:
        clk.__enter__()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for _ in range(steps):
        step(True)
    t1.record(stream)
    torch.cuda.synchronize()
    if clk:
        clk.__exit__(None, None, None)
    barrier(world)
    b2a.check_status(stream)
    ms = reduce_max(t0.elapsed_time(t1) / steps, world)
    n = len(ev)
    qkv_ms = reduce_max(sum(e[0].elapsed_time(e[1]) for e in ev) / n, world)
    att_ms = reduce_max(sum(e[1].elapsed_time(e[2]) for e in ev) / n, world)
    out_ms = reduce_max(sum(e[2].elapsed_time(e[3]) for e in ev) / n, world)
    f_att = 4.0 * S * S * d * H
    f_qkv = 2.0 * S * 3 * h * h
    f_out = 2.0 * S * h * h
    step_flops = w.blocks * (f_att + f_qkv + f_out)
    pk = peaks()

    def tf(f, t):
        return f / (t * 1e-3) / 1e12

    res = {"workload": w.name, "S": S, "H": H, "d": d, "blocks": w.blocks, "ms_per_step": ms,
           "step_flops": step_flops, "tflops": job_throughput(world, step_flops, ms) / 1e12,
           "frac": tf(step_flops, ms) / pk["tc_burst"],
           "qkv_proj_ms": qkv_ms, "qkv_proj_tflops": tf(f_qkv, qkv_ms), "qkv_proj_frac": tf(f_qkv, qkv_ms) / pk["tc_burst"],
           "attn_fwd_ms": att_ms, "attn_fwd_tflops": tf(f_att, att_ms), "attn_fwd_frac": tf(f_att, att_ms) / pk["tc_burst"],
           "attn_kernel": attn_kernel_name(b2a, d, S),
           "out_proj_ms": out_ms, "out_proj_tflops": tf(f_out, out_ms), "out_proj_frac": tf(f_out, out_ms) / pk["tc_burst"],
           "peak": pk["tc_burst"], "peak_source": pk["source"] + "; burst figure"}
    if clk:
        res["clocks"] = clk.summary()
    # The projection with the q/k RMSNorm epilogue (the norm reading of the
    # sample block), timed on its own; not part of the step.
    g_ones = torch.ones(d, dtype=torch.float16, device=dev)
    for _ in range(2):
        b2a.qkv_proj_qknorm(x0, weights[0][0], g_ones, g_ones, H, d, 1e-6, out=qkv_ws, stream=stream)
    torch.cuda.synchronize()
    na = torch.cuda.Event(enable_timing=True)
    nb_ = torch.cuda.Event(enable_timing=True)
    na.record(stream)
    for _ in range(5):
        b2a.qkv_proj_qknorm(x0, weights[0][0], g_ones, g_ones, H, d, 1e-6, out=qkv_ws, stream=stream)
    nb_.record(stream)
    torch.cuda.synchronize()
    b2a.check_status(stream)
    qkn_ms = reduce_max(na.elapsed_time(nb_) / 5, world)
    res["qkv_proj_qknorm_ms"] = qkn_ms
    res["qkv_proj_qknorm_tflops"] = tf(f_qkv, qkn_ms)
    del x0, weights, x, qkv_ws, attn_ws
    return res


def run_stack(args, rank, world, local):
    """Six stacked self-attention blocks (fused QKV GEMM, attention on strided
    views, output GEMM + residual) on x [S, H*d]; value counts attention plus
    both projections."""
    import torch
    import long_context_bidirectional_b200 as b2a

    w = W.STACK_WORKLOADS[args.workload]
    b2a.set_attn_kernel(ATTN_KERNEL_CHOICE[args.attn_kernel])
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream(dev)
    r = measure_stack(b2a, w, dev, stream, args.steps, args.warmup, world, sample_clocks=True)
    pk = peaks()
    line = {
        "metric": METRIC, "value": r["tflops"], "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": r["ms_per_step"], "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f16", "data": "synthetic",
        "config": {"workload": w.name, "S": w.S, "H": w.H, "d": w.d, "blocks": w.blocks, "batch": 1,
                   "step": "per block: qkv_proj, attn_fwd on strided views, out_proj + residual",
                   "step_flops": r["step_flops"], "l2": "inputs larger than L2 (weights 128 MiB per block)",
                   "parallelism": f"replicas x{world}"},
        "kernels": {k: v for k, v in r.items() if k.startswith(("qkv_proj", "attn_fwd", "out_proj"))},
        "roofline": {"bound": "tensor", "kernel": r["attn_kernel"], "achieved": r["attn_fwd_tflops"],
                     "peak": pk["tc_burst"], "unit": "TFLOP/s", "frac": r["attn_fwd_frac"],
                     "peak_source": pk["source"], "traffic": None, "algorithmic": "4*S^2*d*H flops per launch"},
        "cpu_baseline": None, "e2e": None,
        "gpu_launches": args.steps * w.blocks * 3,
        "clocks": r.get("clocks"),
    }
    if rank == 0:
        print(json.dumps(line), flush=True)


# --------------------------------------------------------- reference arm --

def run_reference(args, rank, world):
    if rank != 0:
        return
    if args.workload not in W.ATTN_WORKLOADS:
        print(json.dumps({"impl": "reference", "unavailable": "the CPU reference arm covers the attention "
                          "workloads only"}), flush=True)
        return
    w = W.ATTN_WORKLOADS[args.workload]
    # query rows per head per step: a bounded sample of the workload, large
    # enough that the oracle's arithmetic (not its per-call widening of K and
    # V to FP64) dominates a step (~1-2 s on 16 host cores)
    rows = 32
    for _ in range(args.warmup):
        oracle_sample(w, rows)
    total_flops, total_s = 0.0, 0.0
    for _ in range(args.steps):
        f, dt = oracle_sample(w, rows)
        total_flops += f
        total_s += dt
    value = total_flops / total_s / 1e12
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": 1,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": total_s / args.steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": {"workload": w.name, "S": w.S, "H": w.H, "d": w.d, "P": max(w.P, 1), "batch": 1,
                   "parallelism": "host cores"},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
                         "sample": f"FP64 numpy oracle, {rows} query rows per head x {w.H} heads "
                                   f"against all {w.S} keys per step"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main():
    args = parse()
    if args.impl == "reference":
        rank = int(os.environ.get("RANK", "0"))
        run_reference(args, rank, int(os.environ.get("WORLD_SIZE", "1")))
        return
    rank, world, local = dist_setup(args.gpus)
    try:
        if args.workload in W.STACK_WORKLOADS:
            run_stack(args, rank, world, local)
        else:
            run_ours(args, rank, world, local)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
