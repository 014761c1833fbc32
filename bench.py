#!/usr/bin/env python3
"""Benchmark of the decode step: kv_append + paged GQA decode attention on a B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload I] [--impl ours|reference]

One step = one pass of the whole hot path over one batch: kv_append writes each
sequence's new K/V token into its page, then paged_decode_attn attends over the
paged cache (split-KV with its log-sum-exp merge inside the same launch).  The
default workload is the GQA serving batch (32 sequences, 32 query / 8 KV heads,
head_dim 128, page_size 16, lengths uniform in [512, 4096]).

Prints ONE JSON line on rank 0.  `value` is the step's algorithmic HBM bytes
(all K/V bytes of every context token, plus q, out, the appended rows, block
table and lengths) divided by the step time, in TB/s, summed over ranks.  Each
rank runs its own independent batch (weak scaling, no collective on the data
path).  Inputs are resident in HBM; the working set (two copies of the page
pools, rotated step by step) is several times the 126 MB L2.
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

import torch
import torch.distributed as dist

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from workloads import WORKLOADS, make_inputs, bf16_bits  # noqa: E402

METRIC = "paged GQA decode attn: achieved HBM TB/s (% of B200 peak), tokens/s"
FALLBACK_HBM_GBS = 6650.0
PROFILE_TRAFFIC = os.path.join(ROOT, "profiles", "traffic.json")
_CSRC = "gqa_decode_attention_04_b200/csrc/"
KERNEL_SOURCES = {
    "decode_ws_kernel": [_CSRC + "decode_ws.cu", _CSRC + "ptx.cuh", _CSRC + "internal.cuh"],
    "decode_tc_kernel": [_CSRC + "decode_tc.cu", _CSRC + "ptx.cuh", _CSRC + "internal.cuh"],
}


def decode_kernel_for(inp) -> str:
    """The decode kernel the library picks for this head grouping: the tcgen05 kernel
    for more than 16 query heads per kv head, the mma.sync kernel otherwise."""
    return "decode_tc_kernel" if inp.num_heads // inp.num_kv_heads > 16 else "decode_ws_kernel"


# ------------------------------------------------------------------ helpers

def algorithmic_bytes(inp, with_append: bool, num_seqs=None) -> dict:
    """Bytes the step must move: every cached K/V byte once, q in, out back, plus
    the block-table entries and lengths read, and the appended rows.  With
    num_seqs, only the first num_seqs sequences count."""
    B = inp.num_seqs if num_seqs is None else num_seqs
    H, Hk, D, ps = inp.num_heads, inp.num_kv_heads, inp.head_dim, inp.page_size
    L = inp.seq_lens[:B].to(torch.int64).cpu()
    kv = int(L.sum()) * Hk * D * 2 * 2
    pages = int(((L + ps - 1) // ps).sum())
    qo = 2 * B * H * D * 2
    meta = pages * 4 + B * 4
    decode = kv + qo + meta
    append = 0
    if with_append:
        append = 2 * (B * Hk * D * 2) * 2 + B * 4 + B * 4  # read new rows + write slots, positions, bt
    return {"kv": kv, "decode": decode, "append": append, "step": decode + append}


def measured_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            j = json.load(f)
        return float(j["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def kernel_source_sha(kernel: str) -> str:
    h = hashlib.sha256()
    for rel in KERNEL_SOURCES[kernel]:
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def profiled_traffic(workload_name: str, kernel: str, units_per_launch: int):
    """DRAM bytes per launch from a committed ncu capture, if it was taken of the
    current kernel source; scaled to this launch's units when the capture was of a
    smaller case.  None when absent or stale."""
    try:
        with open(PROFILE_TRAFFIC) as f:
            j = json.load(f)
        e = j[workload_name]
        if not e.get("kernel", "").startswith(kernel) or e.get("kernel_source_sha") != kernel_source_sha(kernel):
            return None
        per_unit = e["dram_bytes_per_launch"] / e["units_per_launch"]
        return int(round(per_unit * units_per_launch))
    except Exception:
        return None


class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu_index = gpu_index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu_index), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        self.lines = []
        if self.proc is not None:
            time.sleep(0.25)
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except Exception:
                self.proc.kill()
                out = ""
            self.lines = [ln for ln in out.splitlines() if ln.strip()]
        return False

    def summary(self):
        sm, mx, reasons = [], None, set()
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx = float(parts[2])
            except ValueError:
                continue
            names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
            for n, v in zip(names, parts[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


def setup_dist(n_gpus: int):
    if n_gpus > 1 or "RANK" in os.environ:
        rank = int(os.environ.get("RANK", "0"))
        world = int(os.environ.get("WORLD_SIZE", "1"))
        local = int(os.environ.get("LOCAL_RANK", "0"))
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if torch.cuda.is_available():
            torch.cuda.set_device(local)
        import datetime
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
        return rank, world, local
    return 0, 1, 0


def rank_seed(workload: int, rank: int) -> int:
    """Seed of the batch rank `rank` runs: rank 0 runs the workload's own batch, the
    others independent batches of the same shape (weak scaling, no data exchange)."""
    return 1000 + workload + 7919 * rank


def reduce_max_sum(t_ms: float, units: float, device):
    """Max of the per-rank times and sum of the per-rank units (whole-job figures)."""
    if not dist.is_initialized():
        return t_ms, units
    t = torch.tensor([t_ms], dtype=torch.float64, device=device)
    u = torch.tensor([units], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    dist.all_reduce(u, op=dist.ReduceOp.SUM)
    return float(t.item()), float(u.item())


def barrier():
    if dist.is_initialized():
        dist.barrier()


# ------------------------------------------------------------------ CPU oracle timing

def time_oracle(inp, min_seconds: float, max_seconds: float):
    """Time the fp64 oracle, as it stands, on the same step (its kv_append, then its
    attention) over the workload, repeated for at least min_seconds, or over a prefix
    of the sequences when one pass would exceed max_seconds.  Returns (bytes/s,
    seqs/s, description).  BLAS is held to one thread: exactly one host core."""
    from threadpoolctl import threadpool_limits
    import oracle

    q, k, v = bf16_bits(inp.q), bf16_bits(inp.k_pages), bf16_bits(inp.v_pages)
    kn, vn = bf16_bits(inp.k_new), bf16_bits(inp.v_new)
    bt, sl, pos = inp.block_table.numpy(), inp.seq_lens.numpy(), inp.positions.numpy()
    B = inp.num_seqs

    def one_step(n):
        k2, v2 = oracle.kv_append(k, v, kn[:n], vn[:n], bt[:n], pos[:n])
        oracle.paged_decode_attention(q[:n], k2, v2, bt[:n], sl[:n], inp.scale)

    with threadpool_limits(1):
        t0 = time.perf_counter()
        one_step(1)
        est_all = (time.perf_counter() - t0) * float(sl.sum()) / max(1, int(sl[0]))
        n = B if est_all <= max_seconds else max(1, int(B * max_seconds / est_all))
        step_bytes = algorithmic_bytes(inp, with_append=True, num_seqs=n)["step"]
        elapsed, passes = 0.0, 0
        while elapsed < min_seconds and elapsed < max_seconds:
            t0 = time.perf_counter()
            one_step(n)
            elapsed += time.perf_counter() - t0
            passes += 1
    desc = (f"{passes} pass(es) of the fp64 oracle step (kv_append + attention) over {n} of "
            f"{B} sequences ({int(sl[:n].sum())} context tokens per pass), single thread")
    return step_bytes * passes / elapsed, n * passes / elapsed, desc


# ------------------------------------------------------------------ arms

def run_reference(args, rank, world):
    """Reference arm: the fp64 CPU oracle on the host, rank 0 only.  Each step is a
    bounded sample of the workload: the oracle's kv_append, then its attention over a
    prefix of the sequences (all of them when that fits the time budget)."""
    if rank != 0:
        return None
    import numpy as np
    from threadpoolctl import threadpool_limits
    import oracle

    seed = 1000 + args.workload
    inp = _with_append(make_inputs(args.workload, seed=seed, poison=False), seed)
    q, k, v = bf16_bits(inp.q), bf16_bits(inp.k_pages), bf16_bits(inp.v_pages)
    kn, vn = bf16_bits(inp.k_new), bf16_bits(inp.v_new)
    bt, sl, pos = inp.block_table.numpy(), inp.seq_lens.numpy(), inp.positions.numpy()
    B = inp.num_seqs

    def one_step(n):
        k2, v2 = oracle.kv_append(k, v, kn[:n], vn[:n], bt[:n], pos[:n])
        oracle.paged_decode_attention(q[:n], k2, v2, bt[:n], sl[:n], inp.scale)

    times, byts, seqs = [], [], []
    with threadpool_limits(1):
        t0 = time.perf_counter()
        one_step(1)
        t_one = time.perf_counter() - t0
        budget = max(0.5, min(4.0, 150.0 / max(1, args.steps + args.warmup)))
        est_all = t_one * float(sl.sum()) / max(1, int(sl[0]))
        n = B if est_all <= budget else max(1, int(B * budget / est_all))
        step_bytes = algorithmic_bytes(inp, with_append=True, num_seqs=n)["step"]
        for i in range(args.warmup + args.steps):
            t0 = time.perf_counter()
            one_step(n)
            dt = time.perf_counter() - t0
            if i >= args.warmup:
                times.append(dt)
                byts.append(step_bytes)
                seqs.append(n)
    total_t = sum(times)
    value = sum(byts) / total_t / 1e12
    sample = (f"each step: fp64 oracle kv_append + attention over the first {n} of {B} sequences "
              f"({int(sl[:n].sum())} context tokens), single thread")
    return {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TB/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * total_t / len(times), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "tokens_per_s": sum(seqs) / total_t,
        "config": {**_config_keys(inp, world), "l2": "host memory (CPU oracle)"},
        "cpu_baseline": {"value": value, "unit": "TB/s", "cores": 1, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": "TB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def _config_keys(inp, world):
    L = inp.seq_lens.to(torch.int64).cpu()
    return {"workload": inp.name, "num_seqs": inp.num_seqs, "num_heads": inp.num_heads,
            "num_kv_heads": inp.num_kv_heads, "head_dim": inp.head_dim, "page_size": inp.page_size,
            "num_pages": inp.num_pages, "context_tokens": int(L.sum()), "seq_len_min": int(L.min()),
            "seq_len_max": int(L.max()), "seed": 1000 + inp.meta.get("workload", 0),
            "step": "kv_append + paged_decode_attn",
            "parallelism": f"dp{world} (independent batch per GPU)" if world > 1 else "single GPU"}


def _with_append(inp, seed):
    """Give a workload without its own append step one new K/V token per sequence
    (positions = seq_len - 1, already counted in seq_lens)."""
    if inp.positions is None:
        g = torch.Generator().manual_seed(seed + 2)
        inp.positions = (inp.seq_lens - 1).clamp(min=0).to(torch.int32)
        inp.k_new = torch.randn(inp.num_seqs, inp.num_kv_heads, inp.head_dim, generator=g).to(torch.bfloat16)
        inp.v_new = torch.randn(inp.num_seqs, inp.num_kv_heads, inp.head_dim, generator=g).to(torch.bfloat16)
    return inp


def run_ours(args, rank, world, local):
    import gqa_decode_attention_04_b200 as gq

    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    seed = rank_seed(args.workload, rank)
    inp_cpu = _with_append(make_inputs(args.workload, seed=seed, poison=False), seed)
    nbytes = algorithmic_bytes(inp_cpu, with_append=True)

    # Rotate between independent copies of the pools so consecutive steps never
    # find their K/V in L2 (each copy alone is larger than L2 for the default workload).
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    kv_bytes = 2 * inp_cpu.k_pages.numel() * 2
    n_sets = max(2, math.ceil(4 * l2 / max(1, kv_bytes)))
    n_sets = min(n_sets, 8)
    base = inp_cpu.to(dev)
    sets = [base]
    for _ in range(n_sets - 1):
        s = inp_cpu.to(dev)
        s.k_pages = base.k_pages.clone()
        s.v_pages = base.v_pages.clone()
        sets.append(s)
    out = torch.empty((inp_cpu.num_seqs, inp_cpu.num_heads, inp_cpu.head_dim), dtype=torch.bfloat16, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step(s):
        # one call: kv_append, then the decode (its launch overlaps the append)
        gq.decode_step(s.q, s.k_new, s.v_new, s.k_pages, s.v_pages, s.block_table, s.positions,
                       s.seq_lens, out=out, scale=s.scale)

    def decode_only(s):
        gq.paged_decode_attn(s.q, s.k_pages, s.v_pages, s.block_table, s.seq_lens, out=out, scale=s.scale)

    for i in range(args.warmup):
        step(sets[i % n_sets])
    torch.cuda.synchronize()
    gq.check_device_error()

    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    launches0 = gq.launch_count()
    visible = [x for x in os.environ.get("CUDA_VISIBLE_DEVICES", "").split(",") if x.strip()]
    smi_index = visible[local] if local < len(visible) else str(local)
    with ClockSampler(smi_index) as clocks:
        barrier()
        torch.cuda.synchronize()
        start.record(stream)
        for i in range(args.steps):
            step(sets[i % n_sets])
        end.record(stream)
        torch.cuda.synchronize()
        barrier()
    launches = gq.launch_count() - launches0
    gq.check_device_error()
    step_ms_local = start.elapsed_time(end) / args.steps
    # The decode kernel alone (roofline figure): the same launches back to back, timed
    # with CUDA events on the launching stream; the average interval per launch.
    d0, d1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    for i in range(3):
        decode_only(sets[i % n_sets])
    torch.cuda.synchronize()
    d0.record(stream)
    for i in range(args.steps):
        decode_only(sets[i % n_sets])
    d1.record(stream)
    torch.cuda.synchronize()
    decode_ms_local = d0.elapsed_time(d1) / args.steps
    total_ms, total_bytes = reduce_max_sum(step_ms_local * args.steps, nbytes["step"] * args.steps, dev)
    _, total_seqs = reduce_max_sum(0.0, inp_cpu.num_seqs * args.steps, dev)
    step_ms = total_ms / args.steps
    value_tbps = total_bytes / (total_ms * 1e-3) / 1e12
    tokens_per_s = total_seqs / (total_ms * 1e-3)

    # ---- end to end through the public API: host inputs in, host result out
    pin = lambda t: t.pin_memory()  # noqa: E731
    host_in = [pin(inp_cpu.q), pin(inp_cpu.k_new), pin(inp_cpu.v_new), pin(inp_cpu.positions),
               pin(inp_cpu.seq_lens), pin(inp_cpu.block_table)]
    host_out = torch.empty(out.shape, dtype=out.dtype).pin_memory()
    h2d = sum(t.numel() * t.element_size() for t in host_in)
    d2h = host_out.numel() * host_out.element_size()

    def e2e_step(s):
        for src, dst in zip(host_in, (s.q, s.k_new, s.v_new, s.positions, s.seq_lens, s.block_table)):
            dst.copy_(src, non_blocking=True)
        step(s)
        host_out.copy_(out, non_blocking=True)
        stream.synchronize()

    for i in range(args.warmup):
        e2e_step(sets[i % n_sets])
    barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for i in range(args.steps):
        e2e_step(sets[i % n_sets])
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms, _ = reduce_max_sum(e0.elapsed_time(e1), 0.0, dev)
    e2e_tbps = total_bytes / (e2e_ms * 1e-3) / 1e12
    gq.check_device_error()

    peak, peak_kind = measured_peak()
    achieved_gbs = nbytes["decode"] / (decode_ms_local * 1e-3) / 1e9
    units = int(inp_cpu.seq_lens.to(torch.int64).sum())
    line = {
        "metric": METRIC,
        "value": value_tbps,
        "unit": "TB/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": step_ms,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic",
        "pct_of_peak": 100.0 * value_tbps * 1e3 / (peak * world),
        "tokens_per_s": tokens_per_s,
        "kv_tbps": nbytes["kv"] * args.steps * world / (total_ms * 1e-3) / 1e12,
        "config": {**_config_keys(inp_cpu, world),
                   "l2": f"inputs larger than L2: {n_sets} rotated pool copies of "
                         f"{kv_bytes / 1e6:.0f} MB each vs {l2 / 1e6:.0f} MB L2"},
        "e2e": {"value": e2e_tbps, "unit": "TB/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "ms_per_step": e2e_ms / args.steps},
        "gpu_launches": int(launches),
        "roofline": {"bound": "hbm", "kernel": decode_kernel_for(inp_cpu),
                     "achieved": achieved_gbs, "peak": peak, "unit": "GB/s",
                     "frac": achieved_gbs / peak, "peak_kind": f"{peak_kind} (hbm_gbs)",
                     "traffic": profiled_traffic(WORKLOADS[args.workload].name, decode_kernel_for(inp_cpu), units),
                     "algorithmic_bytes_per_launch": nbytes["decode"],
                     "decode_ms": decode_ms_local},
        "clocks": clocks.summary(),
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        bps, sps, desc = time_oracle(inp_cpu, min_seconds=10.0, max_seconds=30.0)
        line["cpu_baseline"] = {"value": bps / 1e12, "unit": "TB/s", "cores": 1, "kind": "oracle",
                                "sample": desc, "tokens_per_s": sps}
    return line


def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", type=int, default=2, choices=sorted(WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    if args.impl == "reference":
        # CPU arm: rank 0 alone times the oracle; other ranks exit without work.
        rank = int(os.environ.get("RANK", "0"))
        world = int(os.environ.get("WORLD_SIZE", str(args.gpus)))
        line = run_reference(args, rank, world)
        if line is not None:
            print(json.dumps(line), flush=True)
        return
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA GPU for --impl ours")
    rank, world, local = setup_dist(args.gpus)
    try:
        line = run_ours(args, rank, world, local)
        if rank == 0:
            print(json.dumps(line), flush=True)
    finally:
        if dist.is_initialized():
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
