#!/usr/bin/env python3
"""Benchmark of the decode step: kv_append + paged GQA decode attention on a B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload I] [--impl ours|reference]

One step = one pass of the whole hot path over one batch: kv_append writes each
sequence's new K/V token into its page, then paged_decode_attn attends over the
paged cache (split-KV with its log-sum-exp merge).  The headline workload (default
2) is the GQA serving batch (32 sequences, 32 query / 8 KV heads, head_dim 128,
page_size 16, lengths uniform in [512, 4096]).

Prints ONE JSON line on rank 0.  `value` is the step's algorithmic HBM bytes (all
K/V bytes of every context token, plus q, out, the appended rows, block table and
lengths) divided by the step time, in TB/s, summed over ranks; the step is the public
decode_step call, captured once per pool copy in a CUDA graph and replayed once per
step, as a serving loop issues it (`eager_*`: the same steps as direct calls).  Each rank runs its
own independent batch (weak scaling, no collective on the data path).  Inputs are
resident in HBM; the working set (at least two copies of the page pools, rotated
launch by launch) is several times the 126 MB L2.

On one GPU the line also carries `workloads`: every one of the five synthetic
workloads measured the same way -- its decode launch and its whole step, each
replayed from a CUDA graph of back-to-back launches (so host call overhead is not
what is measured), median over at least five replays and at least 0.2 s of GPU time,
against the measured HBM copy bandwidth.  With --fp8 (the default) each GQA workload
also reports the same decode over an e4m3 copy of its cache.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import math
import os
import platform
import statistics
import subprocess
import sys
import threading
import time

import torch
import torch.distributed as dist

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from workloads import WORKLOADS, make_inputs, make_shrunk_inputs, bf16_bits  # noqa: E402

METRIC = "paged GQA decode attn: achieved HBM TB/s (% of B200 peak), tokens/s"
FALLBACK_HBM_GBS = 6650.0
PROFILE_TRAFFIC = os.path.join(ROOT, "profiles", "traffic.json")
_CSRC = "gqa_decode_attention_04_b200/csrc/"
KERNEL_SOURCES = {
    "decode_ws_kernel": [_CSRC + "decode_ws.cu", _CSRC + "ptx.cuh", _CSRC + "internal.cuh"],
    "decode_tc_kernel": [_CSRC + "decode_tc.cu", _CSRC + "ptx.cuh", _CSRC + "internal.cuh"],
}
# Each timed loop: at least MIN_REPEATS replays of a graph of GRAPH_LAUNCHES calls, and at
# least MIN_LOOP_SECONDS of GPU time (short, so that a compute-heavy decode is timed at
# the clocks it starts with rather than after seconds under the power cap).
MIN_LOOP_SECONDS = 0.03
MIN_REPEATS = 7
GRAPH_LAUNCHES = 100


def decode_kernel_for(inp) -> str:
    """The decode kernel the library picks for this head grouping: the tcgen05 kernel
    for more than 16 query heads per kv head, the mma.sync kernel otherwise."""
    return "decode_tc_kernel" if inp.num_heads // inp.num_kv_heads > 16 else "decode_ws_kernel"


# ------------------------------------------------------------------ helpers

def algorithmic_bytes(inp, with_append: bool, num_seqs=None, kv_elem_bytes: int = 2) -> dict:
    """Bytes the step must move: every cached K/V byte once, q in, out back, plus
    the block-table entries and lengths read, and the appended rows.  With
    num_seqs, only the first num_seqs sequences count.  kv_elem_bytes = 1 for an
    8-bit cache (which also reads one K and one V scale per kv head)."""
    B = inp.num_seqs if num_seqs is None else num_seqs
    H, Hk, D, ps = inp.num_heads, inp.num_kv_heads, inp.head_dim, inp.page_size
    L = inp.seq_lens[:B].to(torch.int64).cpu()
    kv = int(L.sum()) * Hk * D * kv_elem_bytes * 2
    pages = int(((L + ps - 1) // ps).sum())
    qo = 2 * B * H * D * 2
    meta = pages * 4 + B * 4 + (2 * Hk * 4 if kv_elem_bytes == 1 else 0)
    decode = kv + qo + meta
    append = 0
    if with_append:
        # read the new bf16 rows, write them into their slots, positions and block-table entries
        append = B * Hk * D * 2 * 2 + B * Hk * D * kv_elem_bytes * 2 + B * 4 + B * 4
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


def cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as f:
            for ln in f:
                if ln.startswith("model name"):
                    return ln.split(":", 1)[1].strip()
    except OSError:
        pass
    return platform.processor() or "unknown"


class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons.  Samples are kept only if
    their own timestamp falls inside one of the timed windows recorded with window():
    the figures describe the GPU under load, not the set-up around it."""

    FIELDS = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    REASONS = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]

    def __init__(self, gpu_index: str, period_ms: int = 25):
        self.gpu_index = gpu_index
        self.period_ms = period_ms
        self.proc = None
        self.lines = []
        self.windows = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu_index), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", str(self.period_ms)],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self._reader = threading.Thread(target=self._read, daemon=True)
            self._reader.start()
        except Exception:
            self.proc = None
        return self

    def _read(self):
        for ln in self.proc.stdout:
            if ln.strip():
                self.lines.append(ln)

    def window(self):
        """Context manager marking one timed region (host wall clock, with the GPU busy)."""
        sampler = self

        class _W:
            def __enter__(self):
                self.t0 = time.time()

            def __exit__(self, *exc):
                sampler.windows.append((self.t0, time.time()))
                return False
        return _W()

    def __exit__(self, *exc):
        if self.proc is not None:
            time.sleep(2.5 * self.period_ms / 1000.0)  # the last window's final sample
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
            self._reader.join(timeout=5)
        return False

    @staticmethod
    def _stamp(s: str):
        for fmt in ("%Y/%m/%d %H:%M:%S.%f", "%Y/%m/%d %H:%M:%S"):
            try:
                return datetime.datetime.strptime(s.strip(), fmt).timestamp()
            except ValueError:
                continue
        return None

    def summary(self, windows=None):
        """Median SM clock and throttle reasons over the samples inside `windows` (all
        timed windows by default)."""
        windows = self.windows if windows is None else windows
        sm, mx, reasons, n_all = [], None, set(), 0
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 10:
                continue
            n_all += 1
            t = self._stamp(parts[0])
            if t is None or not any(a <= t <= b for a, b in windows):
                continue
            try:
                sm.append(float(parts[2]))
                mx = float(parts[3])
            except ValueError:
                continue
            for n, v in zip(self.REASONS, parts[6:10]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "samples": 0,
                    "samples_total": n_all}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm), "samples_total": n_all, "period_ms": self.period_ms,
                "timed_windows_s": round(sum(b - a for a, b in windows), 3)}


def setup_dist(n_gpus: int):
    if n_gpus > 1 or "RANK" in os.environ:
        rank = int(os.environ.get("RANK", "0"))
        world = int(os.environ.get("WORLD_SIZE", "1"))
        local = int(os.environ.get("LOCAL_RANK", "0"))
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if torch.cuda.is_available():
            torch.cuda.set_device(local)
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

ONE_CORE_REASON = ("the oracle is timed as it stands: plain per-(sequence, head) loops over numpy "
                   "vector operations, which one Python thread drives; BLAS threads would not "
                   "parallelise them, and splitting the batch over processes would be a tuned "
                   "variant of the oracle, not the oracle")


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


def _cpu_fields():
    return {"cpu_model": cpu_model(), "host_cores_available": os.cpu_count(),
            "why_one_core": ONE_CORE_REASON}


# ------------------------------------------------------------------ arms

def run_reference(args, rank, world):
    """Reference arm: the fp64 CPU oracle on the host, rank 0 only.  Each step is a
    bounded sample of the workload: the oracle's kv_append, then its attention over a
    prefix of the sequences (all of them when that fits the time budget)."""
    if rank != 0:
        return None
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
        "cpu_baseline": {"value": value, "unit": "TB/s", "cores": 1, "kind": "oracle", "sample": sample,
                         **_cpu_fields()},
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
        dev = inp.q.device
        inp.positions = (inp.seq_lens - 1).clamp(min=0).to(torch.int32)
        inp.k_new = torch.randn(inp.num_seqs, inp.num_kv_heads, inp.head_dim, generator=g).to(torch.bfloat16).to(dev)
        inp.v_new = torch.randn(inp.num_seqs, inp.num_kv_heads, inp.head_dim, generator=g).to(torch.bfloat16).to(dev)
    return inp


def _pool_sets(inp_dev, dev):
    """The batch plus enough further copies of its page pools that the launches, rotating
    over them, never find their K/V in L2: at least 2 copies and 4x L2 in total (<= 8)."""
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    kv_bytes = 2 * inp_dev.k_pages.numel() * inp_dev.k_pages.element_size()
    n_sets = min(8, max(2, math.ceil(4 * l2 / max(1, kv_bytes))))
    sets = [inp_dev]
    for _ in range(n_sets - 1):
        s = inp_dev.to(dev)
        s.k_pages = inp_dev.k_pages.clone()
        s.v_pages = inp_dev.v_pages.clone()
        sets.append(s)
    desc = (f"inputs larger than L2: {n_sets} rotated pool copies of {kv_bytes / 1e6:.1f} MB each "
            f"vs {l2 / 1e6:.0f} MB L2" if kv_bytes * 2 > l2 else
            f"{n_sets} rotated pool copies of {kv_bytes / 1e3:.1f} KB each (the batch fits in L2)")
    return sets, desc


def graph_time_us(enqueue, n_calls: int, stream, clocks=None):
    """Device time of one call: n_calls back-to-back calls captured once in a CUDA graph,
    the graph replayed at least MIN_REPEATS times and MIN_LOOP_SECONDS, CUDA events on
    the launching stream around each replay.  Returns (median, min, max) in us."""
    for i in range(3):  # first calls set up the workspace, tensor maps and attributes
        enqueue(i)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    cap = torch.cuda.Stream()
    with torch.cuda.graph(g, stream=cap):
        for i in range(n_calls):
            enqueue(i)
    g.replay()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    g.replay()
    e1.record(stream)
    torch.cuda.synchronize()
    one = max(1e-3, e0.elapsed_time(e1) / 1e3)
    reps = max(MIN_REPEATS, math.ceil(MIN_LOOP_SECONDS / one))
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(reps)]
    win = clocks.window() if clocks is not None else None
    if win is not None:
        win.__enter__()
    for a, b in evs:
        a.record(stream)
        g.replay()
        b.record(stream)
    torch.cuda.synchronize()
    if win is not None:
        win.__exit__(None, None, None)
    per = sorted(a.elapsed_time(b) * 1e3 / n_calls for a, b in evs)
    del g
    return statistics.median(per), per[0], per[-1]


def measure_workload(gq, inp_dev, dev, peak, clocks, fp8: bool):
    """One entry of the `workloads` object: the decode launch and the whole step of this
    batch, each from a CUDA graph of back-to-back calls (see graph_time_us)."""
    stream = torch.cuda.current_stream(dev)
    sets, l2_desc = _pool_sets(inp_dev, dev)
    n = len(sets)
    B, H, D = inp_dev.num_seqs, inp_dev.num_heads, inp_dev.head_dim
    w0 = len(clocks.windows) if clocks is not None else 0
    out = torch.empty((B, H, D), dtype=torch.bfloat16, device=dev)
    nb = algorithmic_bytes(inp_dev, with_append=True)

    def decode(i):
        s = sets[i % n]
        gq.paged_decode_attn(s.q, s.k_pages, s.v_pages, s.block_table, s.seq_lens, out=out, scale=s.scale)

    def step(i):
        s = sets[i % n]
        gq.decode_step(s.q, s.k_new, s.v_new, s.k_pages, s.v_pages, s.block_table, s.positions,
                       s.seq_lens, out=out, scale=s.scale)

    d_med, d_min, d_max = graph_time_us(decode, GRAPH_LAUNCHES, stream, clocks)
    s_med, s_min, s_max = graph_time_us(step, GRAPH_LAUNCHES, stream, clocks)
    gq.check_device_error()
    achieved = nb["decode"] / (d_med * 1e-6) / 1e9
    kernel = decode_kernel_for(inp_dev)
    units = int(inp_dev.seq_lens.to(torch.int64).sum())
    entry = {
        "workload": inp_dev.name, "num_seqs": B, "num_heads": H, "num_kv_heads": inp_dev.num_kv_heads,
        "head_dim": D, "page_size": inp_dev.page_size,
        "context_tokens": int(inp_dev.seq_lens.to(torch.int64).sum()),
        "decode_kernel": kernel + (" + merge_tc_kernel" if kernel == "decode_tc_kernel" else ""),
        "decode_us": d_med, "decode_us_min_max": [d_min, d_max],
        "step_us": s_med, "step_us_min_max": [s_min, s_max],
        "algorithmic_bytes_per_decode": nb["decode"], "kv_bytes": nb["kv"],
        "achieved_gbs": achieved, "frac": achieved / peak,
        "kv_tbps": nb["kv"] / (d_med * 1e-6) / 1e12,
        "step_tbps": nb["step"] / (s_med * 1e-6) / 1e12,
        "tokens_per_s": B / (s_med * 1e-6),
        "traffic": profiled_traffic(inp_dev.name, kernel, units),
        "l2": l2_desc, "graph_launches": GRAPH_LAUNCHES,
        "clocks": clocks.summary(clocks.windows[w0:]) if clocks is not None else None,
    }
    if fp8:
        try:
            entry["fp8"] = measure_fp8(gq, sets, dev, peak, clocks)
            entry["fp8"]["traffic"] = profiled_traffic(inp_dev.name + "_fp8", kernel, units)
        except gq.GQAError as e:  # a shape the 8-bit path does not serve
            entry["fp8"] = {"unavailable": str(e)}
    del sets, out
    return entry


def measure_fp8(gq, sets, dev, peak, clocks):
    """The same decode over an e4m3 copy of each pool set (one scale per kv head for K
    and one for V, from the largest magnitude in the pool), and its step with the
    quantising append."""
    stream = torch.cuda.current_stream(dev)
    s0 = sets[0]
    Hk = s0.num_kv_heads
    ks = (s0.k_pages.float().abs().amax(dim=(0, 2, 3)) / 448.0).clamp(min=1e-30).contiguous()
    vs = (s0.v_pages.float().abs().amax(dim=(0, 2, 3)) / 448.0).clamp(min=1e-30).contiguous()
    pools = []
    for s in sets:
        kq = torch.empty(s.k_pages.shape, dtype=torch.uint8, device=dev)
        vq = torch.empty(s.v_pages.shape, dtype=torch.uint8, device=dev)
        gq.quantize_pages_fp8(s.k_pages, kq, ks)
        gq.quantize_pages_fp8(s.v_pages, vq, vs)
        pools.append((kq, vq))
    n = len(sets)
    B, H, D = s0.num_seqs, s0.num_heads, s0.head_dim
    out = torch.empty((B, H, D), dtype=torch.bfloat16, device=dev)
    nb = algorithmic_bytes(s0, with_append=True, kv_elem_bytes=1)

    def decode(i):
        s, (kq, vq) = sets[i % n], pools[i % n]
        gq.paged_decode_attn_fp8(s.q, kq, vq, ks, vs, s.block_table, s.seq_lens, out=out, scale=s.scale)

    def step(i):
        s, (kq, vq) = sets[i % n], pools[i % n]
        gq.decode_step_fp8(s.q, s.k_new, s.v_new, kq, vq, ks, vs, s.block_table, s.positions, s.seq_lens,
                           out=out, scale=s.scale)

    d_med, d_min, d_max = graph_time_us(decode, GRAPH_LAUNCHES, stream, clocks)
    s_med, _, _ = graph_time_us(step, GRAPH_LAUNCHES, stream, clocks)
    gq.check_device_error()
    achieved = nb["decode"] / (d_med * 1e-6) / 1e9
    del pools
    return {"decode_us": d_med, "decode_us_min_max": [d_min, d_max], "step_us": s_med,
            "algorithmic_bytes_per_decode": nb["decode"], "kv_bytes": nb["kv"],
            "achieved_gbs": achieved, "frac": achieved / peak,
            "kv_tbps": nb["kv"] / (d_med * 1e-6) / 1e12, "tokens_per_s": B / (s_med * 1e-6),
            "scales": "one fp32 scale per kv head for K and for V: max |x| / 448 over the pool"}


class PackedInputs:
    """The step's per-call inputs (q, k_new, v_new, positions, seq_lens, block table) in
    one pinned host buffer and one device buffer at 256-byte aligned offsets, so a step
    moves them with a single host-to-device copy; the device tensors are views."""

    def __init__(self, inp_cpu, dev):
        srcs = [inp_cpu.q, inp_cpu.k_new, inp_cpu.v_new, inp_cpu.positions, inp_cpu.seq_lens,
                inp_cpu.block_table]
        offs, off = [], 0
        for t in srcs:
            offs.append(off)
            off += (t.numel() * t.element_size() + 255) // 256 * 256
        self.nbytes = off
        self.host = torch.empty(off, dtype=torch.uint8).pin_memory()
        self.dev = torch.empty(off, dtype=torch.uint8, device=dev)
        self.views = []
        for t, o in zip(srcs, offs):
            nb = t.numel() * t.element_size()
            self.host[o:o + nb].copy_(t.contiguous().view(-1).view(torch.uint8))
            self.views.append(self.dev[o:o + nb].view(t.dtype).view(t.shape))
        self.payload = sum(t.numel() * t.element_size() for t in srcs)

    def upload(self):
        self.dev.copy_(self.host, non_blocking=True)


def e2e_pipelined(gq, args, sets, inp_cpu, dev, stream, out_shape) -> float:
    """End-to-end steps as a serving loop runs them: two sets of packed input and output
    buffers, uploads on one stream, decode_step on the compute stream, downloads on a
    third, each captured once as a CUDA graph; events order the reuse of every buffer.
    Returns the max over ranks of the device time from the first upload to the last
    download, over exactly args.steps steps (after args.warmup untimed ones)."""
    n_sets = len(sets)
    up_s, dn_s = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    packs = [PackedInputs(inp_cpu, dev) for _ in range(2)]
    outs = [torch.empty(out_shape, dtype=torch.bfloat16, device=dev) for _ in range(2)]
    host_outs = [torch.empty(out_shape, dtype=torch.bfloat16).pin_memory() for _ in range(2)]
    cap = torch.cuda.Stream(dev)
    g_up, g_dn, g_step = [], [], {}
    for k in range(2):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=cap):
            packs[k].upload()
        g_up.append(g)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=cap):
            host_outs[k].copy_(outs[k], non_blocking=True)
        g_dn.append(g)
        for j, st in enumerate(sets):
            q, kn, vn, pos, sl, bt = packs[k].views
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=cap):
                gq.decode_step(q, kn, vn, st.k_pages, st.v_pages, bt, pos, sl, out=outs[k], scale=st.scale)
            g_step[(k, j)] = g
    torch.cuda.synchronize()
    ev = lambda: torch.cuda.Event()
    e_up, e_done, e_dl = ([ev() for _ in range(2)] for _ in range(3))
    issued = [False, False]

    def run(i):
        k = i % 2
        if issued[k]:
            up_s.wait_event(e_done[k])       # step i-2 has read these inputs
            stream.wait_event(e_dl[k])       # and its output is downloaded
        with torch.cuda.stream(up_s):
            g_up[k].replay()
            e_up[k].record(up_s)
        stream.wait_event(e_up[k])
        g_step[(k, i % n_sets)].replay()
        e_done[k].record(stream)
        dn_s.wait_event(e_done[k])
        with torch.cuda.stream(dn_s):
            g_dn[k].replay()
            e_dl[k].record(dn_s)
        issued[k] = True
        if i >= 1:
            e_dl[(i - 1) % 2].synchronize()  # the host has step i-1's result

    for i in range(args.warmup):
        run(i)
    torch.cuda.synchronize()
    barrier()
    torch.cuda.synchronize()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    up_s.wait_event(t0)
    for i in range(args.steps):
        run(args.warmup + i)
    stream.wait_event(e_dl[(args.warmup + args.steps - 1) % 2])
    t1.record(stream)
    torch.cuda.synchronize()
    ms, _ = reduce_max_sum(t0.elapsed_time(t1), 0.0, dev)
    del g_up, g_dn, g_step
    return ms


def run_ours(args, rank, world, local):
    import gqa_decode_attention_04_b200 as gq

    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream(dev)
    peak, peak_kind = measured_peak()
    seed = rank_seed(args.workload, rank)
    inp_cpu = _with_append(make_inputs(args.workload, seed=seed, poison=False), seed)
    nbytes = algorithmic_bytes(inp_cpu, with_append=True)
    sets, l2_desc = _pool_sets(inp_cpu.to(dev), dev)
    n_sets = len(sets)
    out = torch.empty((inp_cpu.num_seqs, inp_cpu.num_heads, inp_cpu.head_dim), dtype=torch.bfloat16, device=dev)

    def step(s, ins=None):
        # one call: kv_append, then the decode (its launch overlaps the append)
        q, kn, vn, pos, sl, bt = ins if ins is not None else (s.q, s.k_new, s.v_new, s.positions, s.seq_lens,
                                                               s.block_table)
        gq.decode_step(q, kn, vn, s.k_pages, s.v_pages, bt, pos, sl, out=out, scale=s.scale)

    for i in range(args.warmup):
        step(sets[i % n_sets])
    torch.cuda.synchronize()
    gq.check_device_error()

    visible = [x for x in os.environ.get("CUDA_VISIBLE_DEVICES", "").split(",") if x.strip()]
    smi_index = visible[local] if local < len(visible) else str(local)
    workloads = {}
    # The step as a serving loop issues it: the public decode_step call captured once per
    # pool copy in a CUDA graph, one replay per step (the library's launches per step
    # counted at capture).
    step_graphs = []
    cap_stream = torch.cuda.Stream(dev)
    lc0 = gq.launch_count()
    for s in sets:
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=cap_stream):
            step(s)
        step_graphs.append(g)
    launches_per_step = (gq.launch_count() - lc0) // n_sets
    for i in range(args.warmup):
        step_graphs[i % n_sets].replay()
    torch.cuda.synchronize()
    gq.check_device_error()

    with ClockSampler(smi_index) as clocks:
        # ---- headline: exactly K steps through the public API, device-timed
        start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        barrier()
        torch.cuda.synchronize()
        with clocks.window():
            start.record(stream)
            for i in range(args.steps):
                step_graphs[i % n_sets].replay()
            end.record(stream)
            torch.cuda.synchronize()
        barrier()
        launches = launches_per_step * args.steps
        gq.check_device_error()
        step_ms_local = start.elapsed_time(end) / args.steps
        # the same K steps as direct calls (host call overhead included)
        launches0 = gq.launch_count()
        barrier()
        torch.cuda.synchronize()
        with clocks.window():
            start.record(stream)
            for i in range(args.steps):
                step(sets[i % n_sets])
            end.record(stream)
            torch.cuda.synchronize()
        barrier()
        eager_launches = gq.launch_count() - launches0
        gq.check_device_error()
        step_eager_ms, _ = reduce_max_sum(start.elapsed_time(end), 0.0, dev)
        del step_graphs
        total_ms, total_bytes = reduce_max_sum(step_ms_local * args.steps, nbytes["step"] * args.steps, dev)
        _, total_seqs = reduce_max_sum(0.0, inp_cpu.num_seqs * args.steps, dev)

        # ---- the decode kernel alone (roofline) and every workload (one GPU)
        if world == 1 and not args.headline_only:
            for idx in sorted(WORKLOADS):
                if idx == args.workload:
                    entry = measure_workload(gq, sets[0], dev, peak, clocks, fp8=not args.no_fp8)
                else:
                    wl = _with_append(make_inputs(idx, seed=1000 + idx, device=dev, poison=False), 1000 + idx)
                    entry = measure_workload(gq, wl, dev, peak, clocks, fp8=not args.no_fp8)
                    del wl
                    torch.cuda.empty_cache()
                workloads[str(idx)] = entry
            head = workloads[str(args.workload)]
        else:
            head = measure_workload(gq, sets[0], dev, peak, clocks, fp8=False)
    decode_us = head["decode_us"]

    step_ms = total_ms / args.steps
    value_tbps = total_bytes / (total_ms * 1e-3) / 1e12
    tokens_per_s = total_seqs / (total_ms * 1e-3)

    # ---- end to end through the public API: host inputs in (one packed copy), host result out
    packed = PackedInputs(inp_cpu, dev)
    host_out = torch.empty(out.shape, dtype=out.dtype).pin_memory()
    d2h = host_out.numel() * host_out.element_size()

    def e2e_eager(s):
        packed.upload()
        step(s, packed.views)
        host_out.copy_(out, non_blocking=True)
        stream.synchronize()

    # The same step as a serving loop runs it: the upload, the public decode_step call and
    # the download captured once in a CUDA graph per pool copy, then one replay and one
    # synchronisation per step (host inputs refreshed in the pinned buffer in between).
    graphs = []
    cap = torch.cuda.Stream(dev)
    for s in sets:
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=cap):
            packed.upload()
            step(s, packed.views)
            host_out.copy_(out, non_blocking=True)
        graphs.append(g)

    def e2e_graph(i):
        graphs[i % n_sets].replay()
        stream.synchronize()

    def timed(fn, arg_of):
        for i in range(args.warmup):
            fn(arg_of(i))
        barrier()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for i in range(args.steps):
            fn(arg_of(i))
        e1.record(stream)
        torch.cuda.synchronize()
        ms, _ = reduce_max_sum(e0.elapsed_time(e1), 0.0, dev)
        return ms

    serial_ms = timed(e2e_graph, lambda i: i)
    eager_ms = timed(e2e_eager, lambda i: sets[i % n_sets])
    gq.check_device_error()
    del graphs
    pipe_ms = e2e_pipelined(gq, args, sets, inp_cpu, dev, stream, out.shape)
    e2e_ms = pipe_ms
    e2e_tbps = total_bytes / (e2e_ms * 1e-3) / 1e12
    gq.check_device_error()

    achieved_gbs = nbytes["decode"] / (decode_us * 1e-6) / 1e9
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
        "config": {**_config_keys(inp_cpu, world), "l2": l2_desc},
        "e2e": {"value": e2e_tbps, "unit": "TB/s", "h2d_bytes_per_step": packed.payload,
                "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms / args.steps,
                "copies_per_step": "1 host-to-device (packed inputs) + 1 device-to-host (out)",
                "how": "serving loop, double-buffered: every step uploads its packed inputs on an "
                       "upload stream, runs decode_step on the compute stream and downloads out on a "
                       "download stream (each part a CUDA graph, events between them), so step i+1's "
                       "upload and step i-1's download overlap step i; the host waits for step i-1's "
                       "result on the host after issuing step i; timed from the first upload to the "
                       "last download",
                "serial_ms_per_step": serial_ms / args.steps,
                "serial_value": total_bytes / (serial_ms * 1e-3) / 1e12,
                "serial_how": "upload, decode_step and download in one CUDA graph; one replay and one "
                              "stream synchronisation per step",
                "eager_ms_per_step": eager_ms / args.steps,
                "eager_value": total_bytes / (eager_ms * 1e-3) / 1e12},
        "gpu_launches": int(launches),
        "timing": "the public decode_step call captured once per pool copy in a CUDA graph, one replay "
                  "per step, CUDA events on the launching stream; eager_*: the same steps as direct calls",
        "eager_ms_per_step": step_eager_ms / args.steps,
        "eager_value": total_bytes / (step_eager_ms * 1e-3) / 1e12,
        "eager_gpu_launches": int(eager_launches),
        "roofline": {"bound": "hbm", "kernel": decode_kernel_for(inp_cpu),
                     "achieved": achieved_gbs, "peak": peak, "unit": "GB/s",
                     "frac": achieved_gbs / peak, "peak_kind": f"{peak_kind} (hbm_gbs, burst copy)",
                     "traffic": profiled_traffic(WORKLOADS[args.workload].name, decode_kernel_for(inp_cpu), units),
                     "algorithmic_bytes_per_launch": nbytes["decode"],
                     "decode_us": decode_us, "decode_us_min_max": head["decode_us_min_max"],
                     "timing": f"CUDA graph of {GRAPH_LAUNCHES} back-to-back decode launches, median over "
                               f">= {MIN_REPEATS} replays and >= {MIN_LOOP_SECONDS} s"},
        "clocks": clocks.summary(),
    }
    if workloads:
        line["workloads"] = workloads
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        bps, sps, desc = time_oracle(inp_cpu, min_seconds=10.0, max_seconds=30.0)
        line["cpu_baseline"] = {"value": bps / 1e12, "unit": "TB/s", "cores": 1, "kind": "oracle",
                                "sample": desc, "tokens_per_s": sps, **_cpu_fields()}
    return line


def run_profile(args):
    """Only --warmup + --steps decode launches of the workload (bf16 or e4m3 cache) on two
    rotated pool copies: the small, self-contained case ncu captures are taken of.
    Prints no JSON line."""
    import gqa_decode_attention_04_b200 as gq
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    if args.profile_shrink > 1:  # the same kernel on a smaller case (context lengths / N)
        inp = make_shrunk_inputs(args.workload, args.profile_shrink, seed=1000 + args.workload, device=dev,
                                 poison=False)
    else:
        inp = make_inputs(args.workload, seed=1000 + args.workload, device=dev, poison=False)
    print(f"context tokens per launch: {int(inp.seq_lens.to(torch.int64).sum())}", flush=True)
    sets, _ = _pool_sets(inp, dev)
    sets = sets[:2]
    out = torch.empty((inp.num_seqs, inp.num_heads, inp.head_dim), dtype=torch.bfloat16, device=dev)
    if args.profile == "fp8":
        ks = (inp.k_pages.float().abs().amax(dim=(0, 2, 3)) / 448.0).clamp(min=1e-30).contiguous()
        vs = (inp.v_pages.float().abs().amax(dim=(0, 2, 3)) / 448.0).clamp(min=1e-30).contiguous()
        pools = []
        for st in sets:
            kq = torch.empty(st.k_pages.shape, dtype=torch.uint8, device=dev)
            vq = torch.empty(st.v_pages.shape, dtype=torch.uint8, device=dev)
            gq.quantize_pages_fp8(st.k_pages, kq, ks)
            gq.quantize_pages_fp8(st.v_pages, vq, vs)
            pools.append((kq, vq))
        del sets[1:]
        st = sets[0]
        for i in range(args.warmup + args.steps):
            kq, vq = pools[i % 2]
            gq.paged_decode_attn_fp8(st.q, kq, vq, ks, vs, st.block_table, st.seq_lens, out=out, scale=st.scale)
    else:
        for i in range(args.warmup + args.steps):
            st = sets[i % 2]
            gq.paged_decode_attn(st.q, st.k_pages, st.v_pages, st.block_table, st.seq_lens, out=out, scale=st.scale)
    torch.cuda.synchronize()
    gq.check_device_error()


def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", type=int, default=2, choices=sorted(WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-fp8", action="store_true", help="skip the 8-bit cache entries")
    ap.add_argument("--headline-only", action="store_true", help="skip the other workloads")
    ap.add_argument("--profile", choices=["bf16", "fp8"],
                    help="only run --warmup + --steps decode launches of --workload (ncu captures)")
    ap.add_argument("--profile-shrink", type=int, default=1,
                    help="with --profile: divide every context length by N (a smaller case of the same kernel)")
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
    if args.profile:
        run_profile(args)
        return
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
