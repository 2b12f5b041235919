"""Benchmark of the DSA hot path on B200.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One step = one dsa_prefill of the 128K workload (L = 131072, index dim 160 in
BF16, H = 16, D = 128, top_k = 2048): indexer sample + threshold + causal
indexer with fused filter + exact select + gathered attention.  `value` is
whole-job prefill queries/s (each rank runs its own sequence: weak scaling,
no data-path collective).  The decode rows of the path (64 sequences with
cached lengths in [65536, 131072], top_k 2048) are timed in their own K-step
loop and reported under "decode", and again from a block-paged copy of the
same cache (dsa_decode_paged, 64-row blocks) under "decode.paged".  Inputs
are synthetic and seeded; each step's working set (~9 GB) is far larger than
the 126 MB L2.

--impl reference times the CPU oracle (the plain restatement the tests check
against) on a bounded sample of query rows per step, on the host's cores.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

METRIC = "DSA prefill queries/s @128K (indexer TFLOP/s, gather GB/s); decode tok/s"
PREFILL = "prefill_128k"
DECODE = "decode_64x128k"


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-configs", action="store_true", help="skip the 4K/32K/64K prefill sub-lines")
    ap.add_argument("--no-zigzag", action="store_true", help="skip the row-split (strong scaling) sub-line")
    ap.add_argument("--no-fp8-path", action="store_true", help="skip the FP8 copy of BF16 index inputs")
    ap.add_argument("--cpu-seconds", type=float, default=15.0, help="target CPU-baseline sample time")
    ap.add_argument("--workload", default=PREFILL,
                    choices=["prefill_4k", "prefill_32k", "prefill_64k", "prefill_128k", "prefill_32k_bf16"],
                    help="prefill workload of a step (smaller ones for profiling)")
    ap.add_argument("--decode-batch", type=int, default=0,
                    help="decode only the first B sequences of the batch (profiling)")
    return ap.parse_args()


def rank_info():
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
            int(os.environ.get("LOCAL_RANK", "0")))


def peaks():
    p = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            m = json.load(f)
        p.update({k: float(m[k]) for k in ("hbm_gbs", "bf16_tflops", "bf16_tflops_sustained") if k in m})
        p["source"] = "measured"
    except (OSError, ValueError, KeyError):
        pass
    return p


def measured_peaks_in_run(dev) -> dict:
    """Tensor peaks measured in this run (CUDA events, best of 10): FP8 E4M3 with
    torch._scaled_mm and BF16 with torch.matmul, both 8192^3 (2 N^3 FLOP), as a
    burst on an idle GPU.  The FP8 figure is the denominator for the FP8
    indexer; MEASURED_PEAKS.json holds no FP8 number."""
    import torch
    n = 8192
    out = {}
    a = torch.randn(n, n, device=dev).to(torch.float8_e4m3fn)
    b = torch.randn(n, n, device=dev).to(torch.float8_e4m3fn).t()
    one = torch.ones((), device=dev)
    ab = torch.randn(n, n, device=dev, dtype=torch.bfloat16)
    bb = torch.randn(n, n, device=dev, dtype=torch.bfloat16)
    for name, fn in (("fp8_tflops", lambda: torch._scaled_mm(a, b, scale_a=one, scale_b=one,
                                                              out_dtype=torch.bfloat16)),
                     ("bf16_tflops", lambda: torch.matmul(ab, bb))):
        for _ in range(3):
            fn()
        best = float("inf")
        for _ in range(10):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            fn()
            e1.record()
            e1.synchronize()
            best = min(best, e0.elapsed_time(e1))
        out[name] = 2.0 * n ** 3 / (best / 1000.0) / 1e12
    del a, b, ab, bb
    torch.cuda.empty_cache()
    out["how"] = "torch._scaled_mm FP8 E4M3 and torch.matmul BF16, 8192^3, best of 10 (burst)"
    return out


def gather_ceiling(dsa, idx, K, V, gather_bytes, stream) -> dict:
    """Rate of dsa_gather_probe over the prefill's own indices: the attention's
    exact K/V row reads into shared memory and nothing else, best of a few
    launch shapes (CTAs per SM x 16 KB stages) and three launches each."""
    import torch
    best, shape = float("inf"), None
    sink = torch.zeros(1, dtype=torch.int64, device=idx.device)
    for cps, st in ((2, 3), (4, 3), (5, 2), (6, 2), (7, 2)):
        dsa.dsa_gather_probe(idx, K, V, cps, st, sink=sink, stream=stream)
        for _ in range(3):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            dsa.dsa_gather_probe(idx, K, V, cps, st, sink=sink, stream=stream)
            e1.record(stream)
            e1.synchronize()
            ms = e0.elapsed_time(e1)
            if ms < best:
                best, shape = ms, f"{cps} CTAs/SM x {st} stages of 16 KB"
    return {"gbs": gather_bytes / (best / 1000.0) / 1e9, "ms": best, "shape": shape,
            "how": "dsa_gather_probe: the attention's K and V rows (this step's indices) copied into "
                   "shared memory with 16-byte cp.async and nothing else; best launch shape"}


def reduce_max(x: float, world: int, device) -> float:
    """Max of a per-rank float over all ranks (identity when world == 1)."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def source_sha256(rel_path: str) -> str:
    import hashlib
    with open(os.path.join(ROOT, rel_path), "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()


def profiled_traffic(kernel: str, workload: str, source: str):
    """DRAM bytes per launch from profiles/<kernel>_<workload>.md, or None when the
    summary is missing or the kernel source changed since the counters were taken."""
    path = os.path.join(ROOT, "profiles", f"{kernel}_{workload}.md")
    try:
        fields = {}
        for line in open(path):
            if line.startswith("- ") and ":" in line:
                k, v = line[2:].split(":", 1)
                fields[k.strip()] = v.strip().strip("`")
        if fields.get("source_sha256") != source_sha256(source):
            return None
        return float(fields["dram_bytes_per_launch"])
    except (OSError, KeyError, ValueError):
        return None


# ----------------------------------------------------------------------------- clocks

class ClockSampler:
    """Samples SM clock and throttle reasons of one GPU every 100 ms (NVML)."""

    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown"}

    def __init__(self, device_index: int):
        self.samples, self.reasons, self.max_mhz = [], set(), None
        self._stop = threading.Event()
        self._h = None
        try:
            import pynvml
            pynvml.nvmlInit()
            import torch
            uuid = str(torch.cuda.get_device_properties(device_index).uuid)
            try:
                self._h = pynvml.nvmlDeviceGetHandleByUUID(("GPU-" + uuid).encode())
            except Exception:
                self._h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self._nv = pynvml
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
        except Exception:
            self._h = None
        self._t = threading.Thread(target=self._run, daemon=True)

    def _run(self):
        while not self._stop.is_set():
            try:
                self.samples.append(self._nv.nvmlDeviceGetClockInfo(self._h, self._nv.NVML_CLOCK_SM))
                r = self._nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
                for bit, name in self.REASONS.items():
                    if r & bit:
                        self.reasons.add(name)
            except Exception:
                pass
            self._stop.wait(0.1)

    def __enter__(self):
        if self._h is not None:
            self._t.start()
        return self

    def __exit__(self, *exc):
        self._stop.set()
        if self._h is not None:
            self._t.join()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons),
                    "samples": 0}
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


# ----------------------------------------------------------------------------- work accounting

def prefill_work(w):
    L, k, d, D, H = w.L, w.top_k, w.d_idx, w.D, w.H
    pairs = L * (L + 1) // 2                      # causal pairs, diagonal included
    kept = sum(min(t + 1, k) for t in range(min(L, k))) + max(0, L - k) * k
    return {
        "indexer_flops": 2.0 * d * pairs,
        "gather_bytes": float(kept) * 2 * D * 2,  # one K row + one V row per kept key
        "attn_flops": 4.0 * H * D * kept,
        "attn_bytes": float(kept) * 2 * D * 2 + 2.0 * L * H * D * 2 + 4.0 * L * k,
        "kept": kept,
    }


def decode_work(w, lengths):
    total = int(lengths.sum())
    kept = int(np.minimum(lengths, w.top_k).sum())
    esize = 1 if w.idx_dtype == "fp8" else 2
    return {
        "scan_bytes": float(total) * w.d_idx * esize + total * 4.0,   # read index rows, write scores
        "gather_bytes": float(kept) * 2 * w.D * 2,
        "total_rows": total,
    }


def line_config(w, world: int) -> dict:
    return {"workload": workload_desc(w), "parallelism": f"{world} independent sequences (one per GPU)",
            "l2": "inputs larger than L2 (~9 GB touched per step vs 126 MB L2)"}


def workload_desc(w) -> str:
    return (f"{w.name}: L={w.L} causal, q_idx/k_idx [L,{w.d_idx}] {w.idx_dtype} ints in [-4,4]"
            f"{' with local boost' if w.local_boost else ''}, Q [L,{w.H},{w.D}], K/V [L,{w.D}] bf16 N(0,1), "
            f"top_k={w.top_k}")


def time_prefill_config(dsa, synth, name, steps, warmup, dev, stream, seed, fp8_peak, bf16_peak, max_over_ranks):
    """One prefill workload timed on its own: whole-call time (CUDA events over `steps`
    calls after `warmup`), per-stage times from a second pass, indexer TFLOP/s against the
    peak of its input dtype."""
    import torch
    w = synth.WORKLOADS[name]
    x = synth.prefill_inputs_torch(w, seed=seed, device=dev)
    idt = dsa.IDX_BF16 if w.idx_dtype == "bf16" else dsa.IDX_FP8_E4M3
    ws = torch.empty(dsa.dsa_prefill_workspace_size(w.L, w.d_idx, idt, w.H, w.D, w.top_k),
                     dtype=torch.uint8, device=dev)
    idx = torch.empty((w.L, w.top_k), dtype=torch.int32, device=dev)
    O = torch.empty((w.L, w.H, w.D), dtype=torch.bfloat16, device=dev)

    def step():
        dsa.dsa_prefill(x["q_idx"], x["k_idx"], x["Q"], x["K"], x["V"], w.top_k, indices=idx, O=O,
                        workspace=ws, stream=stream)

    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    if dsa.dsa_sync_status(stream) != 0:
        raise RuntimeError(f"device-side error in {name}")
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize()
    ms = max_over_ranks(e0.elapsed_time(e1)) / steps
    dsa.dsa_stage_timing(True)
    for _ in range(steps):
        step()
    torch.cuda.synchronize()
    dsa.dsa_stage_timing(False)
    st = {k_: v[0] / steps for k_, v in dsa.dsa_stage_times().items() if v[1] > 0}
    work = prefill_work(w)
    idx_ms = st.get("indexer_filter", float("nan"))
    tflops = work["indexer_flops"] / (idx_ms / 1000.0) / 1e12
    peak = fp8_peak if w.idx_dtype == "fp8" else bf16_peak
    out = {"workload": workload_desc(w), "ms_per_step": ms, "queries_per_s": w.L / (ms / 1000.0),
           "stage_ms": st,
           "indexer": {"tflops": tflops, "dtype": w.idx_dtype, "peak": peak, "frac": tflops / peak,
                       "frac_fp8_peak": tflops / fp8_peak, "flops_per_launch": work["indexer_flops"],
                       "peak_source": "FP8 measured in this run" if w.idx_dtype == "fp8"
                       else "BF16 burst, MEASURED_PEAKS.json"},
           "attention_gather_gbs": work["gather_bytes"] / (st.get("attention", float("nan")) / 1000.0) / 1e9,
           "select_stats": dsa.dsa_last_stats(ws, stream)}
    del x, ws, idx, O
    torch.cuda.empty_cache()
    return out


# ----------------------------------------------------------------------------- CPU oracle leg

def cpu_oracle_sample(w, host, target_s, seed=0):
    """Time the oracle on random query rows of the workload, growing the sample
    until one run takes at least half of target_s; returns (queries/s, rows,
    seconds, threads) of that last run."""
    import oracle
    threads = host_threads()
    rng = np.random.default_rng(seed)
    n = max(4, 2 * threads)
    for _ in range(5):
        rows = np.sort(rng.choice(w.L, size=min(n, w.L), replace=False)).astype(np.int64)
        t0 = time.perf_counter()
        oracle.prefill_rows(host, w.idx_dtype, w.top_k, rows=rows, nthreads=threads)
        dt = time.perf_counter() - t0
        if dt >= 0.5 * target_s or len(rows) == w.L:
            break
        n = int(min(w.L, len(rows) * 0.9 * target_s / max(dt, 1e-3)))
    return len(rows) / dt, len(rows), dt, threads


def host_threads() -> int:
    """Host cores this process may run on (torchrun's OMP_NUM_THREADS=1 does not apply
    to the oracle, which is given this count explicitly)."""
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def host_copy(x):
    import torch
    out = {}
    for k, v in x.items():
        if isinstance(v, torch.Tensor):
            t = v.cpu()
            if t.dtype == torch.bfloat16:
                t = t.view(torch.int16)
            out[k] = t.numpy().view(np.uint16) if t.dtype == torch.int16 else t.numpy()
        else:
            out[k] = v
    return out


def run_reference(args):
    import synth
    rank, world, _ = rank_info()
    if rank != 0:
        return
    w = synth.WORKLOADS[PREFILL]
    world_n = max(1, args.gpus)
    host = synth.prefill_inputs(w)
    per_step = max(2.0, min(8.0, 150.0 / max(1, args.steps + args.warmup)))
    # size one step's sample from a calibration run (untimed)
    import oracle
    threads = host_threads()
    probe = np.linspace(0, w.L - 1, max(4, threads), dtype=np.int64)
    t0 = time.perf_counter()
    oracle.prefill_rows(host, w.idx_dtype, w.top_k, rows=probe, nthreads=threads)
    n = int(max(len(probe), len(probe) * per_step / max(time.perf_counter() - t0, 1e-3)))
    rng = np.random.default_rng(1)
    times = []
    for step in range(args.warmup + args.steps):
        rows = np.sort(rng.choice(w.L, size=n, replace=False)).astype(np.int64)
        t0 = time.perf_counter()
        oracle.prefill_rows(host, w.idx_dtype, w.top_k, rows=rows, nthreads=threads)
        if step >= args.warmup:
            times.append(time.perf_counter() - t0)
    total = sum(times)
    value = n * len(times) / total
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "queries/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1000.0 * total / len(times), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": line_config(w, world_n),
        "cpu_baseline": {"value": value, "unit": "queries/s", "cores": threads, "kind": "oracle",
                         "sample": f"{n} random query rows of {PREFILL} per step (full work of each row)"},
        "e2e": {"value": value, "unit": "queries/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ----------------------------------------------------------------------------- GPU leg

def spawn_ranks(args) -> None:
    """`--gpus N` outside torchrun: start N ranks on this node (one process per GPU,
    rendezvous on 127.0.0.1) and exit with their status.  Under torchrun the
    world size must equal N."""
    if "WORLD_SIZE" in os.environ:
        if int(os.environ["WORLD_SIZE"]) != args.gpus:
            raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE={os.environ['WORLD_SIZE']}")
        return
    if args.gpus <= 1:
        return
    import socket
    with socket.socket() as so:
        so.bind(("127.0.0.1", 0))
        port = so.getsockname()[1]
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", f"--nproc-per-node={args.gpus}",
           "--master-addr", "127.0.0.1", f"--master-port={port}", os.path.abspath(__file__)] + sys.argv[1:]
    raise SystemExit(subprocess.call(cmd))


def main():
    args = parse()
    spawn_ranks(args)
    rank, world, local = rank_info()
    if args.impl == "reference":
        run_reference(args)
        return
    import torch
    import torch.distributed as dist

    import synth
    import sparse_attention_10_b200 as dsa
    from sparse_attention_10_b200 import build as dsa_build

    dsa_build.build()
    dsa.load()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=300), device_id=dev)

    def barrier():
        if world > 1:
            dist.barrier()

    def max_over_ranks(x: float) -> float:
        return reduce_max(x, world, dev)

    run_peaks = measured_peaks_in_run(dev)
    w = synth.WORKLOADS[args.workload]
    seed = synth.SEED + rank              # every rank runs its own sequence
    x = synth.prefill_inputs_torch(w, seed=seed, device=dev)
    q, k = x["q_idx"], x["k_idx"]
    Q, K, V = x["Q"], x["K"], x["V"]
    idt = dsa.IDX_BF16 if w.idx_dtype == "bf16" else dsa.IDX_FP8_E4M3
    ws = torch.empty(dsa.dsa_prefill_workspace_size(w.L, w.d_idx, idt, w.H, w.D, w.top_k),
                     dtype=torch.uint8, device=dev)
    idx = torch.empty((w.L, w.top_k), dtype=torch.int32, device=dev)
    O = torch.empty((w.L, w.H, w.D), dtype=torch.bfloat16, device=dev)
    stream = torch.cuda.current_stream()

    def step():
        dsa.dsa_prefill(q, k, Q, K, V, w.top_k, indices=idx, O=O, workspace=ws, stream=stream)

    for _ in range(args.warmup):
        step()
    if dsa.dsa_sync_status(stream) != 0:
        raise RuntimeError("device-side error during warm-up")
    stats = dsa.dsa_last_stats(ws)
    work_cand = 8.0 * stats["candidates"]

    # --- timed region: K prefill steps
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize()
    with ClockSampler(local) as clocks:
        e0.record(stream)
        for _ in range(args.steps):
            step()
        e1.record(stream)
        torch.cuda.synchronize()
    barrier()
    ms = max_over_ranks(e0.elapsed_time(e1))
    if dsa.dsa_sync_status(stream) != 0:
        raise RuntimeError("device-side error in the timed region")
    value = world * w.L * args.steps / (ms / 1000.0)

    # --- per-stage times: the same K steps again with stage events on the stream
    dsa.dsa_stage_timing(True)
    for _ in range(args.steps):
        step()
    torch.cuda.synchronize()
    dsa.dsa_stage_timing(False)
    stages = dsa.dsa_stage_times()
    launches_per_step = sum(v[1] for v in stages.values()) / args.steps
    work = prefill_work(w)
    work["cand_bytes"] = work_cand
    pk = peaks()
    st_ms = {k_: v[0] / args.steps for k_, v in stages.items() if v[1] > 0}
    idx_ms = st_ms.get("indexer_filter", float("nan"))
    att_ms = st_ms.get("attention", float("nan"))
    indexer_tflops = work["indexer_flops"] / (idx_ms / 1000.0) / 1e12
    gather_gbs = work["gather_bytes"] / (att_ms / 1000.0) / 1e9
    dominant = max(("indexer_filter", "attention", "select", "indexer_sample", "threshold"),
                   key=lambda s: st_ms.get(s, 0.0))
    # Peaks: HBM and BF16 from MEASURED_PEAKS.json (measured on this machine), FP8 measured in
    # this run.  The stage kernels are timed one launch at a time inside a ~20 ms step, so the
    # burst figures apply.
    fp8_peak = run_peaks["fp8_tflops"]
    bf16_peak = pk["bf16_tflops"]
    idx_peak = fp8_peak if w.idx_dtype == "fp8" else bf16_peak
    indexer = {"tflops": indexer_tflops, "dtype": w.idx_dtype, "peak_own_dtype": idx_peak,
               "frac_own_dtype": indexer_tflops / idx_peak, "frac_fp8_peak": indexer_tflops / fp8_peak,
               "flops_per_launch": work["indexer_flops"], "ms": idx_ms,
               "peaks": f"own dtype: {'FP8 measured in this run' if w.idx_dtype == 'fp8' else 'BF16 burst, MEASURED_PEAKS.json'}; "
                        f"FP8: measured in this run ({fp8_peak:.0f} TFLOP/s)"}
    ceiling = gather_ceiling(dsa, idx, K, V, work["gather_bytes"], stream)
    att_kernel = "attn_tc_kernel" if w.D == 128 else "attn_kernel"
    att_src = "attention_tc.cu" if w.D == 128 else "attention.cu"
    traffic = profiled_traffic(att_kernel, w.name, "sparse_attention_10_b200/csrc/" + att_src)
    att_s = att_ms / 1000.0
    att_gbs = work["gather_bytes"] / att_s / 1e9
    attention = {
        "kernel": att_kernel, "ms": att_ms,
        "gather": {"achieved": att_gbs, "peak": ceiling["gbs"], "unit": "GB/s", "frac": att_gbs / ceiling["gbs"],
                   "bytes_per_launch": work["gather_bytes"], "peak_source": ceiling["how"],
                   "peak_shape": ceiling["shape"]},
        "hbm": {"achieved": (traffic / att_s / 1e9) if traffic else None, "peak": pk["hbm_gbs"], "unit": "GB/s",
                "frac": (traffic / att_s / 1e9 / pk["hbm_gbs"]) if traffic else None,
                "note": "DRAM bytes of one launch (ncu, profile summary) over this run's launch time"},
        "tensor": {"achieved": work["attn_flops"] / att_s / 1e12, "peak": bf16_peak, "unit": "TFLOP/s",
                   "frac": work["attn_flops"] / att_s / 1e12 / bf16_peak},
    }
    if dominant.startswith("indexer"):
        flops = work["indexer_flops"] if dominant == "indexer_filter" else float("nan")
        ach = flops / (st_ms[dominant] / 1000.0) / 1e12
        roof = {"kernel": "indexer_kernel", "bound": "tensor", "achieved": ach, "peak": idx_peak,
                "unit": "TFLOP/s", "frac": ach / idx_peak,
                "traffic": profiled_traffic("indexer_kernel", w.name, "sparse_attention_10_b200/csrc/indexer.cu")}
    elif dominant == "attention":
        # The gathered K/V rows are random 256-byte rows of tensors that fit in L2: the kernel is
        # bound by the rate the SMs can gather them, measured above by the probe on the same rows.
        roof = {"kernel": att_kernel, "bound": "l2_gather", "achieved": att_gbs, "peak": ceiling["gbs"],
                "unit": "GB/s", "frac": att_gbs / ceiling["gbs"], "bytes_per_launch": work["gather_bytes"],
                "traffic": traffic,
                "peak_source": "measured in this run: " + ceiling["how"],
                "vs_hbm_copy_peak": {"peak": pk["hbm_gbs"], "frac": att_gbs / pk["hbm_gbs"],
                                     "note": "algorithmic gather bytes over the HBM copy peak: above 1 "
                                             "because K and V (67 MB) stay in L2"}}
    else:
        ach = (work["cand_bytes"] + 4.0 * w.L * w.top_k) / (st_ms[dominant] / 1000.0) / 1e9
        roof = {"kernel": "select_kernel", "bound": "hbm", "achieved": ach, "peak": pk["hbm_gbs"], "unit": "GB/s",
                "frac": ach / pk["hbm_gbs"],
                "traffic": profiled_traffic("select_kernel", w.name, "sparse_attention_10_b200/csrc/select.cu")}
    roof.setdefault("peak_source", pk["source"])
    roof["traffic_source"] = ("ncu dram__bytes_read.sum + dram__bytes_write.sum of one launch, from the profile "
                              "summary in profiles/ whose recorded source hash matches this kernel's source "
                              "(null when it does not)")

    # --- the same sequence split over the ranks by query rows (zig-zag chunks, one all-gather
    # of the key rows, dsa_prefill_chunk per chunk): strong scaling of one sequence
    zz = None
    if not args.no_zigzag:
        from sparse_attention_10_b200.zigzag import prefill_sharded, zigzag_chunks
        xs = x if seed == synth.SEED else synth.prefill_inputs_torch(w, seed=synth.SEED, device=dev)
        chunks = zigzag_chunks(w.L, world, rank)
        parts = {n_: [xs[n_][a_:b_].contiguous() for a_, b_ in chunks] for n_ in ("q_idx", "k_idx", "Q", "K", "V")}
        ws_z = [torch.empty(dsa.dsa_prefill_chunk_workspace_size(b_ - a_, b_, w.d_idx, idt, w.H, w.D, w.top_k),
                            dtype=torch.uint8, device=dev) for a_, b_ in chunks]
        wsq = iter(())

        def zchunk(qi, kf, Qi, Kf, Vf, top_k):
            return dsa.dsa_prefill_chunk(qi, kf, Qi, Kf, Vf, top_k, workspace=next(wsq), stream=stream)

        def zstep():
            nonlocal wsq
            wsq = iter(ws_z)
            return prefill_sharded(parts["q_idx"], parts["k_idx"], parts["Q"], parts["K"], parts["V"], w.L,
                                   w.top_k, world, rank, chunk_fn=zchunk)

        for _ in range(max(1, args.warmup)):
            zstep()
        torch.cuda.synchronize()
        nz = max(3, args.steps // 2)
        barrier()
        torch.cuda.synchronize()
        e0.record(stream)
        for _ in range(nz):
            zstep()
        e1.record(stream)
        torch.cuda.synchronize()
        barrier()
        zms = max_over_ranks(e0.elapsed_time(e1)) / nz
        if dsa.dsa_sync_status(stream) != 0:
            raise RuntimeError("device-side error in the row-split prefill")
        zz = {"value": w.L / (zms / 1000.0), "unit": "queries/s", "ms_per_step": zms, "scaling": "strong",
              "chunks_of_rank0": zigzag_chunks(w.L, world, 0),
              "how": f"one {w.name} sequence split over {world} rank(s) by query rows: 2 x {world} zig-zag "
                     f"chunks, all-gather of k_idx/K/V rows (NCCL), dsa_prefill_chunk per chunk; the timed "
                     f"region covers the all-gather and both chunks of every rank (max over ranks)"}
        del parts, ws_z
        if xs is not x:
            del xs
        torch.cuda.empty_cache()

    # --- BF16 index inputs that are exact in FP8 E4M3 (the workload's small integers): the
    # E4M3 copy runs the indexer on the FP8 tensor-core path with identical scores.  Each
    # timed step converts both index tensors (dsa_index_to_fp8) and runs dsa_prefill on the copy.
    fp8_path = None
    if w.idx_dtype == "bf16" and not args.no_fp8_path:
        q8 = torch.empty(q.shape, dtype=torch.uint8, device=dev)
        k8 = torch.empty(k.shape, dtype=torch.uint8, device=dev)
        bad = torch.empty(2, dtype=torch.int64, device=dev)
        dsa.dsa_index_to_fp8(q, out=q8, inexact=bad[0:1], stream=stream)
        dsa.dsa_index_to_fp8(k, out=k8, inexact=bad[1:2], stream=stream)
        torch.cuda.synchronize()
        if int(bad.sum().item()) == 0:
            ws8 = torch.empty(dsa.dsa_prefill_workspace_size(w.L, w.d_idx, dsa.IDX_FP8_E4M3, w.H, w.D, w.top_k),
                              dtype=torch.uint8, device=dev)
            idx8 = torch.empty_like(idx)
            O8 = torch.empty_like(O)

            def step8():
                dsa.dsa_index_to_fp8(q, out=q8, inexact=bad[0:1], stream=stream)
                dsa.dsa_index_to_fp8(k, out=k8, inexact=bad[1:2], stream=stream)
                dsa.dsa_prefill(q8, k8, Q, K, V, w.top_k, indices=idx8, O=O8, workspace=ws8, stream=stream)

            for _ in range(args.warmup):
                step8()
            torch.cuda.synchronize()
            barrier()
            e0.record(stream)
            for _ in range(args.steps):
                step8()
            e1.record(stream)
            torch.cuda.synchronize()
            barrier()
            ms8 = max_over_ranks(e0.elapsed_time(e1)) / args.steps
            dsa.dsa_stage_timing(True)
            for _ in range(args.steps):
                step8()
            torch.cuda.synchronize()
            dsa.dsa_stage_timing(False)
            st8 = {k_: v[0] / args.steps for k_, v in dsa.dsa_stage_times().items() if v[1] > 0}
            if dsa.dsa_sync_status(stream) != 0:
                raise RuntimeError("device-side error on the FP8 index path")
            same = bool(torch.equal(idx8, idx) and torch.equal(O8.view(torch.int16), O.view(torch.int16)))
            t8 = work["indexer_flops"] / (st8["indexer_filter"] / 1000.0) / 1e12
            fp8_path = {"value": world * w.L / (ms8 / 1000.0), "unit": "queries/s", "ms_per_step": ms8,
                        "stage_ms": st8, "matches_bf16_call": same,
                        "indexer": {"tflops": t8, "dtype": "fp8", "peak": fp8_peak, "frac": t8 / fp8_peak,
                                    "peak_source": "FP8 measured in this run"},
                        "how": "per step: dsa_index_to_fp8 on q_idx and k_idx (inside the timed region), "
                               "then dsa_prefill with the E4M3 copies"}
            del ws8, idx8, O8
        del q8, k8, bad
        torch.cuda.empty_cache()

    # --- end to end through the public API with host buffers.  A serving loop
    # pipelines the transfers: while step i computes, step i+1's inputs go up
    # and step i-1's outputs come down (one stream each, double-buffered device
    # tensors, events order the reuse).  Every step still uploads all its inputs
    # from pinned host memory and downloads its full result.
    e2e = None
    if not args.no_e2e:
        hq = q.cpu().pin_memory(); hk = k.cpu().pin_memory()
        hQ = Q.cpu().pin_memory(); hK = K.cpu().pin_memory(); hV = V.cpu().pin_memory()
        hidx = torch.empty(idx.shape, dtype=idx.dtype).pin_memory()
        hO = torch.empty(O.shape, dtype=O.dtype).pin_memory()
        ins = [tuple(torch.empty_like(t, device=dev) for t in (hq, hk, hQ, hK, hV)) for _ in range(2)]
        outs = [(torch.empty_like(idx), torch.empty_like(O)) for _ in range(2)]
        s_up, s_dn = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
        s_cp = torch.cuda.ExternalStream(stream, device=dev) if isinstance(stream, int) else stream
        up_ev = [torch.cuda.Event() for _ in range(2)]
        cp_ev = [torch.cuda.Event() for _ in range(2)]
        dn_ev = [torch.cuda.Event() for _ in range(2)]
        state = {"i": 0}

        def e2e_step():
            i = state["i"]
            b_ = i % 2
            if i >= 2:
                s_up.wait_event(cp_ev[b_])           # step i-2 done with these inputs
            with torch.cuda.stream(s_up):
                for d_, h_ in zip(ins[b_], (hq, hk, hQ, hK, hV)):
                    d_.copy_(h_, non_blocking=True)
                up_ev[b_].record(s_up)
            s_cp.wait_event(up_ev[b_])
            if i >= 2:
                s_cp.wait_event(dn_ev[b_])           # step i-2's outputs are down
            dq_, dk_, dQ_, dK_, dV_ = ins[b_]
            dsa.dsa_prefill(dq_, dk_, dQ_, dK_, dV_, w.top_k, indices=outs[b_][0], O=outs[b_][1],
                            workspace=ws, stream=stream)
            cp_ev[b_].record(s_cp)
            s_dn.wait_event(cp_ev[b_])
            with torch.cuda.stream(s_dn):
                hidx.copy_(outs[b_][0], non_blocking=True)
                hO.copy_(outs[b_][1], non_blocking=True)
                dn_ev[b_].record(s_dn)
            state["i"] = i + 1

        e2e_step()
        torch.cuda.synchronize()
        n_e2e = max(6, args.steps // 2)
        barrier()
        torch.cuda.synchronize()
        state["i"] = 0
        e0.record(s_up)
        for _ in range(n_e2e):
            e2e_step()
        s_dn.wait_event(cp_ev[(n_e2e - 1) % 2])
        e1.record(s_dn)
        torch.cuda.synchronize()
        barrier()
        ems = max_over_ranks(e0.elapsed_time(e1))
        if dsa.dsa_sync_status(stream) != 0:
            raise RuntimeError("device-side error in the end-to-end loop")
        h2d = sum(t.numel() * t.element_size() for t in (hq, hk, hQ, hK, hV))
        d2h = idx.numel() * 4 + O.numel() * 2
        e2e = {"value": world * w.L * n_e2e / (ems / 1000.0), "unit": "queries/s",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": n_e2e,
               "ms_per_step": ems / n_e2e,
               "overlap": "uploads, compute and downloads of consecutive steps on three streams"}
        del ins, outs, hq, hk, hQ, hK, hV, hidx, hO

    # --- decode rows of the path
    decode = None
    if not args.no_decode:
        wd = synth.WORKLOADS[DECODE]
        del ws
        torch.cuda.empty_cache()
        if args.decode_batch:
            import dataclasses
            wd = dataclasses.replace(wd, B=args.decode_batch)
        xd = synth.decode_inputs_torch(wd, seed=seed, device=dev)
        lengths = xd["lengths"]
        wsd = torch.empty(dsa.dsa_decode_workspace_size(wd.B, int(lengths.sum()), wd.d_idx, 0, wd.H, wd.D,
                                                         wd.top_k), dtype=torch.uint8, device=dev)
        Od = torch.empty((wd.B, wd.H, wd.D), dtype=torch.bfloat16, device=dev)
        idd = torch.empty((wd.B, wd.top_k), dtype=torch.int32, device=dev)

        def dstep():
            dsa.dsa_decode(xd["k_idx"], xd["K"], xd["V"], xd["seq_start"], xd["q_idx"], xd["Q"], wd.top_k,
                           int(lengths.max()), O=Od, indices=idd, workspace=wsd, stream=stream)

        for _ in range(args.warmup):
            dstep()
        torch.cuda.synchronize()
        nd = max(args.steps, 20)
        barrier()
        torch.cuda.synchronize()
        e0.record(stream)
        for _ in range(nd):
            dstep()
        e1.record(stream)
        torch.cuda.synchronize()
        barrier()
        dms = max_over_ranks(e0.elapsed_time(e1))
        dsa.dsa_stage_timing(True)
        for _ in range(nd):
            dstep()
        torch.cuda.synchronize()
        dsa.dsa_stage_timing(False)
        dst = {k_: v[0] / nd for k_, v in dsa.dsa_stage_times().items() if v[1] > 0}
        dw = decode_work(wd, lengths)
        scan_ms = dst.get("decode_scan_select", float("nan"))
        decode = {"metric": "decode tok/s", "value": world * wd.B * nd / (dms / 1000.0), "unit": "tok/s",
                  "ms_per_step": dms / nd, "workload": f"{DECODE}: B=64, cached lengths U[65536,131072] "
                  f"(sum {dw['total_rows']}), k_idx fp8 d=128, H=16, D=128, top_k=2048",
                  "stage_ms": dst,
                  "scan_select_gbs": dw["scan_bytes"] / (scan_ms / 1000.0) / 1e9,
                  "scan_select_frac_hbm": dw["scan_bytes"] / (scan_ms / 1000.0) / 1e9 / pk["hbm_gbs"]}
        if dsa.dsa_sync_status(stream) != 0:
            raise RuntimeError("device-side error in decode")

        # the same batch in a block-paged cache: blocks of 64 rows placed by a seeded permutation
        bsz = 64
        xp = synth.paged_decode_inputs_torch(xd, bsz, seed=seed)
        wsp = torch.empty(dsa.dsa_decode_paged_workspace_size(wd.B, int(lengths.max()), wd.d_idx, 0, wd.H,
                                                               wd.D, wd.top_k), dtype=torch.uint8, device=dev)
        Op, idp = torch.empty_like(Od), torch.empty_like(idd)

        def pstep():
            dsa.dsa_decode_paged(xp["k_idx_blocks"], xp["K_blocks"], xp["V_blocks"], xp["block_table"],
                                 xp["seq_lens"], xp["q_idx"], xp["Q"], wd.top_k, int(lengths.max()), O=Op,
                                 indices=idp, workspace=wsp, stream=stream)

        for _ in range(args.warmup):
            pstep()
        torch.cuda.synchronize()
        barrier()
        torch.cuda.synchronize()
        e0.record(stream)
        for _ in range(nd):
            pstep()
        e1.record(stream)
        torch.cuda.synchronize()
        barrier()
        pms = max_over_ranks(e0.elapsed_time(e1))
        if dsa.dsa_sync_status(stream) != 0:
            raise RuntimeError("device-side error in paged decode")
        decode["paged"] = {
            "value": world * wd.B * nd / (pms / 1000.0), "unit": "tok/s", "ms_per_step": pms / nd,
            "layout": f"k_idx/K/V pools of {xp['k_idx_blocks'].shape[0]} blocks x {bsz} rows, "
                      f"block table [{wd.B}, {xp['block_table'].shape[1]}] int32, seeded block order",
            "matches_contiguous": bool(torch.equal(idp, idd) and torch.equal(Op, Od))}

        # several new tokens per sequence (speculative drafts / short chunks) over the same paged
        # cache: T tokens of each sequence are scored in one pass over its index rows
        decode["multi_token"] = {}
        for T in (2, 4):
            mq = synth.multi_queries_torch(wd, wd.B, T, seed=seed, device=dev)
            wsm = torch.empty(dsa.dsa_decode_paged_multi_workspace_size(wd.B, T, int(lengths.max()), wd.d_idx, 0,
                                                                        wd.H, wd.D, wd.top_k),
                              dtype=torch.uint8, device=dev)
            Om = torch.empty((wd.B, T, wd.H, wd.D), dtype=torch.bfloat16, device=dev)
            idm = torch.empty((wd.B, T, wd.top_k), dtype=torch.int32, device=dev)

            def mstep():
                dsa.dsa_decode_paged_multi(xp["k_idx_blocks"], xp["K_blocks"], xp["V_blocks"], xp["block_table"],
                                           xp["seq_lens"], mq["q_idx"], mq["Q"], wd.top_k, int(lengths.max()),
                                           O=Om, indices=idm, workspace=wsm, stream=stream)

            for _ in range(args.warmup):
                mstep()
            torch.cuda.synchronize()
            barrier()
            torch.cuda.synchronize()
            e0.record(stream)
            for _ in range(nd):
                mstep()
            e1.record(stream)
            torch.cuda.synchronize()
            barrier()
            mms = max_over_ranks(e0.elapsed_time(e1))
            if dsa.dsa_sync_status(stream) != 0:
                raise RuntimeError("device-side error in multi-token decode")
            decode["multi_token"][f"T{T}"] = {
                "value": world * wd.B * T * nd / (mms / 1000.0), "unit": "tok/s", "ms_per_step": mms / nd,
                "tokens_per_step": wd.B * T,
                "how": f"dsa_decode_paged_multi, {T} new tokens per sequence, the paged cache above"}
            del mq, wsm, Om, idm
        del xp, wsp

    # --- the other prefill workloads (4K, 32K and 64K), each timed on its own
    configs = None
    if not args.no_configs:
        del idx, O
        torch.cuda.empty_cache()
        configs = {}
        for name in ("prefill_4k", "prefill_32k", "prefill_64k"):
            if name != w.name:
                configs[name] = time_prefill_config(dsa, synth, name, max(5, args.steps // 2), args.warmup,
                                                    dev, stream, seed, run_peaks["fp8_tflops"], pk["bf16_tflops"],
                                                    max_over_ranks)

    # --- CPU oracle baseline (rank 0, one GPU only)
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        host = host_copy(x)
        qps, n, dt, thr = cpu_oracle_sample(w, host, args.cpu_seconds)
        cpu = {"value": qps, "unit": "queries/s", "cores": thr, "kind": "oracle",
               "sample": f"{n} random query rows of {w.name} (full work of each row: indexer over "
                         f"t+1 keys, top-{w.top_k}, attention), {dt:.1f} s"}

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "queries/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16" if w.idx_dtype == "bf16" else "fp8 indexer / bf16 attention", "data": "synthetic",
            "config": line_config(w, world),
            "indexer_tflops": indexer_tflops, "gather_gbs": gather_gbs, "indexer": indexer,
            "attention": attention, "stage_ms": st_ms, "roofline": roof, "cpu_baseline": cpu, "e2e": e2e,
            "peaks_in_run": run_peaks, "configs": configs, "row_split": zz, "fp8_index_path": fp8_path,
            "gpu_launches": int(round(launches_per_step * args.steps)), "clocks": clocks.summary(),
            "decode": decode, "select_stats": stats,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
