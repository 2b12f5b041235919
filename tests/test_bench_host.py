"""Host-side pieces of bench.py: the max-over-ranks reduction across two gloo
ranks on CPU (the N > 1 timing path), work accounting, the profile lookup and
the reference arm (the CPU oracle) with its JSON line."""
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    sys.path.insert(0, ROOT)
    import torch.distributed as dist
    import bench
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world)
    try:
        out[rank] = bench.reduce_max(10.0 * (rank + 1) + 0.5, world, "cpu")
    finally:
        dist.destroy_process_group()


def test_reduce_max_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    out = mgr.dict()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    assert out[0] == out[1] == 20.5


def test_prefill_work_counts():
    sys.path.insert(0, ROOT)
    import bench
    import synth
    w = synth.WORKLOADS["prefill_128k"]
    work = bench.prefill_work(w)
    assert work["indexer_flops"] == 160 * 131072 * 131073
    kept = sum(min(t + 1, 2048) for t in range(131072))
    assert work["kept"] == kept
    assert work["gather_bytes"] == kept * 512


def test_profiled_traffic_requires_matching_source(tmp_path, monkeypatch):
    sys.path.insert(0, ROOT)
    import bench
    assert bench.profiled_traffic("no_such_kernel", "prefill_128k", "bench.py") is None


def _bench(args, env_extra):
    import json
    import subprocess
    env = dict(os.environ, **env_extra)
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py")] + args, cwd=ROOT, env=env,
                       capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    return [json.loads(ln) for ln in lines]


def test_reference_arm_prints_one_contract_line():
    """`bench.py --impl reference` times the oracle on the host and prints one JSON
    line with the contract's keys (no GPU needed)."""
    (line,) = _bench(["--impl", "reference", "--steps", "1", "--warmup", "0"], {"RANK": "0", "WORLD_SIZE": "1"})
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in line, key
    assert line["impl"] == "reference" and line["value"] > 0 and line["steps"] == 1
    assert line["config"]["workload"].startswith("prefill_128k")
    cb = line["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == line["value"] and cb["sample"]
    e2e = line["e2e"]
    assert e2e["value"] == line["value"] and e2e["unit"] == line["unit"]
    assert e2e["h2d_bytes_per_step"] == 0 and e2e["d2h_bytes_per_step"] == 0


def test_reference_arm_other_ranks_do_no_work():
    assert _bench(["--impl", "reference", "--gpus", "2", "--steps", "1", "--warmup", "0"],
                  {"RANK": "1", "WORLD_SIZE": "2"}) == []


def test_bench_starts_its_own_ranks():
    """`--gpus 2` outside torchrun starts two ranks itself (the reference arm needs no
    GPU); exactly one line comes back, from rank 0, and it reports both ranks."""
    clean = {k: v for k, v in os.environ.items() if k not in ("RANK", "WORLD_SIZE", "LOCAL_RANK",
                                                               "MASTER_ADDR", "MASTER_PORT")}
    import json
    import subprocess
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2",
                        "--steps", "1", "--warmup", "0"], cwd=ROOT, env=clean, capture_output=True, text=True,
                       timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [json.loads(ln) for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1 and lines[0]["n_gpus"] == 2


def test_bench_rejects_world_size_other_than_gpus():
    import subprocess
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "4",
                        "--steps", "1", "--warmup", "0"], cwd=ROOT, env=dict(os.environ, RANK="0", WORLD_SIZE="2"),
                       capture_output=True, text=True, timeout=120)
    assert r.returncode != 0 and "WORLD_SIZE" in r.stderr
