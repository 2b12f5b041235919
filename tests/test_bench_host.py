"""Host-side pieces of bench.py: the max-over-ranks reduction across two gloo
ranks on CPU (the N > 1 timing path), work accounting and the profile lookup."""
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
