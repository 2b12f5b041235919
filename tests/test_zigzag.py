"""Query-row split of one sequence over ranks (host logic, CPU, gloo).

The split itself is plumbing (chunk arithmetic and an all-gather of the key
rows); these tests run it on two gloo ranks with the oracle standing in for
the per-chunk CUDA call, and check that the ranks' rows together equal the
single-rank oracle result, row for row.
"""
import os
import socket

import numpy as np
import pytest
import torch

from sparse_attention_10_b200.zigzag import causal_pairs, zigzag_chunks


@pytest.mark.parametrize("L", [16, 17, 300, 4096, 131072])
@pytest.mark.parametrize("world", [1, 2, 3, 4, 8])
def test_chunks_cover_every_row_once_and_balance_work(L, world):
    seen = np.zeros(L, dtype=np.int64)
    work = []
    for r in range(world):
        w = 0
        for a, b in zigzag_chunks(L, world, r):
            assert 0 <= a < b <= L
            seen[a:b] += 1
            w += causal_pairs(a, b)
        work.append(w)
    assert (seen == 1).all()
    assert sum(work) == L * (L + 1) // 2
    if L >= 64 * world:
        c = -(-L // (2 * world))
        # zig-zag pairs a light chunk with a heavy one: ranks differ by at most a chunk's diagonal
        assert max(work) - min(work) <= c * c + c


def test_too_few_rows_rejected():
    with pytest.raises(ValueError):
        zigzag_chunks(7, 4, 0)


def _oracle_chunk(qi, kf, Qi, Kf, Vf, top_k, start=None):
    import oracle
    b = kf.shape[0]
    a = b - qi.shape[0]
    d = qi.shape[1]
    q_full = np.zeros((b, d), dtype=qi.numpy().dtype)
    q_full[a:] = qi.numpy()
    Q_full = np.zeros((b,) + tuple(Qi.shape[1:]), dtype=np.uint16)
    Q_full[a:] = Qi.numpy()
    x = {"q_idx": q_full, "k_idx": kf.numpy(), "Q": Q_full, "K": Kf.numpy(), "V": Vf.numpy()}
    idx, O = oracle.prefill_rows(x, "fp8", top_k, rows=np.arange(a, b, dtype=np.int64))
    return torch.from_numpy(idx), torch.from_numpy(O)


def _rank_main(rank, world, port, out_dir, L, top_k):
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    sys.path.insert(0, root)
    import torch.distributed as dist
    from datetime import timedelta
    import synth
    from sparse_attention_10_b200.zigzag import prefill_sharded, zigzag_chunks
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world,
                            timeout=timedelta(seconds=120))
    try:
        w = synth.WORKLOADS["prefill_4k"]
        x = synth.prefill_inputs(w, L=L)
        chunks = zigzag_chunks(L, world, rank)
        pick = lambda a: [torch.from_numpy(np.ascontiguousarray(a[s:e])) for s, e in chunks]
        res = prefill_sharded(pick(x["q_idx"]), pick(x["k_idx"]), pick(x["Q"]), pick(x["K"]), pick(x["V"]),
                              L, top_k, world, rank, chunk_fn=_oracle_chunk)
        for a, b, idx, O in res:
            np.save(os.path.join(out_dir, f"idx_{a}_{b}.npy"), idx.numpy())
            np.save(os.path.join(out_dir, f"O_{a}_{b}.npy"), O.numpy())
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_equal_the_single_rank_rows(tmp_path):
    import oracle
    import synth
    import torch.multiprocessing as mp
    oracle.build()
    L, top_k, world = 1000, 96, 2
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    mp.spawn(_rank_main, args=(world, port, str(tmp_path), L, top_k), nprocs=world, join=True)
    w = synth.WORKLOADS["prefill_4k"]
    x = synth.prefill_inputs(w, L=L)
    ref_idx, ref_O = oracle.prefill_rows(x, "fp8", top_k)
    got_idx = np.full_like(ref_idx, -7)
    got_O = np.zeros_like(ref_O)
    for r in range(world):
        for a, b in zigzag_chunks(L, world, r):
            got_idx[a:b] = np.load(tmp_path / f"idx_{a}_{b}.npy")
            got_O[a:b] = np.load(tmp_path / f"O_{a}_{b}.npy")
    assert np.array_equal(got_idx, ref_idx)
    assert np.array_equal(got_O, ref_O)
