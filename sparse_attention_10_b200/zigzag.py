"""Query-row split of one causal sequence over the ranks of a process group.

Every query row of DSA prefill depends only on its own query and on the key
rows before it (DeepSeek Sparse Attention, sections 3.2-3.3), so the rows of one
long sequence can be divided among GPUs.  Causal work grows with the row's
position, so the rows are cut into 2 * world equal chunks and rank r takes
chunks r and 2 * world - 1 - r (a zig-zag): every rank then holds the same
amount of causal work.  The only exchange is one all-gather of the key-side
rows (index keys, K and V), after which each rank runs its two chunks with
``dsa_prefill_chunk`` against the key prefix each needs.  Indices and outputs
stay row-sharded.

This module is host-side plumbing (chunk arithmetic and the collective); every
score, selection and attention output is computed by the CUDA library.
"""
from __future__ import annotations

from typing import Callable, List, Optional, Sequence, Tuple

import torch


def zigzag_chunks(L: int, world: int, rank: int) -> List[Tuple[int, int]]:
    """The (start, stop) row ranges of rank `rank`: chunks rank and 2*world-1-rank
    of 2*world chunks of ceil(L / (2*world)) rows (the last ones may be short or empty)."""
    if world < 1 or not 0 <= rank < world or L < 2 * world:
        raise ValueError("need 0 <= rank < world and L >= 2 * world (every rank holds rows)")
    n = 2 * world
    c = -(-L // n)
    out = []
    for k in (rank, n - 1 - rank):
        a, b = min(L, k * c), min(L, (k + 1) * c)
        if b > a:
            out.append((a, b))
    return out


def causal_pairs(start: int, stop: int) -> int:
    """Causal query-key pairs of rows start .. stop-1 (diagonal included)."""
    return (stop * (stop + 1) - start * (start + 1)) // 2


def gather_rows(local: Sequence[torch.Tensor], L: int, world: int, rank: int, group=None) -> torch.Tensor:
    """All-gather key-side rows.  `local` holds this rank's rows of its chunks (in the
    order of zigzag_chunks); the result is the full [L, ...] tensor in position order
    on every rank.  One collective per chunk slot; each rank's data lands directly in
    the rows it covers."""
    import torch.distributed as dist
    dtype, shape = local[0].dtype, tuple(local[0].shape[1:])
    # rows travel as bytes, so any element type (FP8, BF16 bits, ...) goes through any backend
    local = [t.contiguous().view(torch.uint8).reshape(t.shape[0], -1) for t in local]
    ref = local[0]
    full = torch.empty((L,) + tuple(ref.shape[1:]), dtype=ref.dtype, device=ref.device)
    n = 2 * world
    c = -(-L // n)
    for slot in range(2):
        # slot 0: chunk r of rank r; slot 1: chunk 2*world-1-r of rank r
        chunk_of = [r if slot == 0 else n - 1 - r for r in range(world)]
        outs, pads = [], []
        for r in range(world):
            a, b = min(L, chunk_of[r] * c), min(L, (chunk_of[r] + 1) * c)
            if b - a == c:
                outs.append(full[a:b])
            else:                                  # short or empty last chunk: gather padded
                pad = torch.empty((c,) + tuple(ref.shape[1:]), dtype=ref.dtype, device=ref.device)
                outs.append(pad)
                pads.append((pad, a, b))
        mine = zigzag_chunks(L, world, rank)
        k = chunk_of[rank]
        a, b = min(L, k * c), min(L, (k + 1) * c)
        send = torch.zeros((c,) + tuple(ref.shape[1:]), dtype=ref.dtype, device=ref.device)
        src = [t for (ra, rb), t in zip(mine, local) if (ra, rb) == (a, b)]
        if b > a:
            send[:b - a] = src[0]
        if world == 1:
            outs[0].copy_(send)
        else:
            dist.all_gather(outs, send, group=group)
        for pad, a, b in pads:
            if b > a:
                full[a:b] = pad[:b - a]
    return full.view(dtype).reshape((L,) + shape)


def prefill_sharded(q_idx: Sequence[torch.Tensor], k_idx: Sequence[torch.Tensor], Q: Sequence[torch.Tensor],
                    K: Sequence[torch.Tensor], V: Sequence[torch.Tensor], L: int, top_k: int, world: int,
                    rank: int, group=None, chunk_fn: Optional[Callable] = None, **kw):
    """DSA prefill of one sequence of L rows split over `world` ranks.

    Each argument list holds this rank's rows for each of its zig-zag chunks
    (zigzag_chunks order).  Returns [(start, stop, indices, O)] for those chunks.
    `chunk_fn(q_idx, k_idx, Q, K, V, top_k, **kw) -> (indices, O)` runs one chunk
    (default: the library's dsa_prefill_chunk)."""
    if chunk_fn is None:
        from . import dsa_prefill_chunk as chunk_fn
    chunks = zigzag_chunks(L, world, rank)
    kf = gather_rows(k_idx, L, world, rank, group)
    Kf = gather_rows(K, L, world, rank, group)
    Vf = gather_rows(V, L, world, rank, group)
    out = []
    for (a, b), qi, Qi in zip(chunks, q_idx, Q):
        idx, O = chunk_fn(qi, kf[:b], Qi, Kf[:b], Vf[:b], top_k, **kw)
        out.append((a, b, idx, O))
    return out
