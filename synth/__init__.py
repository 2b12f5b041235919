"""Seeded synthetic inputs for DeepSeek Sparse Attention workloads.

This module is shared by the CPU oracle's tests and by the CUDA path's tests and
benchmark.  It only draws and encodes numbers; it holds none of the method's
arithmetic (no dot products, no scaling, no selection, no softmax).

Draws come from a counter-based splitmix64 (Steele, Lea & Flood, "Fast
splittable pseudorandom number generators", OOPSLA 2014): draw i of stream
``key`` is ``mix64(key + (i + 1) * 0x9E3779B97F4A7C15)``, so any slice of a
stream can be regenerated without the rest.

Encodings:
  * small integers in [-4, 4] are written as FP8 E4M3 bytes (OCP 8-bit
    floating point spec) or BF16 bit patterns; every such integer is exact in
    both formats;
  * N(0, 1) values come from Box-Muller in float64 (one 64-bit draw gives the
    two 32-bit uniforms of a pair) and are rounded once to BF16, nearest-even.

The workloads follow the lightning-indexer parameter guide of the DeepSeek
Sparse Attention page (kwkr.cn/news/60693, section 7.2: 32K -> top_k 1024,
index_dim 96, fp8; 64K -> 1536, 128, fp8; 128K -> 2048, 160, bf16) plus a small
4K case and a 64-sequence decode batch.
"""
from __future__ import annotations

import dataclasses
import math
import os
from typing import Optional

import numpy as np

__all__ = [
    "GOLDEN", "SEED", "mix64", "draws", "uniform_ints", "fp8_bytes_of_ints",
    "bf16_bits_of_ints", "bf16_bits_of_f32", "normal_bf16", "Workload",
    "WORKLOADS", "prefill_inputs", "decode_inputs", "decode_lengths", "stream_key",
    "paged_layout", "paged_decode_inputs", "paged_decode_inputs_torch",
]

GOLDEN = np.uint64(0x9E3779B97F4A7C15)
SEED = 20261202

_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)


def mix64(z: np.ndarray) -> np.ndarray:
    """splitmix64 finaliser on a uint64 array (wrapping arithmetic)."""
    z = np.asarray(z, dtype=np.uint64)
    with np.errstate(over="ignore"):
        z = (z ^ (z >> np.uint64(30))) * _M1
        z = (z ^ (z >> np.uint64(27))) * _M2
    return z ^ (z >> np.uint64(31))


def stream_key(*parts: int) -> np.uint64:
    """Key of a named stream: parts are folded through mix64 one at a time."""
    k = np.uint64(0x243F6A8885A308D3)
    for p in parts:
        with np.errstate(over="ignore"):
            k = mix64(np.array([k ^ np.uint64(p & 0xFFFFFFFFFFFFFFFF)], dtype=np.uint64))[0]
            k = np.uint64(k + GOLDEN)
    return np.uint64(k)


def draws(key: np.uint64, start: int, n: int) -> np.ndarray:
    """Draws start .. start+n-1 of stream ``key`` as uint64."""
    i = np.arange(start + 1, start + n + 1, dtype=np.uint64)
    with np.errstate(over="ignore"):
        return mix64(np.uint64(key) + i * GOLDEN)


def uniform_ints(key: np.uint64, n: int, lo: int = -4, hi: int = 4, start: int = 0) -> np.ndarray:
    """n integers uniform on [lo, hi] (multiply-shift on the top 32 bits; bias < 2^-28)."""
    span = np.uint64(hi - lo + 1)
    top = draws(key, start, n) >> np.uint64(32)
    return ((top * span) >> np.uint64(32)).astype(np.int64) + lo


# FP8 E4M3 byte for each integer -4..4 (sign bit 0x80; 1=0x38, 2=0x40, 3=0x44, 4=0x48).
_FP8_OF_INT = {0: 0x00, 1: 0x38, 2: 0x40, 3: 0x44, 4: 0x48}
# BF16 bit pattern of each integer -4..4.
_BF16_OF_INT = {0: 0x0000, 1: 0x3F80, 2: 0x4000, 3: 0x4040, 4: 0x4080}


def fp8_bytes_of_ints(v: np.ndarray) -> np.ndarray:
    """Encode integers in [-4, 4] as FP8 E4M3 bytes (exact)."""
    table = np.zeros(9, dtype=np.uint8)
    for i in range(-4, 5):
        b = _FP8_OF_INT[abs(i)]
        table[i + 4] = b | (0x80 if i < 0 else 0)
    return table[np.asarray(v, dtype=np.int64) + 4]


def bf16_bits_of_ints(v: np.ndarray) -> np.ndarray:
    """Encode integers in [-4, 4] as BF16 bit patterns (exact)."""
    table = np.zeros(9, dtype=np.uint16)
    for i in range(-4, 5):
        b = _BF16_OF_INT[abs(i)]
        table[i + 4] = b | (0x8000 if i < 0 else 0)
    return table[np.asarray(v, dtype=np.int64) + 4]


def bf16_bits_of_f32(x: np.ndarray) -> np.ndarray:
    """Round float32 values (finite) to BF16 bit patterns, nearest-even."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    bias = ((u >> np.uint32(16)) & np.uint32(1)) + np.uint32(0x7FFF)
    with np.errstate(over="ignore"):
        return ((u + bias) >> np.uint32(16)).astype(np.uint16)


def normal_bf16(key: np.uint64, n: int, chunk: int = 1 << 22, workers: int = 0) -> np.ndarray:
    """n N(0,1) values as BF16 bit patterns (Box-Muller, both outputs of a pair).

    Chunks are independent slices of the counter stream, so the result does not
    depend on ``workers`` (threads; 0 = one per CPU, capped at 32).
    """
    out = np.empty(n, dtype=np.uint16)
    npairs = (n + 1) // 2
    starts = list(range(0, npairs, chunk))
    if workers == 0:
        workers = min(32, os.cpu_count() or 1)
    if workers > 1 and len(starts) > 1:
        from concurrent.futures import ThreadPoolExecutor
        with ThreadPoolExecutor(workers) as ex:
            list(ex.map(lambda p0: _normal_chunk(key, p0, min(chunk, npairs - p0), n, out), starts))
    else:
        for p0 in starts:
            _normal_chunk(key, p0, min(chunk, npairs - p0), n, out)
    return out


def _normal_chunk(key, p0, m, n, out):
    """Pairs p0 .. p0+m-1 of the stream into out[2*p0 : 2*(p0+m)] (clipped to n)."""
    z = draws(key, p0, m)
    u1 = ((z >> np.uint64(32)).astype(np.float64) + 0.5) * (1.0 / 4294967296.0)
    u2 = ((z & np.uint64(0xFFFFFFFF)).astype(np.float64) + 0.5) * (1.0 / 4294967296.0)
    r = np.sqrt(-2.0 * np.log(u1))
    th = (2.0 * math.pi) * u2
    pair = np.empty(2 * m, dtype=np.float32)
    pair[0::2] = r * np.cos(th)
    pair[1::2] = r * np.sin(th)
    lo = 2 * p0
    hi = min(n, lo + 2 * m)
    out[lo:hi] = bf16_bits_of_f32(pair[: hi - lo])


@dataclasses.dataclass(frozen=True)
class Workload:
    """One synthetic DSA workload (prefill of one causal sequence, or a decode batch)."""
    name: str
    cid: int                 # stream id of the workload
    kind: str                # "prefill" or "decode"
    L: int                   # prefill length (decode: 0)
    d_idx: int               # index dimension
    idx_dtype: str           # "fp8" (E4M3) or "bf16"
    H: int
    D: int
    top_k: int
    local_boost: bool = False
    B: int = 0               # decode batch
    len_lo: int = 0          # decode cached lengths are uniform on [len_lo, len_hi]
    len_hi: int = 0


WORKLOADS = {
    "prefill_4k": Workload("prefill_4k", 1, "prefill", 4096, 128, "fp8", 4, 64, 256),
    "prefill_32k": Workload("prefill_32k", 2, "prefill", 32768, 96, "fp8", 16, 128, 1024),
    "prefill_64k": Workload("prefill_64k", 3, "prefill", 65536, 128, "fp8", 16, 128, 1536,
                            local_boost=True),
    "prefill_128k": Workload("prefill_128k", 4, "prefill", 131072, 160, "bf16", 16, 128, 2048),
    "decode_64x128k": Workload("decode_64x128k", 5, "decode", 0, 128, "fp8", 16, 128, 2048,
                               B=64, len_lo=65536, len_hi=131072),
    # the 128K per-row settings at 32K length: a capture-sized stand-in for profiling
    "prefill_32k_bf16": Workload("prefill_32k_bf16", 6, "prefill", 32768, 160, "bf16", 16, 128, 2048),
}

# tensor ids inside a workload's streams
_T_QIDX, _T_KIDX, _T_Q, _T_K, _T_V, _T_BOOST, _T_LEN = 1, 2, 3, 4, 5, 6, 7
_T_PAGE, _T_PAD_KIDX, _T_PAD_K, _T_PAD_V = 8, 9, 10, 11
_T_MQIDX, _T_MQ = 12, 13


def _encode_ints(v: np.ndarray, idx_dtype: str) -> np.ndarray:
    if idx_dtype == "fp8":
        return fp8_bytes_of_ints(v)
    if idx_dtype == "bf16":
        return bf16_bits_of_ints(v)
    raise ValueError(idx_dtype)


def _index_ints(w: Workload, seed: int, tid: int, rows: int) -> np.ndarray:
    key = stream_key(seed, w.cid, tid)
    return uniform_ints(key, rows * w.d_idx).reshape(rows, w.d_idx)


def prefill_inputs(w: Workload, seed: int = SEED, L: Optional[int] = None,
                   with_attention: bool = True) -> dict:
    """Host arrays of a prefill workload (optionally truncated to its first L rows).

    Returns q_idx/k_idx as uint8 (fp8) or uint16 (bf16 bits) [L, d_idx];
    Q [L, H, D], K [L, D], V [L, D] as uint16 BF16 bits.  Truncation keeps the
    draws of the full-size workload, so row t is identical at every L.
    """
    assert w.kind == "prefill"
    L = w.L if L is None else L
    qi = _index_ints(w, seed, _T_QIDX, L)
    ki = _index_ints(w, seed, _T_KIDX, L)
    if w.local_boost:
        # 128-aligned position blocks share one seeded vector in dims 0..31 of
        # both the query and key index rows.
        nblk = (L + 127) // 128
        u = uniform_ints(stream_key(seed, w.cid, _T_BOOST), nblk * 32).reshape(nblk, 32)
        blk = np.arange(L) // 128
        qi[:, :32] = u[blk]
        ki[:, :32] = u[blk]
    out = {
        "q_idx": _encode_ints(qi, w.idx_dtype),
        "k_idx": _encode_ints(ki, w.idx_dtype),
        "L": L,
    }
    if with_attention:
        out["Q"] = _prefix_normal(seed, w.cid, _T_Q, L * w.H * w.D).reshape(L, w.H, w.D)
        out["K"] = _prefix_normal(seed, w.cid, _T_K, L * w.D).reshape(L, w.D)
        out["V"] = _prefix_normal(seed, w.cid, _T_V, L * w.D).reshape(L, w.D)
    return out


def _prefix_normal(seed: int, cid: int, tid: int, n: int) -> np.ndarray:
    return normal_bf16(stream_key(seed, cid, tid), n)


def decode_lengths(w: Workload, seed: int = SEED) -> np.ndarray:
    key = stream_key(seed, w.cid, _T_LEN)
    return uniform_ints(key, w.B, w.len_lo, w.len_hi)


def decode_inputs(w: Workload, seed: int = SEED, lengths: Optional[np.ndarray] = None,
                  with_attention: bool = True) -> dict:
    """Host arrays of a decode batch.

    The cache is ragged and contiguous per sequence: rows seq_start[b] ..
    seq_start[b+1]-1 belong to sequence b.  Returns k_idx [sum_len, d_idx],
    K/V [sum_len, D], q_idx [B, d_idx], Q [B, H, D] and seq_start [B+1] int64.
    ``lengths`` overrides the drawn lengths (smaller test cases).
    """
    assert w.kind == "decode"
    if lengths is None:
        lengths = decode_lengths(w, seed)
    lengths = np.asarray(lengths, dtype=np.int64)
    B = lengths.shape[0]
    seq_start = np.zeros(B + 1, dtype=np.int64)
    seq_start[1:] = np.cumsum(lengths)
    total = int(seq_start[-1])
    ki = uniform_ints(stream_key(seed, w.cid, _T_KIDX), total * w.d_idx).reshape(total, w.d_idx)
    qi = uniform_ints(stream_key(seed, w.cid, _T_QIDX), B * w.d_idx).reshape(B, w.d_idx)
    out = {
        "k_idx": _encode_ints(ki, w.idx_dtype),
        "q_idx": _encode_ints(qi, w.idx_dtype),
        "seq_start": seq_start,
        "lengths": lengths,
        "B": B,
    }
    if with_attention:
        out["Q"] = _prefix_normal(seed, w.cid, _T_Q, B * w.H * w.D).reshape(B, w.H, w.D)
        out["K"] = _prefix_normal(seed, w.cid, _T_K, total * w.D).reshape(total, w.D)
        out["V"] = _prefix_normal(seed, w.cid, _T_V, total * w.D).reshape(total, w.D)
    return out


def multi_queries(w: Workload, B: int, T: int, seed: int = SEED) -> dict:
    """Queries of T new tokens per sequence for a decode batch: q_idx [B, T, d_idx]
    (integers in [-4, 4], encoded as the workload's index type) and Q [B, T, H, D]
    BF16 N(0, 1).  Token t of sequence b uses the t-th of T draws of its streams."""
    qi = uniform_ints(stream_key(seed, w.cid, _T_MQIDX, T), B * T * w.d_idx).reshape(B, T, w.d_idx)
    return {"q_idx": _encode_ints(qi, w.idx_dtype),
            "Q": _prefix_normal(seed, w.cid, _T_MQ * 16 + T, B * T * w.H * w.D).reshape(B, T, w.H, w.D)}


def multi_queries_torch(w: Workload, B: int, T: int, seed: int = SEED, device="cuda") -> dict:
    """multi_queries drawn on a device (same numbers)."""
    qi = uniform_ints_torch(stream_key(seed, w.cid, _T_MQIDX, T), B * T * w.d_idx, device=device)
    return {"q_idx": _encode_ints_torch(qi.view(B, T, w.d_idx), w.idx_dtype),
            "Q": normal_bf16_torch(stream_key(seed, w.cid, _T_MQ * 16 + T), B * T * w.H * w.D,
                                   device=device).view(B, T, w.H, w.D)}


def paged_layout(lengths, block_size: int, seed: int = SEED, spare_blocks: int = 3):
    """Placement of a decode batch in a block-paged cache.

    Sequence b occupies ceil(len_b / block_size) blocks of ``block_size`` rows.
    Those blocks, plus ``spare_blocks`` that no sequence uses, are shuffled by a
    seeded permutation (the order of splitmix64 draws), so neighbouring blocks
    of one sequence land at unrelated places in the pool.  Row s of sequence b
    is pool row ``block_table[b, s // block_size] * block_size + s % block_size``.

    Returns ``block_table`` [B, max_blocks] int32 (-1 past each sequence's last
    block) and ``src`` [num_blocks * block_size] int64: for every pool row, the
    row of the contiguous cache (sequences back to back, as decode_inputs lays
    them out) that it holds, or -1 for rows no sequence reaches.
    """
    lengths = np.asarray(lengths, dtype=np.int64)
    assert block_size >= 1 and (block_size & (block_size - 1)) == 0
    nblk = (lengths + block_size - 1) // block_size
    used = int(nblk.sum())
    n_total = used + spare_blocks
    order = np.argsort(draws(stream_key(seed, n_total, block_size, _T_PAGE), 0, n_total), kind="stable")
    B = lengths.shape[0]
    table = np.full((B, max(1, int(nblk.max()))), -1, dtype=np.int32)
    src = np.full(n_total * block_size, -1, dtype=np.int64)
    nxt, first = 0, 0
    for b in range(B):
        for j in range(int(nblk[b])):
            phys = int(order[nxt])
            nxt += 1
            table[b, j] = phys
            n = min(block_size, int(lengths[b]) - j * block_size)
            src[phys * block_size: phys * block_size + n] = first + j * block_size + np.arange(n)
        first += int(lengths[b])
    return table, src


def _fill_pool(rows: np.ndarray, src: np.ndarray, pad: np.ndarray) -> np.ndarray:
    out = pad.copy()
    m = src >= 0
    out[m] = rows[src[m]]
    return out


def paged_decode_inputs(w: Workload, lengths, block_size: int, seed: int = SEED,
                        spare_blocks: int = 3) -> dict:
    """decode_inputs placed in a block-paged cache (paged_layout).

    The rows are those of decode_inputs(w, seed, lengths); pool rows that no
    sequence reaches hold draws of their own streams, so a read of a wrong row
    changes scores and outputs.  Returns k_idx_blocks [num_blocks, block_size,
    d_idx], K_blocks / V_blocks [num_blocks, block_size, D], block_table,
    seq_lens [B] int32, q_idx, Q, lengths, B, block_size, and the contiguous
    inputs under "contiguous".
    """
    xd = decode_inputs(w, seed, lengths=lengths)
    table, src = paged_layout(xd["lengths"], block_size, seed, spare_blocks)
    nrows = src.shape[0]
    nb = nrows // block_size
    pad_i = _encode_ints(uniform_ints(stream_key(seed, w.cid, _T_PAD_KIDX), nrows * w.d_idx)
                         .reshape(nrows, w.d_idx), w.idx_dtype)
    pad_k = _prefix_normal(seed, w.cid, _T_PAD_K, nrows * w.D).reshape(nrows, w.D)
    pad_v = _prefix_normal(seed, w.cid, _T_PAD_V, nrows * w.D).reshape(nrows, w.D)
    return {
        "k_idx_blocks": _fill_pool(xd["k_idx"], src, pad_i).reshape(nb, block_size, w.d_idx),
        "K_blocks": _fill_pool(xd["K"], src, pad_k).reshape(nb, block_size, w.D),
        "V_blocks": _fill_pool(xd["V"], src, pad_v).reshape(nb, block_size, w.D),
        "block_table": table,
        "seq_lens": xd["lengths"].astype(np.int32),
        "q_idx": xd["q_idx"], "Q": xd["Q"], "lengths": xd["lengths"], "B": xd["B"],
        "block_size": block_size, "contiguous": xd,
    }


# ---------------------------------------------------------------------------
# The same generators written with torch integer/float ops, so large inputs can
# be drawn directly on a device.  Definitions match the numpy ones above draw
# for draw (64-bit wrapping arithmetic in int64, logical shifts emulated).

def _to_i64(u: int) -> int:
    u &= 0xFFFFFFFFFFFFFFFF
    return u - (1 << 64) if u >= (1 << 63) else u


_M1_I, _M2_I, _G_I = _to_i64(0xBF58476D1CE4E5B9), _to_i64(0x94D049BB133111EB), _to_i64(0x9E3779B97F4A7C15)


def _srl(x, s: int):
    return (x >> s) & ((1 << (64 - s)) - 1)


def draws_torch(key, start: int, n: int, device):
    import torch
    i = torch.arange(start + 1, start + n + 1, dtype=torch.int64, device=device)
    z = i * _G_I + _to_i64(int(key))
    z = (z ^ _srl(z, 30)) * _M1_I
    z = (z ^ _srl(z, 27)) * _M2_I
    return z ^ _srl(z, 31)


def uniform_ints_torch(key, n: int, lo: int = -4, hi: int = 4, device="cuda", chunk: int = 1 << 26):
    import torch
    out = torch.empty(n, dtype=torch.int8, device=device)
    for s in range(0, n, chunk):
        m = min(chunk, n - s)
        top = _srl(draws_torch(key, s, m, device), 32)
        out[s:s + m] = ((top * (hi - lo + 1)) >> 32).to(torch.int8) + lo
    return out


def normal_bf16_torch(key, n: int, device="cuda", chunk: int = 1 << 25):
    """N(0,1) as a torch.bfloat16 tensor on `device` (same draws as normal_bf16)."""
    import torch
    out = torch.empty(n, dtype=torch.bfloat16, device=device)
    npairs = (n + 1) // 2
    for p0 in range(0, npairs, chunk):
        m = min(chunk, npairs - p0)
        z = draws_torch(key, p0, m, device)
        u1 = (_srl(z, 32).to(torch.float64) + 0.5) * (1.0 / 4294967296.0)
        u2 = ((z & 0xFFFFFFFF).to(torch.float64) + 0.5) * (1.0 / 4294967296.0)
        r = torch.sqrt(-2.0 * torch.log(u1))
        th = (2.0 * math.pi) * u2
        pair = torch.stack([(r * torch.cos(th)).to(torch.float32),
                            (r * torch.sin(th)).to(torch.float32)], dim=1).reshape(-1)
        lo = 2 * p0
        hi = min(n, lo + 2 * m)
        out[lo:hi] = pair[: hi - lo].to(torch.bfloat16)
    return out


def _encode_ints_torch(v, idx_dtype: str):
    import torch
    if idx_dtype == "fp8":
        return v.to(torch.float8_e4m3fn).view(torch.uint8)
    return v.to(torch.bfloat16)


def prefill_inputs_torch(w: Workload, seed: int = SEED, device="cuda") -> dict:
    """prefill_inputs drawn on a device: uint8 / bfloat16 torch tensors."""
    import torch
    L = w.L
    qi = uniform_ints_torch(stream_key(seed, w.cid, _T_QIDX), L * w.d_idx, device=device).view(L, w.d_idx)
    ki = uniform_ints_torch(stream_key(seed, w.cid, _T_KIDX), L * w.d_idx, device=device).view(L, w.d_idx)
    if w.local_boost:
        nblk = (L + 127) // 128
        u = uniform_ints_torch(stream_key(seed, w.cid, _T_BOOST), nblk * 32, device=device).view(nblk, 32)
        blk = torch.arange(L, device=device) // 128
        qi[:, :32] = u[blk]
        ki[:, :32] = u[blk]
    return {
        "q_idx": _encode_ints_torch(qi, w.idx_dtype), "k_idx": _encode_ints_torch(ki, w.idx_dtype), "L": L,
        "Q": normal_bf16_torch(stream_key(seed, w.cid, _T_Q), L * w.H * w.D, device).view(L, w.H, w.D),
        "K": normal_bf16_torch(stream_key(seed, w.cid, _T_K), L * w.D, device).view(L, w.D),
        "V": normal_bf16_torch(stream_key(seed, w.cid, _T_V), L * w.D, device).view(L, w.D),
    }


def decode_inputs_torch(w: Workload, seed: int = SEED, device="cuda") -> dict:
    """decode_inputs drawn on a device (drawn lengths)."""
    import torch
    lengths = decode_lengths(w, seed)
    B = lengths.shape[0]
    seq_start = np.zeros(B + 1, dtype=np.int64)
    seq_start[1:] = np.cumsum(lengths)
    total = int(seq_start[-1])
    ki = uniform_ints_torch(stream_key(seed, w.cid, _T_KIDX), total * w.d_idx, device=device)
    qi = uniform_ints_torch(stream_key(seed, w.cid, _T_QIDX), B * w.d_idx, device=device)
    return {
        "k_idx": _encode_ints_torch(ki, w.idx_dtype).view(total, w.d_idx),
        "q_idx": _encode_ints_torch(qi, w.idx_dtype).view(B, w.d_idx),
        "seq_start": torch.from_numpy(seq_start).to(device), "lengths": lengths, "B": B,
        "Q": normal_bf16_torch(stream_key(seed, w.cid, _T_Q), B * w.H * w.D, device).view(B, w.H, w.D),
        "K": normal_bf16_torch(stream_key(seed, w.cid, _T_K), total * w.D, device).view(total, w.D),
        "V": normal_bf16_torch(stream_key(seed, w.cid, _T_V), total * w.D, device).view(total, w.D),
    }


def paged_decode_inputs_torch(xd: dict, block_size: int, seed: int = SEED, spare_blocks: int = 3) -> dict:
    """A device copy of a decode batch (decode_inputs_torch) placed in a block-paged
    cache by paged_layout; rows no sequence reaches are zero."""
    import torch
    table, src = paged_layout(xd["lengths"], block_size, seed, spare_blocks)
    dev = xd["k_idx"].device
    s = torch.from_numpy(src).to(dev)
    m = s >= 0

    def pool(x):
        out = x.new_zeros((s.numel(),) + tuple(x.shape[1:]))
        out[m] = x[s[m]]
        return out.view((s.numel() // block_size, block_size) + tuple(x.shape[1:]))

    return {
        "k_idx_blocks": pool(xd["k_idx"]), "K_blocks": pool(xd["K"]), "V_blocks": pool(xd["V"]),
        "block_table": torch.from_numpy(table).to(dev),
        "seq_lens": torch.from_numpy(np.asarray(xd["lengths"], dtype=np.int32)).to(dev),
        "q_idx": xd["q_idx"], "Q": xd["Q"], "lengths": xd["lengths"], "B": xd["B"],
        "block_size": block_size,
    }
