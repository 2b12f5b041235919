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
from typing import Optional

import numpy as np

__all__ = [
    "GOLDEN", "SEED", "mix64", "draws", "uniform_ints", "fp8_bytes_of_ints",
    "bf16_bits_of_ints", "bf16_bits_of_f32", "normal_bf16", "Workload",
    "WORKLOADS", "prefill_inputs", "decode_inputs", "decode_lengths", "stream_key",
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


def normal_bf16(key: np.uint64, n: int, chunk: int = 1 << 24) -> np.ndarray:
    """n N(0,1) values as BF16 bit patterns (Box-Muller, both outputs of a pair)."""
    out = np.empty(n, dtype=np.uint16)
    npairs = (n + 1) // 2
    two_pi = 2.0 * math.pi
    for p0 in range(0, npairs, chunk):
        m = min(chunk, npairs - p0)
        z = draws(key, p0, m)
        u1 = ((z >> np.uint64(32)).astype(np.float64) + 0.5) * (1.0 / 4294967296.0)
        u2 = ((z & np.uint64(0xFFFFFFFF)).astype(np.float64) + 0.5) * (1.0 / 4294967296.0)
        r = np.sqrt(-2.0 * np.log(u1))
        th = two_pi * u2
        pair = np.empty(2 * m, dtype=np.float32)
        pair[0::2] = r * np.cos(th)
        pair[1::2] = r * np.sin(th)
        lo = 2 * p0
        hi = min(n, lo + 2 * m)
        out[lo:hi] = bf16_bits_of_f32(pair[: hi - lo])
    return out


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
}

# tensor ids inside a workload's streams
_T_QIDX, _T_KIDX, _T_Q, _T_K, _T_V, _T_BOOST, _T_LEN = 1, 2, 3, 4, 5, 6, 7


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
