"""DSA oracle — test infrastructure only.

Python access (ctypes) to ``dsa_oracle.cpp``, the plain CPU restatement of
DeepSeek Sparse Attention (lightning indexer -> top-k -> softmax attention over
the selected keys, one MQA-shared K/V) from the DeepSeek Sparse Attention page
(kwkr.cn/news/60693, sections 3.2, 3.3, 4.1 and 4.2).

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline leg
may import this module.  The CUDA path never does.  Parity status: pinned.
"""
from __future__ import annotations

import ctypes
import math
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "dsa_oracle.cpp")
_LIB = os.path.join(_HERE, "libdsa_oracle.so")

IDX_DTYPES = {"fp8": 0, "bf16": 1}

_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle (g++ -O2, OpenMP, no FP contraction) next to its source."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        cmd = ["g++", "-std=c++17", "-O2", "-fopenmp", "-ffp-contract=off", "-fno-fast-math",
               "-shared", "-fPIC", _SRC, "-o", _LIB + ".tmp"]
        subprocess.check_call(cmd)
        os.replace(_LIB + ".tmp", _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB)
        P, I, I64, F, D = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_float, ctypes.c_double
        lib.oracle_fp8_e4m3_value.argtypes = [ctypes.c_uint8]
        lib.oracle_fp8_e4m3_value.restype = D
        lib.oracle_bf16_value.argtypes = [ctypes.c_uint16]
        lib.oracle_bf16_value.restype = D
        lib.oracle_bf16_round.argtypes = [D]
        lib.oracle_bf16_round.restype = ctypes.c_uint16
        lib.oracle_indexer_scores.argtypes = [P, P, I, I, F, I64, I64, P, I]
        lib.oracle_indexer_scores.restype = None
        lib.oracle_prefill_rows.argtypes = [P, P, I, I, F, P, P, P, I64, I, I, D, I, P, I64, P, P, I]
        lib.oracle_prefill_rows.restype = None
        lib.oracle_decode.argtypes = [P, P, P, P, I, I, I, I, P, P, I, I, F, D, P, P, I]
        lib.oracle_decode.restype = None
        lib.oracle_max_threads.argtypes = []
        lib.oracle_max_threads.restype = I
        _lib = lib
    return _lib


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def default_index_scale(d: int) -> float:
    """d^-0.5 rounded to float32 (the indexer's scale, section 3.2)."""
    return float(np.float32(1.0 / math.sqrt(d)))


def max_threads() -> int:
    return _load().oracle_max_threads()


def fp8_e4m3_value(b: int) -> float:
    return _load().oracle_fp8_e4m3_value(b)


def bf16_value(h: int) -> float:
    return _load().oracle_bf16_value(h)


def bf16_round(x: float) -> int:
    return _load().oracle_bf16_round(x)


def indexer_scores(q_idx, k_idx, idx_dtype: str, scale=None, nthreads: int = 0) -> np.ndarray:
    """Dense [Lq, Lk] relu(fp32(q.k) * scale) with no mask."""
    q_idx = np.ascontiguousarray(q_idx)
    k_idx = np.ascontiguousarray(k_idx)
    Lq, d = q_idx.shape
    Lk = k_idx.shape[0]
    scale = default_index_scale(d) if scale is None else scale
    out = np.empty((Lq, Lk), dtype=np.float32)
    _load().oracle_indexer_scores(_ptr(q_idx), _ptr(k_idx), IDX_DTYPES[idx_dtype], d, scale,
                                  Lq, Lk, _ptr(out), nthreads)
    return out


def prefill_rows(inp: dict, idx_dtype: str, top_k: int, rows=None, H=None, D=None,
                 idx_scale=None, attn_scale=None, want_o: bool = True, nthreads: int = 0):
    """Indices [n, top_k] int32 and O [n, H, D] (BF16 bits) for the listed rows."""
    q_idx = np.ascontiguousarray(inp["q_idx"])
    k_idx = np.ascontiguousarray(inp["k_idx"])
    L, d = q_idx.shape
    rows = np.arange(L, dtype=np.int64) if rows is None else np.ascontiguousarray(rows, dtype=np.int64)
    n = rows.shape[0]
    idx_scale = default_index_scale(d) if idx_scale is None else idx_scale
    indices = np.empty((n, top_k), dtype=np.int32)
    O = None
    Q = K = V = None
    if want_o:
        Q = np.ascontiguousarray(inp["Q"])
        K = np.ascontiguousarray(inp["K"])
        V = np.ascontiguousarray(inp["V"])
        H = Q.shape[1] if H is None else H
        D = Q.shape[2] if D is None else D
        O = np.empty((n, H, D), dtype=np.uint16)
    else:
        H = H or 1
        D = D or 1
    attn_scale = 1.0 / math.sqrt(D) if attn_scale is None else attn_scale
    _load().oracle_prefill_rows(_ptr(q_idx), _ptr(k_idx), IDX_DTYPES[idx_dtype], d, idx_scale,
                                _ptr(Q), _ptr(K), _ptr(V), L, H, D, attn_scale, top_k,
                                _ptr(rows), n, _ptr(indices), _ptr(O), nthreads)
    return indices, O


def decode(inp: dict, idx_dtype: str, top_k: int, idx_scale=None, attn_scale=None,
           want_o: bool = True, nthreads: int = 0):
    """Indices [B, top_k] int32 and O [B, H, D] (BF16 bits) of one decode step."""
    k_idx = np.ascontiguousarray(inp["k_idx"])
    q_idx = np.ascontiguousarray(inp["q_idx"])
    seq_start = np.ascontiguousarray(inp["seq_start"], dtype=np.int64)
    B, d = q_idx.shape
    idx_scale = default_index_scale(d) if idx_scale is None else idx_scale
    indices = np.empty((B, top_k), dtype=np.int32)
    Q = K = V = O = None
    H = D = 1
    if want_o:
        Q = np.ascontiguousarray(inp["Q"])
        K = np.ascontiguousarray(inp["K"])
        V = np.ascontiguousarray(inp["V"])
        H, D = Q.shape[1], Q.shape[2]
        O = np.empty((B, H, D), dtype=np.uint16)
    attn_scale = 1.0 / math.sqrt(D) if attn_scale is None else attn_scale
    _load().oracle_decode(_ptr(k_idx), _ptr(K), _ptr(V), _ptr(seq_start), B, IDX_DTYPES[idx_dtype],
                          d, D, _ptr(q_idx), _ptr(Q), H, top_k, idx_scale, attn_scale,
                          _ptr(indices), _ptr(O), nthreads)
    return indices, O


def decode_multi(inp: dict, idx_dtype: str, top_k: int, idx_scale=None, attn_scale=None,
                 want_o: bool = True, nthreads: int = 0):
    """One decode step with T new tokens per sequence: indices [B, T, top_k], O [B, T, H, D].

    inp holds the contiguous cache (k_idx, K, V, seq_start) and q_idx [B, T, d],
    Q [B, T, H, D].  The new tokens are the last T rows of each sequence; token j
    sits at position len_b - T + j and, as any query of the DeepSeek Sparse
    Attention page (sections 3.2-3.3), sees the rows up to its own position.
    Each token is an ordinary decode over its causal prefix of the sequence.
    """
    q_idx = np.asarray(inp["q_idx"])
    B, T, d = q_idx.shape
    ss = np.asarray(inp["seq_start"], dtype=np.int64)
    rows, starts = [], [0]
    for b in range(B):
        n_b = int(ss[b + 1] - ss[b])
        for j in range(T):
            n = n_b - T + 1 + j
            rows.append(np.arange(ss[b], ss[b] + n, dtype=np.int64))
            starts.append(starts[-1] + n)
    rows = np.concatenate(rows)
    flat = {"k_idx": np.asarray(inp["k_idx"])[rows], "q_idx": q_idx.reshape(B * T, d),
            "seq_start": np.asarray(starts, dtype=np.int64)}
    if want_o:
        Q = np.asarray(inp["Q"])
        flat["K"] = np.asarray(inp["K"])[rows]
        flat["V"] = np.asarray(inp["V"])[rows]
        flat["Q"] = Q.reshape((B * T,) + Q.shape[2:])
    idx, O = decode(flat, idx_dtype, top_k, idx_scale, attn_scale, want_o, nthreads)
    return idx.reshape(B, T, top_k), (None if O is None else O.reshape((B, T) + O.shape[1:]))


def decode_paged(inp: dict, idx_dtype: str, top_k: int, idx_scale=None, attn_scale=None,
                 want_o: bool = True, nthreads: int = 0):
    """One decode step over a block-paged cache: indices [B, top_k] and O [B, H, D].

    The DeepSeek Sparse Attention page (section 4.2) keeps the cache in token
    blocks laid out on 128-byte boundaries.  Read here as: row s of sequence b
    lives in block ``block_table[b, s // block_size]`` at offset
    ``s % block_size`` of pools shaped [num_blocks, block_size, ...].  The
    oracle reads each sequence's rows out in order and takes the ordinary
    decode step on them; indices are positions within the sequence.
    """
    table = np.asarray(inp["block_table"])
    lens = np.asarray(inp["seq_lens"], dtype=np.int64)
    bs = inp["k_idx_blocks"].shape[1]
    rows = []
    for b in range(lens.shape[0]):
        s = np.arange(int(lens[b]))
        rows.append(table[b, s // bs].astype(np.int64) * bs + s % bs)
    rows = np.concatenate(rows)
    seq_start = np.zeros(lens.shape[0] + 1, dtype=np.int64)
    seq_start[1:] = np.cumsum(lens)
    flat = {"k_idx": inp["k_idx_blocks"].reshape(-1, inp["k_idx_blocks"].shape[2])[rows],
            "q_idx": inp["q_idx"], "seq_start": seq_start}
    if want_o:
        D = inp["K_blocks"].shape[2]
        flat["K"] = inp["K_blocks"].reshape(-1, D)[rows]
        flat["V"] = inp["V_blocks"].reshape(-1, D)[rows]
        flat["Q"] = inp["Q"]
    return decode(flat, idx_dtype, top_k, idx_scale, attn_scale, want_o, nthreads)
