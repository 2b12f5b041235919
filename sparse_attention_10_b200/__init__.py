"""B200 (sm_100a) DeepSeek Sparse Attention: lightning indexer -> top-k -> sparse MQA attention.

Thin Python binding of the C ABI in ``include/dsa.h`` (``libdsa.so``).  Every
function here only marshals arguments: all arithmetic runs in the library's
CUDA kernels.  PyTorch provides device memory and streams.  There is no CPU
path: a missing library or a CPU tensor raises.
"""
from __future__ import annotations

import ctypes
import math
import os
from typing import Optional, Tuple

import torch

__all__ = [
    "DsaError", "load", "dsa_version", "dsa_status_string", "dsa_indexer_scores",
    "dsa_prefill_workspace_size", "dsa_prefill", "dsa_decode_workspace_size", "dsa_decode",
    "dsa_sync_status", "dsa_last_stats", "dsa_debug_wait_timeout", "dsa_debug_force_fallback", "IDX_FP8_E4M3", "IDX_BF16",
    "LIB_PATH", "dsa_stage_timing", "dsa_stage_times", "STAGES", "dsa_decode_static",
    "dsa_decode_paged_workspace_size", "dsa_decode_paged", "dsa_gather_probe",
    "dsa_prefill_chunk_workspace_size", "dsa_prefill_chunk", "dsa_index_to_fp8",
    "dsa_decode_multi_workspace_size", "dsa_decode_multi", "dsa_decode_paged_multi_workspace_size",
    "dsa_decode_paged_multi",
]

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libdsa.so")
IDX_FP8_E4M3 = 0
IDX_BF16 = 1
STATUS = {0: "DSA_OK", 1: "DSA_ERR_INVALID_ARG", 2: "DSA_ERR_UNSUPPORTED", 3: "DSA_ERR_WORKSPACE",
          4: "DSA_ERR_CUDA", 5: "DSA_ERR_TIMEOUT", 6: "DSA_ERR_DEVICE"}

_lib = None


class DsaError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {STATUS.get(status, status)}")


def load() -> ctypes.CDLL:
    """Load libdsa.so (build it first with ``sparse_attention_10_b200.build``)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"CUDA library not built: {LIB_PATH} (run __graft_entry__.build())")
    lib = ctypes.CDLL(LIB_PATH)
    P, I, I64, F, SZ = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_float, ctypes.c_size_t
    sigs = {
        "dsa_status_string": ([I], ctypes.c_char_p),
        "dsa_version": ([], ctypes.c_char_p),
        "dsa_indexer_scores": ([P, P, I, I, F, I64, I64, P, P], I),
        "dsa_prefill_workspace_size": ([I64, I, I, I, I, I], SZ),
        "dsa_prefill": ([P, P, I, I, F, P, P, P, I64, I, I, F, I, P, P, P, SZ, P], I),
        "dsa_prefill_chunk_workspace_size": ([I64, I64, I, I, I, I, I], SZ),
        "dsa_prefill_chunk": ([P, P, I, I, F, P, P, P, I64, I64, I, I, F, I, P, P, P, SZ, P], I),
        "dsa_decode_workspace_size": ([I, I64, I, I, I, I, I], SZ),
        "dsa_decode_multi_workspace_size": ([I, I, I64, I, I, I, I, I], SZ),
        "dsa_decode_multi": ([P, P, P, P, I, I, I64, I64, I, I, I, P, P, I, I, F, F, P, P, P, SZ, P], I),
        "dsa_decode_paged_multi_workspace_size": ([I, I, I64, I, I, I, I, I], SZ),
        "dsa_decode_paged_multi": ([P, P, P, I64, I, P, I, P, I, I, I64, I, I, I, P, P, I, I, F, F, P, P, P,
                                    SZ, P], I),
        "dsa_decode": ([P, P, P, P, I, I64, I64, I, I, I, P, P, I, I, F, F, P, P, P, SZ, P], I),
        "dsa_sync_status": ([P], I),
        "dsa_last_stats": ([P, ctypes.POINTER(ctypes.c_int64), P], I),
        "dsa_debug_wait_timeout": ([ctypes.c_uint64, P], I),
        "dsa_debug_force_fallback": ([I], I),
        "dsa_decode_static": ([P, P, P, P, I, I64, I64, I, I, I, P, P, I, I, F, F, P, P, P], I),
        "dsa_decode_paged_workspace_size": ([I, I64, I, I, I, I, I], SZ),
        "dsa_decode_paged": ([P, P, P, I64, I, P, I, P, I, I64, I, I, I, P, P, I, I, F, F, P, P, P, SZ,
                              P], I),
        "dsa_gather_probe": ([P, I64, I, P, P, I, I, I, P, P], I),
        "dsa_index_to_fp8": ([P, I64, P, P, P], I),
        "dsa_stage_timing": ([I], I),
        "dsa_stage_times": ([ctypes.POINTER(ctypes.c_double), ctypes.POINTER(ctypes.c_int64), I], I),
    }
    for name, (args, res) in sigs.items():
        fn = getattr(lib, name)
        fn.argtypes = args
        fn.restype = res
    _lib = lib
    return lib


def _check(status: int, where: str) -> None:
    if status != 0:
        raise DsaError(status, where)


def _dev(t: torch.Tensor, name: str) -> int:
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t.data_ptr()


def _stream(stream) -> int:
    s = torch.cuda.current_stream() if stream is None else stream
    return s.cuda_stream


def _idx_dtype(t: torch.Tensor) -> int:
    if t.dtype in (torch.uint8, torch.float8_e4m3fn):
        return IDX_FP8_E4M3
    if t.dtype in (torch.bfloat16, torch.int16, torch.uint16):
        return IDX_BF16
    raise ValueError(f"index tensors must be FP8 E4M3 (uint8) or BF16, got {t.dtype}")


def _scale(x: Optional[float]) -> float:
    return float("nan") if x is None else float(x)


def dsa_version() -> str:
    return load().dsa_version().decode()


def dsa_status_string(status: int) -> str:
    return load().dsa_status_string(status).decode()


def dsa_indexer_scores(q_idx: torch.Tensor, k_idx: torch.Tensor, idx_scale: Optional[float] = None,
                       out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """Dense relu(fp32(q_idx @ k_idx^T) * scale), [Lq, Lk] float32 (no mask)."""
    lib = load()
    Lq, d = q_idx.shape
    Lk = k_idx.shape[0]
    if out is None:
        out = torch.empty((Lq, Lk), dtype=torch.float32, device=q_idx.device)
    st = lib.dsa_indexer_scores(_dev(q_idx, "q_idx"), _dev(k_idx, "k_idx"), _idx_dtype(q_idx), d,
                                _scale(idx_scale), Lq, Lk, _dev(out, "out"), _stream(stream))
    _check(st, "dsa_indexer_scores")
    return out


def dsa_prefill_workspace_size(L: int, d_idx: int, idx_dtype: int, H: int, D: int, top_k: int) -> int:
    return int(load().dsa_prefill_workspace_size(L, d_idx, idx_dtype, H, D, top_k))


def dsa_prefill(q_idx: torch.Tensor, k_idx: torch.Tensor, Q: torch.Tensor, K: torch.Tensor,
                V: torch.Tensor, top_k: int, idx_scale: Optional[float] = None,
                attn_scale: Optional[float] = None, indices: Optional[torch.Tensor] = None,
                O: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None,
                stream=None) -> Tuple[torch.Tensor, torch.Tensor]:
    """DSA prefill of one causal sequence -> (indices [L, top_k] int32, O [L, H, D] bf16)."""
    lib = load()
    L, d = q_idx.shape
    _, H, D = Q.shape
    idt = _idx_dtype(q_idx)
    dev = q_idx.device
    if indices is None:
        indices = torch.empty((L, top_k), dtype=torch.int32, device=dev)
    if O is None:
        O = torch.empty((L, H, D), dtype=torch.bfloat16, device=dev)
    need = dsa_prefill_workspace_size(L, d, idt, H, D, top_k)
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=dev)
    st = lib.dsa_prefill(_dev(q_idx, "q_idx"), _dev(k_idx, "k_idx"), idt, d, _scale(idx_scale),
                         _dev(Q, "Q"), _dev(K, "K"), _dev(V, "V"), L, H, D, _scale(attn_scale), top_k,
                         _dev(indices, "indices"), _dev(O, "O"), _dev(workspace, "workspace"),
                         workspace.numel() * workspace.element_size(), _stream(stream))
    _check(st, "dsa_prefill")
    return indices, O


def dsa_prefill_chunk_workspace_size(Lq: int, Lk: int, d_idx: int, idx_dtype: int, H: int, D: int,
                                     top_k: int) -> int:
    return int(load().dsa_prefill_chunk_workspace_size(Lq, Lk, d_idx, idx_dtype, H, D, top_k))


def dsa_prefill_chunk(q_idx: torch.Tensor, k_idx: torch.Tensor, Q: torch.Tensor, K: torch.Tensor,
                      V: torch.Tensor, top_k: int, idx_scale: Optional[float] = None,
                      attn_scale: Optional[float] = None, indices: Optional[torch.Tensor] = None,
                      O: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None,
                      stream=None) -> Tuple[torch.Tensor, torch.Tensor]:
    """DSA for the last Lq positions of a causal sequence of Lk = k_idx.shape[0] tokens
    (query row i at key position Lk - Lq + i) -> (indices [Lq, top_k], O [Lq, H, D])."""
    lib = load()
    Lq, d = q_idx.shape
    Lk = k_idx.shape[0]
    _, H, D = Q.shape
    idt = _idx_dtype(q_idx)
    dev = q_idx.device
    if indices is None:
        indices = torch.empty((Lq, top_k), dtype=torch.int32, device=dev)
    if O is None:
        O = torch.empty((Lq, H, D), dtype=torch.bfloat16, device=dev)
    if workspace is None:
        workspace = torch.empty(dsa_prefill_chunk_workspace_size(Lq, Lk, d, idt, H, D, top_k),
                                dtype=torch.uint8, device=dev)
    st = lib.dsa_prefill_chunk(_dev(q_idx, "q_idx"), _dev(k_idx, "k_idx"), idt, d, _scale(idx_scale),
                               _dev(Q, "Q"), _dev(K, "K"), _dev(V, "V"), Lq, Lk, H, D, _scale(attn_scale),
                               top_k, _dev(indices, "indices"), _dev(O, "O"), _dev(workspace, "workspace"),
                               workspace.numel() * workspace.element_size(), _stream(stream))
    _check(st, "dsa_prefill_chunk")
    return indices, O


def dsa_decode_workspace_size(B: int, total_rows: int, d_idx: int, idx_dtype: int, H: int, D: int,
                              top_k: int) -> int:
    return int(load().dsa_decode_workspace_size(B, total_rows, d_idx, idx_dtype, H, D, top_k))


def dsa_decode(k_idx: torch.Tensor, K: torch.Tensor, V: torch.Tensor, seq_start: torch.Tensor,
               q_idx: torch.Tensor, Q: torch.Tensor, top_k: int, max_len: int,
               idx_scale: Optional[float] = None, attn_scale: Optional[float] = None,
               O: Optional[torch.Tensor] = None, indices: Optional[torch.Tensor] = None,
               want_indices: bool = True, workspace: Optional[torch.Tensor] = None,
               stream=None) -> Tuple[torch.Tensor, Optional[torch.Tensor]]:
    """One decode step over a ragged cache -> (O [B, H, D] bf16, indices [B, top_k] or None)."""
    lib = load()
    B, d = q_idx.shape
    _, H, D = Q.shape
    total = k_idx.shape[0]
    idt = _idx_dtype(q_idx)
    dev = q_idx.device
    if O is None:
        O = torch.empty((B, H, D), dtype=torch.bfloat16, device=dev)
    if indices is None and want_indices:
        indices = torch.empty((B, top_k), dtype=torch.int32, device=dev)
    need = dsa_decode_workspace_size(B, total, d, idt, H, D, top_k)
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=dev)
    if seq_start.dtype != torch.int64:
        raise ValueError("seq_start must be int64")
    st = lib.dsa_decode(_dev(k_idx, "k_idx"), _dev(K, "K"), _dev(V, "V"), _dev(seq_start, "seq_start"),
                        B, total, int(max_len), idt, d, D, _dev(q_idx, "q_idx"), _dev(Q, "Q"), H, top_k,
                        _scale(idx_scale), _scale(attn_scale), _dev(O, "O"),
                        _dev(indices, "indices") if indices is not None else None,
                        _dev(workspace, "workspace"), workspace.numel() * workspace.element_size(),
                        _stream(stream))
    _check(st, "dsa_decode")
    return O, indices


def dsa_decode_paged_workspace_size(B: int, max_len: int, d_idx: int, idx_dtype: int, H: int, D: int,
                                    top_k: int) -> int:
    return int(load().dsa_decode_paged_workspace_size(B, max_len, d_idx, idx_dtype, H, D, top_k))


def dsa_decode_paged(k_idx: torch.Tensor, K: torch.Tensor, V: torch.Tensor, block_table: torch.Tensor,
                     seq_lens: torch.Tensor, q_idx: torch.Tensor, Q: torch.Tensor, top_k: int, max_len: int,
                     idx_scale: Optional[float] = None, attn_scale: Optional[float] = None,
                     O: Optional[torch.Tensor] = None, indices: Optional[torch.Tensor] = None,
                     want_indices: bool = True, workspace: Optional[torch.Tensor] = None,
                     stream=None) -> Tuple[torch.Tensor, Optional[torch.Tensor]]:
    """One decode step over a block-paged cache -> (O [B, H, D] bf16, indices [B, top_k] or None).

    k_idx [num_blocks, block_size, d_idx], K/V [num_blocks, block_size, D],
    block_table [B, max_blocks] int32, seq_lens [B] int32 (all on the device)."""
    lib = load()
    B, d = q_idx.shape
    _, H, D = Q.shape
    num_blocks, block_size = k_idx.shape[0], k_idx.shape[1]
    if block_table.dtype != torch.int32 or seq_lens.dtype != torch.int32:
        raise ValueError("block_table and seq_lens must be int32")
    if block_table.dim() != 2 or block_table.shape[0] != B or seq_lens.shape != (B,):
        raise ValueError("block_table must be [B, max_blocks] and seq_lens [B]")
    idt = _idx_dtype(q_idx)
    dev = q_idx.device
    if O is None:
        O = torch.empty((B, H, D), dtype=torch.bfloat16, device=dev)
    if indices is None and want_indices:
        indices = torch.empty((B, top_k), dtype=torch.int32, device=dev)
    if workspace is None:
        need = dsa_decode_paged_workspace_size(B, int(max_len), d, idt, H, D, top_k)
        workspace = torch.empty(need, dtype=torch.uint8, device=dev)
    st = lib.dsa_decode_paged(_dev(k_idx, "k_idx"), _dev(K, "K"), _dev(V, "V"), num_blocks, block_size,
                              _dev(block_table, "block_table"), block_table.shape[1],
                              _dev(seq_lens, "seq_lens"), B, int(max_len), idt, d, D, _dev(q_idx, "q_idx"),
                              _dev(Q, "Q"), H, top_k, _scale(idx_scale), _scale(attn_scale), _dev(O, "O"),
                              _dev(indices, "indices") if indices is not None else None,
                              _dev(workspace, "workspace"), workspace.numel() * workspace.element_size(),
                              _stream(stream))
    _check(st, "dsa_decode_paged")
    return O, indices


def dsa_decode_multi_workspace_size(B: int, T: int, total_rows: int, d_idx: int, idx_dtype: int, H: int, D: int,
                                    top_k: int) -> int:
    return int(load().dsa_decode_multi_workspace_size(B, T, total_rows, d_idx, idx_dtype, H, D, top_k))


def dsa_decode_paged_multi_workspace_size(B: int, T: int, max_len: int, d_idx: int, idx_dtype: int, H: int,
                                          D: int, top_k: int) -> int:
    return int(load().dsa_decode_paged_multi_workspace_size(B, T, max_len, d_idx, idx_dtype, H, D, top_k))


def dsa_decode_multi(k_idx: torch.Tensor, K: torch.Tensor, V: torch.Tensor, seq_start: torch.Tensor,
                     q_idx: torch.Tensor, Q: torch.Tensor, top_k: int, max_len: int,
                     idx_scale: Optional[float] = None, attn_scale: Optional[float] = None,
                     O: Optional[torch.Tensor] = None, indices: Optional[torch.Tensor] = None,
                     want_indices: bool = True, workspace: Optional[torch.Tensor] = None,
                     stream=None) -> Tuple[torch.Tensor, Optional[torch.Tensor]]:
    """One decode step with T new tokens per sequence (q_idx [B, T, d], Q [B, T, H, D]) over a
    ragged contiguous cache -> (O [B, T, H, D] bf16, indices [B, T, top_k] or None)."""
    lib = load()
    B, T, d = q_idx.shape
    _, _, H, D = Q.shape
    total = k_idx.shape[0]
    idt = _idx_dtype(q_idx)
    dev = q_idx.device
    if O is None:
        O = torch.empty((B, T, H, D), dtype=torch.bfloat16, device=dev)
    if indices is None and want_indices:
        indices = torch.empty((B, T, top_k), dtype=torch.int32, device=dev)
    if workspace is None:
        workspace = torch.empty(int(lib.dsa_decode_multi_workspace_size(B, T, total, d, idt, H, D, top_k)),
                                dtype=torch.uint8, device=dev)
    if seq_start.dtype != torch.int64:
        raise ValueError("seq_start must be int64")
    st = lib.dsa_decode_multi(_dev(k_idx, "k_idx"), _dev(K, "K"), _dev(V, "V"), _dev(seq_start, "seq_start"),
                              B, T, total, int(max_len), idt, d, D, _dev(q_idx, "q_idx"), _dev(Q, "Q"), H, top_k,
                              _scale(idx_scale), _scale(attn_scale), _dev(O, "O"),
                              _dev(indices, "indices") if indices is not None else None,
                              _dev(workspace, "workspace"), workspace.numel() * workspace.element_size(),
                              _stream(stream))
    _check(st, "dsa_decode_multi")
    return O, indices


def dsa_decode_paged_multi(k_idx: torch.Tensor, K: torch.Tensor, V: torch.Tensor, block_table: torch.Tensor,
                           seq_lens: torch.Tensor, q_idx: torch.Tensor, Q: torch.Tensor, top_k: int,
                           max_len: int, idx_scale: Optional[float] = None,
                           attn_scale: Optional[float] = None, O: Optional[torch.Tensor] = None,
                           indices: Optional[torch.Tensor] = None, want_indices: bool = True,
                           workspace: Optional[torch.Tensor] = None,
                           stream=None) -> Tuple[torch.Tensor, Optional[torch.Tensor]]:
    """dsa_decode_multi over a block-paged cache (layout of dsa_decode_paged)."""
    lib = load()
    B, T, d = q_idx.shape
    _, _, H, D = Q.shape
    num_blocks, block_size = k_idx.shape[0], k_idx.shape[1]
    if block_table.dtype != torch.int32 or seq_lens.dtype != torch.int32:
        raise ValueError("block_table and seq_lens must be int32")
    if block_table.dim() != 2 or block_table.shape[0] != B or seq_lens.shape != (B,):
        raise ValueError("block_table must be [B, max_blocks] and seq_lens [B]")
    idt = _idx_dtype(q_idx)
    dev = q_idx.device
    if O is None:
        O = torch.empty((B, T, H, D), dtype=torch.bfloat16, device=dev)
    if indices is None and want_indices:
        indices = torch.empty((B, T, top_k), dtype=torch.int32, device=dev)
    if workspace is None:
        workspace = torch.empty(int(lib.dsa_decode_paged_multi_workspace_size(B, T, int(max_len), d, idt, H, D,
                                                                              top_k)),
                                dtype=torch.uint8, device=dev)
    st = lib.dsa_decode_paged_multi(_dev(k_idx, "k_idx"), _dev(K, "K"), _dev(V, "V"), num_blocks, block_size,
                                    _dev(block_table, "block_table"), block_table.shape[1],
                                    _dev(seq_lens, "seq_lens"), B, T, int(max_len), idt, d, D,
                                    _dev(q_idx, "q_idx"), _dev(Q, "Q"), H, top_k, _scale(idx_scale),
                                    _scale(attn_scale), _dev(O, "O"),
                                    _dev(indices, "indices") if indices is not None else None,
                                    _dev(workspace, "workspace"), workspace.numel() * workspace.element_size(),
                                    _stream(stream))
    _check(st, "dsa_decode_paged_multi")
    return O, indices


def dsa_decode_static(k_idx: torch.Tensor, K: torch.Tensor, V: torch.Tensor, seq_start: torch.Tensor,
                      q_idx: torch.Tensor, Q: torch.Tensor, top_k: int, max_len: int,
                      O: torch.Tensor, indices: Optional[torch.Tensor] = None,
                      idx_scale: Optional[float] = None, attn_scale: Optional[float] = None,
                      stream=None) -> Tuple[torch.Tensor, Optional[torch.Tensor]]:
    """dsa_decode with the library's built-in scratch: for callers that must not allocate.

    O (and indices, if wanted) are passed in by the caller; nothing is allocated here.
    """
    lib = load()
    B, d = q_idx.shape
    _, H, D = Q.shape
    if seq_start.dtype != torch.int64:
        raise ValueError("seq_start must be int64")
    st = lib.dsa_decode_static(_dev(k_idx, "k_idx"), _dev(K, "K"), _dev(V, "V"), _dev(seq_start, "seq_start"),
                               B, k_idx.shape[0], int(max_len), _idx_dtype(q_idx), d, D, _dev(q_idx, "q_idx"),
                               _dev(Q, "Q"), H, top_k, _scale(idx_scale), _scale(attn_scale), _dev(O, "O"),
                               _dev(indices, "indices") if indices is not None else None, _stream(stream))
    _check(st, "dsa_decode_static")
    return O, indices


def dsa_gather_probe(indices: torch.Tensor, K: torch.Tensor, V: torch.Tensor, ctas_per_sm: int, stages: int,
                     sink: Optional[torch.Tensor] = None, stream=None) -> None:
    """Diagnostic: gather the K and V rows listed in indices into shared memory
    and nothing else (the memory ceiling of the attention's gather)."""
    L, top_k = indices.shape
    D = K.shape[1]
    if sink is None:
        sink = torch.zeros(1, dtype=torch.int64, device=indices.device)
    _check(load().dsa_gather_probe(_dev(indices, "indices"), L, top_k, _dev(K, "K"), _dev(V, "V"), D,
                                   int(ctas_per_sm), int(stages), _dev(sink, "sink"), _stream(stream)),
           "dsa_gather_probe")


def dsa_index_to_fp8(x: torch.Tensor, out: Optional[torch.Tensor] = None,
                     inexact: Optional[torch.Tensor] = None, stream=None) -> Tuple[torch.Tensor, torch.Tensor]:
    """E4M3 copy of a BF16 index tensor -> (copy as uint8, device count of values it changed).
    The copy gives the same indexer scores only when the count is zero."""
    if x.dtype != torch.bfloat16:
        raise ValueError("x must be bfloat16")
    if out is None:
        out = torch.empty(x.shape, dtype=torch.uint8, device=x.device)
    if inexact is None:
        inexact = torch.empty(1, dtype=torch.int64, device=x.device)
    _check(load().dsa_index_to_fp8(_dev(x, "x"), x.numel(), _dev(out, "out"), _dev(inexact, "inexact"),
                                   _stream(stream)), "dsa_index_to_fp8")
    return out, inexact


def dsa_sync_status(stream=None) -> int:
    """Synchronise and return (then clear) the device status word (0 = ok)."""
    return int(load().dsa_sync_status(_stream(stream)))


def dsa_last_stats(workspace: torch.Tensor, stream=None) -> dict:
    out = (ctypes.c_int64 * 4)()
    _check(load().dsa_last_stats(_dev(workspace, "workspace"), out, _stream(stream)), "dsa_last_stats")
    return {"fallback_rows": out[0], "overflow_rows": out[1], "candidates": out[2]}


def dsa_debug_force_fallback(period: int) -> None:
    """Send every prefill row t with t % period == 0 to the select's exact
    fallback (period 0: off).  Test hook; results are unchanged."""
    _check(load().dsa_debug_force_fallback(int(period)), "dsa_debug_force_fallback")


def dsa_debug_wait_timeout(limit_ns: int, stream=None) -> None:
    _check(load().dsa_debug_wait_timeout(int(limit_ns), _stream(stream)), "dsa_debug_wait_timeout")


STAGES = ["indexer_sample", "threshold", "indexer_filter", "select", "attention",
          "decode_scan_select", "unused", "decode_attention"]


def dsa_stage_timing(enable: bool) -> None:
    _check(load().dsa_stage_timing(1 if enable else 0), "dsa_stage_timing")


def dsa_stage_times() -> dict:
    """{stage: (milliseconds, kernel launches)} summed since the last read (then reset)."""
    n = len(STAGES)
    ms = (ctypes.c_double * n)()
    ln = (ctypes.c_int64 * n)()
    _check(load().dsa_stage_times(ms, ln, n), "dsa_stage_times")
    return {STAGES[i]: (ms[i], int(ln[i])) for i in range(n)}


def default_index_scale(d: int) -> float:
    return float(torch.tensor(1.0 / math.sqrt(d), dtype=torch.float32))
