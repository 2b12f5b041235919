"""dsa_decode_static: the decode entry point for callers that cannot allocate
device memory (a plugin whose host application owns every allocation, or a
serving loop that must not call cudaMalloc once running).  It takes its
scratch from a block built into the library instead of a caller workspace.

This file is collected last so that a run stopping at the first failure has
already run every other test; it must also pass on its own in a fresh process.
"""
import numpy as np
import pytest
import torch

import synth

pytestmark = pytest.mark.gpu
ATOL = 2e-2


@pytest.fixture(scope="module")
def dsa():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from sparse_attention_10_b200 import build
    build.build()
    import sparse_attention_10_b200 as m
    m.load()
    return m


def test_static_scratch_decode_matches_workspace_decode_twice(dsa):
    w = synth.WORKLOADS["decode_64x128k"]
    lens = np.array([3, 700, 2048, 9000, 131072, 70001], dtype=np.int64)   # 213k rows < 2^20
    xd = synth.decode_inputs(w, lengths=lens)
    t = {k: torch.from_numpy(np.ascontiguousarray(xd[k])).cuda()
         for k in ("k_idx", "K", "V", "q_idx", "Q", "seq_start")}
    K, V, Q = (t[k].view(torch.bfloat16) for k in ("K", "V", "Q"))
    max_len = int(lens.max())
    O_ref, idx_ref = dsa.dsa_decode(t["k_idx"], K, V, t["seq_start"], t["q_idx"], Q, w.top_k, max_len)
    assert dsa.dsa_sync_status() == 0
    for call in range(2):
        O = torch.full_like(O_ref, float("nan"))
        idx = torch.full_like(idx_ref, -7)
        dsa.dsa_decode_static(t["k_idx"], K, V, t["seq_start"], t["q_idx"], Q, w.top_k, max_len,
                              O=O, indices=idx)
        assert dsa.dsa_sync_status() == 0, f"call {call}"
        assert torch.equal(idx, idx_ref), f"call {call}: indices differ"
        err = (O.float() - O_ref.float()).abs().max().item()
        assert err <= ATOL, f"call {call}: max-abs {err}"


def small_batch(B=64, H=16, D=128, d=128):
    """Real device buffers for a batch of B one-row sequences (seq_start = 0..B)."""
    return {
        "k_idx": torch.zeros((B, d), dtype=torch.uint8, device="cuda"),
        "K": torch.zeros((B, D), dtype=torch.bfloat16, device="cuda"),
        "V": torch.zeros((B, D), dtype=torch.bfloat16, device="cuda"),
        "seq_start": torch.arange(B + 1, dtype=torch.int64, device="cuda"),
        "q_idx": torch.zeros((B, d), dtype=torch.uint8, device="cuda"),
        "Q": torch.zeros((B, H, D), dtype=torch.bfloat16, device="cuda"),
        "O": torch.zeros((B, H, D), dtype=torch.bfloat16, device="cuda"),
    }


def test_static_scratch_rejects_sizes_beyond_its_block(dsa):
    import ctypes
    lib = dsa.load()
    too_many_rows = 1 << 22
    # the size bound alone: such a call needs more scratch than the block holds
    assert dsa.dsa_decode_workspace_size(64, too_many_rows, 128, 0, 16, 128, 2048) > (18 << 20)
    # Every pointer is a real device buffer of a small batch, so even a call
    # that got past the host-side size check would meet the device-side check
    # (seq_start[B] != total_rows) and read nothing out of bounds.
    t = small_batch()
    st = lib.dsa_decode_static(*(ctypes.c_void_p(t[n].data_ptr()) for n in ("k_idx", "K", "V", "seq_start")),
                               64, too_many_rows, 131072, 0, 128, 128,
                               ctypes.c_void_p(t["q_idx"].data_ptr()), ctypes.c_void_p(t["Q"].data_ptr()),
                               16, 2048, float("nan"), float("nan"), ctypes.c_void_p(t["O"].data_ptr()),
                               None, None)
    assert st == 3   # DSA_ERR_WORKSPACE: the built-in scratch is too small for these sizes
    assert dsa.dsa_sync_status() == 0   # nothing was enqueued


def test_static_scratch_rejects_output_off_the_current_device(dsa):
    # The block is per device: an output in host memory is refused before any launch.
    t = small_batch()
    O_host = torch.zeros((64, 16, 128), dtype=torch.bfloat16).pin_memory()
    import ctypes
    lib = dsa.load()
    st = lib.dsa_decode_static(*(ctypes.c_void_p(t[n].data_ptr()) for n in ("k_idx", "K", "V", "seq_start")),
                               64, 64, 1, 0, 128, 128,
                               ctypes.c_void_p(t["q_idx"].data_ptr()), ctypes.c_void_p(t["Q"].data_ptr()),
                               16, 2048, float("nan"), float("nan"), ctypes.c_void_p(O_host.data_ptr()),
                               None, None)
    assert st == 1   # DSA_ERR_INVALID_ARG
    assert dsa.dsa_sync_status() == 0
    assert bool((O_host == 0).all())
