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


def test_static_scratch_rejects_sizes_beyond_its_block(dsa):
    import ctypes
    lib = dsa.load()
    P = ctypes.c_void_p
    too_many_rows = 1 << 22
    st = lib.dsa_decode_static(P(16), P(16), P(16), P(16), 64, too_many_rows, 131072, 0, 128, 128,
                               P(16), P(16), 16, 2048, float("nan"), float("nan"), P(16), None, None)
    assert st == 3   # DSA_ERR_WORKSPACE: the built-in scratch is too small for these sizes
