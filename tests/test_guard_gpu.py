"""Guard regions around every buffer a call writes: outputs and workspace.

A memory checker cannot run here, so each buffer the library writes is placed
between two 4 KB guard regions filled with a fixed byte pattern (the buffer's
own tail, up to the next 256 bytes, is guarded too).  After the call and a
synchronise the guards must be unchanged, and the results must equal those of
the same call on plainly allocated buffers.
"""
import numpy as np
import pytest
import torch

import synth

pytestmark = pytest.mark.gpu

G = 4096
PAT = 0xA5


@pytest.fixture(scope="module")
def dsa():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    import sparse_attention_10_b200 as m
    m.load()
    return m


class Guarded:
    """One device allocation: [guard | buffer, padded to 256 bytes | guard]."""

    def __init__(self, nbytes: int):
        self.nbytes = nbytes
        padded = (nbytes + 255) // 256 * 256
        self.buf = torch.full((G + padded + G,), PAT, dtype=torch.uint8, device="cuda")

    def tensor(self, dtype=torch.uint8, shape=None):
        t = self.buf[G:G + self.nbytes].view(dtype)
        return t if shape is None else t.view(shape)

    def intact(self) -> bool:
        return bool((self.buf[:G] == PAT).all()) and bool((self.buf[G + self.nbytes:] == PAT).all())


def dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def prefill_case(name, L, top_k):
    w = synth.WORKLOADS[name]
    x = synth.prefill_inputs(w, L=L)
    q, k = dev(x["q_idx"]), dev(x["k_idx"])
    if w.idx_dtype == "bf16":
        q, k = q.view(torch.bfloat16), k.view(torch.bfloat16)
    return w, q, k, dev(x["Q"]).view(torch.bfloat16), dev(x["K"]).view(torch.bfloat16), \
        dev(x["V"]).view(torch.bfloat16), top_k or w.top_k


@pytest.mark.parametrize("name,L,top_k,force", [
    ("prefill_4k", 4096, None, 0),       # FP8 index, 4 heads of 64
    ("prefill_4k", 3001, None, 3),       # every third row through the exact fallback
    ("prefill_128k", 5000, None, 0),     # BF16 index dim 160, 16 heads of 128 (tcgen05 attention)
])
def test_prefill_writes_stay_inside_buffers(dsa, name, L, top_k, force):
    w, q, k, Q, K, V, top_k = prefill_case(name, L, top_k)
    H, D = Q.shape[1], Q.shape[2]
    need = dsa.dsa_prefill_workspace_size(L, q.shape[1], 0 if w.idx_dtype == "fp8" else 1, H, D, top_k)
    g_idx, g_o, g_ws = Guarded(L * top_k * 4), Guarded(L * H * D * 2), Guarded(need)
    dsa.dsa_debug_force_fallback(force)
    try:
        idx, O = dsa.dsa_prefill(q, k, Q, K, V, top_k, indices=g_idx.tensor(torch.int32, (L, top_k)),
                                 O=g_o.tensor(torch.bfloat16, (L, H, D)), workspace=g_ws.tensor())
        assert dsa.dsa_sync_status() == 0
        ref_idx, ref_o = dsa.dsa_prefill(q, k, Q, K, V, top_k)
        assert dsa.dsa_sync_status() == 0
    finally:
        dsa.dsa_debug_force_fallback(0)
    assert g_idx.intact() and g_o.intact() and g_ws.intact()
    assert torch.equal(idx, ref_idx)
    assert torch.equal(O.view(torch.int16), ref_o.view(torch.int16))


def decode_case(lens):
    w = synth.WORKLOADS["decode_64x128k"]
    return w, synth.decode_inputs(w, lengths=np.array(lens, dtype=np.int64))


@pytest.mark.parametrize("want_indices,zero_q", [(True, False), (False, False), (True, True)])
def test_decode_writes_stay_inside_buffers(dsa, want_indices, zero_q):
    # zero_q: every score +0, so sequences longer than 8192 rows take the
    # select's many-candidate path (compaction in the workspace's key scratch)
    w, xd = decode_case([1, 2, 100, 2049, 9000, 70000])
    if zero_q:
        xd["q_idx"] = np.zeros_like(xd["q_idx"])
    t = {n: dev(xd[n]) for n in ("k_idx", "K", "V", "q_idx", "Q", "seq_start")}
    B, total, mx = xd["B"], int(xd["seq_start"][-1]), int(xd["lengths"].max())
    need = dsa.dsa_decode_workspace_size(B, total, w.d_idx, 0, w.H, w.D, w.top_k)
    g_idx, g_o, g_ws = Guarded(B * w.top_k * 4), Guarded(B * w.H * w.D * 2), Guarded(need)
    args = (t["k_idx"], t["K"].view(torch.bfloat16), t["V"].view(torch.bfloat16), t["seq_start"],
            t["q_idx"], t["Q"].view(torch.bfloat16), w.top_k, mx)
    O, idx = dsa.dsa_decode(*args, O=g_o.tensor(torch.bfloat16, (B, w.H, w.D)),
                            indices=g_idx.tensor(torch.int32, (B, w.top_k)) if want_indices else None,
                            want_indices=want_indices, workspace=g_ws.tensor())
    assert dsa.dsa_sync_status() == 0
    ref_o, ref_idx = dsa.dsa_decode(*args)
    assert dsa.dsa_sync_status() == 0
    assert g_idx.intact() and g_o.intact() and g_ws.intact()
    if want_indices:
        assert torch.equal(idx, ref_idx)
    assert torch.equal(O.view(torch.int16), ref_o.view(torch.int16))


@pytest.mark.parametrize("zero_q", [False, True])
def test_paged_decode_writes_stay_inside_buffers(dsa, zero_q):
    w = synth.WORKLOADS["decode_64x128k"]
    lens = np.array([1, 2, 100, 2049, 9000, 70000], dtype=np.int64)
    xp = synth.paged_decode_inputs(w, lens, 16)
    if zero_q:
        xp["q_idx"] = np.zeros_like(xp["q_idx"])
    t = {n: dev(xp[n]) for n in ("k_idx_blocks", "K_blocks", "V_blocks", "block_table", "seq_lens",
                                 "q_idx", "Q")}
    B, mx = xp["B"], int(lens.max())
    need = dsa.dsa_decode_paged_workspace_size(B, mx, w.d_idx, 0, w.H, w.D, w.top_k)
    g_idx, g_o, g_ws = Guarded(B * w.top_k * 4), Guarded(B * w.H * w.D * 2), Guarded(need)
    args = (t["k_idx_blocks"], t["K_blocks"].view(torch.bfloat16), t["V_blocks"].view(torch.bfloat16),
            t["block_table"], t["seq_lens"], t["q_idx"], t["Q"].view(torch.bfloat16), w.top_k, mx)
    O, idx = dsa.dsa_decode_paged(*args, O=g_o.tensor(torch.bfloat16, (B, w.H, w.D)),
                                  indices=g_idx.tensor(torch.int32, (B, w.top_k)), workspace=g_ws.tensor())
    assert dsa.dsa_sync_status() == 0
    ref_o, ref_idx = dsa.dsa_decode_paged(*args)
    assert dsa.dsa_sync_status() == 0
    assert g_idx.intact() and g_o.intact() and g_ws.intact()
    assert torch.equal(idx, ref_idx)
    assert torch.equal(O.view(torch.int16), ref_o.view(torch.int16))


def test_paged_multi_token_decode_writes_stay_inside_buffers(dsa):
    import dataclasses
    w = synth.WORKLOADS["decode_64x128k"]
    lens = np.array([4, 100, 2049, 9000], dtype=np.int64)
    T = 4
    xp = synth.paged_decode_inputs(w, lens, 16)
    mq = synth.multi_queries(w, len(lens), T)
    t = {n: dev(xp[n]) for n in ("k_idx_blocks", "K_blocks", "V_blocks", "block_table", "seq_lens")}
    B, mx = len(lens), int(lens.max())
    need = dsa.dsa_decode_paged_multi_workspace_size(B, T, mx, w.d_idx, 0, w.H, w.D, w.top_k)
    g_idx, g_o, g_ws = Guarded(B * T * w.top_k * 4), Guarded(B * T * w.H * w.D * 2), Guarded(need)
    args = (t["k_idx_blocks"], t["K_blocks"].view(torch.bfloat16), t["V_blocks"].view(torch.bfloat16),
            t["block_table"], t["seq_lens"], dev(mq["q_idx"]), dev(mq["Q"]).view(torch.bfloat16), w.top_k, mx)
    O, idx = dsa.dsa_decode_paged_multi(*args, O=g_o.tensor(torch.bfloat16, (B, T, w.H, w.D)),
                                        indices=g_idx.tensor(torch.int32, (B, T, w.top_k)),
                                        workspace=g_ws.tensor())
    assert dsa.dsa_sync_status() == 0
    ref_o, ref_idx = dsa.dsa_decode_paged_multi(*args)
    assert dsa.dsa_sync_status() == 0
    assert g_idx.intact() and g_o.intact() and g_ws.intact()
    assert torch.equal(idx, ref_idx)
    assert torch.equal(O.view(torch.int16), ref_o.view(torch.int16))
