"""The synthetic workloads against the figures the DSA page prints."""
import os

import numpy as np

import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def test_prefill_workloads_follow_the_parameter_guide():
    # DeepSeek Sparse Attention page, section 7.2: top_k / index_dim / precision per length.
    rows = [l.split() for l in open(os.path.join(GOLDEN, "param_guide.txt")) if l.strip() and l[0] != "#"]
    by_len = {w.L: w for w in synth.WORKLOADS.values() if w.kind == "prefill" and w.cid <= 5}
    assert len(rows) == 3
    for L, k, d, prec in rows:
        w = by_len[int(L)]
        assert (w.top_k, w.d_idx, w.idx_dtype) == (int(k), int(d), prec)


def test_generator_is_counter_based_and_prefix_stable():
    key = synth.stream_key(1, 2, 3)
    a = synth.draws(key, 0, 1000)
    b = synth.draws(key, 400, 600)
    assert np.array_equal(a[400:], b)
    w = synth.WORKLOADS["prefill_4k"]
    small = synth.prefill_inputs(w, L=300)
    big = synth.prefill_inputs(w, L=600)
    assert np.array_equal(small["q_idx"], big["q_idx"][:300])


def test_integer_draws_uniform_on_minus4_to_4():
    v = synth.uniform_ints(synth.stream_key(5), 90000)
    assert v.min() == -4 and v.max() == 4
    counts = np.bincount(v + 4)
    assert np.all(np.abs(counts - 10000) < 500)


def test_normal_draws_moments():
    x = synth.normal_bf16(synth.stream_key(9), 200001)
    f = (x.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    assert abs(f.mean()) < 0.01 and abs(f.std() - 1.0) < 0.01


def test_local_boost_shares_32_dims_within_128_blocks():
    w = synth.WORKLOADS["prefill_64k"]
    x = synth.prefill_inputs(w, L=512, with_attention=False)
    q, k = x["q_idx"], x["k_idx"]
    assert np.array_equal(q[:128, :32], np.broadcast_to(q[0, :32], (128, 32)))
    assert np.array_equal(k[130, :32], q[255, :32])
    assert not np.array_equal(q[127, :32], q[128, :32])


def test_decode_lengths_in_range():
    w = synth.WORKLOADS["decode_64x128k"]
    n = synth.decode_lengths(w)
    assert n.shape == (64,) and n.min() >= 65536 and n.max() <= 131072


def test_paged_inputs_torch_match_numpy():
    """The device-side builder of a paged cache (used by the benchmark) places the
    rows exactly as the numpy one the parity tests use."""
    import torch
    w = synth.WORKLOADS["decode_64x128k"]
    lens = np.array([5, 130, 64, 1], dtype=np.int64)
    xp = synth.paged_decode_inputs(w, lens, 16)
    xd = xp["contiguous"]
    xt = {"k_idx": torch.from_numpy(xd["k_idx"]), "K": torch.from_numpy(xd["K"].view(np.int16)),
          "V": torch.from_numpy(xd["V"].view(np.int16)), "q_idx": torch.from_numpy(xd["q_idx"]),
          "Q": torch.from_numpy(xd["Q"].view(np.int16)), "lengths": lens, "B": 4}
    pt = synth.paged_decode_inputs_torch(xt, 16)
    assert np.array_equal(pt["block_table"].numpy(), xp["block_table"])
    assert np.array_equal(pt["seq_lens"].numpy(), xp["seq_lens"])
    table = xp["block_table"]
    for name, ref in (("k_idx_blocks", xp["k_idx_blocks"]), ("K_blocks", xp["K_blocks"].view(np.int16)),
                      ("V_blocks", xp["V_blocks"].view(np.int16))):
        got = pt[name].numpy()
        assert got.shape == ref.shape
        for b, n in enumerate(lens):     # every row a sequence reaches is the same
            s = np.arange(int(n))
            blk, off = table[b, s // 16], s % 16
            assert np.array_equal(got[blk, off], ref[blk, off])
