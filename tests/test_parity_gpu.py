"""CUDA path vs the CPU oracle, through the C ABI (needs a B200).

Bar: indices bit-exact (integer-valued indexer inputs make every score exact
on both sides); attention outputs within max-abs 2e-2 of the oracle's FP64
result rounded to BF16.  Small cases compare every row; the full-size
workloads compare every row at 32K and, at 64K and 128K, the first rows,
tile and capacity boundaries, the last rows and 2048 seeded random rows, and
check properties of all rows.
"""
import numpy as np
import pytest
import torch

import oracle
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


def to_dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def bf16(a):
    return to_dev(a).view(torch.bfloat16)


def bits_to_f32(a):
    return (np.asarray(a, dtype=np.uint32) << 16).view(np.float32)


def run_prefill(dsa, x, top_k, **kw):
    q, k = to_dev(x["q_idx"]), to_dev(x["k_idx"])
    if q.dtype == torch.uint16:
        q, k = q.view(torch.bfloat16), k.view(torch.bfloat16)
    ws = torch.empty(dsa.dsa_prefill_workspace_size(q.shape[0], q.shape[1], 0 if q.dtype == torch.uint8 else 1,
                                                    x["Q"].shape[1], x["Q"].shape[2], top_k),
                     dtype=torch.uint8, device="cuda")
    idx, O = dsa.dsa_prefill(q, k, bf16(x["Q"]), bf16(x["K"]), bf16(x["V"]), top_k, workspace=ws, **kw)
    assert dsa.dsa_sync_status() == 0
    stats = dsa.dsa_last_stats(ws)
    return idx.cpu().numpy(), O.view(torch.int16).cpu().numpy().view(np.uint16), stats


def small_inputs(L, d, H, D, idx_dtype="fp8", seed=3, lo=-4, hi=4):
    key = synth.stream_key(seed, 500, L, d)
    qi = synth.uniform_ints(key, L * d, lo, hi).reshape(L, d)
    ki = synth.uniform_ints(key, L * d, lo, hi, start=L * d).reshape(L, d)
    enc = synth.fp8_bytes_of_ints if idx_dtype == "fp8" else synth.bf16_bits_of_ints
    return {
        "q_idx": enc(qi), "k_idx": enc(ki), "L": L,
        "Q": synth.normal_bf16(synth.stream_key(seed, 1, L), L * H * D).reshape(L, H, D),
        "K": synth.normal_bf16(synth.stream_key(seed, 2, L), L * D).reshape(L, D),
        "V": synth.normal_bf16(synth.stream_key(seed, 3, L), L * D).reshape(L, D),
    }


def compare(x, idx_dtype, top_k, idx, O, rows=None):
    ri, ro = oracle.prefill_rows(x, idx_dtype, top_k, rows=rows)
    sel = slice(None) if rows is None else rows
    gi = idx[sel]
    bad = np.nonzero((gi != ri).any(axis=1))[0]
    assert bad.size == 0, f"indices differ on rows {np.asarray(rows if rows is not None else np.arange(len(ri)))[bad[:10]]}"
    err = np.abs(bits_to_f32(O[sel]) - bits_to_f32(ro)).max()
    assert err <= ATOL, f"max-abs error {err}"


# ------------------------------------------------------------------ indexer

@pytest.mark.parametrize("idx_dtype,d,Lq,Lk", [
    ("fp8", 128, 300, 517), ("fp8", 96, 129, 257), ("bf16", 160, 200, 300),
    ("fp8", 32, 1, 1), ("bf16", 16, 130, 70), ("fp8", 256, 64, 1000), ("bf16", 256, 40, 260),
])
def test_indexer_scores_bit_exact(dsa, idx_dtype, d, Lq, Lk):
    key = synth.stream_key(77, d, Lq, Lk)
    enc = synth.fp8_bytes_of_ints if idx_dtype == "fp8" else synth.bf16_bits_of_ints
    q = enc(synth.uniform_ints(key, Lq * d).reshape(Lq, d))
    k = enc(synth.uniform_ints(key, Lk * d, start=Lq * d).reshape(Lk, d))
    qt, kt = to_dev(q), to_dev(k)
    if idx_dtype == "bf16":
        qt, kt = qt.view(torch.bfloat16), kt.view(torch.bfloat16)
    got = dsa.dsa_indexer_scores(qt, kt).cpu().numpy()
    assert dsa.dsa_sync_status() == 0
    ref = oracle.indexer_scores(q, k, idx_dtype)
    assert np.array_equal(got.view(np.uint32), ref.view(np.uint32))


def test_indexer_scores_general_fp8_close(dsa):
    rng = np.random.default_rng(1)
    b = rng.integers(0, 256, size=(200, 128), dtype=np.uint8)
    b = np.where((b & 0x7F) == 0x7F, np.uint8(0x3C), b)
    c = rng.integers(0, 256, size=(300, 128), dtype=np.uint8)
    c = np.where((c & 0x7F) == 0x7F, np.uint8(0x3C), c)
    got = dsa.dsa_indexer_scores(to_dev(b), to_dev(c)).cpu().numpy()
    ref = oracle.indexer_scores(b, c, "fp8")
    assert np.allclose(got, ref, rtol=1e-5, atol=1e-5 * np.abs(ref).max())


# ------------------------------------------------------------------ prefill, small

@pytest.mark.parametrize("L,top_k", [(1, 16), (5, 16), (129, 64), (700, 256), (2000, 256), (1500, 64)])
def test_prefill_small_all_rows(dsa, L, top_k):
    x = small_inputs(L, 128, 4, 64)
    idx, O, _ = run_prefill(dsa, x, top_k)
    compare(x, "fp8", top_k, idx, O)


@pytest.mark.parametrize("L,top_k,H", [(1, 16, 16), (5, 16, 1), (129, 64, 16), (300, 300, 3), (777, 128, 16)])
def test_prefill_small_head_dim_128(dsa, L, top_k, H):
    # Head dim 128 runs the tcgen05 attention: single-key items, items shorter
    # than one 128-key tile, fewer heads than the MMA's 16.
    x = small_inputs(L, 128, H, 128, seed=17)
    idx, O, _ = run_prefill(dsa, x, top_k)
    compare(x, "fp8", top_k, idx, O)


def test_prefill_d96_ragged(dsa):
    x = small_inputs(2333, 96, 16, 128, seed=5)
    idx, O, _ = run_prefill(dsa, x, 128)
    compare(x, "fp8", 128, idx, O)


def test_prefill_bf16_index(dsa):
    x = small_inputs(1900, 160, 16, 128, idx_dtype="bf16", seed=6)
    idx, O, _ = run_prefill(dsa, x, 300)
    compare(x, "bf16", 300, idx, O)


def test_prefill_bf16_index_dim_256_single_stage(dsa):
    # 512-byte index rows leave room for one pipeline stage in the indexer.
    x = small_inputs(1500, 256, 2, 64, idx_dtype="bf16", seed=13)
    idx, O, _ = run_prefill(dsa, x, 128)
    compare(x, "bf16", 128, idx, O)


def test_prefill_fp8_index_dim_256(dsa):
    x = small_inputs(1700, 256, 2, 64, seed=14)
    idx, O, _ = run_prefill(dsa, x, 96)
    compare(x, "fp8", 96, idx, O)


def test_prefill_many_ties(dsa):
    # Index values in {-1, 0, 1}: scores take few values, so ties cross the k-th place.
    x = small_inputs(3000, 32, 2, 64, seed=8, lo=-1, hi=1)
    idx, O, _ = run_prefill(dsa, x, 200)
    compare(x, "fp8", 200, idx, O)


def test_prefill_large_accumulators_tie_after_scaling(dsa):
    # BF16 integers in [244, 256], index dim 256: dot products in [2^23, 2^24)
    # stay exact in FP32, but with idx_scale 0.55 neighbouring accumulators
    # round to the same score, so the select must rank by score (ties by
    # index), not by accumulator.
    x = small_inputs(1500, 256, 4, 64, idx_dtype="bf16", seed=15)
    key = synth.stream_key(15, 501, 1500, 256)
    for name, start in (("q_idx", 0), ("k_idx", 1500 * 256)):
        v = synth.uniform_ints(key, 1500 * 256, 244, 256, start=start).reshape(1500, 256)
        x[name] = synth.bf16_bits_of_f32(v.astype(np.float32))   # exact: |v| <= 256
    idx, O, _ = run_prefill(dsa, x, 64, idx_scale=0.55)
    ri, ro = oracle.prefill_rows(x, "bf16", 64, idx_scale=0.55)
    assert np.array_equal(idx, ri)
    assert np.abs(bits_to_f32(O) - bits_to_f32(ro)).max() <= ATOL


def test_prefill_attention_large_norm_key(dsa):
    # One K row with 64 times the others' norm: queries that keep it get
    # scores far above the rest, so softmax weights span a wide range.
    x = small_inputs(1500, 96, 16, 128, seed=16)
    K = bits_to_f32(x["K"]).reshape(1500, 128)
    K[7] *= 64.0                              # a power of two: still exact in BF16
    x["K"] = synth.bf16_bits_of_f32(K)
    idx, O, _ = run_prefill(dsa, x, 256)
    compare(x, "fp8", 256, idx, O)


def test_prefill_all_zero_scores(dsa):
    x = small_inputs(2500, 128, 4, 64, seed=9)
    x["q_idx"] = np.zeros_like(x["q_idx"])
    idx, O, stats = run_prefill(dsa, x, 256)
    for t in (0, 10, 255, 256, 2499):
        m = min(256, t + 1)
        assert idx[t, :m].tolist() == list(range(m))
    compare(x, "fp8", 256, idx, O, rows=np.array([0, 1, 300, 1000, 2499]))


# ------------------------------------------------------------------ exact fallback of the select

@pytest.fixture
def force_fallback(dsa):
    yield dsa.dsa_debug_force_fallback
    dsa.dsa_debug_force_fallback(0)


def test_prefill_forced_fallback_many_rows(dsa, force_fallback):
    # Every 7th row through the fallback: more rows than the grid-wide slots
    # (one per SM), so the shared-memory select and the one-CTA path both run.
    x = small_inputs(3000, 96, 4, 128, seed=12)
    force_fallback(7)
    idx, O, stats = run_prefill(dsa, x, 256)
    assert stats["fallback_rows"] == len(range(0, 3000, 7)), stats
    compare(x, "fp8", 256, idx, O)


def test_prefill_forced_fallback_zero_ties(dsa, force_fallback):
    # All scores zero: the boundary bin is the ReLU zeros', the shared-memory
    # select declines and the one-CTA path ranks the ties by index.
    x = small_inputs(1200, 128, 4, 64, seed=13)
    x["q_idx"] = np.zeros_like(x["q_idx"])
    force_fallback(5)
    idx, O, stats = run_prefill(dsa, x, 128)
    assert stats["fallback_rows"] == len(range(0, 1200, 5)), stats
    for t in (0, 5, 130, 1195):
        m = min(128, t + 1)
        assert idx[t, :m].tolist() == list(range(m))
    compare(x, "fp8", 128, idx, O, rows=np.array([0, 5, 10, 127, 130, 600, 1195, 1199]))


def test_prefill_forced_fallback_bf16_long_rows(dsa, force_fallback):
    # BF16 index rows of 160, top_k 2048, rows spanning several scoring chunks.
    x = small_inputs(9000, 160, 16, 128, idx_dtype="bf16", seed=14)
    force_fallback(1000)
    idx, O, stats = run_prefill(dsa, x, 2048)
    assert stats["fallback_rows"] == 9, stats
    compare(x, "bf16", 2048, idx, O, rows=np.array([0, 1000, 2000, 2047, 4000, 7000, 8000, 8999]))


def test_prefill_top_k_2048_small(dsa):
    x = small_inputs(5000, 128, 16, 128, seed=10)
    idx, O, _ = run_prefill(dsa, x, 2048)
    rows = np.unique(np.concatenate([np.arange(0, 5000, 97), [2047, 2048, 4095, 4096, 4999]]))
    compare(x, "fp8", 2048, idx, O, rows=rows)


def test_prefill_explicit_scales(dsa):
    x = small_inputs(900, 128, 4, 64, seed=11)
    idx, O, _ = run_prefill(dsa, x, 100, idx_scale=0.25, attn_scale=0.05)
    ri, ro = oracle.prefill_rows(x, "fp8", 100, idx_scale=0.25, attn_scale=0.05)
    assert np.array_equal(idx, ri)
    assert np.abs(bits_to_f32(O) - bits_to_f32(ro)).max() <= ATOL


def test_prefill_workload_4k_all_rows(dsa):
    w = synth.WORKLOADS["prefill_4k"]
    x = synth.prefill_inputs(w)
    idx, O, stats = run_prefill(dsa, x, w.top_k)
    compare(x, w.idx_dtype, w.top_k, idx, O)


# ------------------------------------------------------------------ FP8 copy of BF16 index inputs

def test_index_to_fp8_is_exact_on_integers_and_counts_the_rest(dsa):
    v = torch.tensor([0, 1, -1, 2, -3, 4, 0.5, 448, -448, 0.1, 3.3, 1000, float("nan"), -0.0, 17, 2 ** -9],
                     dtype=torch.bfloat16, device="cuda")
    out, bad = dsa.dsa_index_to_fp8(v)
    torch.cuda.synchronize()
    back = out.view(torch.float8_e4m3fn).float()
    exact = (back == v.float())
    # 0.1, 3.3, 1000 (beyond 448), NaN and 17 (needs 4 mantissa bits) do not survive
    assert int(bad.item()) == 5
    assert exact[:9].all() and exact[13] and exact[15]
    ref = v.float().to(torch.float8_e4m3fn).view(torch.uint8)
    fin = torch.isfinite(v.float()) & (v.float().abs() <= 448)
    assert torch.equal(out[fin], ref[fin])


def test_prefill_on_the_fp8_copy_of_bf16_integer_inputs_is_identical(dsa):
    """The 128K workload's settings (BF16 index dim 160, top_k 2048) at L = 9000:
    the E4M3 copy of the integer inputs runs the FP8 indexer and gives the same
    indices and outputs as the BF16 call, and the oracle's."""
    x = small_inputs(9000, 160, 16, 128, idx_dtype="bf16", seed=23)
    q, k = bf16(x["q_idx"]), bf16(x["k_idx"])
    q8, bq = dsa.dsa_index_to_fp8(q)
    k8, bk = dsa.dsa_index_to_fp8(k)
    assert int(bq.item()) == 0 and int(bk.item()) == 0
    Q, K, V = bf16(x["Q"]), bf16(x["K"]), bf16(x["V"])
    i16, o16 = dsa.dsa_prefill(q, k, Q, K, V, 2048)
    i8, o8 = dsa.dsa_prefill(q8, k8, Q, K, V, 2048)
    assert dsa.dsa_sync_status() == 0
    assert torch.equal(i8, i16)
    assert torch.equal(o8.view(torch.int16), o16.view(torch.int16))
    rows = np.unique(np.concatenate([np.arange(0, 9000, 211), [2047, 2048, 8999]])).astype(np.int64)
    compare(x, "bf16", 2048, i8.cpu().numpy(), o8.view(torch.int16).cpu().numpy().view(np.uint16), rows=rows)


# ------------------------------------------------------------------ prefill of a chunk of rows

def run_chunk(dsa, x, q0, top_k, **kw):
    """Rows q0 .. Lk-1 of x against keys 0 .. Lk-1 through dsa_prefill_chunk."""
    Lk = x["q_idx"].shape[0]
    q, k = to_dev(x["q_idx"][q0:]), to_dev(x["k_idx"])
    if q.dtype == torch.uint16:
        q, k = q.view(torch.bfloat16), k.view(torch.bfloat16)
    idx, O = dsa.dsa_prefill_chunk(q, k, bf16(x["Q"][q0:]), bf16(x["K"]), bf16(x["V"]), top_k, **kw)
    assert dsa.dsa_sync_status() == 0
    return idx.cpu().numpy(), O.view(torch.int16).cpu().numpy().view(np.uint16)


@pytest.mark.parametrize("Lk,q0,top_k,H,D,d,idx_dtype", [
    (2333, 1633, 256, 16, 128, 96, "fp8"),     # chunk start off every tile boundary
    (5000, 4999, 2048, 16, 128, 128, "fp8"),   # one new token (decode as a chunk)
    (3000, 64, 300, 4, 64, 160, "bf16"),       # most rows of the sequence, head dim 64
    (4100, 2048, 1024, 3, 128, 128, "fp8"),    # chunk starting on a key-tile boundary
])
def test_prefill_chunk_matches_oracle_rows(dsa, Lk, q0, top_k, H, D, d, idx_dtype):
    x = small_inputs(Lk, d, H, D, idx_dtype=idx_dtype, seed=21)
    idx, O = run_chunk(dsa, x, q0, top_k)
    rows = np.arange(q0, Lk, dtype=np.int64)
    ri, ro = oracle.prefill_rows(x, idx_dtype, top_k, rows=rows)
    assert np.array_equal(idx, ri)
    assert np.abs(bits_to_f32(O) - bits_to_f32(ro)).max() <= ATOL


def test_prefill_chunk_forced_fallback(dsa, force_fallback):
    x = small_inputs(6000, 128, 16, 128, seed=22)
    force_fallback(9)
    idx, O = run_chunk(dsa, x, 3500, 2048)
    ri, ro = oracle.prefill_rows(x, "fp8", 2048, rows=np.arange(3500, 6000, dtype=np.int64))
    assert np.array_equal(idx, ri)
    assert np.abs(bits_to_f32(O) - bits_to_f32(ro)).max() <= ATOL


def test_prefill_chunks_in_zigzag_order_equal_the_whole_prefill(dsa):
    """The 32K workload split as for 4 ranks (8 zig-zag chunks): every chunk
    through dsa_prefill_chunk against its key prefix gives, row for row, the
    indices and outputs of the whole-sequence call."""
    from sparse_attention_10_b200.zigzag import zigzag_chunks
    w = synth.WORKLOADS["prefill_32k"]
    x = synth.prefill_inputs_torch(w, device="cuda")
    idx_all, O_all = dsa.dsa_prefill(x["q_idx"], x["k_idx"], x["Q"], x["K"], x["V"], w.top_k)
    assert dsa.dsa_sync_status() == 0
    for r in range(4):
        for a, b in zigzag_chunks(w.L, 4, r):
            idx, O = dsa.dsa_prefill_chunk(x["q_idx"][a:b], x["k_idx"][:b], x["Q"][a:b], x["K"][:b],
                                           x["V"][:b], w.top_k)
            assert dsa.dsa_sync_status() == 0
            assert torch.equal(idx, idx_all[a:b]), (a, b)
            assert torch.equal(O.view(torch.int16), O_all[a:b].view(torch.int16)), (a, b)


# ------------------------------------------------------------------ prefill, full size

def sampled_rows(L, k, n=2048, seed=0):
    rng = np.random.default_rng(seed)
    fixed = [0, 1, 127, 128, k - 2, k - 1, k, k + 1, 2 * k, 4 * k, L // 2, L - 129, L - 128, L - 2, L - 1]
    rows = np.concatenate([np.array([r for r in fixed if 0 <= r < L]), rng.integers(0, L, n)])
    return np.unique(rows).astype(np.int64)


def check_index_properties(idx, top_k):
    t = torch.from_numpy(idx).cuda()
    L = t.shape[0]
    m = torch.clamp(torch.arange(L, device="cuda") + 1, max=top_k)
    col = torch.arange(top_k, device="cuda")[None, :]
    valid = col < m[:, None]
    assert bool(((t >= 0) == valid).all()), "-1 padding in the wrong place"
    assert bool((t[valid] <= torch.arange(L, device="cuda")[:, None].expand_as(t)[valid]).all()), "non-causal index"
    s, _ = torch.sort(torch.where(valid, t, torch.full_like(t, -1)), dim=1)
    dup = (s[:, 1:] == s[:, :-1]) & (s[:, 1:] >= 0)
    assert not bool(dup.any()), "duplicate index in a row"


def host_copy(x):
    out = {}
    for k, v in x.items():
        if isinstance(v, torch.Tensor):
            t = v.cpu()
            if t.dtype == torch.bfloat16:
                t = t.view(torch.int16)
            out[k] = t.numpy().view(np.uint16) if t.dtype == torch.int16 else t.numpy()
        else:
            out[k] = v
    return out


@pytest.mark.parametrize("name,every_row", [("prefill_32k", True), ("prefill_64k", False),
                                            ("prefill_128k", False)])
def test_prefill_full_workloads(dsa, name, every_row):
    """The full-size workloads: every row of the 32K one against the oracle;
    at 64K and 128K the fixed boundary rows plus 2048 seeded random rows (the
    oracle runs on every host thread), and properties of every row."""
    w = synth.WORKLOADS[name]
    x = host_copy(synth.prefill_inputs_torch(w, device="cuda"))
    idx, O, stats = run_prefill(dsa, x, w.top_k)
    check_index_properties(idx, w.top_k)
    rows = None if every_row else sampled_rows(w.L, w.top_k)
    compare(x, w.idx_dtype, w.top_k, idx, O, rows=rows)
    assert stats["fallback_rows"] < w.L // 100, stats


def test_prefill_128k_forced_fallback_rows(dsa, force_fallback):
    # Full-size rows (up to 131072 keys each) through the grid-wide fallback:
    # every 10007th row is forced there and compared with the oracle.
    w = synth.WORKLOADS["prefill_128k"]
    x = host_copy(synth.prefill_inputs_torch(w, device="cuda"))
    force_fallback(10007)
    idx, O, stats = run_prefill(dsa, x, w.top_k)
    forced = np.arange(0, w.L, 10007, dtype=np.int64)
    assert stats["fallback_rows"] >= len(forced), stats
    check_index_properties(idx, w.top_k)
    compare(x, w.idx_dtype, w.top_k, idx, O, rows=forced)


# ------------------------------------------------------------------ decode

def run_decode(dsa, xd, top_k):
    t = {k: to_dev(xd[k]) for k in ("k_idx", "K", "V", "q_idx", "Q", "seq_start")}
    O, idx = dsa.dsa_decode(t["k_idx"], t["K"].view(torch.bfloat16), t["V"].view(torch.bfloat16),
                            t["seq_start"], t["q_idx"], t["Q"].view(torch.bfloat16), top_k,
                            int(xd["lengths"].max()))
    assert dsa.dsa_sync_status() == 0
    return idx.cpu().numpy(), O.view(torch.int16).cpu().numpy().view(np.uint16)


def test_decode_small_ragged(dsa):
    w = synth.WORKLOADS["decode_64x128k"]
    lens = np.array([1, 2, 100, 2047, 2048, 2049, 4097, 9000, 70000], dtype=np.int64)
    xd = synth.decode_inputs(w, lengths=lens)
    idx, O = run_decode(dsa, xd, w.top_k)
    ri, ro = oracle.decode(xd, w.idx_dtype, w.top_k)
    assert np.array_equal(idx, ri)
    assert np.abs(bits_to_f32(O) - bits_to_f32(ro)).max() <= ATOL


def test_decode_small_top_k(dsa):
    w = synth.WORKLOADS["decode_64x128k"]
    lens = np.array([3, 50, 777], dtype=np.int64)
    xd = synth.decode_inputs(w, lengths=lens)
    idx, O = run_decode(dsa, xd, 40)
    ri, ro = oracle.decode(xd, w.idx_dtype, 40)
    assert np.array_equal(idx, ri)
    assert np.abs(bits_to_f32(O) - bits_to_f32(ro)).max() <= ATOL


@pytest.mark.parametrize("idx_dtype,d,top_k", [("fp8", 64, 300), ("fp8", 256, 512), ("bf16", 128, 256),
                                               ("bf16", 160, 128)])
def test_decode_index_formats(dsa, idx_dtype, d, top_k):
    import dataclasses
    w = dataclasses.replace(synth.WORKLOADS["decode_64x128k"], d_idx=d, idx_dtype=idx_dtype)
    lens = np.array([7, 513, 4100, 20000], dtype=np.int64)
    xd = synth.decode_inputs(w, lengths=lens)
    idx, O = run_decode(dsa, xd, top_k)
    ri, ro = oracle.decode(xd, idx_dtype, top_k)
    assert np.array_equal(idx, ri)
    assert np.abs(bits_to_f32(O) - bits_to_f32(ro)).max() <= ATOL


@pytest.mark.parametrize("B", [75, 100, 200])
def test_decode_batch_sizes(dsa, B):
    """Batches that take 3, 2 and 2 key splits per sequence on 148 SMs; lengths 1..3000 leave
    splits with no keys (a sequence shorter than its split count) and ragged last splits."""
    w = synth.WORKLOADS["decode_64x128k"]
    lens = np.array([1 + (i * 977) % 3000 for i in range(B)], dtype=np.int64)
    lens[:3] = [1, 2, 3]
    xd = synth.decode_inputs(w, lengths=lens)
    idx, O = run_decode(dsa, xd, 512)
    ri, ro = oracle.decode(xd, w.idx_dtype, 512)
    assert np.array_equal(idx, ri)
    assert np.abs(bits_to_f32(O) - bits_to_f32(ro)).max() <= ATOL


def test_decode_full_workload(dsa):
    w = synth.WORKLOADS["decode_64x128k"]
    xd = host_copy(synth.decode_inputs_torch(w, device="cuda"))
    idx, O = run_decode(dsa, xd, w.top_k)
    ri, ro = oracle.decode(xd, w.idx_dtype, w.top_k)
    assert np.array_equal(idx, ri)
    assert np.abs(bits_to_f32(O) - bits_to_f32(ro)).max() <= ATOL


def tie_queries(B, d, mode):
    """Decode queries whose scores tie widely: "zero" makes every score +0;
    "e0" puts a single 1 in dimension 0, so a score is relu(k_idx[s, 0] * scale)
    and takes one of nine values (about len/9 keys share each)."""
    q = np.zeros((B, d), dtype=np.int64)
    if mode == "e0":
        q[:, 0] = 1
    return synth.fp8_bytes_of_ints(q)


def boundary_bin_count(xd, top_k, scale):
    """Keys at or above the bin of each sequence's m-th best score, binning by
    the top bits of the FP32 score (bits 30..20), as the decode select does:
    above 8192 the select takes its many-candidate path."""
    out = []
    ss = xd["seq_start"]
    q = synth_fp8_values(xd["q_idx"])
    for b in range(len(ss) - 1):
        k = synth_fp8_values(xd["k_idx"][ss[b]:ss[b + 1]])
        sc = np.maximum(np.float32(k @ q[b]) * np.float32(scale), np.float32(0)).astype(np.float32)
        bins = sc.view(np.uint32) >> 20
        m = min(top_k, sc.size)
        kth = np.sort(bins)[::-1][m - 1]
        out.append(int((bins >= kth).sum()))
    return out


def synth_fp8_values(a):
    # the test inputs are exact small integers: decode E4M3 codes of -4..4
    table = {int(c): v for v, c in zip(range(-4, 5), synth.fp8_bytes_of_ints(np.arange(-4, 5)))}
    lut = np.zeros(256, dtype=np.float64)
    for c, v in table.items():
        lut[c] = v
    return lut[np.asarray(a)]


@pytest.mark.parametrize("mode,lens", [
    ("zero", [1, 5000, 8193, 20000, 131072]),
    ("e0", [9000, 30000, 100000, 131072]),
])
def test_decode_wide_ties_many_candidates(dsa, mode, lens):
    """Scores that tie across the k-th place on long sequences: more than 8192
    keys fall in the boundary bin, so the select compacts its candidates in
    global scratch and selects there; ties must still go to the lower index."""
    w = synth.WORKLOADS["decode_64x128k"]
    lens = np.array(lens, dtype=np.int64)
    xd = synth.decode_inputs(w, lengths=lens)
    xd["q_idx"] = tie_queries(len(lens), w.d_idx, mode)
    scale = oracle.default_index_scale(w.d_idx)
    assert max(boundary_bin_count(xd, w.top_k, scale)) > 8192
    idx, O = run_decode(dsa, xd, w.top_k)
    ri, ro = oracle.decode(xd, w.idx_dtype, w.top_k)
    assert np.array_equal(idx, ri)
    assert np.abs(bits_to_f32(O) - bits_to_f32(ro)).max() <= ATOL
    if mode == "zero":
        for b, n in enumerate(lens):
            m = min(int(n), w.top_k)
            assert idx[b, :m].tolist() == list(range(m))


# ------------------------------------------------------------------ several new tokens per sequence

def multi_case(lens, T, idx_dtype="fp8", d=128, D=128, seed=None):
    import dataclasses
    w = dataclasses.replace(synth.WORKLOADS["decode_64x128k"], d_idx=d, idx_dtype=idx_dtype, D=D)
    lens = np.array(lens, dtype=np.int64)
    xd = synth.decode_inputs(w, lengths=lens)
    mq = synth.multi_queries(w, len(lens), T)
    return w, dict(xd, q_idx=mq["q_idx"], Q=mq["Q"])


@pytest.mark.parametrize("T,idx_dtype,d,D,top_k,lens", [
    (2, "fp8", 128, 128, 2048, [2, 3, 100, 2049, 9000, 70000]),
    (4, "fp8", 128, 128, 512, [4, 5, 2048, 4100, 30000]),
    (3, "fp8", 64, 64, 300, [3, 777, 5000]),          # 64-byte index rows, head dim 64
    (4, "bf16", 64, 128, 1024, [4, 1500, 20000]),     # BF16 index rows of 128 bytes
])
def test_decode_multi_matches_oracle(dsa, T, idx_dtype, d, D, top_k, lens):
    w, x = multi_case(lens, T, idx_dtype, d, D)
    t = {k: to_dev(x[k]) for k in ("k_idx", "K", "V", "q_idx", "Q", "seq_start")}
    O, idx = dsa.dsa_decode_multi(t["k_idx"], t["K"].view(torch.bfloat16), t["V"].view(torch.bfloat16),
                                  t["seq_start"], t["q_idx"], t["Q"].view(torch.bfloat16), top_k, max(lens))
    assert dsa.dsa_sync_status() == 0
    ri, ro = oracle.decode_multi(x, idx_dtype, top_k)
    assert np.array_equal(idx.cpu().numpy(), ri)
    got = O.view(torch.int16).cpu().numpy().view(np.uint16)
    assert np.abs(bits_to_f32(got) - bits_to_f32(ro)).max() <= ATOL


@pytest.mark.parametrize("T,block_size", [(2, 64), (4, 16), (3, 1)])
def test_decode_paged_multi_matches_oracle(dsa, T, block_size):
    w, x = multi_case([4, 64, 2049, 20001], T)       # every length >= T
    xp = synth.paged_decode_inputs(w, x["lengths"], block_size)
    t = {k: to_dev(xp[k]) for k in ("k_idx_blocks", "K_blocks", "V_blocks", "block_table", "seq_lens")}
    O, idx = dsa.dsa_decode_paged_multi(t["k_idx_blocks"], t["K_blocks"].view(torch.bfloat16),
                                        t["V_blocks"].view(torch.bfloat16), t["block_table"], t["seq_lens"],
                                        to_dev(x["q_idx"]), bf16(x["Q"]), w.top_k, int(x["lengths"].max()))
    assert dsa.dsa_sync_status() == 0
    ri, ro = oracle.decode_multi(x, w.idx_dtype, w.top_k)
    assert np.array_equal(idx.cpu().numpy(), ri)
    got = O.view(torch.int16).cpu().numpy().view(np.uint16)
    assert np.abs(bits_to_f32(got) - bits_to_f32(ro)).max() <= ATOL


def test_decode_multi_full_batch_equals_single_token_steps(dsa):
    """The 64-sequence batch (65K-131K rows each) with T = 2: token 1 sees every row and
    is the single-token decode of the same query; token 0 is the single-token decode of the
    batch with each sequence's last row dropped."""
    w = synth.WORKLOADS["decode_64x128k"]
    xd = synth.decode_inputs_torch(w, device="cuda")
    mq = synth.multi_queries_torch(w, w.B, 2, device="cuda")
    ss, lens = xd["seq_start"], xd["lengths"]
    mx = int(lens.max())
    O, idx = dsa.dsa_decode_multi(xd["k_idx"], xd["K"], xd["V"], ss, mq["q_idx"], mq["Q"], w.top_k, mx)
    assert dsa.dsa_sync_status() == 0
    O1, i1 = dsa.dsa_decode(xd["k_idx"], xd["K"], xd["V"], ss, mq["q_idx"][:, 1].contiguous(),
                            mq["Q"][:, 1].contiguous(), w.top_k, mx)
    assert torch.equal(idx[:, 1], i1)
    assert (O[:, 1].float() - O1.float()).abs().max().item() <= ATOL
    keep = torch.ones(xd["k_idx"].shape[0], dtype=torch.bool, device="cuda")
    keep[ss[1:] - 1] = False                               # drop each sequence's last row
    ss0 = ss - torch.arange(ss.shape[0], device="cuda", dtype=torch.int64)
    O0, i0 = dsa.dsa_decode(xd["k_idx"][keep].contiguous(), xd["K"][keep].contiguous(), xd["V"][keep].contiguous(),
                            ss0, mq["q_idx"][:, 0].contiguous(), mq["Q"][:, 0].contiguous(), w.top_k, mx)
    assert dsa.dsa_sync_status() == 0
    assert torch.equal(idx[:, 0], i0)
    assert (O[:, 0].float() - O0.float()).abs().max().item() <= ATOL


def test_decode_multi_checks(dsa):
    import ctypes
    lib = dsa.load()
    w, x = multi_case([5, 9], 2, d=96)          # 96-byte FP8 index rows: no multi-token scan
    t = {k: to_dev(x[k]) for k in ("k_idx", "K", "V", "q_idx", "Q", "seq_start")}
    P = lambda a: ctypes.c_void_p(a.data_ptr())
    args = lambda T: (P(t["k_idx"]), P(t["K"]), P(t["V"]), P(t["seq_start"]), 2, T, 14, 9, 0, 96, 128,
                      P(t["q_idx"]), P(t["Q"]), 16, 64, float("nan"), float("nan"), P(t["Q"]), None)
    ws = torch.empty(1 << 24, dtype=torch.uint8, device="cuda")
    assert lib.dsa_decode_multi(*args(2), P(ws), ws.numel(), None) == 2   # DSA_ERR_UNSUPPORTED
    assert lib.dsa_decode_multi(*args(5), P(ws), ws.numel(), None) == 1   # T outside [1, 4]
    assert lib.dsa_decode_multi_workspace_size(2, 5, 14, 96, 0, 16, 128, 64) == 0
    # lengths shorter than T are caught on the device: the call records DSA_ERR_INVALID_ARG
    w, x = multi_case([1, 9], 1)
    mq = synth.multi_queries(w, 2, 2)
    t = {k: to_dev(x[k]) for k in ("k_idx", "K", "V", "seq_start")}
    dsa.dsa_decode_multi(t["k_idx"], t["K"].view(torch.bfloat16), t["V"].view(torch.bfloat16), t["seq_start"],
                         to_dev(mq["q_idx"]), bf16(mq["Q"]), 64, 9)
    assert dsa.dsa_sync_status() == 1
    assert dsa.dsa_sync_status() == 0


# ------------------------------------------------------------------ paged decode

def run_decode_paged(dsa, xp, top_k, max_len=None):
    t = {k: to_dev(xp[k]) for k in ("k_idx_blocks", "K_blocks", "V_blocks", "block_table", "seq_lens",
                                    "q_idx", "Q")}
    O, idx = dsa.dsa_decode_paged(t["k_idx_blocks"], t["K_blocks"].view(torch.bfloat16),
                                  t["V_blocks"].view(torch.bfloat16), t["block_table"], t["seq_lens"],
                                  t["q_idx"], t["Q"].view(torch.bfloat16), top_k,
                                  int(xp["lengths"].max()) if max_len is None else max_len)
    return idx, O


@pytest.mark.parametrize("idx_dtype,d,H,D,top_k", [("bf16", 160, 16, 128, 2048), ("fp8", 128, 4, 64, 256)])
def test_prefill_step_replays_from_a_cuda_graph(dsa, idx_dtype, d, H, D, top_k):
    """A prefill step (threshold sample, filter, select with its queued large-row
    and fallback passes, attention) captured in a CUDA graph replays to the
    results of an ordinary call: every decision between the kernels is taken on
    the device."""
    L = 5000
    x = small_inputs(L, d, H, D, idx_dtype)
    q, k = to_dev(x["q_idx"]), to_dev(x["k_idx"])
    if q.dtype == torch.uint16:
        q, k = q.view(torch.bfloat16), k.view(torch.bfloat16)
    Q, K, V = bf16(x["Q"]), bf16(x["K"]), bf16(x["V"])
    ws = torch.empty(dsa.dsa_prefill_workspace_size(L, d, 0 if idx_dtype == "fp8" else 1, H, D, top_k),
                     dtype=torch.uint8, device="cuda")
    idx = torch.empty((L, top_k), dtype=torch.int32, device="cuda")
    O = torch.empty((L, H, D), dtype=torch.bfloat16, device="cuda")

    def step():
        dsa.dsa_prefill(q, k, Q, K, V, top_k, indices=idx, O=O, workspace=ws)

    step()
    torch.cuda.synchronize()
    assert dsa.dsa_sync_status() == 0
    ref_idx, ref_o = idx.clone(), O.clone()
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        step()
    torch.cuda.current_stream().wait_stream(side)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        step()
    idx.zero_()
    O.zero_()
    g.replay()
    torch.cuda.synchronize()
    assert dsa.dsa_sync_status() == 0
    assert torch.equal(idx, ref_idx)
    assert torch.equal(O.view(torch.int16), ref_o.view(torch.int16))
    del g


def test_decode_step_replays_from_a_cuda_graph(dsa):
    """A decode step (memsets and programmatically launched kernels) captured in
    a CUDA graph replays to the results of an ordinary call, contiguous and
    paged cache."""
    w = synth.WORKLOADS["decode_64x128k"]
    lens = np.array([2, 100, 2049, 9000, 70000], dtype=np.int64)
    xd = synth.decode_inputs(w, lengths=lens)
    xp = synth.paged_decode_inputs(w, lens, 64)
    t = {k: to_dev(xd[k]) for k in ("k_idx", "K", "V", "q_idx", "Q", "seq_start")}
    tp = {k: to_dev(xp[k]) for k in ("k_idx_blocks", "K_blocks", "V_blocks", "block_table", "seq_lens",
                                     "q_idx", "Q")}
    B, mx = len(lens), int(lens.max())
    O = torch.empty((B, w.H, w.D), dtype=torch.bfloat16, device="cuda")
    idx = torch.empty((B, w.top_k), dtype=torch.int32, device="cuda")
    Op, idxp = torch.empty_like(O), torch.empty_like(idx)
    ws = torch.empty(dsa.dsa_decode_workspace_size(B, int(lens.sum()), w.d_idx, 0, w.H, w.D, w.top_k),
                     dtype=torch.uint8, device="cuda")
    wsp = torch.empty(dsa.dsa_decode_paged_workspace_size(B, mx, w.d_idx, 0, w.H, w.D, w.top_k),
                      dtype=torch.uint8, device="cuda")

    def step():
        dsa.dsa_decode(t["k_idx"], t["K"].view(torch.bfloat16), t["V"].view(torch.bfloat16), t["seq_start"],
                       t["q_idx"], t["Q"].view(torch.bfloat16), w.top_k, mx, O=O, indices=idx, workspace=ws)
        dsa.dsa_decode_paged(tp["k_idx_blocks"], tp["K_blocks"].view(torch.bfloat16),
                             tp["V_blocks"].view(torch.bfloat16), tp["block_table"], tp["seq_lens"],
                             tp["q_idx"], tp["Q"].view(torch.bfloat16), w.top_k, mx, O=Op, indices=idxp,
                             workspace=wsp)

    step()
    torch.cuda.synchronize()
    assert dsa.dsa_sync_status() == 0
    ref = [x.clone() for x in (idx, O, idxp, Op)]
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        step()
    torch.cuda.current_stream().wait_stream(side)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        step()
    for x in (idx, O, idxp, Op):
        x.zero_()
    g.replay()
    torch.cuda.synchronize()
    assert dsa.dsa_sync_status() == 0
    for x, y in zip((idx, O, idxp, Op), ref):
        assert torch.equal(x.view(torch.int16) if x.dtype == torch.bfloat16 else x,
                           y.view(torch.int16) if y.dtype == torch.bfloat16 else y)
    del g


def test_decode_with_stage_timing_matches_plain_calls(dsa):
    """The decode kernels follow one another by programmatic launches; stage
    timing records CUDA events between them.  Results with and without the
    events must be identical (contiguous, paged and two-token steps), and the
    decode stages must be timed."""
    w = synth.WORKLOADS["decode_64x128k"]
    lens = np.array([2, 100, 2049, 9000, 70000], dtype=np.int64)
    xd = synth.decode_inputs(w, lengths=lens)
    xp = synth.paged_decode_inputs(w, lens, 64)
    mq = synth.multi_queries(w, len(lens), 2)
    t = {k: to_dev(xd[k]) for k in ("k_idx", "K", "V", "seq_start")}
    tm = {k: to_dev(mq[k]) for k in ("q_idx", "Q")}

    def calls():
        a = run_decode(dsa, xd, w.top_k)
        idx, O = run_decode_paged(dsa, xp, w.top_k)
        b = (idx.cpu().numpy(), O.view(torch.int16).cpu().numpy())
        O2, idx2 = dsa.dsa_decode_multi(t["k_idx"], t["K"].view(torch.bfloat16), t["V"].view(torch.bfloat16),
                                        t["seq_start"], tm["q_idx"], tm["Q"].view(torch.bfloat16), w.top_k,
                                        int(lens.max()))
        assert dsa.dsa_sync_status() == 0
        return a + b + (idx2.cpu().numpy(), O2.view(torch.int16).cpu().numpy())

    plain = calls()
    dsa.dsa_stage_times()   # reset
    dsa.dsa_stage_timing(True)
    try:
        timed = calls()
        times = dsa.dsa_stage_times()
    finally:
        dsa.dsa_stage_timing(False)
    for x, y in zip(plain, timed):
        assert np.array_equal(x, y)
    assert times["decode_scan_select"][1] > 0 and times["decode_scan_select"][0] > 0
    assert times["decode_attention"][1] > 0 and times["decode_attention"][0] > 0


@pytest.mark.parametrize("block_size,idx_dtype,d,D,top_k", [
    (1, "fp8", 128, 128, 256),       # one row per block
    (16, "fp8", 128, 128, 2048),
    (64, "bf16", 160, 128, 512),     # rows of 320 bytes: the generic scan kernel
    (2048, "bf16", 128, 128, 128),   # one block per scan chunk
    (4096, "fp8", 64, 64, 300),      # blocks longer than a scan chunk; head dim 64
])
def test_decode_paged_matches_oracle(dsa, block_size, idx_dtype, d, D, top_k):
    import dataclasses
    w = dataclasses.replace(synth.WORKLOADS["decode_64x128k"], d_idx=d, idx_dtype=idx_dtype, D=D)
    lens = np.array([1, 2, 100, 2047, 2048, 2049, 4097, 9000, 20001], dtype=np.int64)
    xp = synth.paged_decode_inputs(w, lens, block_size)
    idx, O = run_decode_paged(dsa, xp, top_k)
    assert dsa.dsa_sync_status() == 0
    ri, ro = oracle.decode_paged(xp, idx_dtype, top_k)
    assert np.array_equal(idx.cpu().numpy(), ri)
    got = O.view(torch.int16).cpu().numpy().view(np.uint16)
    assert np.abs(bits_to_f32(got) - bits_to_f32(ro)).max() <= ATOL


@pytest.mark.parametrize("mode", ["zero", "e0"])
def test_decode_paged_wide_ties_many_candidates(dsa, mode):
    """The wide-tie decode of test_decode_wide_ties_many_candidates over a
    block-paged cache (blocks of 64 rows in seeded order)."""
    w = synth.WORKLOADS["decode_64x128k"]
    lens = np.array([3000, 20000, 131072], dtype=np.int64)
    xp = synth.paged_decode_inputs(w, lens, 64)
    xp["q_idx"] = tie_queries(len(lens), w.d_idx, mode)
    c = dict(xp["contiguous"], q_idx=xp["q_idx"])
    assert max(boundary_bin_count(c, w.top_k, oracle.default_index_scale(w.d_idx))) > 8192
    idx, O = run_decode_paged(dsa, xp, w.top_k)
    assert dsa.dsa_sync_status() == 0
    ri, ro = oracle.decode_paged(xp, w.idx_dtype, w.top_k)
    assert np.array_equal(idx.cpu().numpy(), ri)
    got = O.view(torch.int16).cpu().numpy().view(np.uint16)
    assert np.abs(bits_to_f32(got) - bits_to_f32(ro)).max() <= ATOL


def test_decode_paged_shared_blocks(dsa):
    """Two sequences whose block tables point at the same blocks (a shared
    prefix) read the same rows: equal inputs give equal results."""
    w = synth.WORKLOADS["decode_64x128k"]
    lens = np.array([3000, 5000], dtype=np.int64)
    xp = synth.paged_decode_inputs(w, lens, 64)
    table = xp["block_table"].copy()
    n0 = -(-3000 // 64)
    table[1, :n0] = table[0, :n0]          # sequence 1 starts with sequence 0's blocks
    shared = dict(xp, block_table=table)
    idx, O = run_decode_paged(dsa, shared, 2048)
    assert dsa.dsa_sync_status() == 0
    ri, ro = oracle.decode_paged(shared, "fp8", 2048)
    assert np.array_equal(idx.cpu().numpy(), ri)
    got = O.view(torch.int16).cpu().numpy().view(np.uint16)
    assert np.abs(bits_to_f32(got) - bits_to_f32(ro)).max() <= ATOL


def test_decode_paged_rejects_bad_table_on_device(dsa):
    """A block id outside the pool, or a length past max_len, is caught by the
    device-side check before any kernel reads through the table: the call
    records DSA_ERR_INVALID_ARG and the next valid call is unaffected."""
    w = synth.WORKLOADS["decode_64x128k"]
    lens = np.array([100, 700, 50], dtype=np.int64)
    xp = synth.paged_decode_inputs(w, lens, 64)
    nb = xp["k_idx_blocks"].shape[0]
    bad = xp["block_table"].copy()
    bad[1, 5] = nb                          # sequence 1 reaches block 5 (rows 320..383)
    run_decode_paged(dsa, dict(xp, block_table=bad), 256)
    assert dsa.dsa_sync_status() == 1
    run_decode_paged(dsa, xp, 256, max_len=600)   # sequence 1 is longer than max_len
    assert dsa.dsa_sync_status() == 1
    idx, O = run_decode_paged(dsa, xp, 256)
    assert dsa.dsa_sync_status() == 0
    ri, _ = oracle.decode_paged(xp, "fp8", 256, want_o=False)
    assert np.array_equal(idx.cpu().numpy(), ri)


def test_decode_paged_full_workload(dsa):
    """The 64-sequence decode batch (65K-131K cached rows each) in blocks of 64
    rows placed by a seeded permutation."""
    w = synth.WORKLOADS["decode_64x128k"]
    xd = synth.decode_inputs_torch(w, device="cuda")
    xp = synth.paged_decode_inputs_torch(xd, 64)
    O, idx = dsa.dsa_decode_paged(xp["k_idx_blocks"], xp["K_blocks"].view(torch.bfloat16),
                                  xp["V_blocks"].view(torch.bfloat16), xp["block_table"], xp["seq_lens"],
                                  xp["q_idx"], xp["Q"].view(torch.bfloat16), w.top_k,
                                  int(xp["lengths"].max()))
    assert dsa.dsa_sync_status() == 0
    idx, O = idx.cpu().numpy(), O.view(torch.int16).cpu().numpy().view(np.uint16)
    del xp
    ri, ro = oracle.decode(host_copy(xd), w.idx_dtype, w.top_k)
    assert np.array_equal(idx, ri)
    assert np.abs(bits_to_f32(O) - bits_to_f32(ro)).max() <= ATOL


def test_device_generator_matches_numpy_definition():
    k = synth.stream_key(5, 6)
    a = synth.normal_bf16(k, 3_000_001)
    b = synth.normal_bf16_torch(k, 3_000_001, device="cuda").view(torch.int16).cpu().numpy().view(np.uint16)
    assert (a == b).mean() > 0.999999
    a = synth.uniform_ints(k, 1_000_000)
    b = synth.uniform_ints_torch(k, 1_000_000, device="cuda").cpu().numpy()
    assert np.array_equal(a, b)


# ------------------------------------------------------------------ failure detection

def test_bounded_wait_reports_timeout_and_context_survives(dsa):
    assert dsa.dsa_sync_status() == 0
    dsa.dsa_debug_wait_timeout(1_000_000)   # 1 ms, nothing completes the barrier
    assert dsa.dsa_sync_status() == 5       # DSA_ERR_TIMEOUT, read and cleared
    assert dsa.dsa_sync_status() == 0
    x = small_inputs(300, 128, 4, 64, seed=12)
    idx, O, _ = run_prefill(dsa, x, 32)
    compare(x, "fp8", 32, idx, O)
