"""Pins of the CPU oracle against things other than itself.

Each test ties one part of the oracle to a library routine, a closed form, a
special case or brute force, so that a dropped term, a wrong sign or index, or
a transposed operand in the oracle fails at least one of them.  The method is
DeepSeek Sparse Attention as the DeepSeek Sparse Attention page
(kwkr.cn/news/60693) describes it: lightning indexer (section 3.2), top-k
token selection (section 3.3), BF16 attention over the kept keys with one
shared K/V (sections 4.1, 4.2).
"""
import math

import numpy as np
import pytest
import torch

import synth

pytestmark = pytest.mark.filterwarnings("ignore::DeprecationWarning")


# ---------------------------------------------------------------- helpers

def f32(x):
    return np.float32(x)


def ints_as(idx_dtype, v):
    return synth.fp8_bytes_of_ints(v) if idx_dtype == "fp8" else synth.bf16_bits_of_ints(v)


def ref_scores_from_ints(qi, ki, scale):
    """relu(fp32(fp32(q.k) * scale)) for integer matrices, via numpy int64 matmul."""
    dot = (qi.astype(np.int64) @ ki.astype(np.int64).T).astype(np.float32)
    s = dot * np.float32(scale)
    return np.where(s > 0, s, np.float32(0.0)).astype(np.float32)


def within_half_bf16_ulp(got, ref):
    """|got - ref| <= half a BF16 ulp of ref (plus 1e-12 relative fp64 slack)."""
    _, e = np.frexp(ref)                      # ref = m * 2^e, m in [0.5, 1)
    half_ulp = np.ldexp(1.0, e - 9)           # bf16 keeps 8 significant bits
    return np.all(np.abs(got - ref) <= half_ulp + np.abs(ref) * 1e-12 + 1e-300)


def bf16_bits_to_f64(b):
    return (np.asarray(b, dtype=np.uint32) << 16).view(np.float32).astype(np.float64)


def stable_topk(row_scores, k):
    """First k of a stable descending sort (ties -> lower index), -1 padded."""
    order = np.argsort(-row_scores, kind="stable")[:k]
    out = np.full(k, -1, dtype=np.int32)
    out[: order.shape[0]] = order
    return out


def small_prefill(L, d, H, D, idx_dtype="fp8", seed=7, lo=-4, hi=4):
    key = synth.stream_key(seed, 99, L, d)
    qi = synth.uniform_ints(key, L * d, lo, hi).reshape(L, d)
    ki = synth.uniform_ints(key, L * d, lo, hi, start=L * d).reshape(L, d)
    inp = {
        "q_idx": ints_as(idx_dtype, qi), "k_idx": ints_as(idx_dtype, ki),
        "Q": synth.normal_bf16(synth.stream_key(seed, 1, L), L * H * D).reshape(L, H, D),
        "K": synth.normal_bf16(synth.stream_key(seed, 2, L), L * D).reshape(L, D),
        "V": synth.normal_bf16(synth.stream_key(seed, 3, L), L * D).reshape(L, D),
    }
    return inp, qi, ki


# ---------------------------------------------------------------- formats

def test_fp8_decoder_matches_torch_e4m3fn(oracle_mod):
    ref = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = np.array([oracle_mod.fp8_e4m3_value(b) for b in range(256)])
    nan = np.isnan(ref)
    assert np.array_equal(nan, np.isnan(got))
    assert np.array_equal(got[~nan], ref[~nan])
    # OCP FP8 spec anchors: max normal, min normal, min subnormal, one.
    assert oracle_mod.fp8_e4m3_value(0x7E) == 448.0
    assert oracle_mod.fp8_e4m3_value(0x08) == 2.0 ** -6
    assert oracle_mod.fp8_e4m3_value(0x01) == 2.0 ** -9
    assert oracle_mod.fp8_e4m3_value(0x38) == 1.0
    assert oracle_mod.fp8_e4m3_value(0xC4) == -3.0


def test_small_int_encodings_are_exact(oracle_mod):
    v = np.arange(-4, 5)
    for b, x in zip(synth.fp8_bytes_of_ints(v), v):
        assert oracle_mod.fp8_e4m3_value(int(b)) == float(x)
    for h, x in zip(synth.bf16_bits_of_ints(v), v):
        assert oracle_mod.bf16_value(int(h)) == float(x)


def test_bf16_decoder_matches_torch(oracle_mod):
    bits = np.arange(0, 65536, 97, dtype=np.uint16)
    ref = torch.from_numpy(bits.astype(np.int16)).view(torch.bfloat16).to(torch.float64).numpy()
    got = np.array([oracle_mod.bf16_value(int(b)) for b in bits])
    nan = np.isnan(ref)
    assert np.array_equal(got[~nan], ref[~nan])


def test_bf16_round_matches_torch_on_float32_values(oracle_mod):
    rng = np.random.default_rng(3)
    x = np.concatenate([rng.standard_normal(4000).astype(np.float32),
                        (rng.standard_normal(500) * 1e-39).astype(np.float32),  # subnormals
                        np.float32([0.0, -0.0, 1.0, 3e38, -3e38])])
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().astype(np.uint16)
    got = np.array([oracle_mod.bf16_round(float(v)) for v in x], dtype=np.uint16)
    assert np.array_equal(got, ref)


def test_bf16_round_is_a_single_rounding(oracle_mod):
    # 1 + 2^-8 is the exact midpoint between bf16 neighbours 1 and 1 + 2^-7; a
    # value just above it must round up, which a detour through float32 gets wrong.
    assert oracle_mod.bf16_round(1.0 + 2.0 ** -8 + 2.0 ** -40) == 0x3F81
    assert oracle_mod.bf16_round(1.0 + 2.0 ** -8) == 0x3F80        # tie -> even
    assert oracle_mod.bf16_round(1.0 + 3 * 2.0 ** -8) == 0x3F82    # tie -> even (up)
    assert oracle_mod.bf16_round(-2.0) == 0xC000


# ---------------------------------------------------------------- indexer

@pytest.mark.parametrize("idx_dtype,d", [("fp8", 96), ("fp8", 128), ("bf16", 160), ("fp8", 32)])
def test_indexer_scores_integer_inputs_bit_exact(oracle_mod, idx_dtype, d):
    Lq, Lk = 37, 53
    key = synth.stream_key(11, d)
    qi = synth.uniform_ints(key, Lq * d).reshape(Lq, d)
    ki = synth.uniform_ints(key, Lk * d, start=Lq * d).reshape(Lk, d)
    scale = oracle_mod.default_index_scale(d)
    got = oracle_mod.indexer_scores(ints_as(idx_dtype, qi), ints_as(idx_dtype, ki), idx_dtype, scale)
    ref = ref_scores_from_ints(qi, ki, scale)
    assert got.view(np.uint32).tolist() == ref.view(np.uint32).tolist()  # +0, never -0


def test_indexer_scores_general_fp8_inputs_bit_exact(oracle_mod):
    # Arbitrary finite E4M3 bytes: a float64 dot of d <= 256 FP8 products is
    # exact, so numpy's float64 matmul gives the same fp32 score.
    rng = np.random.default_rng(5)
    d = 64
    def finite_bytes(n):
        b = rng.integers(0, 256, n, dtype=np.uint8)
        return np.where((b & 0x7F) == 0x7F, np.uint8(0x38), b).astype(np.uint8)
    q = finite_bytes(20 * d).reshape(20, d)
    k = finite_bytes(30 * d).reshape(30, d)
    dec = torch.from_numpy(np.arange(256, dtype=np.uint8)).view(torch.float8_e4m3fn).double().numpy()
    scale = 0.125
    dot = (dec[q] @ dec[k].T).astype(np.float32)
    s = dot * np.float32(scale)
    ref = np.where(s > 0, s, np.float32(0.0)).astype(np.float32)
    got = oracle_mod.indexer_scores(q, k, "fp8", scale)
    assert got.view(np.uint32).tolist() == ref.view(np.uint32).tolist()


def test_indexer_closed_form_unit_query(oracle_mod):
    # q = e_0 and k[s, 0] = a_s (other dims 0) -> I[s] = relu(a_s * scale).
    d = 128
    a = np.arange(-4, 5)
    q = np.zeros((1, d), dtype=np.int64); q[0, 0] = 1
    k = np.zeros((9, d), dtype=np.int64); k[:, 0] = a
    scale = oracle_mod.default_index_scale(d)
    got = oracle_mod.indexer_scores(synth.fp8_bytes_of_ints(q), synth.fp8_bytes_of_ints(k), "fp8", scale)[0]
    expect = [max(0.0, float(f32(x) * f32(scale))) for x in a]
    assert got.tolist() == expect
    assert scale == float(f32(2.0 ** -3.5))


# ---------------------------------------------------------------- selection

@pytest.mark.parametrize("k", [1, 7, 64, 300])
def test_selection_equals_stable_full_sort(oracle_mod, k):
    L, d = 200, 32
    inp, qi, ki = small_prefill(L, d, 2, 64, lo=-2, hi=2)   # narrow range -> many ties
    scale = oracle_mod.default_index_scale(d)
    idx, _ = oracle_mod.prefill_rows(inp, "fp8", k, want_o=False)
    S = ref_scores_from_ints(qi, ki, scale)
    for t in range(L):
        assert idx[t].tolist() == stable_topk(S[t, : t + 1], k).tolist(), t


def test_selection_all_zero_scores_keeps_lowest_indices(oracle_mod):
    L, d, k = 50, 32, 20
    inp, _, _ = small_prefill(L, d, 1, 64)
    inp["q_idx"] = np.zeros_like(inp["q_idx"])          # every score is +0
    idx, _ = oracle_mod.prefill_rows(inp, "fp8", k, want_o=False)
    for t in range(L):
        m = min(k, t + 1)
        assert idx[t, :m].tolist() == list(range(m))
        assert (idx[t, m:] == -1).all()


def test_selection_positives_first_then_zeros_by_index(oracle_mod):
    # Row of 10 keys with 3 positive scores: positives by value, then zeros by index.
    d = 32
    q = np.zeros((10, d), dtype=np.int64); q[:, 0] = 1
    k = np.zeros((10, d), dtype=np.int64)
    k[:, 0] = [0, -3, 2, 0, 4, -1, 0, 2, -4, 0]
    inp = {"q_idx": synth.fp8_bytes_of_ints(q), "k_idx": synth.fp8_bytes_of_ints(k)}
    idx, _ = oracle_mod.prefill_rows(inp, "fp8", 8, rows=[9], want_o=False)
    assert idx[0].tolist() == [4, 2, 7, 0, 1, 3, 5, 6]


def test_selection_k_at_least_length_is_permutation(oracle_mod):
    L = 40
    inp, _, _ = small_prefill(L, 32, 1, 64)
    idx, _ = oracle_mod.prefill_rows(inp, "fp8", 64, want_o=False)
    for t in range(L):
        assert sorted(idx[t, : t + 1].tolist()) == list(range(t + 1))
        assert (idx[t, t + 1:] == -1).all()


# ---------------------------------------------------------------- attention

def test_dense_limit_equals_torch_sdpa(oracle_mod):
    # With k >= L the sparse attention is dense causal attention.
    L, d, H, D = 48, 32, 3, 64
    inp, _, _ = small_prefill(L, d, H, D)
    _, O = oracle_mod.prefill_rows(inp, "fp8", 64)
    q = torch.from_numpy(bf16_bits_to_f64(inp["Q"])).permute(1, 0, 2)            # [H, L, D]
    kk = torch.from_numpy(bf16_bits_to_f64(inp["K"]))[None].expand(H, L, D)
    vv = torch.from_numpy(bf16_bits_to_f64(inp["V"]))[None].expand(H, L, D)
    ref = torch.nn.functional.scaled_dot_product_attention(q, kk, vv, is_causal=True)
    ref = ref.permute(1, 0, 2).numpy()
    got = bf16_bits_to_f64(O)
    # one rounding to bf16: within half an ulp of the fp64 value
    assert within_half_bf16_ulp(got, ref)


def test_constant_value_rows_give_that_row(oracle_mod):
    L, d, H, D = 30, 32, 2, 64
    inp, _, _ = small_prefill(L, d, H, D)
    inp["V"] = np.broadcast_to(inp["V"][5], (L, D)).copy()
    _, O = oracle_mod.prefill_rows(inp, "fp8", 8)
    assert np.array_equal(O, np.broadcast_to(inp["V"][5], (L, H, D)))


def test_first_query_attends_only_to_itself(oracle_mod):
    L, d, H, D = 16, 32, 4, 128
    inp, _, _ = small_prefill(L, d, H, D)
    idx, O = oracle_mod.prefill_rows(inp, "fp8", 4, rows=[0])
    assert idx[0].tolist() == [0, -1, -1, -1]
    assert np.array_equal(O[0], np.broadcast_to(inp["V"][0], (H, D)))


def test_two_equal_keys_split_weight(oracle_mod):
    # Keys 0 and 1 identical (index and attention), k = 2 -> O = (V0 + V1) / 2.
    L, d, H, D = 2, 32, 1, 64
    inp, _, _ = small_prefill(L, d, H, D)
    inp["K"][1] = inp["K"][0]
    _, O = oracle_mod.prefill_rows(inp, "fp8", 2, rows=[1])
    v = bf16_bits_to_f64(inp["V"])
    expect = np.array([oracle_mod.bf16_round(x) for x in (v[0] + v[1]) / 2], dtype=np.uint16)
    assert np.array_equal(O[0, 0], expect)


# ---------------------------------------------------------------- brute force

def brute_force_prefill(qi, ki, Qf, Kf, Vf, k, idx_scale, attn_scale):
    """Pure-Python restatement on tiny inputs: explicit mask matrix, lists, math."""
    L, d = qi.shape
    H, D = Qf.shape[1], Qf.shape[2]
    mask = [[s <= t for s in range(L)] for t in range(L)]
    out_idx, out_o = [], []
    for t in range(L):
        row = []
        for s in range(L):
            if not mask[t][s]:
                continue
            dot = sum(int(qi[t, j]) * int(ki[s, j]) for j in range(d))
            sc = float(f32(f32(dot) * f32(idx_scale)))
            row.append((sc if sc > 0 else 0.0, s))
        row.sort(key=lambda p: (-p[0], p[1]))
        keep = [s for _, s in row[:k]]
        out_idx.append(keep + [-1] * (k - len(keep)))
        o = []
        for h in range(H):
            lg = [sum(Qf[t, h, j] * Kf[s, j] for j in range(D)) * attn_scale for s in keep]
            m = max(lg)
            w = [math.exp(x - m) for x in lg]
            z = sum(w)
            o.append([sum(w[i] * Vf[s, j] for i, s in enumerate(keep)) / z for j in range(D)])
        out_o.append(o)
    return np.array(out_idx, dtype=np.int32), np.array(out_o)


@pytest.mark.parametrize("L,k", [(24, 5), (40, 16), (64, 64)])
def test_brute_force_tiny(oracle_mod, L, k):
    d, H, D = 32, 2, 64
    inp, qi, ki = small_prefill(L, d, H, D, lo=-3, hi=3, seed=L)
    idx_scale = oracle_mod.default_index_scale(d)
    bi, bo = brute_force_prefill(qi, ki, bf16_bits_to_f64(inp["Q"]), bf16_bits_to_f64(inp["K"]),
                                 bf16_bits_to_f64(inp["V"]), k, idx_scale, 1.0 / math.sqrt(D))
    idx, O = oracle_mod.prefill_rows(inp, "fp8", k)
    assert np.array_equal(idx, bi)
    got = bf16_bits_to_f64(O)
    assert within_half_bf16_ulp(got, bo)


# ---------------------------------------------------------------- decode

def test_decode_is_last_row_of_each_sequence(oracle_mod):
    w = synth.WORKLOADS["decode_64x128k"]
    lengths = np.array([1, 5, 300, 129, 2048 + 3], dtype=np.int64)
    inp = synth.decode_inputs(w, lengths=lengths)
    k = 256
    idx, O = oracle_mod.decode(inp, "fp8", k)
    st = inp["seq_start"]
    for b, n in enumerate(lengths):
        qi = np.zeros((n, w.d_idx), dtype=np.uint8)
        qi[n - 1] = inp["q_idx"][b]
        Qb = np.zeros((n, w.H, w.D), dtype=np.uint16)
        Qb[n - 1] = inp["Q"][b]
        sub = {"q_idx": qi, "k_idx": inp["k_idx"][st[b]:st[b + 1]], "Q": Qb,
               "K": inp["K"][st[b]:st[b + 1]], "V": inp["V"][st[b]:st[b + 1]]}
        pi, po = oracle_mod.prefill_rows(sub, "fp8", k, rows=[n - 1])
        assert np.array_equal(idx[b], pi[0])
        assert np.array_equal(O[b], po[0])
        dec = torch.from_numpy(np.arange(256, dtype=np.uint8)).view(torch.float8_e4m3fn).double().numpy()
        sc = (dec[sub["k_idx"]] @ dec[inp["q_idx"][b]]).astype(np.float32) * np.float32(
            oracle_mod.default_index_scale(w.d_idx))
        sc = np.where(sc > 0, sc, np.float32(0))
        assert idx[b].tolist() == stable_topk(sc, k).tolist()


# ---------------------------------------------------------------- paged decode

def test_paged_decode_literal_layout(oracle_mod):
    """A block-paged cache written out by hand (block size 2): the paged step equals
    the step over the same rows stored back to back."""
    w = synth.WORKLOADS["decode_64x128k"]
    flat = synth.decode_inputs(w, lengths=np.array([3, 5], dtype=np.int64))
    # sequence 0 (rows 0..2 of the flat cache) in blocks 4, 1;
    # sequence 1 (rows 3..7) in blocks 0, 5, 2; block 3 is unused
    table = np.array([[4, 1, -1], [0, 5, 2]], dtype=np.int32)
    holds = [3, 4, 2, None, 7, None, None, None, 0, 1, 5, 6]   # pool row -> flat row
    rng = np.random.default_rng(5)

    def pool(x):
        out = rng.integers(0, 1 << (8 * x.itemsize), size=(12,) + x.shape[1:]).astype(x.dtype)
        for r, f in enumerate(holds):
            if f is not None:
                out[r] = x[f]
        return out.reshape((6, 2) + x.shape[1:])

    paged = {"k_idx_blocks": pool(flat["k_idx"]), "K_blocks": pool(flat["K"]),
             "V_blocks": pool(flat["V"]), "block_table": table,
             "seq_lens": np.array([3, 5], dtype=np.int32), "q_idx": flat["q_idx"], "Q": flat["Q"]}
    for k in (1, 4, 16):
        pi, po = oracle_mod.decode_paged(paged, "fp8", k)
        ri, ro = oracle_mod.decode(flat, "fp8", k)
        assert np.array_equal(pi, ri) and np.array_equal(po, ro)
    # a wrong block (sequence 1's middle block pointed at the unused one) changes the result
    bad = dict(paged, block_table=np.array([[4, 1, -1], [0, 3, 2]], dtype=np.int32))
    bi, bo = oracle_mod.decode_paged(bad, "fp8", 4)
    ri, ro = oracle_mod.decode(flat, "fp8", 4)
    assert not (np.array_equal(bi, ri) and np.array_equal(bo, ro))


@pytest.mark.parametrize("block_size", [1, 4, 64])
def test_paged_layout_places_every_row_once(block_size):
    lengths = np.array([1, 63, 64, 65, 200], dtype=np.int64)
    table, src = synth.paged_layout(lengths, block_size, spare_blocks=2)
    starts = np.concatenate([[0], np.cumsum(lengths)])
    placed = src[src >= 0]
    assert np.array_equal(np.sort(placed), np.arange(int(lengths.sum())))
    for b, n in enumerate(lengths):
        s = np.arange(int(n))
        assert np.array_equal(src[table[b, s // block_size].astype(np.int64) * block_size + s % block_size],
                              starts[b] + s)
        used = -(-int(n) // block_size)
        assert (table[b, used:] == -1).all()
    nb = src.shape[0] // block_size
    assert nb == int((-(-lengths // block_size)).sum()) + 2
    assert sorted(table[table >= 0].tolist()) == sorted(set(table[table >= 0].tolist()))


def test_paged_decode_inputs_match_contiguous(oracle_mod):
    w = synth.WORKLOADS["decode_64x128k"]
    lengths = np.array([1, 2, 100, 2049, 300], dtype=np.int64)
    for bs in (1, 16, 4096):
        xp = synth.paged_decode_inputs(w, lengths, bs)
        pi, po = oracle_mod.decode_paged(xp, "fp8", 256)
        ri, ro = oracle_mod.decode(xp["contiguous"], "fp8", 256)
        assert np.array_equal(pi, ri) and np.array_equal(po, ro)


# ---------------------------------------------------------------- scale overrides

def _fp8_of_ints(v):
    return torch.from_numpy(np.asarray(v, dtype=np.float32)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def _bf16_times2(bits):
    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16) * 2
    return t.view(torch.int16).numpy().view(np.uint16)


def test_scale_overrides_are_applied(oracle_mod):
    """Doubling an operand (exact in FP8 and BF16) and halving its scale leaves every
    result unchanged bit for bit, while the default scale on the doubled operand does not:
    so a supplied idx_scale / attn_scale is used, not replaced by the default."""
    L, d, H, D, k = 48, 64, 2, 32, 8
    key = synth.stream_key(11, 48, 64)
    qi = synth.uniform_ints(key, L * d).reshape(L, d)
    ki = synth.uniform_ints(key, L * d, start=L * d).reshape(L, d)
    x = {"q_idx": _fp8_of_ints(qi), "k_idx": _fp8_of_ints(ki),
         "Q": synth.normal_bf16(synth.stream_key(11, 1), L * H * D).reshape(L, H, D),
         "K": synth.normal_bf16(synth.stream_key(11, 2), L * D).reshape(L, D),
         "V": synth.normal_bf16(synth.stream_key(11, 3), L * D).reshape(L, D)}
    s_idx, s_att = oracle_mod.default_index_scale(d), 1.0 / np.sqrt(D)
    q2 = _fp8_of_ints(2 * qi)
    a = oracle_mod.indexer_scores(x["q_idx"], x["k_idx"], "fp8")
    assert np.array_equal(oracle_mod.indexer_scores(q2, x["k_idx"], "fp8", scale=s_idx / 2), a)
    assert np.array_equal(oracle_mod.indexer_scores(q2, x["k_idx"], "fp8"), 2 * a) and a.max() > 0

    x2 = dict(x, Q=_bf16_times2(x["Q"]))
    ri, ro = oracle_mod.prefill_rows(x, "fp8", k)
    si, so = oracle_mod.prefill_rows(x2, "fp8", k, attn_scale=s_att / 2)
    assert np.array_equal(si, ri) and np.array_equal(so, ro)
    _, to = oracle_mod.prefill_rows(x2, "fp8", k)
    assert not np.array_equal(to, ro)

    lens = np.array([1, 7, 40], dtype=np.int64)
    xd = synth.decode_inputs(synth.WORKLOADS["decode_64x128k"], lengths=lens)
    xd2 = dict(xd, Q=_bf16_times2(xd["Q"]))
    di, do = oracle_mod.decode(xd, "fp8", k)
    ei, eo = oracle_mod.decode(xd2, "fp8", k, attn_scale=1.0 / np.sqrt(xd["Q"].shape[2]) / 2)
    assert np.array_equal(ei, di) and np.array_equal(eo, do)


# ---------------------------------------------------------------- several new tokens per sequence

def test_decode_multi_token_equals_prefill_rows_at_its_position():
    """Token j of sequence b (T new tokens, the last T rows of the sequence) is the
    prefill query at position len_b - T + j of that sequence: checked against the
    prefill oracle on the sequence's own rows, and T = 1 is the single-token decode."""
    import numpy as np
    import oracle
    import synth
    w = synth.WORKLOADS["decode_64x128k"]
    lens = np.array([4, 40, 300, 1000], dtype=np.int64)
    T = 3
    xd = synth.decode_inputs(w, lengths=lens)
    mq = synth.multi_queries(w, len(lens), T)
    x = dict(xd, q_idx=mq["q_idx"], Q=mq["Q"])
    idx, O = oracle.decode_multi(x, w.idx_dtype, 128)
    ss = xd["seq_start"]
    for b, n in enumerate(lens):
        rows = slice(ss[b], ss[b + 1])
        for j in range(T):
            pos = int(n) - T + j
            qf = np.zeros((int(n), w.d_idx), dtype=xd["k_idx"].dtype)
            qf[pos] = mq["q_idx"][b, j]
            Qf = np.zeros((int(n), w.H, w.D), dtype=np.uint16)
            Qf[pos] = mq["Q"][b, j]
            p = {"q_idx": qf, "k_idx": xd["k_idx"][rows], "Q": Qf, "K": xd["K"][rows], "V": xd["V"][rows]}
            ri, ro = oracle.prefill_rows(p, w.idx_dtype, 128, rows=np.array([pos], dtype=np.int64))
            assert np.array_equal(idx[b, j], ri[0]), (b, j)
            assert np.array_equal(O[b, j], ro[0]), (b, j)
    x1 = dict(xd, q_idx=xd["q_idx"][:, None, :], Q=xd["Q"][:, None])
    i1, o1 = oracle.decode_multi(x1, w.idx_dtype, 128)
    i0, o0 = oracle.decode(xd, w.idx_dtype, 128)
    assert np.array_equal(i1[:, 0], i0) and np.array_equal(o1[:, 0], o0)
