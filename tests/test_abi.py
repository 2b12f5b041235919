"""Host-side checks of the C ABI: the library loads, exports what the header
declares, and rejects bad arguments synchronously (no GPU work is enqueued)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    from sparse_attention_10_b200 import build
    build.build()
    import sparse_attention_10_b200 as dsa
    return dsa.load()


def declared_functions():
    text = open(os.path.join(ROOT, "include", "dsa.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(dsa_[a-z_0-9]+)\s*\(", text)))


def test_header_declares_the_two_calls():
    names = declared_functions()
    assert "dsa_prefill" in names and "dsa_decode" in names


def test_library_exports_every_declared_symbol(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name


def test_status_strings_and_version(lib):
    import sparse_attention_10_b200 as dsa
    assert dsa.dsa_status_string(0) == "ok"
    assert dsa.dsa_status_string(5) == "device-side wait timed out"
    assert re.match(r"\d+\.\d+\.\d+", dsa.dsa_version())


P = ctypes.c_void_p


def prefill(lib, q=16, k=16, Qp=16, Kp=16, Vp=16, idx=16, O=16, ws=256, L=128, H=4, D=64, top_k=16,
            d=128, dtype=0, ws_bytes=1 << 40):
    return lib.dsa_prefill(P(q), P(k), dtype, d, float("nan"), P(Qp), P(Kp), P(Vp), L, H, D,
                           float("nan"), top_k, P(idx), P(O), P(ws), ws_bytes, None)


def test_prefill_rejects_bad_arguments(lib):
    assert prefill(lib, q=0) == 1                    # null
    assert prefill(lib, k=8) == 1                    # misaligned
    assert prefill(lib, ws=16 + 256) == 1            # workspace not 256-aligned
    assert prefill(lib, L=0) == 1
    assert prefill(lib, top_k=0) == 1
    assert prefill(lib, top_k=2049) == 1
    assert prefill(lib, H=17) == 1
    assert prefill(lib, D=96) == 2                   # unsupported head dim
    assert prefill(lib, d=100) == 2                  # fp8 rows not a multiple of 32 bytes
    assert prefill(lib, d=257) == 1
    assert prefill(lib, dtype=7) == 1
    assert prefill(lib, ws_bytes=1) == 3             # workspace too small


def test_workspace_sizes_grow_with_length(lib):
    a = lib.dsa_prefill_workspace_size(4096, 128, 0, 4, 64, 256)
    b = lib.dsa_prefill_workspace_size(8192, 128, 0, 4, 64, 256)
    assert 0 < a < b
    assert lib.dsa_prefill_workspace_size(0, 128, 0, 4, 64, 256) == 0
    assert lib.dsa_decode_workspace_size(64, 1 << 20, 128, 0, 16, 128, 2048) > 8 << 20


def test_decode_rejects_bad_arguments(lib):
    def dec(seq=16, B=2, total=100, max_len=50, top_k=64, H=16, D=128, d=128, ws_bytes=1 << 40):
        return lib.dsa_decode(P(16), P(16), P(16), P(seq), B, total, max_len, 0, d, D, P(16), P(16),
                              H, top_k, float("nan"), float("nan"), P(16), None, P(256), ws_bytes,
                              None)
    assert dec(seq=0) == 1
    assert dec(seq=20) == 1        # int64 array must be 8-byte aligned
    assert dec(B=0) == 1
    assert dec(B=65536, total=1 << 20) == 1   # sequences are a grid dimension
    assert dec(max_len=0) == 1
    assert dec(top_k=4096) == 1
    assert dec(D=80) == 2
    assert dec(ws_bytes=10) == 3


def test_decode_paged_rejects_bad_arguments(lib):
    def dec(bt=16, lens=16, nb=100, bs=64, mb=8, B=2, max_len=500, top_k=64, H=16, D=128, d=128,
            kidx=16, ws_bytes=1 << 40):
        return lib.dsa_decode_paged(P(kidx), P(16), P(16), nb, bs, P(bt), mb, P(lens), B, max_len, 0, d,
                                    D, P(16), P(16), H, top_k, float("nan"), float("nan"), P(16), None,
                                    P(256), ws_bytes, None)
    assert dec(bt=0) == 1 and dec(lens=0) == 1        # null
    assert dec(bt=18) == 1 and dec(lens=6) == 1       # int32 arrays must be 4-byte aligned
    assert dec(kidx=8) == 1                           # pools 16-byte aligned
    assert dec(bs=0) == 1 and dec(bs=48) == 1 and dec(bs=1 << 17) == 1   # power of two <= 65536
    assert dec(nb=0) == 1
    assert dec(nb=1 << 26, bs=64) == 1                # pool rows beyond 2^31 - 1
    assert dec(mb=0) == 1
    assert dec(B=0) == 1 and dec(B=65536) == 1
    assert dec(max_len=0) == 1 and dec(max_len=1 << 31) == 1
    assert dec(top_k=4096) == 1 and dec(H=0) == 1
    assert dec(D=80) == 2
    assert dec(ws_bytes=10) == 3
    need = lib.dsa_decode_paged_workspace_size(2, 500, 128, 0, 16, 128, 64)
    assert need > lib.dsa_decode_workspace_size(2, 1000, 128, 0, 16, 128, 64)   # + the length sums
    assert dec(ws_bytes=need - 1) == 3
    assert lib.dsa_decode_paged_workspace_size(0, 500, 128, 0, 16, 128, 64) == 0
    assert lib.dsa_decode_paged_workspace_size(2, 0, 128, 0, 16, 128, 64) == 0


def test_indexer_scores_rejects_bad_arguments(lib):
    f = lib.dsa_indexer_scores
    assert f(None, P(16), 0, 128, float("nan"), 4, 4, P(16), None) == 1
    assert f(P(16), P(16), 0, 128, float("nan"), 0, 4, P(16), None) == 1
    assert f(P(16), P(16), 1, 8, float("nan"), 4, 4, P(16), None) == 2   # 16 bytes per row


def test_python_binding_refuses_cpu_tensors(lib):
    import torch
    import sparse_attention_10_b200 as dsa
    q = torch.zeros((4, 128), dtype=torch.uint8)
    with pytest.raises(ValueError):
        dsa.dsa_indexer_scores(q, q)


def test_force_fallback_hook_validates_and_resets(lib):
    import sparse_attention_10_b200 as dsa
    assert lib.dsa_debug_force_fallback(-1) == 1     # negative period rejected
    dsa.dsa_debug_force_fallback(7)
    dsa.dsa_debug_force_fallback(0)                  # back to normal


def test_binding_exports_what_it_lists():
    import sparse_attention_10_b200 as m
    assert [n for n in m.__all__ if not hasattr(m, n)] == []
