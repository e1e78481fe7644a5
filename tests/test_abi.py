"""The C ABI without a GPU: the library loads, exports every entry point the
header declares, and rejects bad arguments on the host before enqueuing work."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def header_functions():
    txt = open(os.path.join(ROOT, "include", "qsa.h")).read()
    return re.findall(r"QSA_API\s+[\w\s\*]+?\b(qsa_\w+)\s*\(", txt)


def test_header_declares_the_five_calls():
    names = set(header_functions())
    for n in ("qsa_append_kv", "qsa_index_scores", "qsa_topk_blocks", "qsa_sparse_decode", "qsa_combine"):
        assert n in names


def test_library_exports_every_declared_symbol():
    import sparse_attention_decode_03_b200 as qsa
    lib = ctypes.CDLL(qsa.LIB_PATH)
    for n in header_functions():
        assert hasattr(lib, n), n
    assert qsa.ABI_VERSION == 7
    assert qsa.status_string(0) == "QSA_OK" and qsa.status_string(-3) == "QSA_ERR_CUDA"


def test_decode_plan():
    import sparse_attention_decode_03_b200 as qsa
    c, s = qsa.qsa_decode_plan(32, 2, 512, 148)
    assert c == -(-32 * 2 * 513 // 148) and s == qsa.splits_bound(512, c)
    c, s = qsa.qsa_decode_plan(1, 2, 512, 148)
    assert c == 16 and s == (513 + 14) // 16 + 1
    with pytest.raises(qsa.QSAError):
        qsa.qsa_decode_plan(1, 0, 512, 148)
    with pytest.raises(qsa.QSAError):
        qsa.qsa_decode_plan(1, 1, 4096, 148)


def test_host_validation_returns_before_any_cuda_call():
    import sparse_attention_decode_03_b200 as qsa
    L = qsa.qsa.LIB
    fake = ctypes.c_void_p(0x1000)
    cache = qsa.qsa.qsa_cache_t(0x1000, 0x1000, 0x1000, 0x1000, 10, 2, 4, 2)
    cp = ctypes.byref(cache)
    # sparse decode: Hq not a multiple of Hkv; group too large; K too large; too few split slots
    args = lambda hq, k, chunk, ms: (cp, fake, 1, hq, fake, fake, fake, fake, k, 0.0625, chunk, ms, fake, fake, None, None)
    assert L.qsa_sparse_decode(*args(3, 16, 16, 4)) == -1
    assert L.qsa_sparse_decode(*args(64, 16, 16, 4)) == -2
    assert L.qsa_sparse_decode(*args(16, 4096, 16, 400)) == -1
    assert L.qsa_sparse_decode(*args(16, 512, 16, 2)) == -1
    assert L.qsa_sparse_decode(None, fake, 1, 16, fake, fake, fake, fake, 16, 0.0625, 16, 4, fake, fake, None, None) == -1
    assert L.qsa_sparse_decode(cp, fake, 1, 16, fake, fake, fake, fake, 16, 0.0, 16, 4, fake, fake, None, None) == -1
    # zero queries is a no-op
    assert L.qsa_sparse_decode(cp, fake, 0, 16, fake, fake, fake, fake, 16, 0.0625, 16, 4, fake, fake, None, None) == 0
    assert L.qsa_topk_blocks(fake, 100, fake, 1, 4096, fake, fake, None, None) == -1
    assert L.qsa_topk_blocks(fake, 0, fake, 1, 16, fake, fake, None, None) == -1
    assert L.qsa_append_kv(cp, fake, fake, fake, fake, fake, -1, None, None) == -1
    assert L.qsa_append_kv(cp, fake, fake, fake, fake, fake, 0, None, None) == 0
    assert L.qsa_append_kv(None, fake, fake, fake, fake, fake, 5, None, None) == -1
    assert L.qsa_index_scores(cp, None, fake, fake, fake, 1, fake, 16, None, None) == -1
    assert L.qsa_combine(ctypes.c_void_p(0x1004), fake, 1, 4, 16, fake, fake, None) == -1  # misaligned
    assert L.qsa_combine(fake, fake, 1, 0, 16, fake, fake, None) == -1
    # strided merge: output type, 16-byte strides of part_o, fp32 output alignment
    assert L.qsa_combine_strided(fake, fake, 1, 2, 4, 2048, 1024, 8, 4, fake, 2, fake, None) == -1
    assert L.qsa_combine_strided(fake, fake, 1, 2, 4, 2046, 1024, 8, 4, fake, 0, fake, None) == -1
    assert L.qsa_combine_strided(fake, fake, 1, 2, 4, 2048, 1024, 8, 4, ctypes.c_void_p(0x1008), 1, fake, None) == -1
    assert L.qsa_combine_strided(fake, fake, 0, 2, 4, 2048, 1024, 8, 4, fake, 1, fake, None) == 0
    # DCP localisation: the shard must be well formed
    assert L.qsa_dcp_localize_tokens(fake, fake, 4, 2, 2, 1, fake, fake, None) == -1
    assert L.qsa_dcp_localize_tokens(fake, fake, 4, 0, 0, 1, fake, fake, None) == -1
    assert L.qsa_dcp_localize_tokens(fake, fake, 4, 2, 1, 0, fake, fake, None) == -1
    assert L.qsa_dcp_localize_tokens(fake, fake, 0, 2, 1, 1, fake, fake, None) == 0
    assert L.qsa_dcp_localize_selection(fake, fake, fake, 1, 16, 2, -1, 1, fake, fake, fake, None, None) == -1
    assert L.qsa_dcp_localize_selection(fake, fake, fake, 1, 4096, 2, 0, 1, fake, fake, fake, None, None) == -1
    # a cache group needs at least one of main K/V and side cache
    empty = qsa.qsa.qsa_cache_t(None, None, 0x1000, 0x1000, 10, 2, 4, 2)
    assert L.qsa_append_kv(ctypes.byref(empty), fake, fake, fake, fake, fake, 5, None, None) == -1
    kv_only = qsa.qsa.qsa_cache_t(0x1000, None, None, 0x1000, 10, 2, 4, 2)
    assert L.qsa_index_scores(ctypes.byref(kv_only), fake, fake, fake, fake, 1, fake, 16, None, None) == -1
    kc_only = qsa.qsa.qsa_cache_t(None, 0x1000, 0x1000, 0x1000, 10, 2, 4, 2)
    assert L.qsa_sparse_decode(ctypes.byref(kc_only), fake, 1, 16, fake, fake, fake, fake, 16, 0.0625, 16, 4, fake,
                               fake, None, None) == -1
    # attention with the in-kernel merge: the decode checks plus its own buffers
    m_args = lambda nq, pd, out: (cp, fake, nq, 16, fake, fake, fake, fake, 16, 0.0625, 16, 4, fake, fake, pd, out, fake,
                                  None, None)
    assert L.qsa_sparse_attention(*m_args(1, None, fake)) == -1
    assert L.qsa_sparse_attention(*m_args(1, fake, None)) == -1
    assert L.qsa_sparse_attention(*m_args(1, fake, ctypes.c_void_p(0x1004))) == -1   # out not 8-byte aligned
    assert L.qsa_sparse_attention(*m_args(0, None, None)) == 0
    assert L.qsa_sparse_attention(cp, fake, 1, 3, fake, fake, fake, fake, 16, 0.0625, 16, 4, fake, fake, fake, fake,
                                  fake, None, None) == -1                            # Hq not a multiple of Hkv
    # fused indexer + selection: the checks of both separate calls
    assert L.qsa_index_topk(cp, fake, fake, fake, fake, 1, 4096, fake, 16, fake, fake, None, None) == -1
    assert L.qsa_index_topk(cp, fake, fake, fake, fake, 1, 16, fake, 0, fake, fake, None, None) == -1
    assert L.qsa_index_topk(cp, fake, fake, fake, fake, 1, 16, fake, 16, None, fake, None, None) == -1
    assert L.qsa_index_topk(cp, ctypes.c_void_p(0x1008), fake, fake, fake, 1, 16, fake, 16, fake, fake, None,
                            None) == -1
    assert L.qsa_index_topk(ctypes.byref(kv_only), fake, fake, fake, fake, 1, 16, fake, 16, fake, fake, None,
                            None) == -1
    assert L.qsa_index_topk(cp, fake, fake, fake, fake, 0, 16, fake, 16, fake, fake, None, None) == 0
    # its shared memory: a fixed part plus 68 B (page id + 16 score keys) per page of a CTA's eighth of the row
    wide = qsa.qsa.qsa_cache_t(0x1000, 0x1000, 0x1000, 0x1000, 10, 2, 4096, 2)
    wp = ctypes.byref(wide)
    b_long, b_short = L.qsa_index_topk_smem_bytes(wp, 65536), L.qsa_index_topk_smem_bytes(wp, 1024)
    assert b_long - b_short == (512 - 8) * 68 and 64 << 10 < b_short < 72 << 10
    assert L.qsa_index_topk_smem_bytes(wp, 1 << 30) == L.qsa_index_topk_smem_bytes(wp, 65536)  # capped by the table
    assert L.qsa_index_topk_smem_bytes(wp, 0) == -1
    # K/V storage types: BF16 and FP8 e4m3 only
    bad = qsa.qsa.qsa_cache_t(0x1000, 0x1000, 0x1000, 0x1000, 10, 2, 4, 2, 7)
    bp = ctypes.byref(bad)
    assert L.qsa_append_kv(bp, fake, fake, fake, fake, fake, 5, None, None) == -2
    assert L.qsa_sparse_decode(bp, fake, 1, 16, fake, fake, fake, fake, 16, 0.0625, 16, 4, fake, fake, None, None) == -2


def test_binding_rejects_host_tensors():
    import torch

    import sparse_attention_decode_03_b200 as qsa
    with pytest.raises(ValueError):
        qsa.qsa_combine(torch.zeros(1, 2, 4, 256), torch.zeros(1, 2, 4), torch.zeros(1, 4, 256, dtype=torch.bfloat16),
                        torch.zeros(1, 4))
    i32 = dict(dtype=torch.int32)
    with pytest.raises(ValueError):  # checked before the cache is touched
        qsa.qsa_index_topk(None, torch.zeros(2, 8, 128, dtype=torch.bfloat16), torch.zeros(2, 8),
                           torch.zeros(2, **i32), torch.zeros(2, **i32), 16, torch.zeros(2, 64),
                           torch.zeros(2, 16, **i32), torch.zeros(2, **i32))
    with pytest.raises(ValueError):
        qsa.qsa_sparse_attention(None, torch.zeros(2, 4, 256, dtype=torch.bfloat16), torch.zeros(2, **i32),
                                 torch.zeros(2, **i32), torch.zeros(2, 16, **i32), torch.zeros(2, **i32), 16, 0.0625,
                                 16, 4, torch.zeros(2, 4, 4, 256), torch.zeros(2, 4, 4), torch.zeros(2, **i32),
                                 torch.zeros(2, 4, 256, dtype=torch.bfloat16), torch.zeros(2, 4))


def test_fused_selection_rule():
    """The Decoder's choice of the fused indexer + selection: enough clusters
    to fill the SMs, all resident at once, and a decode-shaped call."""
    import sparse_attention_decode_03_b200 as qsa
    pays = qsa.fused_selection_pays
    assert pays(32, 32, 148, 33)          # batch-32 decode: 256 CTAs, one wave
    assert not pays(64, 64, 148, 33)      # two waves of clusters
    assert not pays(8, 8, 148, 33)        # 64 CTAs leave most SMs idle
    assert not pays(24, 2, 148, 33)       # 12 queries per sequence: prefill-shaped, the tensor-core indexer
    assert not pays(32, 32, 148, 0)       # shared memory does not fit


def test_fused_default_falls_back_only_when_clusters_cannot_be_placed(monkeypatch):
    """The Decoder's default keeps the two-call selection when the occupancy
    query fails (QSA_ERR_CUDA) or is unsupported, and raises a caller error
    (QSA_ERR_INVALID_ARG) instead of hiding it."""
    import sparse_attention_decode_03_b200 as qsa
    from sparse_attention_decode_03_b200 import qsa as Q

    class FakeCache:
        kc_pages = object()
        max_seqs = 32

    def failing(code):
        def f(cache, scores_ld):
            raise qsa.QSAError("qsa_index_topk_resident_queries", code)
        return f

    monkeypatch.setattr(Q, "index_topk_resident_queries", failing(Q.QSA_ERR_CUDA))
    assert Q.fused_default(FakeCache(), 8192, 32, 148) is False
    monkeypatch.setattr(Q, "index_topk_resident_queries", failing(Q.QSA_ERR_UNSUPPORTED))
    assert Q.fused_default(FakeCache(), 8192, 32, 148) is False
    monkeypatch.setattr(Q, "index_topk_resident_queries", failing(Q.QSA_ERR_INVALID_ARG))
    with pytest.raises(qsa.QSAError):
        Q.fused_default(FakeCache(), 8192, 32, 148)
    monkeypatch.setattr(Q, "index_topk_resident_queries", lambda cache, ld: 33)
    assert Q.fused_default(FakeCache(), 8192, 32, 148) is True


def test_bf16_cache_views_follow_the_header_layout():
    """PagedCache.k_view / v_view undo the BF16 cache's operand layout stated in
    include/qsa.h: per micro-block [4 dim atoms][8 rows: K 0-3, V 0-3][64], the
    16-byte chunk c of row r stored at chunk position c ^ r."""
    import torch
    from sparse_attention_decode_03_b200 import qsa as Q

    class Cache(Q.PagedCache):
        def __init__(self):  # host buffers only: no device needed
            self.num_pages, self.num_kv_heads, self.kv_dtype = 2, 2, Q.KV_BF16
            self.kv_pages = torch.zeros((2, 2, 16, 4, 8, 64), dtype=torch.int32)

    c = Cache()
    g = torch.Generator().manual_seed(3)
    K = torch.randint(0, 1 << 30, (2, 2, 64, 256), dtype=torch.int32, generator=g)
    V = torch.randint(0, 1 << 30, (2, 2, 64, 256), dtype=torch.int32, generator=g)
    raw = c.kv_pages.view(2, 2, 16, 4, 8, 8, 8)
    for t in range(64):
        blk, i = t // 4, t % 4
        for d in range(256):
            atom, ch, e = d // 64, (d % 64) // 8, d % 8
            raw[:, :, blk, atom, i, ch ^ i, e] = K[:, :, t, d]
            raw[:, :, blk, atom, 4 + i, ch ^ (4 + i), e] = V[:, :, t, d]
    assert torch.equal(c.k_view(), K) and torch.equal(c.v_view(), V)
