"""The fused indexer + selection (qsa_index_topk) through the C ABI against the
oracle: bit-exact scores and selections across the cluster's slice
boundaries, ragged last pages, rows at or under K, K = 0 and the largest K,
the general path the selection falls back to when its sample misleads, an
out-of-range query, and whole decode steps (full size included) that must
equal the two-call pipeline bit for bit."""
import numpy as np
import pytest
import torch

from oracle import qsa_oracle as O
from tests import oracle_ref as R
from workloads import configs as C

pytestmark = pytest.mark.gpu

qsa = pytest.importorskip("sparse_attention_decode_03_b200")
H = pytest.importorskip("workloads.harness")


@pytest.fixture(autouse=True, scope="module")
def _need_cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")


def _step(wl, k, fused, cache=None, chunk=None):
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    if cache is None:
        cache = H.build_cache(wl, dev_status=st)
    inp = H.step_inputs(wl)
    qsa.qsa_append_kv(cache, inp["k_new"], inp["v_new"], inp["kidx_new"], inp["seq_id"], inp["pos"], st)
    dec = qsa.Decoder(cache, wl.hq, wl.nq, k=k, scale=wl.scale, chunk_units=chunk, fused=fused)
    dec.dev_status = st
    dec.run(inp["q"], inp["q_idx"], inp["w"], inp["q_seq"], inp["q_pos"])
    torch.cuda.synchronize()
    return cache, dec, int(st.item())


def _check_rows(wl, dec, k, rows=None):
    sc = dec.scores.cpu().numpy()
    sel = dec.sel.cpu().numpy()
    cnt = dec.count.cpu().numpy()
    for row in (range(wl.nq) if rows is None else rows):
        d = R.query_inputs(wl, row)
        nb, _ = O.visible(d["p"])
        kc = O.compress_keys(R.kidx_seq(wl, d["seq"], d["p"] + 1))
        s_ref = O.block_scores(d["q_idx"], d["w"], kc)
        assert np.array_equal(sc[row, :nb], s_ref.astype(np.float32)), f"scores row {row}"
        sel_ref = O.select_blocks(s_ref, k)
        assert cnt[row] == len(sel_ref), f"count row {row}"
        assert np.array_equal(sel[row, :cnt[row]], sel_ref), f"selection row {row}"
        assert np.all(sel[row, cnt[row]:] == -1)


@pytest.mark.parametrize("name,lengths,k", [
    ("quarter", [4000, 999, 66, 5], 64),   # one-page slices, idle CTAs, a row under K
    ("long", [3000, 2050], 512),           # a row of exactly K blocks
    ("long", [20001, 9003], 512),          # several pages per CTA, ragged last page
    ("batched", [1500], 16),
    ("quarter", [700, 3], 0),              # K = 0
    ("long", [36000], 2048),               # the largest K
])
def test_fused_index_topk_bit_exact(name, lengths, k):
    wl = C.shrink(C.get(name), lengths, page_perm=True, k_top=k)
    _, dec, st = _step(wl, k, fused=True)
    assert dec.fused and st == 0
    _check_rows(wl, dec, k)


def test_fused_all_ties_take_the_general_path():
    """Every score equal: the sampled threshold admits all 5,000 blocks, more
    than the gathered lists hold, so the leader CTA runs the general exact
    path over the scores row; ties go to the lowest indices."""
    wl = C.shrink(C.get("quarter"), [20000], k_top=700)
    cache = H.new_cache(wl)
    pos = torch.arange(0, 20000, device="cuda")
    k = C.k_rows(wl, 0, pos, "cuda")
    ki = torch.ones((20000, 128), dtype=torch.bfloat16, device="cuda")
    qsa.qsa_append_kv(cache, k, k, ki, torch.zeros(20000, dtype=torch.int32, device="cuda"), pos.to(torch.int32))
    qs = C.queries(wl, device="cuda")
    qs["q_pos"].fill_(19999)
    dec = qsa.Decoder(cache, wl.hq, 1, k=700, fused=True)
    dec.run(qs["q"], qs["q_idx"], qs["w"], qs["q_seq"], qs["q_pos"])
    torch.cuda.synchronize()
    assert int(dec.dev_status.item()) == 0
    assert dec.count.item() == 700
    assert dec.sel[0].tolist() == list(range(700))
    s = dec.scores[0, :5000]
    assert torch.all(s == s[0])


def test_fused_out_of_range_query_is_flagged_and_empty():
    wl = C.shrink(C.get("long"), [3000, 2500], page_perm=True, k_top=64)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    cache = H.build_cache(wl, dev_status=st)
    qs = C.queries(wl, device="cuda")
    qs["q_seq"][1] = wl.batch + 5
    scores = torch.zeros((wl.nq, cache.max_pages_per_seq * 16), dtype=torch.float32, device="cuda")
    sel = torch.zeros((wl.nq, 64), dtype=torch.int32, device="cuda")
    count = torch.full((wl.nq,), 7, dtype=torch.int32, device="cuda")
    qsa.qsa_index_topk(cache, qs["q_idx"], qs["w"], qs["q_seq"], qs["q_pos"], 64, scores, sel, count, st)
    torch.cuda.synchronize()
    assert "BAD_SEQ" in qsa.dev_status_names(int(st.item()))
    assert count[1].item() == 0 and torch.all(sel[1] == -1)
    assert count[0].item() == 64


@pytest.mark.parametrize("name,lengths", [("long", [9000, 4100, 777]), ("quarter", [16000, 2000, 50, 6000])])
def test_fused_decode_step_equals_two_call_step(name, lengths):
    """The whole step (append, select, attend, combine) with the fused call
    gives the same selections and bit-identical outputs as with the two calls."""
    wl = C.shrink(C.get(name), lengths, page_perm=True)
    _, a, st_a = _step(wl, wl.k_top, fused=False)
    _, b, st_b = _step(wl, wl.k_top, fused=True)
    assert st_a == 0 and st_b == 0
    assert torch.equal(a.count, b.count) and torch.equal(a.sel, b.sel)
    nq = wl.nq
    assert torch.equal(a.out[:nq].view(torch.int16), b.out[:nq].view(torch.int16))
    assert torch.equal(a.lse[:nq].view(torch.int32), b.lse[:nq].view(torch.int32))


@pytest.mark.parametrize("name", ["long", "quarter", "long-fp8"])
def test_fused_full_size_matches_oracle_rows(name):
    """Full-size decode workloads in the benchmark's launch configuration:
    every row's selection equals the two-call pipeline's, sampled rows equal
    the oracle's."""
    wl = C.get(name)
    cache = None
    _, a, st_a = _step(wl, wl.k_top, fused=False, chunk=H.chunk_units_for(wl))
    sel_a, cnt_a = a.sel.clone(), a.count.clone()
    del a
    torch.cuda.empty_cache()
    _, b, st_b = _step(wl, wl.k_top, fused=True, cache=cache, chunk=H.chunk_units_for(wl))
    assert st_a == 0 and st_b == 0
    assert torch.equal(cnt_a, b.count) and torch.equal(sel_a, b.sel)
    L = np.array(wl.total_lengths)
    rows = sorted({0, int(L.argmin()), int(L.argmax()), wl.nq - 1})
    sel = b.sel.cpu().numpy()
    cnt = b.count.cpu().numpy()
    for row in rows:
        r = R.expect_query(wl, row)
        assert np.array_equal(sel[row, :cnt[row]], r["sel"]), f"{name} row {row}"


def test_fused_bad_page_flags_and_matches_two_calls():
    """A block-table entry outside the page pool: both forms set BAD_PAGE,
    score that page's 16 blocks -inf and select the same blocks."""
    wl = C.shrink(C.get("long"), [6000, 3000], page_perm=True, k_top=64)
    st0 = torch.zeros(1, dtype=torch.int32, device="cuda")
    cache = H.build_cache(wl, dev_status=st0)
    inp = H.step_inputs(wl)
    qsa.qsa_append_kv(cache, inp["k_new"], inp["v_new"], inp["kidx_new"], inp["seq_id"], inp["pos"], st0)
    torch.cuda.synchronize()
    assert int(st0.item()) == 0
    cache.block_table[0, 5] = 10 ** 7
    ld = cache.max_pages_per_seq * 16
    res = []
    for fused in (False, True):
        st = torch.zeros(1, dtype=torch.int32, device="cuda")
        sc = torch.full((wl.nq, ld), 3.0, dtype=torch.float32, device="cuda")
        sel = torch.zeros((wl.nq, 64), dtype=torch.int32, device="cuda")
        cnt = torch.zeros((wl.nq,), dtype=torch.int32, device="cuda")
        if fused:
            qsa.qsa_index_topk(cache, inp["q_idx"], inp["w"], inp["q_seq"], inp["q_pos"], 64, sc, sel, cnt, st)
        else:
            qsa.qsa_index_scores(cache, inp["q_idx"], inp["w"], inp["q_seq"], inp["q_pos"], sc, st)
            qsa.qsa_topk_blocks(sc, inp["q_pos"], 64, sel, cnt, st)
        torch.cuda.synchronize()
        res.append((int(st.item()), sc, sel, cnt))
    (s0, sc0, se0, c0), (s1, sc1, se1, c1) = res
    assert s0 & 1 and s1 & 1
    nb = ((inp["q_pos"].long() + 1) // 4).tolist()
    assert torch.all(torch.isneginf(sc1[0, 80:96]))
    for r in range(wl.nq):
        assert torch.equal(sc0[r, :nb[r]].view(torch.int32), sc1[r, :nb[r]].view(torch.int32)), f"scores row {r}"
    assert torch.equal(se0, se1) and torch.equal(c0, c1)
