"""Parity of the CUDA path (through the C ABI) with the CPU oracle on small
cases that still span several tiles, chunks and pages, plus the edge cases the
pages' operator tests list ([CANN] "Negen tests ..."): unordered physical
slots, several selection widths, default and explicit scales, fully masked
rows, selection width zero, causal tail remainders 0..3, two requests sharing
a prefix's physical pages, cache reuse, and the five local head shapes at 1 and
257 query rows."""
import dataclasses
import json
import os

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


def _status():
    return torch.zeros(1, dtype=torch.int32, device="cuda")


def run_step(wl, cache=None, k=None, chunk=None, scale=None, target_ctas=None):
    st = _status()
    if cache is None:
        cache = H.build_cache(wl, dev_status=st)
    inp = H.step_inputs(wl)
    qsa.qsa_append_kv(cache, inp["k_new"], inp["v_new"], inp["kidx_new"], inp["seq_id"], inp["pos"], st)
    dec = qsa.Decoder(cache, wl.hq, wl.nq, k=wl.k_top if k is None else k, scale=wl.scale if scale is None else scale,
                      chunk_units=chunk, target_ctas=target_ctas)
    dec.dev_status = st
    dec.run(inp["q"], inp["q_idx"], inp["w"], inp["q_seq"], inp["q_pos"])
    torch.cuda.synchronize()
    return cache, dec, int(st.item())


def bits16(t):
    return t.contiguous().view(torch.int16).cpu()


# ---------------------------------------------------------------- append


def _append_irregular(cache, wl, st):
    """Append every sequence's positions in irregular chunks, several
    sequences per call, with padding tokens (seq_id -1) between the runs."""
    sizes = [1, 3, 2, 64, 5, 100, 7, 250, 4, 1, 33]
    cursor = [0] * wl.batch
    it = 0
    while any(c < L for c, L in zip(cursor, wl.lengths)):
        parts = []
        for b, L in enumerate(wl.lengths):
            if cursor[b] >= L:
                continue
            n = min(sizes[(it + b) % len(sizes)], L - cursor[b])
            pos = torch.arange(cursor[b], cursor[b] + n, device="cuda")
            parts.append((C.k_rows(wl, b, pos, "cuda"), C.v_rows(wl, b, pos, "cuda"), C.kidx_rows(wl, b, pos, "cuda"),
                          torch.full((n,), b, dtype=torch.int32, device="cuda"), pos.to(torch.int32)))
            cursor[b] += n
            # a padding token: garbage data, must write nothing
            parts.append((torch.full((1, wl.hkv, 256), 999.0, dtype=torch.bfloat16, device="cuda"),
                          torch.full((1, wl.hkv, 256), 999.0, dtype=torch.bfloat16, device="cuda"),
                          torch.full((1, 128), 999.0, dtype=torch.bfloat16, device="cuda"),
                          torch.full((1,), -1, dtype=torch.int32, device="cuda"),
                          torch.zeros((1,), dtype=torch.int32, device="cuda")))
        cat = [torch.cat([p[i] for p in parts]) for i in range(5)]
        qsa.qsa_append_kv(cache, *cat, st)
        it += 1


@pytest.mark.parametrize("name,lengths", [("quarter", [301, 64, 130, 7]), ("long", [197, 260])])
def test_append_kv_bit_exact(name, lengths):
    wl = C.shrink(C.get(name), lengths, page_perm=True)
    cache = H.new_cache(wl)
    cache.kv_pages.fill_(1024.0)
    cache.kc_pages.fill_(512.0)
    st = _status()
    _append_irregular(cache, wl, st)
    torch.cuda.synchronize()
    assert st.item() == 0
    bt = cache.block_table.cpu()
    for b, L in enumerate(wl.lengths):
        pos = torch.arange(L)
        pg, row = bt[b, pos // 64].long(), pos % 64
        k_gpu = cache.k_view().cpu()[pg, :, row]
        v_gpu = cache.v_view().cpu()[pg, :, row]
        assert torch.equal(k_gpu.view(torch.int16), C.k_rows(wl, b, pos).view(torch.int16))
        assert torch.equal(v_gpu.view(torch.int16), C.v_rows(wl, b, pos).view(torch.int16))
        kid = C.kidx_rows(wl, b, pos).float().numpy()
        kc_ref = O.compress_keys(kid)
        nb = L // 4
        j = torch.arange(nb)
        kc_gpu = cache.kc_pages.cpu()[bt[b, j // 16].long(), j % 16].float().numpy()
        assert np.array_equal(kc_gpu.view(np.uint32), kc_ref.view(np.uint32))
        if L % 4:
            part = cache.kc_partial[b].cpu().numpy()
            assert np.array_equal(part.view(np.uint32), O.open_block_partial(kid).view(np.uint32))
        # untouched slots keep their sentinel
        last = int(bt[b, (L - 1) // 64])
        if L % 64:
            assert torch.all(cache.k_view()[last, :, L % 64:].float() == 1024.0)
            assert torch.all(cache.v_view()[last, :, L % 64:].float() == 1024.0)
        if nb % 16:
            assert torch.all(cache.kc_pages[last, nb % 16:].float() == 512.0)


def test_append_order_rules():
    """The stated order rules of qsa_append_kv: a token whose predecessor in the
    arrays is the same sequence at a non-consecutive position sets
    QSA_DEV_BAD_ORDER; a sequence split into two runs within one call is not
    detected, but every K/V row is written and the other sequence's rows, kc and
    open-block sum stay exact."""
    wl = C.shrink(C.get("tiny"), [40, 40])
    # detected: sequence 0 jumps from position 5 to 7 inside one run
    cache = H.new_cache(wl)
    st = _status()
    pos = torch.tensor([4, 5, 7], dtype=torch.int32)
    qsa.qsa_append_kv(cache, C.k_rows(wl, 0, pos).cuda(), C.v_rows(wl, 0, pos).cuda(), C.kidx_rows(wl, 0, pos).cuda(),
                      torch.zeros(3, dtype=torch.int32, device="cuda"), pos.cuda(), st)
    torch.cuda.synchronize()
    assert "BAD_ORDER" in qsa.dev_status_names(int(st.item()))
    # not detected: A 0..5, B 0..9, A 6..9 in one call
    cache = H.new_cache(wl)
    st = _status()
    runs = [(0, 0, 6), (1, 0, 10), (0, 6, 10)]
    parts = []
    for b, p0, p1 in runs:
        pos = torch.arange(p0, p1)
        parts.append((C.k_rows(wl, b, pos), C.v_rows(wl, b, pos), C.kidx_rows(wl, b, pos),
                      torch.full((p1 - p0,), b, dtype=torch.int32), pos.to(torch.int32)))
    cat = [torch.cat([p[i] for p in parts]).cuda() for i in range(5)]
    qsa.qsa_append_kv(cache, *cat, st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    bt = cache.block_table.cpu()
    for b in range(2):
        pos = torch.arange(10)
        pg, row = bt[b, pos // 64].long(), pos % 64
        assert torch.equal(cache.k_view().cpu()[pg, :, row].view(torch.int16), C.k_rows(wl, b, pos).view(torch.int16))
        assert torch.equal(cache.v_view().cpu()[pg, :, row].view(torch.int16), C.v_rows(wl, b, pos).view(torch.int16))
    kid = C.kidx_rows(wl, 1, torch.arange(10)).float().numpy()
    j = torch.arange(2)
    kc_b = cache.kc_pages.cpu()[bt[1, j // 16].long(), j % 16].float().numpy()
    assert np.array_equal(kc_b.view(np.uint32), O.compress_keys(kid).view(np.uint32))
    assert np.array_equal(cache.kc_partial[1].cpu().numpy().view(np.uint32),
                          O.open_block_partial(kid).view(np.uint32))


def test_append_chunking_is_bitwise_invariant():
    """kc and the open-block partial do not depend on how the tokens are split
    into calls (all at once vs one token per call)."""
    wl = C.shrink(C.get("tiny"), [203])
    a = H.new_cache(wl)
    H.append_range(a, wl, 0, 0, 203)
    b = H.new_cache(wl)
    for p in range(203):
        H.append_range(b, wl, 0, p, p + 1)
    torch.cuda.synchronize()
    bt = a.block_table.cpu()
    j = torch.arange(203 // 4)
    pos = torch.arange(203)
    assert torch.equal(bits16(a.kc_pages.cpu()[bt[0, j // 16].long(), j % 16]),
                       bits16(b.kc_pages.cpu()[bt[0, j // 16].long(), j % 16]))
    assert torch.equal(a.kc_partial[0].cpu().view(torch.int32), b.kc_partial[0].cpu().view(torch.int32))
    assert torch.equal(bits16(a.k_view().cpu()[bt[0, pos // 64].long(), :, pos % 64]),
                       bits16(b.k_view().cpu()[bt[0, pos // 64].long(), :, pos % 64]))
    assert torch.equal(bits16(a.v_view().cpu()[bt[0, pos // 64].long(), :, pos % 64]),
                       bits16(b.v_view().cpu()[bt[0, pos // 64].long(), :, pos % 64]))


# ---------------------------------------------------------------- indexer + top-k


@pytest.mark.parametrize("name,lengths,k", [
    ("quarter", [4000, 999, 66, 5], 64),
    ("long", [3000, 2050], 512),
    ("batched", [1500], 16),
    ("quarter", [700, 3], 0),
])
def test_index_scores_and_topk_bit_exact(name, lengths, k):
    wl = C.shrink(C.get(name), lengths, page_perm=True, k_top=k)
    cache, dec, st = run_step(wl, k=k)
    assert st == 0
    sc = dec.scores.cpu().numpy()
    sel = dec.sel.cpu().numpy()
    cnt = dec.count.cpu().numpy()
    for row in range(wl.nq):
        d = R.query_inputs(wl, row)
        nb, _ = O.visible(d["p"])
        kc = O.compress_keys(R.kidx_seq(wl, d["seq"], d["p"] + 1))
        s_ref = O.block_scores(d["q_idx"], d["w"], kc)
        assert np.array_equal(sc[row, :nb], s_ref.astype(np.float32)), f"scores row {row}"
        sel_ref = O.select_blocks(s_ref, k)
        assert cnt[row] == len(sel_ref)
        assert np.array_equal(sel[row, :cnt[row]], sel_ref), f"selection row {row}"
        assert np.all(sel[row, cnt[row]:] == -1)


@pytest.mark.parametrize("lengths,new,k", [
    ([700, 2900, 33], 37, 64),     # 111 queries: ragged last tile, tiles spanning two sequences
    ([36000], 40, 512),            # rows longer than one CTA's 8,192-block chunk, ragged tile
])
def test_query_tiled_index_scores_bit_exact(lengths, new, k):
    """Chunked-prefill calls (many queries per sequence) take the query-tiled
    indexer; its scores and the selections must match the oracle exactly."""
    wl = C.shrink(C.get("prefill"), lengths, new_tokens=new, page_perm=True, k_top=k)
    assert wl.nq >= 8 * wl.batch and wl.nq >= 32
    cache, dec, st = run_step(wl, k=k)
    assert st == 0
    sc = dec.scores.cpu().numpy()
    sel = dec.sel.cpu().numpy()
    cnt = dec.count.cpu().numpy()
    for row in range(wl.nq):
        d = R.query_inputs(wl, row)
        nb, _ = O.visible(d["p"])
        kc = O.compress_keys(R.kidx_seq(wl, d["seq"], d["p"] + 1))
        s_ref = O.block_scores(d["q_idx"], d["w"], kc)
        assert np.array_equal(sc[row, :nb], s_ref.astype(np.float32)), f"scores row {row}"
        sel_ref = O.select_blocks(s_ref, k)
        assert cnt[row] == len(sel_ref)
        assert np.array_equal(sel[row, :cnt[row]], sel_ref), f"selection row {row}"


def test_query_tiled_scores_any_row_pitch():
    """The query-tiled indexer stores aligned score rows with bulk copies and
    falls back to element stores when a row's start is not 16-byte aligned (an
    odd pitch, or an offset base).  All three give the same scores, and no
    element past a query's nb_q is written."""
    wl = C.shrink(C.get("prefill"), [700, 2900, 33], new_tokens=37, page_perm=True, k_top=64)
    cache, dec, st = run_step(wl, k=64)
    assert st == 0
    nq = wl.nq
    inp = H.step_inputs(wl)
    nb = ((inp["q_pos"].long() + 1) // 4).cpu()
    width = int(nb.max()) + 40
    ref = dec.scores[:nq, :int(nb.max())].cpu()
    for ld, offset in [(width - width % 4, 0), (width - width % 4 + 3, 0), (width - width % 4, 1)]:
        flat = torch.full((nq * ld + 8,), float("nan"), dtype=torch.float32, device="cuda")
        scores = flat[offset:offset + nq * ld].view(nq, ld)
        status = _status()
        qsa.qsa_index_scores(cache, inp["q_idx"], inp["w"], inp["q_seq"], inp["q_pos"], scores, status)
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        got = scores.cpu()
        for row in range(nq):
            n = int(nb[row])
            assert torch.equal(got[row, :n].view(torch.int32), ref[row, :n].view(torch.int32)), (ld, offset, row)
            assert torch.isnan(got[row, n:]).all(), f"ld {ld} offset {offset}: row {row} written past nb_q"


def test_topk_all_ties_take_lowest_indices():
    wl = C.shrink(C.get("quarter"), [2000], k_top=100)
    cache = H.new_cache(wl)
    pos = torch.arange(0, 2000, device="cuda")
    k = C.k_rows(wl, 0, pos, "cuda")
    ki = torch.ones((2000, 128), dtype=torch.bfloat16, device="cuda")  # every kc equal
    qsa.qsa_append_kv(cache, k, k, ki, torch.zeros(2000, dtype=torch.int32, device="cuda"), pos.to(torch.int32))
    qs = C.queries(wl, device="cuda")
    qs["q_pos"].fill_(1999)
    dec = qsa.Decoder(cache, wl.hq, 1, k=100)
    dec.run(qs["q"], qs["q_idx"], qs["w"], qs["q_seq"], qs["q_pos"])
    torch.cuda.synchronize()
    assert dec.count.item() == 100
    assert dec.sel[0].tolist() == list(range(100))


def _topk_rows(kind, n, gen):
    if kind == "random":
        return torch.randn(n, generator=gen) * 100
    if kind == "ascending":
        return torch.arange(n, dtype=torch.float32) * 0.5
    if kind == "descending":
        return -torch.arange(n, dtype=torch.float32)
    if kind == "ties":          # few distinct values: ties straddle the K-th key
        return torch.randint(0, 7, (n,), generator=gen).float()
    if kind == "fine_ties":     # about 20 equal keys per value near the cut: a small last bin with ties
        return torch.round(torch.randn(n, generator=gen) * 64) / 64
    if kind == "neg_inf":       # blocks whose page was rejected score -inf
        x = torch.randn(n, generator=gen)
        x[torch.rand(n, generator=gen) < 0.5] = float("-inf")
        return x
    if kind == "hot_tail":      # the best blocks crowd into the last 5% of the row
        x = torch.randn(n, generator=gen)
        x[int(0.95 * n):] += 50
        return x
    raise ValueError(kind)


@pytest.mark.parametrize("nrows", [2, 300])
@pytest.mark.parametrize("kind", ["random", "ascending", "descending", "ties", "fine_ties", "neg_inf", "hot_tail"])
@pytest.mark.parametrize("n,k,pad", [(513, 512, 0), (1024, 512, 3), (1025, 1, 0), (4095, 2048, 1),
                                     (32768, 512, 0), (65536, 512, 5), (100000, 512, 0)])
def test_topk_rows_match_oracle_on_every_path(kind, n, k, pad, nrows):
    """Sampled-threshold path (random rows; rows whose last radix bin is small
    and holds ties straddling the K-th key) and its fallback (sorted rows, heavy
    ties, crowded tails overflow a warp's candidate list), aligned and
    misaligned row strides, -inf scores, rows of 513 .. 100,000 blocks; with
    few queries (1024-thread blocks) and many (300 rows, more than two per SM:
    256-thread blocks), the long rows of a 256K-token context included."""
    gen = torch.Generator().manual_seed(n * 7 + k + pad)
    rows = [_topk_rows(kind, n, gen), _topk_rows("random", n, gen)]
    rows += [rows[i % 2] if i % 5 else _topk_rows(kind, n, gen) for i in range(2, nrows)]
    ld = n + pad
    scores = torch.full((len(rows), ld), float("nan"), dtype=torch.float32)
    for i, r in enumerate(rows):
        scores[i, :n] = r
    q_pos = torch.full((len(rows),), 4 * n - 1, dtype=torch.int32, device="cuda")
    sel = torch.full((len(rows), k), -7, dtype=torch.int32, device="cuda")
    cnt = torch.zeros(len(rows), dtype=torch.int32, device="cuda")
    st = _status()
    qsa.qsa_topk_blocks(scores.cuda(), q_pos, k, sel, cnt, st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    sel_h, cnt_h = sel.cpu().numpy(), cnt.cpu().numpy()
    refs = {}
    for i, r in enumerate(rows):
        key = id(r)
        if key not in refs:
            refs[key] = O.select_blocks(r.double().numpy(), k)
        ref = refs[key]
        assert int(cnt_h[i]) == len(ref)
        assert np.array_equal(sel_h[i][:len(ref)], ref), f"{kind} row {i}"


# ---------------------------------------------------------------- attention


def _check_decode(wl, dec, rows, k=None, scale=None, chunk=None, prefix_from=None, partials=True):
    out = dec.out.float().cpu().numpy()
    lse = dec.lse.cpu().numpy()
    po = dec.part_o.cpu().numpy()
    pl = dec.part_lse.cpu().numpy()
    sel = dec.sel.cpu().numpy()
    for row in rows:
        r = R.expect_query(wl, row, k=k, scale=scale, chunk=dec.chunk_units if partials else None,
                           prefix_from=prefix_from)
        assert np.array_equal(sel[row, :len(r["sel"])], r["sel"]), f"selection row {row}"
        R.assert_close(out[row], r["o"], f"out row {row}")
        R.assert_close(lse[row], r["lse"], f"lse row {row}")
        if partials:
            R.assert_close(po[row], r["part_o"], f"part_o row {row}")
            R.assert_close(pl[row], r["part_lse"], f"part_lse row {row}")


def _head_cases():
    g = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "head_shapes.json")))
    return [(hq, hkv, n) for hq, hkv in g["head_pairs"] for n in g["query_rows"]]


@pytest.mark.parametrize("hq,hkv,nrows", _head_cases())
def test_decode_head_shapes(hq, hkv, nrows):
    base = C.get("quarter")
    if nrows == 1:
        wl = C.shrink(base, [3001], name=f"h{hq}x{hkv}", k_top=64)
    else:  # 257 query rows: an extend of 257 tokens, every tail remainder
        wl = C.shrink(base, [1200], new_tokens=nrows, name=f"h{hq}x{hkv}-extend", k_top=64)
    wl = dataclasses.replace(wl, hq=hq, hkv=hkv, page_perm=True)
    cache, dec, st = run_step(wl, k=64)
    assert st == 0
    rows = range(wl.nq) if wl.nq <= 8 else [0, 1, 2, 3, 100, 255, 256]
    _check_decode(wl, dec, rows, k=64)


@pytest.mark.parametrize("chunk", [1, 3, 16, 77, 513, 100000])
def test_decode_chunk_sizes(chunk):
    wl = C.shrink(C.get("long"), [2600, 1303], k_top=96)
    cache, dec, st = run_step(wl, k=96, chunk=chunk)
    assert st == 0
    _check_decode(wl, dec, range(wl.nq), k=96)


@pytest.mark.parametrize("k", [1, 15, 16, 17, 65])
@pytest.mark.parametrize("tail", [0, 1, 2, 3])
def test_decode_widths_and_tails(k, tail):
    L = 4 * 300 + tail  # context incl. the query's own token
    wl = C.shrink(C.get("batched"), [L - 1], k_top=k, page_perm=True)
    cache, dec, st = run_step(wl, k=k)
    assert st == 0
    assert int(dec.count[0]) == k
    _check_decode(wl, dec, [0], k=k)


def test_explicit_scale():
    wl = C.shrink(C.get("tiny"), [1999], k_top=40)
    cache, dec, st = run_step(wl, k=40, scale=0.0371)
    _check_decode(wl, dec, [0], k=40, scale=0.0371)


def test_zero_budget_and_fully_masked_rows():
    # K = 0: attention over the tail only; with t = 0 the row is fully masked
    for L, t in ((4 * 50 + 2, 2), (4 * 50, 0)):
        wl = C.shrink(C.get("tiny"), [L - 1], k_top=0)
        cache, dec, st = run_step(wl, k=0)
        assert st == 0 and int(dec.count[0]) == 0
        if t == 0:
            assert torch.all(dec.out == 0)
            assert torch.all(torch.isneginf(dec.lse))
        _check_decode(wl, dec, [0], k=0)


def test_short_context_equals_dense():
    # nb < K: every visible block is selected -> dense causal attention
    wl = C.shrink(C.get("long"), [57, 6], k_top=512)
    cache, dec, st = run_step(wl)
    assert st == 0
    assert dec.count.tolist() == [58 // 4, 7 // 4]
    _check_decode(wl, dec, range(2))


def test_shared_prefix_pages_and_cache_reuse():
    """Two requests map a shared prefix onto the same physical pages; then the
    cache is reused by a second decode step after more tokens are appended."""
    wl = C.shrink(C.get("quarter"), [640 + 300, 640 + 901], k_top=48, page_perm=False)
    wl2 = dataclasses.replace(wl, lengths=tuple(L + 1 + 37 for L in wl.lengths))
    P = 10  # shared pages = 640 tokens
    n0 = (wl2.total_lengths[0] + 63) // 64
    n1 = (wl2.total_lengths[1] + 63) // 64
    pps = max(n0, n1)
    bt = torch.full((2, pps), -1, dtype=torch.int32)
    bt[0, :n0] = torch.arange(n0)
    bt[1, :P] = torch.arange(P)
    bt[1, P:n1] = torch.arange(n0, n0 + n1 - P)
    cache = qsa.PagedCache(num_pages=n0 + n1 - P, max_seqs=2, max_pages_per_seq=pps, num_kv_heads=wl.hkv,
                           block_table=bt)
    H.append_range(cache, wl, 0, 0, wl.lengths[0])          # writes the prefix once
    H.append_range(cache, wl, 1, P * 64, wl.lengths[1])     # seq 1 only its own suffix
    _, dec, st = run_step(wl, cache=cache, k=48)
    assert st == 0
    _check_decode(wl, dec, [0], k=48)
    _check_decode(wl, dec, [1], k=48, prefix_from=(0, P * 64))
    first = dec.out.clone()
    # reuse: append 37 more tokens to both sequences and decode again
    for b in range(2):
        H.append_range(cache, wl, b, wl.lengths[b] + 1, wl2.lengths[b])
    _, dec2, st = run_step(wl2, cache=cache, k=48)
    assert st == 0
    _check_decode(wl2, dec2, [0], k=48)
    _check_decode(wl2, dec2, [1], k=48, prefix_from=(0, P * 64))
    assert not torch.equal(first, dec2.out)


def test_outputs_are_deterministic():
    wl = C.shrink(C.get("long"), [5000, 4097, 2222], k_top=256)
    cache, dec, st = run_step(wl, k=256)
    inp = C.queries(wl, device="cuda")
    outs = []
    for _ in range(3):
        dec.run(inp["q"], inp["q_idx"], inp["w"], inp["q_seq"], inp["q_pos"])
        torch.cuda.synchronize()
        outs.append((dec.out.clone(), dec.lse.clone(), dec.sel.clone(), dec.part_o.clone()))
    for o in outs[1:]:
        for a, b in zip(outs[0], o):
            assert torch.equal(a.view(torch.uint8) if a.dtype != torch.int32 else a,
                               b.view(torch.uint8) if b.dtype != torch.int32 else b)


def test_device_status_flags_bad_data_without_faulting():
    wl = C.shrink(C.get("quarter"), [900], k_top=32)
    cache, dec, st = run_step(wl, k=32)
    assert st == 0
    inp = C.queries(wl, device="cuda")
    # a selection index beyond the visible blocks and a count beyond K
    sel = dec.sel.clone()
    sel[0, 3] = 10 ** 6
    s2 = _status()
    qsa.qsa_sparse_decode(cache, inp["q"], inp["q_seq"], inp["q_pos"], sel, dec.count, 32, 1 / 16,
                          dec.chunk_units, dec.max_splits, dec.part_o, dec.part_lse, s2)
    torch.cuda.synchronize()
    assert int(s2.item()) & 8
    bad_count = torch.full_like(dec.count, 10 ** 6)
    s3 = _status()
    qsa.qsa_sparse_decode(cache, inp["q"], inp["q_seq"], inp["q_pos"], dec.sel, bad_count, 32, 1 / 16,
                          dec.chunk_units, dec.max_splits, dec.part_o, dec.part_lse, s3)
    torch.cuda.synchronize()
    assert int(s3.item()) & 16
    # a block-table entry outside the page pool
    cache.block_table[0, 2] = 10 ** 7
    s4 = _status()
    qsa.qsa_index_scores(cache, inp["q_idx"], inp["w"], inp["q_seq"], inp["q_pos"], dec.scores, s4)
    qsa.qsa_topk_blocks(dec.scores, inp["q_pos"], 32, dec.sel, dec.count, s4)
    qsa.qsa_sparse_decode(cache, inp["q"], inp["q_seq"], inp["q_pos"], dec.sel, dec.count, 32, 1 / 16,
                          dec.chunk_units, dec.max_splits, dec.part_o, dec.part_lse, s4)
    torch.cuda.synchronize()
    assert int(s4.item()) & 1
    # the context is still usable
    cache.block_table[0, 2] = C.block_table(wl)[0, 2]
    dec.run(inp["q"], inp["q_idx"], inp["w"], inp["q_seq"], inp["q_pos"])
    torch.cuda.synchronize()
    _check_decode(wl, dec, [0], k=32)


def test_host_errors_enqueue_nothing():
    wl = C.shrink(C.get("tiny"), [300], k_top=16)
    cache, dec, st = run_step(wl, k=16)
    inp = C.queries(wl, device="cuda")
    with pytest.raises(qsa.QSAError) as e:
        qsa.qsa_sparse_decode(cache, inp["q"], inp["q_seq"], inp["q_pos"], dec.sel, dec.count, 16, 1 / 16,
                              dec.chunk_units, 1, dec.part_o[:, :1], dec.part_lse[:, :1])
    assert e.value.status == -1
    with pytest.raises(ValueError):
        qsa.qsa_index_scores(cache, inp["q_idx"].cpu(), inp["w"], inp["q_seq"], inp["q_pos"], dec.scores)


def test_split_pipeline_stress_no_expired_waits():
    """Hundreds of decode launches with an L2 flush between them: the copy /
    consumer pipeline never loses a phase (a wait that named a stale phase
    would consume unarrived data and later expire with the TIMEOUT bit), and
    every launch reproduces the first one bit for bit."""
    wl = C.shrink(C.get("long"), [16383] * 16, k_top=512)
    cache, dec, st = run_step(wl)
    assert st == 0
    inp = C.queries(wl, device="cuda")
    calls = dec.bind(inp["q"], inp["q_idx"], inp["w"], inp["q_seq"], inp["q_pos"])
    ref_o, ref_l = dec.out.clone(), dec.part_lse.clone()
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")
    for _ in range(300):
        calls[2]()
        calls[3]()
        flush.zero_()
    torch.cuda.synchronize()
    assert int(dec.dev_status.item()) == 0, qsa.dev_status_names(int(dec.dev_status.item()))
    assert torch.equal(dec.out.view(torch.int16), ref_o.view(torch.int16))
    assert torch.equal(dec.part_lse, ref_l)


def test_step_io_staging_and_readback():
    """The staged step inputs (one host-to-device copy) drive the same step as
    separately allocated inputs, bit for bit, and the output read-back (one
    copy for a full batch, two for a partial one) returns the device values."""
    wl = C.shrink(C.get("long"), [3000, 2050, 777], k_top=64)
    st = _status()
    cache = H.build_cache(wl, dev_status=st)
    ref_in = H.step_inputs(wl)
    io = qsa.StepIO(wl.batch * wl.new_tokens, wl.nq, wl.hq, wl.hkv)
    for k, t in H.step_inputs(wl, device="cpu").items():
        io.host[k].copy_(t)
    io.upload()
    torch.cuda.synchronize()
    for k, t in ref_in.items():
        assert torch.equal(io.dev[k], t), k
    saved = cache.kc_partial.clone()
    outs = []
    for inp in (ref_in, io.dev):
        cache.kc_partial.copy_(saved)
        qsa.qsa_append_kv(cache, inp["k_new"], inp["v_new"], inp["kidx_new"], inp["seq_id"], inp["pos"], st)
        dec = qsa.Decoder(cache, wl.hq, wl.nq, k=64)
        dec.dev_status = st
        dec.run(inp["q"], inp["q_idx"], inp["w"], inp["q_seq"], inp["q_pos"])
        host = dec.host_outputs()
        nbytes = dec.download(host, wl.nq)
        torch.cuda.synchronize()
        assert nbytes == host[0].numel()
        assert torch.equal(host[1].view(torch.int16), dec.out.cpu().view(torch.int16))
        assert torch.equal(host[2], dec.lse.cpu())
        outs.append(dec.out.clone())
    assert int(st.item()) == 0
    assert torch.equal(outs[0].view(torch.int16), outs[1].view(torch.int16))
    # a partial batch reads back its rows only
    dec2 = qsa.Decoder(cache, wl.hq, wl.nq + 5, k=64)
    dec2.dev_status = st
    dec2.run(io.dev["q"], io.dev["q_idx"], io.dev["w"], io.dev["q_seq"], io.dev["q_pos"])
    host = dec2.host_outputs()
    host[1].zero_()
    nbytes = dec2.download(host, wl.nq)
    torch.cuda.synchronize()
    assert nbytes == wl.nq * wl.hq * 256 * 2 + wl.nq * wl.hq * 4
    assert torch.equal(host[1][:wl.nq].view(torch.int16), dec2.out[:wl.nq].cpu().view(torch.int16))
    assert torch.all(host[1][wl.nq:] == 0)


@pytest.mark.parametrize("hq,hkv,k,L", [
    (16, 1, 2048, 4 * 2300 + 2),    # the largest group (16 Q heads per KV head) and the largest budget
    (2, 2, 2048, 4 * 2048 + 3),     # one Q head per KV head; budget = every complete block but none spare
    (32, 2, 700, 4 * 3000),         # group 16 at two KV heads, no tail
])
def test_decode_limits_budget_and_group(hq, hkv, k, L):
    wl = dataclasses.replace(C.shrink(C.get("quarter"), [L - 1], k_top=k, page_perm=True), hq=hq, hkv=hkv)
    cache, dec, st = run_step(wl, k=k)
    assert st == 0
    assert int(dec.count[0]) == min(k, L // 4)
    _check_decode(wl, dec, [0], k=k)


def test_noalloc_call_on_an_fp8_cache():
    wl = dataclasses.replace(C.shrink(C.get("long"), [4000, 2500], k_top=256, page_perm=True), kv_fp8=True)
    cache, dec, st = run_step(wl, k=256)
    assert st == 0
    s2 = _status()
    out = torch.empty_like(dec.out[:wl.nq])
    lse = torch.empty_like(dec.lse[:wl.nq])
    inp = H.step_inputs(wl)
    qsa.qsa_sparse_attention_noalloc(cache, inp["q"], inp["q_seq"], inp["q_pos"], dec.sel[:wl.nq], dec.count[:wl.nq],
                                     256, wl.scale, dec.chunk_units, out, lse, s2)
    torch.cuda.synchronize()
    assert int(s2.item()) == 0
    assert torch.equal(out.view(torch.int16), dec.out[:wl.nq].view(torch.int16))
    for row in range(wl.nq):
        ref = R.expect_query(wl, row, k=256)
        R.assert_close(out[row].float().cpu().numpy(), ref["o"], f"noalloc fp8 row {row}")
