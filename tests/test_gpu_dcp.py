"""Decode context parallelism on one GPU: the localisation kernels bit-exact
against the shard rule, the strided / fp32 merge against the oracle's combine,
and whole DCP steps with N ranks run one after another on the same GPU (the
all-gather emulated by copies): every rank's selection equals the oracle's,
every rank's share matches the oracle's share, and the merged output matches
the oracle and the unsharded path."""
import dataclasses

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


@pytest.mark.parametrize("nranks,rank,interleave", [(2, 0, 1), (2, 1, 1), (3, 2, 1), (4, 1, 2), (1, 0, 1)])
def test_localize_tokens_bit_exact(nranks, rank, interleave):
    sh = qsa.DCPShard(nranks, rank, interleave)
    g = torch.Generator().manual_seed(nranks * 7 + rank)
    n = 3001
    seq = torch.randint(-1, 5, (n,), generator=g, dtype=torch.int32)
    pos = torch.randint(0, 64 * 50, (n,), generator=g, dtype=torch.int32)
    sl = torch.full((n,), 77, dtype=torch.int32, device="cuda")
    pl = torch.full((n,), 77, dtype=torch.int32, device="cuda")
    qsa.qsa_dcp_localize_tokens(seq.cuda(), pos.cuda(), nranks, rank, interleave, sl, pl)
    torch.cuda.synchronize()
    want_s = [int(s) if s >= 0 and sh.owner(int(p) // 64) == rank else -1 for s, p in zip(seq, pos)]
    want_p = [sh.local_page(int(p) // 64) * 64 + int(p) % 64 if w >= 0 else 0 for w, p in zip(want_s, pos)]
    assert sl.cpu().tolist() == want_s
    assert pl.cpu().tolist() == want_p


def _host_localize(sel, cnt, p, K, sh):
    """The localisation the header states, written out on the host."""
    if p < 0:
        return [-1] * K, 0, p
    nb, t = (p + 1) // 4, (p + 1) % 4
    loc = [sh.local_page(j // 16) * 16 + j % 16 for j in sel[:cnt] if sh.owner(j // 16) == sh.r]
    Pt = nb // 16
    tail_page = sh.owner(Pt) == sh.r
    nb_l = sh.local_pages(Pt) * 16 + (nb % 16 if tail_page else 0)
    if tail_page and t > 0:
        pl = 4 * nb_l + t - 1
    elif nb_l > 0:
        pl = 4 * nb_l - 1
    else:
        pl = 3
    return loc + [-1] * (K - len(loc)), len(loc), pl


@pytest.mark.parametrize("nranks,interleave", [(2, 1), (3, 1), (2, 3), (5, 1)])
def test_localize_selection_bit_exact(nranks, interleave):
    g = np.random.default_rng(nranks * 11 + interleave)
    K = 40
    rows, counts, qpos = [], [], []
    for i in range(60):
        p = int(g.integers(0, 64 * 40)) if i > 3 else [0, 2, 4 * 16 * nranks * interleave + 1, 63][i]
        nb = (p + 1) // 4
        c = min(K, nb, int(g.integers(0, K + 1)))
        s = np.sort(g.choice(nb, size=c, replace=False)) if c else np.zeros(0, np.int64)
        rows.append(list(s) + [-1] * (K - c))
        counts.append(c)
        qpos.append(p)
    qpos[5] = -1
    counts[5] = 0
    sel = torch.tensor(rows, dtype=torch.int32).cuda()
    cnt = torch.tensor(counts, dtype=torch.int32).cuda()
    qp = torch.tensor(qpos, dtype=torch.int32).cuda()
    for rank in range(nranks):
        sh = qsa.DCPShard(nranks, rank, interleave)
        st = _status()
        sl = torch.full_like(sel, 99)
        cl = torch.full_like(cnt, 99)
        pl = torch.full_like(qp, 99)
        qsa.qsa_dcp_localize_selection(sel, cnt, qp, K, nranks, rank, interleave, sl, cl, pl, st)
        torch.cuda.synchronize()
        assert int(st.item()) == 0
        for i in range(len(rows)):
            s_w, c_w, p_w = _host_localize(rows[i], counts[i], qpos[i], K, sh)
            assert sl[i].tolist() == s_w and int(cl[i]) == c_w and int(pl[i]) == p_w, (rank, i)
    # bad entries are dropped and flagged; a bad count is clamped and flagged
    bad = sel.clone()
    bad[7, 0] = 10 ** 6
    cnt2 = cnt.clone()
    cnt2[8] = K + 5
    st = _status()
    sl, cl, pl = torch.empty_like(sel), torch.empty_like(cnt), torch.empty_like(qp)
    qsa.qsa_dcp_localize_selection(bad, cnt2, qp, K, nranks, 0, interleave, sl, cl, pl, st)
    torch.cuda.synchronize()
    assert int(st.item()) & 8 and int(st.item()) & 16  # QSA_DEV_BAD_SEL, QSA_DEV_BAD_COUNT


def test_strided_merge_f32_and_rank_major_match_the_oracle():
    g = torch.Generator().manual_seed(5)
    nq, S, hq = 7, 5, 12
    po = torch.randn(nq, S, hq, 256, generator=g)
    pl = torch.randn(nq, S, hq, generator=g) * 3
    pl[0, :, 3] = float("-inf")       # a fully empty row
    pl[1, 2] = float("-inf")          # one empty split
    out = torch.empty(nq, hq, 256, device="cuda")
    lse = torch.empty(nq, hq, device="cuda")
    qsa.qsa_combine_f32(po.cuda(), pl.cuda(), out, lse)
    # the same splits laid out split-major, merged into bf16
    out_b = torch.empty(nq, hq, 256, dtype=torch.bfloat16, device="cuda")
    lse_b = torch.empty(nq, hq, device="cuda")
    qsa.qsa_combine_ranks(po.permute(1, 0, 2, 3).contiguous().cuda(), pl.permute(1, 0, 2).contiguous().cuda(),
                          out_b, lse_b)
    torch.cuda.synchronize()
    for q in range(nq):
        o_ref, l_ref = O.combine(po[q].double().numpy(), pl[q].double().numpy())
        R.assert_close(out[q].cpu().numpy(), o_ref, f"fp32 merge row {q}")
        R.assert_close(lse[q].cpu().numpy(), l_ref, f"lse row {q}")
        R.assert_close(out_b[q].float().cpu().numpy(), o_ref, f"bf16 rank-major merge row {q}")
        R.assert_close(lse_b[q].cpu().numpy(), l_ref, f"rank-major lse row {q}")
    assert torch.all(out[0, 3] == 0) and torch.isneginf(lse[0, 3])


def _build_ranks(wl, nranks, interleave, k, st):
    pages = [-(-L // 64) for L in wl.total_lengths]
    ranks = []
    for r in range(nranks):
        sh = qsa.DCPShard(nranks, r, interleave)
        sel_cache = qsa.PagedCache(wl.num_pages(), wl.batch, wl.pages_per_seq(), wl.hkv,
                                   block_table=C.block_table(wl), with_kv=False)
        bt, used = sh.shard_block_table(pages)
        shard = qsa.PagedCache(max(1, used), wl.batch, bt.shape[1], wl.hkv, block_table=bt, with_kc=False,
                               kv_dtype=qsa.KV_FP8_E4M3 if wl.kv_fp8 else qsa.KV_BF16)
        rk = qsa.DCPRank(sel_cache, shard, wl.hq, wl.nq, nranks, r, interleave, k=k, scale=wl.scale)
        rk.dev_status = st
        ranks.append(rk)
    for b, L in enumerate(wl.lengths):     # the cached context, in chunks
        for a0 in range(0, L, 1000):
            a1 = min(L, a0 + 1000)
            pos = torch.arange(a0, a1, device="cuda")
            args = (C.k_rows(wl, b, pos, "cuda"), C.v_rows(wl, b, pos, "cuda"), C.kidx_rows(wl, b, pos, "cuda"),
                    torch.full((a1 - a0,), b, dtype=torch.int32, device="cuda"), pos.to(torch.int32))
            for rk in ranks:
                rk.append(*args)
    return ranks


@pytest.mark.parametrize("nranks,interleave,name,lengths,k,new", [
    (2, 1, "long", [5000, 3001], 64, 1),
    (3, 1, "quarter", [4100, 777, 130], 32, 1),
    (2, 2, "batched", [2600], 512, 1),
    (4, 1, "long", [1300, 64 * 9 + 2], 16, 1),
    (2, 1, "prefill", [3000, 700], 64, 37),    # chunked prefill: the query-tiled indexer on the selector
])
def test_dcp_step_matches_the_oracle_and_the_unsharded_path(nranks, interleave, name, lengths, k, new):
    wl = C.shrink(C.get(name), lengths, new_tokens=new, k_top=k, page_perm=True)
    st = _status()
    ranks = _build_ranks(wl, nranks, interleave, k, st)
    inp = H.step_inputs(wl)
    for rk in ranks:
        rk.append(inp["k_new"], inp["v_new"], inp["kidx_new"], inp["seq_id"], inp["pos"])
    for rk in ranks:
        rk.attend(inp["q"], inp["q_idx"], inp["w"], inp["q_seq"], inp["q_pos"])
    for rk in ranks:              # the all-gather, emulated: every rank's result into every rank's buffer
        for j, other in enumerate(ranks):
            rk.o_all[j].copy_(other.o_rank)
            rk.lse_all[j].copy_(other.lse_rank)
    outs = [rk.merge(wl.nq) for rk in ranks]
    torch.cuda.synchronize()
    assert int(st.item()) == 0, qsa.dev_status_names(int(st.item()))
    # unsharded path on the same inputs
    _, dec, st1 = _unsharded(wl, k)
    assert st1 == 0
    rows = range(wl.nq) if wl.nq <= 8 else [0, 1, 2, 3, 36, 37, 50, wl.nq - 1]
    for row in rows:
        ref = R.expect_query(wl, row, k=k)
        for rk in ranks:
            assert np.array_equal(rk.sel[row, :int(rk.count[row])].cpu().numpy(), ref["sel"])
        d = R.query_inputs(wl, row)
        rows = R.kv_reader(wl, d["seq"])
        for r, rk in enumerate(ranks):
            o_r, l_r = O.dcp_rank_partial(d["q"], ref["sel"], d["p"], rows, wl.scale, nranks, r, interleave)
            R.assert_close(rk.o_rank[row].cpu().numpy(), o_r, f"rank {r} share row {row}")
            R.assert_close(rk.lse_rank[row].cpu().numpy(), l_r, f"rank {r} lse row {row}")
        for r, (out, lse) in enumerate(outs):
            R.assert_close(out[row].float().cpu().numpy(), ref["o"], f"merged out row {row} on rank {r}")
            R.assert_close(lse[row].cpu().numpy(), ref["lse"], f"merged lse row {row} on rank {r}")
            R.assert_close(out[row].float().cpu().numpy(), dec.out[row].float().cpu().numpy(),
                           f"merged vs unsharded row {row}")


def _unsharded(wl, k):
    st = _status()
    cache = H.build_cache(wl, dev_status=st)
    inp = H.step_inputs(wl)
    qsa.qsa_append_kv(cache, inp["k_new"], inp["v_new"], inp["kidx_new"], inp["seq_id"], inp["pos"], st)
    dec = qsa.Decoder(cache, wl.hq, wl.nq, k=k, scale=wl.scale)
    dec.dev_status = st
    dec.run(inp["q"], inp["q_idx"], inp["w"], inp["q_seq"], inp["q_pos"])
    torch.cuda.synchronize()
    return cache, dec, int(st.item())


def test_dcp_step_with_fp8_shards():
    wl = dataclasses.replace(C.shrink(C.get("long"), [3000, 2222], k_top=64, page_perm=True), kv_fp8=True)
    st = _status()
    ranks = _build_ranks(wl, 2, 1, 64, st)
    inp = H.step_inputs(wl)
    for rk in ranks:
        rk.append(inp["k_new"], inp["v_new"], inp["kidx_new"], inp["seq_id"], inp["pos"])
        rk.attend(inp["q"], inp["q_idx"], inp["w"], inp["q_seq"], inp["q_pos"])
    for j, other in enumerate(ranks):
        ranks[0].o_all[j].copy_(other.o_rank)
        ranks[0].lse_all[j].copy_(other.lse_rank)
    out, lse = ranks[0].merge(wl.nq)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    for row in range(wl.nq):
        ref = R.expect_query(wl, row, k=64)
        R.assert_close(out[row].float().cpu().numpy(), ref["o"], f"fp8 merged out row {row}")
