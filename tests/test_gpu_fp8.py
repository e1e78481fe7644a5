"""The FP8 e4m3 main K/V cache: the append stores e4m3 of every BF16 row
exactly (round to nearest even, saturated), and sparse attention over the FP8
cache matches the oracle run on the same e4m3 values, across tile counts,
ragged tails, chunkings and head shapes."""
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


def _fp8(wl):
    return dataclasses.replace(wl, kv_fp8=True)


def _status():
    return torch.zeros(1, dtype=torch.int32, device="cuda")


def _run(wl, k, chunk=None, scale=None):
    st = _status()
    cache = H.build_cache(wl, dev_status=st)
    assert cache.kv_pages.dtype == torch.float8_e4m3fn
    inp = H.step_inputs(wl)
    qsa.qsa_append_kv(cache, inp["k_new"], inp["v_new"], inp["kidx_new"], inp["seq_id"], inp["pos"], st)
    dec = qsa.Decoder(cache, wl.hq, wl.nq, k=k, scale=wl.scale if scale is None else scale, chunk_units=chunk)
    dec.dev_status = st
    dec.run(inp["q"], inp["q_idx"], inp["w"], inp["q_seq"], inp["q_pos"])
    torch.cuda.synchronize()
    assert int(st.item()) == 0, qsa.dev_status_names(int(st.item()))
    return dec


def _check(wl, dec, rows, k, scale=None, partials=True):
    out = dec.out.float().cpu().numpy()
    lse = dec.lse.cpu().numpy()
    sel = dec.sel.cpu().numpy()
    po, pl = dec.part_o.cpu().numpy(), dec.part_lse.cpu().numpy()
    for row in rows:
        r = R.expect_query(wl, row, k=k, scale=scale, chunk=dec.chunk_units if partials else None)
        assert np.array_equal(sel[row, :len(r["sel"])], r["sel"]), f"selection row {row}"
        R.assert_close(out[row], r["o"], f"out row {row}")
        R.assert_close(lse[row], r["lse"], f"lse row {row}")
        if partials:
            R.assert_close(po[row], r["part_o"], f"part_o row {row}")
            R.assert_close(pl[row], r["part_lse"], f"part_lse row {row}")


@pytest.mark.parametrize("name,lengths", [("quarter", [301, 64, 130, 7]), ("long", [197, 260])])
def test_append_fp8_matches_oracle_rounding(name, lengths):
    wl = _fp8(C.shrink(C.get(name), lengths, page_perm=True))
    cache = H.new_cache(wl)
    cache.kv_pages.view(torch.uint8).fill_(0x7E)  # sentinel: 448
    st = _status()
    for b, L in enumerate(wl.lengths):  # two calls per sequence, the second starting mid-block
        for a, z in ((0, L // 2 + 1), (L // 2 + 1, L)):
            if z > a:
                H.append_range(cache, wl, b, a, z, st)
    torch.cuda.synchronize()
    assert st.item() == 0
    bt = cache.block_table.cpu()
    kv = cache.kv_pages.cpu()
    for b, L in enumerate(wl.lengths):
        pos = torch.arange(L)
        pg, row = bt[b, pos // 64].long(), pos % 64
        for view, rows in ((0, C.k_rows(wl, b, pos)), (1, C.v_rows(wl, b, pos))):
            got = kv[:, :, :, view].reshape(wl.num_pages(), wl.hkv, 64, 256)[pg, :, row].double().numpy()
            want = O.e4m3_round(rows.float().numpy())
            assert np.array_equal(got, want), f"seq {b} {'KV'[view]} values"
            assert np.array_equal(np.signbit(got), np.signbit(want)), f"seq {b} {'KV'[view]} signs of zero"
        last = int(bt[b, (L - 1) // 64])
        if L % 64:
            untouched = kv.view(torch.uint8)[last, :, :, :, :, :].reshape(wl.hkv, 16, 2, 4, 256)
            t = torch.arange(L % 64, 64)
            assert torch.all(untouched[:, t // 4, :, t % 4] == 0x7E)


def test_append_fp8_saturates_and_rounds_ties_to_even():
    wl = _fp8(C.shrink(C.get("tiny"), [4]))
    cache = H.new_cache(wl)
    st = _status()
    vals = torch.tensor([448.0, 464.0, 1000.0, -3e38, 1.0625, 1.1875, 2.0 ** -10, 3 * 2.0 ** -10, -0.0, 17.0, 0.1, -7.5])
    k = torch.zeros(4, wl.hkv, 256)
    k.view(-1)[: vals.numel()] = vals
    k = k.to(torch.bfloat16).cuda()
    v = (-k).contiguous()
    ki = torch.zeros(4, 128, dtype=torch.bfloat16, device="cuda")
    qsa.qsa_append_kv(cache, k, v, ki, torch.zeros(4, dtype=torch.int32, device="cuda"),
                      torch.arange(4, dtype=torch.int32, device="cuda"), st)
    torch.cuda.synchronize()
    assert st.item() == 0
    got_k = cache.k_view()[0, :, :4].cpu().double().numpy().transpose(1, 0, 2)
    got_v = cache.v_view()[0, :, :4].cpu().double().numpy().transpose(1, 0, 2)
    assert np.array_equal(got_k, O.e4m3_round(k.float().cpu().numpy()))
    assert np.array_equal(got_v, O.e4m3_round(v.float().cpu().numpy()))
    head = got_k.reshape(-1)[:vals.numel()]
    # 448, saturated 464 / 1000 / -3e38, ties 1.0625 -> 1.0 and 1.1875 -> 1.25, 2^-10 -> 0, 3*2^-10 -> 2^-8
    assert head[:8].tolist() == [448.0, 448.0, 448.0, -448.0, 1.0, 1.25, 0.0, 2.0 ** -8]


@pytest.mark.parametrize("k", [1, 16, 17, 65])
@pytest.mark.parametrize("tail", [0, 3])
def test_fp8_decode_widths_and_tails(k, tail):
    L = 4 * 300 + tail
    wl = _fp8(C.shrink(C.get("batched"), [L - 1], k_top=k, page_perm=True))
    dec = _run(wl, k)
    assert int(dec.count[0]) == k
    _check(wl, dec, [0], k)


@pytest.mark.parametrize("chunk", [1, 3, 77, 100000])
def test_fp8_decode_chunk_sizes(chunk):
    wl = _fp8(C.shrink(C.get("long"), [2600, 1303], k_top=96))
    dec = _run(wl, 96, chunk=chunk)
    _check(wl, dec, range(wl.nq), 96)


@pytest.mark.parametrize("hq,hkv", [(16, 2), (24, 2), (12, 1), (6, 1), (16, 1)])
def test_fp8_decode_head_shapes(hq, hkv):
    wl = _fp8(dataclasses.replace(C.shrink(C.get("quarter"), [3001, 777], k_top=64, page_perm=True), hq=hq, hkv=hkv))
    dec = _run(wl, 64)
    _check(wl, dec, range(wl.nq), 64)


def test_fp8_extend_rows_and_dense_short_context():
    wl = _fp8(C.shrink(C.get("quarter"), [1200], new_tokens=37, k_top=64, page_perm=True))
    dec = _run(wl, 64)
    _check(wl, dec, [0, 1, 2, 3, 17, 36], 64)
    wl = _fp8(C.shrink(C.get("long"), [57, 6], k_top=512))
    dec = _run(wl, 512)
    _check(wl, dec, range(2), 512)


def test_fp8_zero_budget_and_fully_masked_row():
    for L, t in ((4 * 50 + 2, 2), (4 * 50, 0)):
        wl = _fp8(C.shrink(C.get("tiny"), [L - 1], k_top=0))
        dec = _run(wl, 0)
        if t == 0:
            assert torch.all(dec.out == 0) and torch.all(torch.isneginf(dec.lse))
        _check(wl, dec, [0], 0)


def test_fp8_outputs_are_deterministic():
    wl = _fp8(C.shrink(C.get("long"), [5000, 4097, 2222], k_top=256))
    a = _run(wl, 256)
    o1 = a.out.clone()
    a.run(*[H.step_inputs(wl)[n] for n in ("q", "q_idx", "w", "q_seq", "q_pos")])
    torch.cuda.synchronize()
    assert torch.equal(o1.view(torch.int16), a.out.view(torch.int16))
