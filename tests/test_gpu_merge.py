"""The attention call with the in-kernel split merge (qsa_sparse_attention)
through the C ABI: out and lse equal the split kernel + qsa_combine bit for
bit (BF16 and FP8 K/V, one and many splits per (query, KV head) pair, K = 0,
an out-of-range query), the pair counters are left at zero so calls can
repeat, and the outputs stay within the oracle's tolerance."""
import numpy as np
import pytest
import torch

from tests import oracle_ref as R
from workloads import configs as C

pytestmark = pytest.mark.gpu

qsa = pytest.importorskip("sparse_attention_decode_03_b200")
H = pytest.importorskip("workloads.harness")


@pytest.fixture(autouse=True, scope="module")
def _need_cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")


def _pipelines(wl, k, chunk):
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    cache = H.build_cache(wl, dev_status=st)
    inp = H.step_inputs(wl)
    qsa.qsa_append_kv(cache, inp["k_new"], inp["v_new"], inp["kidx_new"], inp["seq_id"], inp["pos"], st)
    decs = []
    for merged in (False, True):
        d = qsa.Decoder(cache, wl.hq, wl.nq, k=k, scale=wl.scale, chunk_units=chunk, merged=merged)
        d.dev_status = st
        decs.append(d)
    return cache, inp, st, decs


def _run(d, inp):
    d.run(inp["q"], inp["q_idx"], inp["w"], inp["q_seq"], inp["q_pos"])


@pytest.mark.parametrize("name,lengths,k,chunk", [
    ("long", [9000, 4100, 777], 512, 37),     # many splits per pair, ragged chunks
    ("long", [9000, 4100, 777], 512, 4096),   # one split per pair
    ("quarter", [16000, 2000, 50, 6000], 64, 11),
    ("batched", [1500, 900], 16, 5),
    ("long-fp8", [6000, 3001], 512, 100),
    ("quarter", [700, 3], 0, 3),               # K = 0: the trailing tokens only
])
def test_merged_equals_separate_combine(name, lengths, k, chunk):
    wl = C.shrink(C.get(name), lengths, page_perm=True, k_top=k)
    cache, inp, st, (sep, mer) = _pipelines(wl, k, chunk)
    nq = wl.nq
    for rep in range(3):  # the counters return to zero: the call repeats
        _run(sep, inp)
        mer.out.fill_(7.0)
        mer.lse.fill_(7.0)
        _run(mer, inp)
        torch.cuda.synchronize()
        assert int(st.item()) == 0, qsa.dev_status_names(int(st.item()))
        assert torch.equal(sep.sel[:nq], mer.sel[:nq])
        assert torch.equal(sep.out[:nq].view(torch.int16), mer.out[:nq].view(torch.int16)), f"out, call {rep}"
        assert torch.equal(sep.lse[:nq].view(torch.int32), mer.lse[:nq].view(torch.int32)), f"lse, call {rep}"
        assert torch.count_nonzero(mer.pair_done) == 0
    # and the oracle's tolerance on every row
    out = mer.out[:nq].float().cpu().numpy()
    lse = mer.lse[:nq].cpu().numpy()
    for row in range(nq):
        r = R.expect_query(wl, row)
        R.assert_close(out[row], r["o"], f"out row {row}")
        R.assert_close(lse[row], r["lse"], f"lse row {row}")


def test_merged_out_of_range_query():
    """A query whose sequence id is out of range: status bit, zero output and
    lse = -inf for it (every split empty), the other rows unchanged."""
    wl = C.shrink(C.get("long"), [3000, 2500, 1800], page_perm=True, k_top=64)
    cache, inp, st, (sep, mer) = _pipelines(wl, 64, 29)
    inp["q_seq"][1] = wl.batch + 9
    _run(sep, inp)
    _run(mer, inp)
    torch.cuda.synchronize()
    assert "BAD_SEQ" in qsa.dev_status_names(int(st.item()))
    nq = wl.nq
    assert torch.equal(sep.out[:nq].view(torch.int16), mer.out[:nq].view(torch.int16))
    assert torch.equal(sep.lse[:nq].view(torch.int32), mer.lse[:nq].view(torch.int32))
    assert torch.all(mer.out[1] == 0) and torch.all(torch.isneginf(mer.lse[1]))
    assert torch.count_nonzero(mer.pair_done) == 0


@pytest.mark.parametrize("name", ["long", "quarter"])
def test_merged_full_size(name):
    """Full-size workloads in the benchmark's launch configuration: the merged
    call equals the separate combine bit for bit on every row."""
    wl = C.get(name)
    cache, inp, st, (sep, mer) = _pipelines(wl, wl.k_top, H.chunk_units_for(wl))
    _run(sep, inp)
    _run(mer, inp)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    nq = wl.nq
    assert torch.equal(sep.out[:nq].view(torch.int16), mer.out[:nq].view(torch.int16))
    assert torch.equal(sep.lse[:nq].view(torch.int32), mer.lse[:nq].view(torch.int32))
    assert torch.count_nonzero(mer.pair_done) == 0
    rows = [0, nq - 1]
    out = mer.out[:nq].float().cpu().numpy()
    for row in rows:
        r = R.expect_query(wl, row)
        R.assert_close(out[row], r["o"], f"{name} out row {row}")
