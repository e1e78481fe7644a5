"""The five workloads at full size, in the launch configuration the benchmark
times: bit-exact selections and toleranced outputs on sampled query rows (the
oracle regenerates each sampled row's inputs on the host), and properties that
hold for every row at any size."""
import numpy as np
import pytest
import torch

from oracle import qsa_oracle as O
from tests import oracle_ref as R
from workloads import configs as C

pytestmark = pytest.mark.gpu

qsa = pytest.importorskip("sparse_attention_decode_03_b200")
H = pytest.importorskip("workloads.harness")

SAMPLES = {
    "tiny": [0],
    "batched": [0, 5, 7],
    "long": [0, 17, 31],
    "quarter": None,            # shortest, longest and two more
    "prefill": [0, 1, 2, 3, 4095, 4096, 6001, 8191],
    "long-fp8": [0, 17, 31],
    "quarter-fp8": None,
}


@pytest.fixture(autouse=True, scope="module")
def _need_cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")


@pytest.mark.parametrize("name", list(C.ALL) + list(C.FP8))
def test_workload_full_size(name):
    wl = C.get(name)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    cache = H.build_cache(wl, dev_status=st)
    inp = H.step_inputs(wl)
    dec = qsa.Decoder(cache, wl.hq, wl.nq, k=wl.k_top, scale=wl.scale, chunk_units=H.chunk_units_for(wl))
    dec.dev_status = st
    qsa.qsa_append_kv(cache, inp["k_new"], inp["v_new"], inp["kidx_new"], inp["seq_id"], inp["pos"], st)
    dec.run(inp["q"], inp["q_idx"], inp["w"], inp["q_seq"], inp["q_pos"])
    torch.cuda.synchronize()
    assert int(st.item()) == 0, qsa.dev_status_names(int(st.item()))

    # every row: count = min(K, nb), strictly increasing in-range selection, finite outputs
    q_pos = inp["q_pos"].cpu().numpy().astype(np.int64)
    nb = (q_pos + 1) // 4
    cnt = dec.count.cpu().numpy()
    assert np.array_equal(cnt, np.minimum(wl.k_top, nb))
    sel = dec.sel.cpu().numpy()
    for r in range(wl.nq):
        s = sel[r, :cnt[r]]
        assert np.all(np.diff(s) > 0) and s[0] >= 0 and s[-1] < nb[r]
    assert torch.isfinite(dec.out.float()).all()

    rows = SAMPLES[name]
    if rows is None:
        L = np.array(wl.total_lengths)
        rows = sorted({int(L.argmin()), int(L.argmax()), 0, 40})
    errs = []
    for row in rows:
        r = R.expect_query(wl, row)
        assert np.array_equal(sel[row, :cnt[row]], r["sel"]), f"{name} row {row}: selection differs"
        out = dec.out[row].float().cpu().numpy()
        R.assert_close(out, r["o"], f"{name} out row {row}")
        R.assert_close(dec.lse[row].cpu().numpy(), r["lse"], f"{name} lse row {row}")
        errs.append(R.rel_l2(out, r["o"]))
    print(f"{name}: rows {rows} relative L2 max {max(errs):.2e}")
    assert max(errs) < 8e-3   # the pages' operator-test threshold
