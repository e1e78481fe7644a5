"""qsa_sparse_attention_noalloc: sparse attention + combine for callers that
cannot allocate device memory.

Some callers cannot call cudaMalloc: a serving engine that gives nearly all
device memory to its KV-cache pool at start-up, a plug-in whose host program
owns every allocation, or a latency-critical loop that must not take
cudaMalloc's implicit device synchronisation.  For them libqsa keeps the split
partials in a fixed device array of its own, so the call takes only inputs and
outputs.

The GPU test runs the call twice in a row, with different split layouts and
scales, and checks each result against the two-call path with caller-owned
partial buffers (qsa_sparse_decode, then qsa_combine) on the same inputs.
The array is shared by every call and keeps the previous call's contents, so
the second call also checks that nothing from the first one leaks into it.
The file name puts it last in collection order.
"""
import ctypes

import numpy as np
import pytest
import torch

from tests import oracle_ref as R
from workloads import configs as C

qsa = pytest.importorskip("sparse_attention_decode_03_b200")


def _two_call_path(cache, inp, sel, count, k, scale, chunk, hq):
    nq = int(inp["q_seq"].shape[0])
    splits = qsa.splits_bound(k, chunk)
    part_o = torch.empty((nq, splits, hq, 256), dtype=torch.float32, device="cuda")
    part_lse = torch.empty((nq, splits, hq), dtype=torch.float32, device="cuda")
    out = torch.empty((nq, hq, 256), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((nq, hq), dtype=torch.float32, device="cuda")
    qsa.qsa_sparse_decode(cache, inp["q"], inp["q_seq"], inp["q_pos"], sel, count, k, scale, chunk, splits,
                          part_o, part_lse)
    qsa.qsa_combine(part_o, part_lse, out, lse)
    return out, lse


@pytest.mark.gpu
def test_noalloc_matches_two_call_path_on_two_calls_in_a_row():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from workloads import harness as H
    torch.cuda.set_device(0)
    wl = C.shrink(C.get("long"), [3001, 1998, 4098], k_top=128, name="noalloc")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    cache = H.build_cache(wl, dev_status=st)
    inp = H.step_inputs(wl)
    qsa.qsa_append_kv(cache, inp["k_new"], inp["v_new"], inp["kidx_new"], inp["seq_id"], inp["pos"], st)
    dec = qsa.Decoder(cache, wl.hq, wl.nq, k=wl.k_top, scale=wl.scale)
    dec.dev_status = st
    dec.run(inp["q"], inp["q_idx"], inp["w"], inp["q_seq"], inp["q_pos"])
    sel, count = dec.sel[:wl.nq], dec.count[:wl.nq]

    calls = [(dec.chunk_units, wl.scale), (37, 0.05)]
    outs = []
    for chunk, scale in calls:   # back to back on one stream, no host sync between them
        out = torch.full((wl.nq, wl.hq, 256), float("nan"), dtype=torch.bfloat16, device="cuda")
        lse = torch.full((wl.nq, wl.hq), float("nan"), dtype=torch.float32, device="cuda")
        qsa.qsa_sparse_attention_noalloc(cache, inp["q"], inp["q_seq"], inp["q_pos"], sel, count, wl.k_top, scale,
                                         chunk, out, lse, st)
        outs.append((out, lse))
    refs = [_two_call_path(cache, inp, sel, count, wl.k_top, scale, chunk, wl.hq) for chunk, scale in calls]
    torch.cuda.synchronize()
    assert int(st.item()) == 0, qsa.dev_status_names(int(st.item()))
    for i, ((out, lse), (ref_out, ref_lse)) in enumerate(zip(outs, refs)):
        R.assert_close(out.float().cpu().numpy(), ref_out.float().cpu().numpy(), f"call {i + 1}: out")
        R.assert_close(lse.cpu().numpy(), ref_lse.cpu().numpy(), f"call {i + 1}: lse")
    # the two calls differ (scale), so the second result is its own
    assert not torch.equal(outs[0][0], outs[1][0])
    # the first call agrees with the full decode step's own output too
    R.assert_close(outs[0][0].float().cpu().numpy(), dec.out[:wl.nq].float().cpu().numpy(), "call 1 vs Decoder")


def test_noalloc_rejects_calls_beyond_its_scratch_before_any_cuda_call():
    L = qsa.qsa.LIB
    fake = ctypes.c_void_p(0x1000)
    cache = qsa.qsa.qsa_cache_t(0x1000, 0x1000, 0x1000, 0x1000, 10, 2, 4, 2)
    cp = ctypes.byref(cache)

    def call(nq, hq, k, chunk, out=fake):
        return L.qsa_sparse_attention_noalloc(cp, fake, nq, hq, fake, fake, fake, fake, k, 0.0625, chunk, out, fake,
                                              None, None)
    splits = qsa.splits_bound(512, 16)
    fits = qsa.qsa.NOALLOC_SCRATCH_BYTES // (splits * 24 * 1028)
    assert call(fits + 1, 24, 512, 16) == -2        # QSA_ERR_UNSUPPORTED: partials exceed the array
    assert call(10 ** 6, 24, 512, 16) == -2
    assert call(4, 24, 512, 16, out=None) == -1     # no output buffer
    assert call(4, 24, 4096, 16) == -1              # k above QSA_MAX_TOPK
    assert call(0, 24, 512, 16) == 0                # nothing to do
    assert np.int64(fits) * splits * 24 * 1028 <= qsa.qsa.NOALLOC_SCRATCH_BYTES
