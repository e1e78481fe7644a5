"""qsa.StepPipeline (two slots of staged inputs, Decoder buffers and step
graphs; uploads, steps and downloads on three streams ordered by events):
after a burst of steps enqueued without any host synchronisation, each slot's
host outputs equal a plain Decoder.run on that slot's inputs, bit for bit."""
import pytest
import torch

from workloads import configs as C

pytestmark = pytest.mark.gpu

qsa = pytest.importorskip("sparse_attention_decode_03_b200")
H = pytest.importorskip("workloads.harness")


@pytest.fixture(autouse=True, scope="module")
def _need_cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")


@pytest.mark.parametrize("name,lengths", [("long", [9000, 4100, 777]), ("quarter", [16000, 2000, 50, 6000])])
def test_pipeline_slots_match_plain_steps(name, lengths):
    wl = C.shrink(C.get(name), lengths, page_perm=True)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    cache = H.build_cache(wl, dev_status=st)
    saved = cache.kc_partial.clone()
    base = H.step_inputs(wl, device="cpu")
    stream = torch.cuda.Stream()
    ios, decs, calls = [], [], []
    for slot in range(2):
        io = qsa.StepIO(wl.batch * wl.new_tokens, wl.nq, wl.hq, wl.hkv, "cuda")
        for k, t in base.items():
            io.host[k].copy_(t)
        io.host["q"].mul_(1.0 + 0.5 * slot)  # the two slots attend with different queries
        d = qsa.Decoder(cache, wl.hq, wl.nq, k=wl.k_top, scale=wl.scale)
        d.dev_status = st
        v = io.dev
        calls.append([qsa.bind_append_kv(cache, v["k_new"], v["v_new"], v["kidx_new"], v["seq_id"], v["pos"], st,
                                         stream=stream)]
                     + d.bind(v["q"], v["q_idx"], v["w"], v["q_seq"], v["q_pos"], stream=stream))
        ios.append(io)
        decs.append(d)

    def restore(cs):
        with torch.cuda.stream(cs):
            cache.kc_partial.copy_(saved)

    pipe = qsa.StepPipeline(ios, decs, calls, stream, before=restore)
    n = 7
    for i in range(n):
        pipe.step(i)
    got = {}
    for i in (n - 2, n - 1):
        out, lse = pipe.wait_outputs(i)
        got[i % 2] = (out[:wl.nq].clone(), lse[:wl.nq].clone())
    torch.cuda.synchronize()
    assert int(st.item()) == 0, qsa.dev_status_names(int(st.item()))
    for slot in range(2):
        cache.kc_partial.copy_(saved)
        ref = qsa.Decoder(cache, wl.hq, wl.nq, k=wl.k_top, scale=wl.scale)
        ref.dev_status = st
        v = {k: t.to("cuda") for k, t in base.items()}
        v["q"] = v["q"] * (1.0 + 0.5 * slot)
        qsa.qsa_append_kv(cache, v["k_new"], v["v_new"], v["kidx_new"], v["seq_id"], v["pos"], st)
        ref.run(v["q"], v["q_idx"], v["w"], v["q_seq"], v["q_pos"])
        torch.cuda.synchronize()
        assert torch.equal(got[slot][0].view(torch.int16), ref.out[:wl.nq].cpu().view(torch.int16)), f"slot {slot}"
        assert torch.equal(got[slot][1].view(torch.int32), ref.lse[:wl.nq].cpu().view(torch.int32)), f"slot {slot}"
