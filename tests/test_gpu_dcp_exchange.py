"""The DCP cross-rank exchange as the library runs it: two rank processes on
one GPU, each with its own replicated selector and K/V shard, run a whole step
through the C ABI -- append, scores, top-K, localisation, attention over the
shard, merge of the rank's splits -- then DCPRank.gather over a gloo process
group (staged through host memory; no kernel of one rank waits for another's)
and DCPRank.merge.  Every rank's selection equals the oracle's, every rank's
share equals the oracle's share of that rank, and the merged output on every
rank equals the oracle's unsharded result."""
import os
import socket

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, interleave, name, lengths, k):
    import datetime

    import torch.distributed as dist

    import sparse_attention_decode_03_b200 as qsa
    from oracle import qsa_oracle as O
    from tests import oracle_ref as R
    from workloads import configs as C
    from workloads import harness as H

    torch.cuda.set_device(0)
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=120))
    try:
        wl = C.shrink(C.get(name), lengths, k_top=k, page_perm=True)
        st = torch.zeros(1, dtype=torch.int32, device="cuda")
        sh = qsa.DCPShard(world, rank, interleave)
        pages = [-(-L // 64) for L in wl.total_lengths]
        selector = qsa.PagedCache(wl.num_pages(), wl.batch, wl.pages_per_seq(), wl.hkv,
                                  block_table=C.block_table(wl), with_kv=False)
        bt, used = sh.shard_block_table(pages)
        shard = qsa.PagedCache(max(1, used), wl.batch, bt.shape[1], wl.hkv, block_table=bt, with_kc=False)
        rk = qsa.DCPRank(selector, shard, wl.hq, wl.nq, world, rank, interleave, k=k, scale=wl.scale)
        rk.dev_status = st
        for b, L in enumerate(wl.lengths):   # this rank's copy of the cached context
            pos = torch.arange(0, L)
            up = lambda t: t.cuda()
            rk.append(up(C.k_rows(wl, b, pos)), up(C.v_rows(wl, b, pos)), up(C.kidx_rows(wl, b, pos)),
                      torch.full((L,), b, dtype=torch.int32, device="cuda"), up(pos.to(torch.int32)))
        inp = {n: t.cuda() for n, t in H.step_inputs(wl, device="cpu").items()}
        rk.append(inp["k_new"], inp["v_new"], inp["kidx_new"], inp["seq_id"], inp["pos"])
        rk.attend(inp["q"], inp["q_idx"], inp["w"], inp["q_seq"], inp["q_pos"])
        rk.gather(nq=wl.nq)
        out, lse = rk.merge(wl.nq)
        torch.cuda.synchronize()
        assert int(st.item()) == 0, qsa.dev_status_names(int(st.item()))
        for row in range(wl.nq):
            ref = R.expect_query(wl, row, k=k)
            assert np.array_equal(rk.sel[row, :int(rk.count[row])].cpu().numpy(), ref["sel"]), (rank, row)
            d = R.query_inputs(wl, row)
            o_r, l_r = O.dcp_rank_partial(d["q"], ref["sel"], d["p"], R.kv_reader(wl, d["seq"]), wl.scale, world,
                                          rank, interleave)
            R.assert_close(rk.o_rank[row].cpu().numpy(), o_r, f"rank {rank} share row {row}")
            R.assert_close(rk.lse_rank[row].cpu().numpy(), l_r, f"rank {rank} lse row {row}")
            R.assert_close(out[row].float().cpu().numpy(), ref["o"], f"rank {rank} merged out row {row}")
            R.assert_close(lse[row].cpu().numpy(), ref["lse"], f"rank {rank} merged lse row {row}")
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("interleave,name,lengths,k", [
    (1, "long", [3000, 1701], 64),
    (2, "quarter", [2600, 900, 130], 32),
])
def test_two_rank_processes_exchange_through_the_library(interleave, name, lengths, k):
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import torch.multiprocessing as mp
    mp.start_processes(_rank_main, args=(2, _free_port(), interleave, name, lengths, k), nprocs=2, join=True,
                       start_method="spawn")
