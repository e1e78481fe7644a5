"""DCP host logic on the CPU: the shard rule of the binding against the
oracle's, shard block tables, and the cross-rank exchange with two gloo ranks
(each rank computes its share with the oracle, the shares are all-gathered
rank-major -- by torch.distributed and by the library's DCPRank.gather -- and
merged by log-sum-exp, which must give the unsharded result)."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from oracle import qsa_oracle as O


def _shard_cls():
    from sparse_attention_decode_03_b200.dcp import DCPShard
    return DCPShard


@pytest.mark.parametrize("nranks,interleave", [(1, 1), (2, 1), (3, 1), (2, 2), (4, 3)])
def test_shard_rule_matches_the_oracle_and_numbers_local_pages_in_order(nranks, interleave):
    DCPShard = _shard_cls()
    pages = 41
    seen = {}
    for rank in range(nranks):
        sh = DCPShard(nranks, rank, interleave)
        mine = [P for P in range(pages) if sh.owner(P) == rank]
        assert all(O.dcp_owner(P * 64, nranks, interleave) == rank for P in mine)
        # local pages are 0, 1, 2, ... in context order
        assert [sh.local_page(P) for P in mine] == list(range(len(mine)))
        for n in range(pages + 1):
            assert sh.local_pages(n) == sum(1 for P in mine if P < n)
        for P in mine:
            seen[P] = rank
    assert sorted(seen) == list(range(pages))   # every page on exactly one rank


def test_shard_block_table():
    DCPShard = _shard_cls()
    sh = DCPShard(2, 1, 1)
    bt, used = sh.shard_block_table([5, 1, 4], first_page=3)
    assert used == 2 + 0 + 2
    assert bt.tolist() == [[3, 4], [-1, -1], [5, 6]]


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _toy(L, hq, hkv, seed):
    r = np.random.default_rng(seed)
    K = r.standard_normal((L, hkv, 256))
    V = r.standard_normal((L, hkv, 256))
    kidx = r.integers(-8, 9, size=(L, 128)).astype(np.float32)
    q = r.standard_normal((hq, 256))
    qi = r.integers(-8, 9, size=(8, 128)).astype(np.float64)
    w = r.choice([0.5, 1.0, 2.0], size=8)
    return K, V, kidx, q, qi, w


def _rank_main(rank, world, port, interleave):
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world)
    try:
        hq, hkv, k = 12, 2, 16
        L = 64 * 6 + 7
        K, V, kidx, q, qi, w = _toy(L, hq, hkv, seed=3)   # the same replicated inputs on every rank
        rows = lambda pos: (K[pos], V[pos])
        queries = [L - 1, 64 * 4 + 2, 65, 3]
        mine_o, mine_l, refs = [], [], []
        for p in queries:
            r = O.decode_query(q, qi, w, p, kidx, rows, k=k, scale=1 / 16)   # every rank selects the same blocks
            o, lse = O.dcp_rank_partial(q, r["sel"], p, rows, 1 / 16, world, rank, interleave)
            mine_o.append(o)
            mine_l.append(lse)
            refs.append(r)
        o_r = torch.from_numpy(np.stack(mine_o))     # [nq][Hq][256]
        l_r = torch.from_numpy(np.stack(mine_l))     # [nq][Hq]
        o_all = [torch.empty_like(o_r) for _ in range(world)]
        l_all = [torch.empty_like(l_r) for _ in range(world)]
        dist.all_gather(o_all, o_r)
        dist.all_gather(l_all, l_r)
        o_all = torch.stack(o_all).numpy()           # rank-major [R][nq][Hq][256]
        l_all = torch.stack(l_all).numpy()
        # the library's exchange (DCPRank.gather, gloo: staged through host memory) on the same shares
        from types import SimpleNamespace
        from sparse_attention_decode_03_b200.dcp import DCPRank, DCPShard
        nq, max_nq = len(queries), len(queries) + 2
        fake = SimpleNamespace(sh=DCPShard(world, rank, interleave), max_nq=max_nq,
                               o_rank=torch.zeros((max_nq,) + tuple(o_r.shape[1:]), dtype=o_r.dtype),
                               lse_rank=torch.zeros((max_nq,) + tuple(l_r.shape[1:]), dtype=l_r.dtype),
                               o_all=torch.full((world, max_nq) + tuple(o_r.shape[1:]), 7.0, dtype=o_r.dtype),
                               lse_all=torch.full((world, max_nq) + tuple(l_r.shape[1:]), 7.0, dtype=l_r.dtype))
        fake.o_rank[:nq] = o_r
        fake.lse_rank[:nq] = l_r
        DCPRank.gather(fake, nq=nq)
        assert np.array_equal(fake.o_all[:, :nq].numpy(), o_all) and np.array_equal(fake.lse_all[:, :nq].numpy(), l_all)
        assert torch.all(fake.o_all[:, nq:] == 7.0)    # rows past nq are not touched
        for i, r in enumerate(refs):
            o, lse = O.combine(o_all[:, i], l_all[:, i])
            assert np.allclose(o, r["o"], rtol=1e-12, atol=1e-12), (rank, i)
            assert np.allclose(lse, r["lse"], rtol=1e-12), (rank, i)
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("interleave", [1, 2])
def test_two_gloo_ranks_exchange_and_merge(interleave):
    mp.start_processes(_rank_main, args=(2, _free_port(), interleave), nprocs=2, join=True, start_method="spawn")
