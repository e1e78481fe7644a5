"""Decode context parallelism (DCP) for QSA decode.

[DCP] "Qwen 4 QSA krijgt decode-contextparallellisme ...", section "Wat de pull
request daadwerkelijk verandert": the main K/V is sharded by context over the
ranks, each rank reads its own slice, the selector (indexer side cache and
top-K) stays together with the main KV in one cache group and is replicated,
the split attention results are combined across ranks, and a localisation
step maps the globally selected blocks to each rank's slots.

One rank per GPU holds
  * a selector group (side cache only, every page of every sequence),
    identical on every rank, so every rank computes the same selection;
  * its K/V shard (main K/V only): logical page P of a sequence lives on rank
    (P // I) % N at local page (P // (I N)) * I + P % I (I = interleave_pages).
A step is: append (side cache: every token; shard: the rank's tokens at local
positions) -> scores -> top-K -> localise -> sparse attention on the shard ->
merge of the rank's own splits (fp32) -> all-gather of every rank's
(o, lse) -> log-sum-exp merge over the ranks.  Every step runs in libqsa's
kernels; torch.distributed only moves the per-query results between ranks.
"""
from __future__ import annotations

import torch

from . import qsa as _q


class DCPShard:
    """The shard rule on the host (the kernels apply the same one)."""

    def __init__(self, nranks: int, rank: int, interleave_pages: int = 1):
        if nranks < 1 or not 0 <= rank < nranks or interleave_pages < 1:
            raise ValueError("need nranks >= 1, 0 <= rank < nranks, interleave_pages >= 1")
        self.n, self.r, self.I = int(nranks), int(rank), int(interleave_pages)

    def owner(self, page: int) -> int:
        return (page // self.I) % self.n

    def local_page(self, page: int) -> int:
        return (page // (self.I * self.n)) * self.I + page % self.I

    def local_pages(self, n_pages: int) -> int:
        """Pages among the first n_pages of a sequence that this rank holds."""
        cyc = self.I * self.n
        return (n_pages // cyc) * self.I + max(0, min(n_pages % cyc, (self.r + 1) * self.I) - self.r * self.I)

    def shard_block_table(self, pages_per_seq: list[int], max_local_pages: int | None = None,
                          first_page: int = 0) -> tuple[torch.Tensor, int]:
        """A block table for this rank's shard: each sequence's local pages get
        consecutive physical pages.  Returns (table [B][max_local_pages], pages used)."""
        loc = [self.local_pages(n) for n in pages_per_seq]
        width = max_local_pages or max(1, max(loc))
        bt = torch.full((len(loc), width), -1, dtype=torch.int32)
        nxt = first_page
        for b, m in enumerate(loc):
            bt[b, :m] = torch.arange(nxt, nxt + m, dtype=torch.int32)
            nxt += m
        return bt, nxt - first_page


class DCPRank:
    """One rank's buffers and calls for a DCP decode step over up to max_nq queries."""

    def __init__(self, selector: _q.PagedCache, shard: _q.PagedCache, hq: int, max_nq: int, nranks: int,
                 rank: int, interleave_pages: int = 1, k: int = 512, scale: float = 1.0 / 16.0,
                 target_ctas: int | None = None, chunk_units: int | None = None):
        if selector.kc_pages is None or shard.kv_pages is None:
            raise ValueError("the selector group needs a side cache and the shard group main K/V")
        dev = selector.device
        self.sh = DCPShard(nranks, rank, interleave_pages)
        self.selector, self.shard = selector, shard
        self.hq, self.k, self.scale, self.max_nq = hq, k, scale, max_nq
        if target_ctas is None:
            target_ctas = torch.cuda.get_device_properties(dev).multi_processor_count
        if chunk_units is None:
            chunk_units, self.max_splits = _q.qsa_decode_plan(max_nq, shard.num_kv_heads, k, target_ctas)
        else:
            self.max_splits = _q.splits_bound(k, chunk_units)
        self.chunk_units = chunk_units
        self.scores_ld = selector.max_pages_per_seq * _q.BLOCKS_PER_PAGE
        i32 = dict(dtype=torch.int32, device=dev)
        f32 = dict(dtype=torch.float32, device=dev)
        self.scores = torch.empty((max_nq, self.scores_ld), **f32)
        self.sel = torch.empty((max_nq, k), **i32)
        self.count = torch.empty((max_nq,), **i32)
        self.sel_local = torch.empty((max_nq, k), **i32)
        self.count_local = torch.empty((max_nq,), **i32)
        self.q_pos_local = torch.empty((max_nq,), **i32)
        self.part_o = torch.empty((max_nq, self.max_splits, hq, _q.HEAD_DIM), **f32)
        self.part_lse = torch.empty((max_nq, self.max_splits, hq), **f32)
        self.o_rank = torch.empty((max_nq, hq, _q.HEAD_DIM), **f32)     # this rank's merged result
        self.lse_rank = torch.empty((max_nq, hq), **f32)
        self.o_all = torch.empty((nranks, max_nq, hq, _q.HEAD_DIM), **f32)  # every rank's, rank-major
        self.lse_all = torch.empty((nranks, max_nq, hq), **f32)
        self.out = torch.empty((max_nq, hq, _q.HEAD_DIM), dtype=torch.bfloat16, device=dev)
        self.lse = torch.empty((max_nq, hq), **f32)
        self.dev_status = torch.zeros((1,), **i32)
        self._tok = None

    # -- the step, in order

    def append(self, k_new, v_new, kidx_new, seq_id, pos, stream=None):
        """Side cache: every token; K/V shard: this rank's tokens at local positions."""
        n = int(seq_id.shape[0])
        if self._tok is None or self._tok[0].shape[0] < n:
            self._tok = (torch.empty(n, dtype=torch.int32, device=seq_id.device),
                         torch.empty(n, dtype=torch.int32, device=seq_id.device))
        seq_l, pos_l = self._tok[0][:n], self._tok[1][:n]
        _q.qsa_append_kv(self.selector, k_new, v_new, kidx_new, seq_id, pos, self.dev_status, stream)
        _q.qsa_dcp_localize_tokens(seq_id, pos, self.sh.n, self.sh.r, self.sh.I, seq_l, pos_l, stream)
        _q.qsa_append_kv(self.shard, k_new, v_new, kidx_new, seq_l, pos_l, self.dev_status, stream)

    def attend(self, q, q_idx, w, q_seq, q_pos, stream=None):
        """Selection (replicated), localisation, attention over this rank's blocks,
        merge of its splits: (o_rank [nq][hq][256] fp32, lse_rank [nq][hq])."""
        nq = int(q_seq.shape[0])
        assert nq <= self.max_nq
        sc, se, cn = self.scores[:nq], self.sel[:nq], self.count[:nq]
        sl, cl, pl = self.sel_local[:nq], self.count_local[:nq], self.q_pos_local[:nq]
        po, plse = self.part_o[:nq], self.part_lse[:nq]
        _q.qsa_index_scores(self.selector, q_idx, w, q_seq, q_pos, sc, self.dev_status, stream)
        _q.qsa_topk_blocks(sc, q_pos, self.k, se, cn, self.dev_status, stream)
        _q.qsa_dcp_localize_selection(se, cn, q_pos, self.k, self.sh.n, self.sh.r, self.sh.I, sl, cl, pl,
                                      self.dev_status, stream)
        _q.qsa_sparse_decode(self.shard, q, q_seq, pl, sl, cl, self.k, self.scale, self.chunk_units,
                             self.max_splits, po, plse, self.dev_status, stream)
        _q.qsa_combine_f32(po, plse, self.o_rank[:nq], self.lse_rank[:nq], stream)
        return self.o_rank[:nq], self.lse_rank[:nq]

    def gather(self, group=None, nq: int | None = None):
        """All-gather every rank's (o, lse) into o_all / lse_all, rank-major.

        On an NCCL group the whole max_nq-row device buffers go through one
        all_gather_into_tensor each.  On a gloo group (host transport, e.g. ranks
        sharing one GPU or a CPU-only test) the rank's first nq rows (default
        max_nq) are copied to the host, all-gathered there and copied back into
        o_all / lse_all; the device-to-host copy waits for the attention of the
        current stream."""
        import torch.distributed as dist
        if dist.get_backend(group) != "gloo":
            dist.all_gather_into_tensor(self.o_all, self.o_rank, group=group)
            dist.all_gather_into_tensor(self.lse_all, self.lse_rank, group=group)
            return
        n = self.max_nq if nq is None else int(nq)
        o, lse = self.o_rank[:n].cpu(), self.lse_rank[:n].cpu()
        o_parts = [torch.empty_like(o) for _ in range(self.sh.n)]
        l_parts = [torch.empty_like(lse) for _ in range(self.sh.n)]
        dist.all_gather(o_parts, o, group=group)
        dist.all_gather(l_parts, lse, group=group)
        for j in range(self.sh.n):
            self.o_all[j, :n].copy_(o_parts[j], non_blocking=False)
            self.lse_all[j, :n].copy_(l_parts[j], non_blocking=False)

    def merge(self, nq: int, stream=None):
        """Log-sum-exp merge over the ranks: (out bf16 [nq][hq][256], lse [nq][hq])."""
        H, D = self.hq, _q.HEAD_DIM
        _q._check("qsa_combine_strided", _q.LIB.qsa_combine_strided(
            _q._ptr(self.o_all), _q._ptr(self.lse_all), nq, self.sh.n, H, H * D, self.max_nq * H * D, H,
            self.max_nq * H, _q._ptr(self.out), _q.OUT_BF16, _q._ptr(self.lse), _q._stream(stream)))
        return self.out[:nq], self.lse[:nq]
