"""Device-side set-up of a workload for the CUDA path (tests and benchmark).

Builds the paged cache group of a workload by generating its logical rows on
the device (``workloads.configs``) and appending them with ``qsa_append_kv``,
and prepares the inputs of one timed step: the new tokens each sequence
appends and the queries at their positions.
"""
from __future__ import annotations

import torch

import sparse_attention_decode_03_b200 as qsa

from . import configs as C


def new_cache(wl: C.Workload, device="cuda", block_table=None) -> qsa.PagedCache:
    bt = C.block_table(wl) if block_table is None else block_table
    return qsa.PagedCache(num_pages=wl.num_pages(), max_seqs=wl.batch, max_pages_per_seq=wl.pages_per_seq(),
                          num_kv_heads=wl.hkv, block_table=bt, device=device,
                          kv_dtype=qsa.KV_FP8_E4M3 if wl.kv_fp8 else qsa.KV_BF16)


def append_range(cache: qsa.PagedCache, wl: C.Workload, seq: int, start: int, stop: int, dev_status=None,
                 device="cuda"):
    pos = torch.arange(start, stop, dtype=torch.int64, device=device)
    k = C.k_rows(wl, seq, pos, device)
    v = C.v_rows(wl, seq, pos, device)
    ki = C.kidx_rows(wl, seq, pos, device)
    sid = torch.full((stop - start,), seq, dtype=torch.int32, device=device)
    qsa.qsa_append_kv(cache, k, v, ki, sid, pos.to(torch.int32), dev_status)


def build_cache(wl: C.Workload, device="cuda", chunk_tokens: int = 32768, dev_status=None) -> qsa.PagedCache:
    """The cache group holding every sequence's cached context (positions
    0 .. lengths[b]-1), written through qsa_append_kv in chunks."""
    cache = new_cache(wl, device)
    for b, L in enumerate(wl.lengths):
        for s in range(0, L, chunk_tokens):
            append_range(cache, wl, b, s, min(L, s + chunk_tokens), dev_status, device)
    return cache


def build_cache_from_host(wl: C.Workload, device="cuda", dev_status=None) -> qsa.PagedCache:
    """The same cache group as build_cache, for small workloads: every row is
    generated on the host and uploaded in one copy per tensor and sequence, so
    the device runs only the library's append kernels (no generator kernels)."""
    cache = new_cache(wl, device)
    for b, L in enumerate(wl.lengths):
        pos = torch.arange(0, L, dtype=torch.int64)
        up = lambda t: t.to(device, non_blocking=False)
        qsa.qsa_append_kv(cache, up(C.k_rows(wl, b, pos)), up(C.v_rows(wl, b, pos)), up(C.kidx_rows(wl, b, pos)),
                          up(torch.full((L,), b, dtype=torch.int32)), up(pos.to(torch.int32)), dev_status)
    return cache


def step_tokens(wl: C.Workload, device="cuda") -> dict:
    """The tokens one step appends: positions lengths[b] .. lengths[b]+new-1 of
    every sequence, sequence-major."""
    ks, vs, kis, sids, poss = [], [], [], [], []
    for b, L in enumerate(wl.lengths):
        pos = torch.arange(L, L + wl.new_tokens, dtype=torch.int64, device=device)
        ks.append(C.k_rows(wl, b, pos, device))
        vs.append(C.v_rows(wl, b, pos, device))
        kis.append(C.kidx_rows(wl, b, pos, device))
        sids.append(torch.full((wl.new_tokens,), b, dtype=torch.int32, device=device))
        poss.append(pos.to(torch.int32))
    return {"k_new": torch.cat(ks), "v_new": torch.cat(vs), "kidx_new": torch.cat(kis),
            "seq_id": torch.cat(sids), "pos": torch.cat(poss)}


def step_inputs(wl: C.Workload, device="cuda") -> dict:
    d = step_tokens(wl, device)
    d.update(C.queries(wl, device=device))
    return d


def chunk_units_for(wl: C.Workload):
    """KV chunk size for a workload: about `splits_per_query` chunks per query
    when the workload names one, else None (balance over the SMs)."""
    if wl.splits_per_query > 0:
        slots = wl.hkv * (wl.k_top + 1)
        return -(-slots // wl.splits_per_query)
    return None
