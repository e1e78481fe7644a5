"""The five QSA workloads and their logical (unpaged) input tensors.

Shapes follow the decode and prefill scenarios on the pages (contexts up to a
quarter-million tokens, a 512-block budget, head dim 256, GQA head pairs
(16,2) (24,2) (12,1) (6,1)).  Every tensor is produced from ``workloads.synth``
counters, so any row can be regenerated on any device.

Logical layouts (no paging):
  K, V      [n_pos][Hkv][256]  bf16  rows of one sequence
  k_idx     [n_pos][128]       bf16  integer-valued
  q         [nq][Hq][256]      bf16
  q_idx     [nq][8][128]       bf16  integer-valued
  w         [nq][8]            fp32  in {0.5, 1, 2}
  q_seq     [nq]               int32 sequence of each query
  q_pos     [nq]               int32 absolute position of each query
"""
from __future__ import annotations

import dataclasses
import math
from functools import lru_cache

import torch

from . import synth

HEAD_DIM = 256
IDX_HEADS = 8
IDX_DIM = 128
RATIO = 4
PAGE = 64


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    batch: int
    hq: int
    hkv: int
    lengths: tuple            # cached context per sequence BEFORE the timed step's tokens
    new_tokens: int = 1       # tokens appended (and queried) per sequence by one step
    k_top: int = 512
    scale: float = 1.0 / 16.0
    page_perm: bool = False
    spikes: bool = False
    seed: int = 0
    splits_per_query: int = 0  # 0 = balance over the SMs; >0 = about this many KV chunks per query
    kv_fp8: bool = False       # main K/V cache stored as FP8 e4m3 (the side cache stays BF16)

    @property
    def total_lengths(self) -> list[int]:
        return [L + self.new_tokens for L in self.lengths]

    @property
    def nq(self) -> int:
        return self.batch * self.new_tokens

    def pages_per_seq(self) -> int:
        return math.ceil(max(self.total_lengths) / PAGE)

    def num_pages(self) -> int:
        return sum(math.ceil(L / PAGE) for L in self.total_lengths)

    def describe(self) -> dict:
        return {"workload": self.name, "batch": self.batch, "hq": self.hq, "hkv": self.hkv,
                "context": (self.total_lengths[0] if len(set(self.total_lengths)) == 1
                            else [min(self.total_lengths), max(self.total_lengths)]),
                "new_tokens_per_seq": self.new_tokens, "top_k_blocks": self.k_top,
                "head_dim": HEAD_DIM, "indexer": f"{IDX_HEADS}x{IDX_DIM}", "page_tokens": PAGE,
                "page_permutation": self.page_perm, "kv_cache": "fp8_e4m3" if self.kv_fp8 else "bf16"}


def _decode(name, batch, ctx, hq, hkv, **kw):
    lengths = tuple(c - 1 for c in ctx)   # the step appends the current token
    return Workload(name=name, batch=batch, hq=hq, hkv=hkv, lengths=lengths, new_tokens=1, **kw)


@lru_cache(maxsize=None)
def get(name: str) -> Workload:
    if name == "tiny":
        return _decode("decode-b1-ctx4096-h16x2", 1, [4096], 16, 2)
    if name == "batched":
        return _decode("decode-b8-ctx32768-h16x2-paged", 8, [32768] * 8, 16, 2,
                       page_perm=True, splits_per_query=8)
    if name == "long":
        return _decode("decode-b32-ctx131072-h24x2-spiked", 32, [131072] * 32, 24, 2, spikes=True)
    if name == "quarter":
        lens = synth.sequence_lengths(0, 64, 16384, 262144)
        return _decode("decode-b64-ctx16k-262k-h12x1-paged", 64, lens, 12, 1, page_perm=True)
    if name == "long-fp8":
        return dataclasses.replace(get("long"), name="decode-b32-ctx131072-h24x2-spiked-fp8kv", kv_fp8=True)
    if name == "quarter-fp8":
        return dataclasses.replace(get("quarter"), name="decode-b64-ctx16k-262k-h12x1-paged-fp8kv", kv_fp8=True)
    if name == "prefill":
        return Workload(name="extend-b2-ctx65536+4096-h6x1", batch=2, hq=6, hkv=1,
                        lengths=(65536, 65536), new_tokens=4096)
    raise KeyError(name)


ALL = ("tiny", "batched", "long", "quarter", "prefill")
FP8 = ("long-fp8", "quarter-fp8")   # the same decode workloads with an FP8 e4m3 main K/V cache


def shrink(wl: Workload, lengths, new_tokens=None, k_top=None, name=None, **kw) -> Workload:
    """A smaller workload with the same head geometry and value recipe."""
    return dataclasses.replace(
        wl, name=name or (wl.name + "-small"), batch=len(lengths), lengths=tuple(lengths),
        new_tokens=new_tokens if new_tokens is not None else wl.new_tokens,
        k_top=k_top if k_top is not None else wl.k_top, **kw)


# ----------------------------------------------------------------------------
# logical tensors


def _spike_pos(wl: Workload, seq: int, pos: torch.Tensor) -> torch.Tensor:
    return synth.spike_mask(wl.seed, seq, pos, 5)


@lru_cache(maxsize=256)
def _spike_shift_k(wl: Workload, seq: int) -> torch.Tensor:
    # fp32(3 * u_g) per KV head, computed once on the host: [Hkv][256]
    return torch.stack([(3.0 * synth.spike_direction(wl.seed, seq, g)).to(torch.float32)
                        for g in range(wl.hkv)])


@lru_cache(maxsize=256)
def _spike_shift_q(wl: Workload, seq: int) -> torch.Tensor:
    return torch.stack([synth.spike_direction(wl.seed, seq, g).to(torch.float32)
                        for g in range(wl.hkv)])


def _kv_rows(wl: Workload, tag: int, seq: int, positions, device) -> torch.Tensor:
    pos = synth._positions(positions, device)
    keys = synth.row_keys(wl.seed, tag, seq, pos)
    z = synth.normal_f32(keys, wl.hkv * HEAD_DIM).view(-1, wl.hkv, HEAD_DIM)
    if wl.spikes and tag == synth.TAG_K:
        m = _spike_pos(wl, seq, pos)
        shift = _spike_shift_k(wl, seq).to(device)
        z = torch.where(m[:, None, None], z + shift[None], z)
    return z.to(torch.bfloat16)


def k_rows(wl: Workload, seq: int, positions, device="cpu") -> torch.Tensor:
    """Main keys K[seq][positions] -> [n][Hkv][256] bf16 (post-RoPE values)."""
    return _kv_rows(wl, synth.TAG_K, seq, positions, device)


def v_rows(wl: Workload, seq: int, positions, device="cpu") -> torch.Tensor:
    return _kv_rows(wl, synth.TAG_V, seq, positions, device)


def kidx_rows(wl: Workload, seq: int, positions, device="cpu") -> torch.Tensor:
    """Indexer keys k_idx[seq][positions] -> [n][128] bf16, integers in [-8, 8]."""
    pos = synth._positions(positions, device)
    keys = synth.row_keys(wl.seed, synth.TAG_KIDX, seq, pos)
    v = synth.int_uniform(keys, IDX_DIM, -8, 8)
    if wl.spikes:
        m = _spike_pos(wl, seq, pos)
        s = synth.spike_sign(wl.seed, seq).to(device)
        v = torch.where(m[:, None], torch.clamp(v + 4 * s[None], -8, 8), v)
    return v.to(torch.bfloat16)


def query_positions(wl: Workload) -> tuple[torch.Tensor, torch.Tensor]:
    """(q_seq, q_pos), both int32 [nq]: each sequence's new tokens, in order."""
    seqs, poss = [], []
    for b, L in enumerate(wl.lengths):
        seqs.append(torch.full((wl.new_tokens,), b, dtype=torch.int32))
        poss.append(torch.arange(L, L + wl.new_tokens, dtype=torch.int32))
    return torch.cat(seqs), torch.cat(poss)


def queries(wl: Workload, rows=None, device="cpu") -> dict:
    """Query-side tensors for the query rows ``rows`` (default: all nq)."""
    q_seq, q_pos = query_positions(wl)
    if rows is not None:
        rows = torch.as_tensor(rows, dtype=torch.int64)
        q_seq, q_pos = q_seq[rows], q_pos[rows]
    q_seq_d = q_seq.to(device)
    q_pos_d = q_pos.to(device)
    kq = synth.row_keys(wl.seed, synth.TAG_Q, q_seq_d, q_pos_d)
    q = synth.normal_f32(kq, wl.hq * HEAD_DIM).view(-1, wl.hq, HEAD_DIM)
    ki = synth.row_keys(wl.seed, synth.TAG_QIDX, q_seq_d, q_pos_d)
    qi = synth.int_uniform(ki, IDX_HEADS * IDX_DIM, -8, 8).view(-1, IDX_HEADS, IDX_DIM)
    kw = synth.row_keys(wl.seed, synth.TAG_W, q_seq_d, q_pos_d)
    wi = synth.int_uniform(kw, IDX_HEADS, 0, 2)
    w = torch.tensor([0.5, 1.0, 2.0], device=device)[wi]
    if wl.spikes:
        g_of_h = torch.arange(wl.hq, device=device) // (wl.hq // wl.hkv)
        for b in sorted(set(int(x) for x in q_seq)):
            sel = (q_seq_d == b)
            shift = _spike_shift_q(wl, b).to(device)[g_of_h]          # [Hq][256]
            q[sel] = q[sel] + shift[None]
            s = synth.spike_sign(wl.seed, b).to(device)
            qi[sel] = torch.clamp(qi[sel] + 2 * s[None, None], -8, 8)
    return {"q": q.to(torch.bfloat16), "q_idx": qi.to(torch.bfloat16), "w": w.to(torch.float32),
            "q_seq": q_seq_d.to(torch.int32), "q_pos": q_pos_d.to(torch.int32)}


def block_table(wl: Workload) -> torch.Tensor:
    """[B][pages_per_seq] int32 logical->physical page map (identity order or a
    seeded random permutation); unused entries are -1."""
    pps = wl.pages_per_seq()
    n = wl.num_pages()
    phys = synth.page_permutation(wl.seed, n) if wl.page_perm else torch.arange(n, dtype=torch.int32)
    bt = torch.full((wl.batch, pps), -1, dtype=torch.int32)
    o = 0
    for b, L in enumerate(wl.total_lengths):
        c = math.ceil(L / PAGE)
        bt[b, :c] = phys[o:o + c]
        o += c
    return bt
