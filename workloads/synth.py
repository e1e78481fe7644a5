"""Seeded, counter-based synthetic inputs for the QSA decode path.

This module is the one piece shared by the CUDA path's tests/benchmark and the
CPU oracle's callers.  It holds none of the method's arithmetic: it only
produces input tensors (keys, values, queries, indexer keys/queries, indexer
weights, sequence lengths, page tables) from a seed.

Every value is a pure function of (seed, tensor tag, sequence, position,
element), computed with integer arithmetic only, so the same call returns
bit-identical tensors on the CPU and on a CUDA device.  That lets the GPU side
build a multi-GB cache on the device while the oracle regenerates, on the host,
exactly the rows it needs.

Hash: the 32-bit PCG-RXS-M-XS output permutation used as a stateless hash
("pcg_hash" in Jarzynski & Olano, "Hash Functions for GPU Rendering", JCGT 9(3),
2020).  It is evaluated on int64 tensors holding values in [0, 2^32); every
product stays below 2^63, so there is no signed overflow anywhere.

Value recipes (the workload shapes come from the pages' decode / prefill
scenarios; see ``workloads.configs``):
  * main K, V, query Q: approximately N(0, 1) -- the sum of twelve 16-bit
    uniforms minus its mean, divided by 2^16 (variance exactly 1) -- rounded to
    BF16 (round-to-nearest-even, torch's conversion).
  * indexer keys k_idx and indexer queries q_idx: integers uniform in [-8, 8],
    stored exactly in BF16.
  * indexer weights w: uniform over {0.5, 1, 2}, fp32.
"""
from __future__ import annotations

import torch

MASK32 = 0xFFFFFFFF

# tensor tags (arbitrary distinct 32-bit constants)
TAG_K = 0x4B4B4B01
TAG_V = 0x56565602
TAG_KIDX = 0x4B494403
TAG_Q = 0x51515104
TAG_QIDX = 0x51494405
TAG_W = 0x57575706
TAG_SPIKE = 0x53504B07
TAG_SPIKE_DIR = 0x53444908
TAG_SPIKE_SIGN = 0x53534909
TAG_LEN = 0x4C454E0A
TAG_PERM = 0x5045520B


def pcg_hash(x: torch.Tensor) -> torch.Tensor:
    """PCG-RXS-M-XS 32-bit hash of an int64 tensor holding values in [0, 2^32)."""
    state = (x * 747796405 + 2891336453) & MASK32
    shift = (state >> 28) + 4
    word = ((torch.bitwise_right_shift(state, shift) ^ state) * 277803737) & MASK32
    return (word >> 22) ^ word


def pcg_hash_int(x: int) -> int:
    """Scalar version of :func:`pcg_hash` for host-side key derivation."""
    state = (x * 747796405 + 2891336453) & MASK32
    word = (((state >> ((state >> 28) + 4)) ^ state) * 277803737) & MASK32
    return ((word >> 22) ^ word) & MASK32


def stream_key(seed: int, tag: int) -> int:
    return pcg_hash_int(pcg_hash_int(seed & MASK32) ^ (tag & MASK32))


def row_keys(seed: int, tag: int, seq, pos: torch.Tensor) -> torch.Tensor:
    """One 32-bit key per (sequence, position) row.  ``seq`` is an int or a
    tensor broadcastable against ``pos``."""
    base = stream_key(seed, tag)
    pos = pos.to(torch.int64)
    if isinstance(seq, torch.Tensor):
        s = seq.to(device=pos.device, dtype=torch.int64)
    else:
        s = torch.full_like(pos, int(seq))
    h = pcg_hash(s ^ base)
    return pcg_hash(h ^ pos)


def _element_hash(keys: torch.Tensor, width: int, k: int) -> torch.Tensor:
    e = torch.arange(width, device=keys.device, dtype=torch.int64)
    return pcg_hash(keys[:, None] ^ ((e[None, :] << 4) | k))


def normal_f32(keys: torch.Tensor, width: int, max_elems: int = 1 << 24) -> torch.Tensor:
    """[n, width] fp32, approximately N(0,1), exactly representable in fp32."""
    n = keys.shape[0]
    out = torch.empty((n, width), dtype=torch.float32, device=keys.device)
    rows = max(1, max_elems // max(width, 1))
    for r0 in range(0, n, rows):
        kk = keys[r0:r0 + rows]
        acc = torch.zeros((kk.shape[0], width), dtype=torch.int64, device=keys.device)
        for k in range(6):
            u = _element_hash(kk, width, k)
            acc += (u & 0xFFFF) + (u >> 16)
        acc -= 393210  # 12 * (65536 - 1) / 2
        out[r0:r0 + rows] = acc.to(torch.float32) * (1.0 / 65536.0)
    return out


def int_uniform(keys: torch.Tensor, width: int, lo: int, hi: int, salt: int = 0) -> torch.Tensor:
    """[n, width] int64 uniform in [lo, hi]."""
    span = hi - lo + 1
    u = _element_hash(keys, width, 8 + salt)
    return ((u * span) >> 32) + lo


def uniform_u32(keys: torch.Tensor, salt: int = 0) -> torch.Tensor:
    return pcg_hash(keys ^ (0x9E3779B9 ^ salt))


def _positions(positions, device) -> torch.Tensor:
    if isinstance(positions, torch.Tensor):
        return positions.to(device=device, dtype=torch.int64)
    return torch.as_tensor(positions, dtype=torch.int64, device=device)


def spike_mask(seed: int, seq: int, positions: torch.Tensor, percent: int) -> torch.Tensor:
    keys = row_keys(seed, TAG_SPIKE, seq, positions)
    return ((uniform_u32(keys) * 100) >> 32) < percent


def spike_direction(seed: int, seq: int, kv_head: int) -> torch.Tensor:
    """Unit vector u_g (fp64, CPU) for one (sequence, KV head)."""
    keys = row_keys(seed, TAG_SPIKE_DIR, seq, torch.tensor([kv_head]))
    v = normal_f32(keys, 256)[0].to(torch.float64)
    return v / torch.linalg.vector_norm(v)


def spike_sign(seed: int, seq: int) -> torch.Tensor:
    """Random +-1 vector s (int64, CPU) of length 128 for one sequence."""
    keys = row_keys(seed, TAG_SPIKE_SIGN, seq, torch.tensor([0]))
    return int_uniform(keys, 128, 0, 1)[0] * 2 - 1


def sequence_lengths(seed: int, batch: int, lo: int, hi: int) -> list[int]:
    keys = row_keys(seed, TAG_LEN, 0, torch.arange(batch))
    span = hi - lo + 1
    return [int(x) for x in (((uniform_u32(keys) * span) >> 32) + lo)]


def page_permutation(seed: int, num_pages: int) -> torch.Tensor:
    """A seeded random permutation of physical page ids (CPU, int32)."""
    g = torch.Generator().manual_seed(stream_key(seed, TAG_PERM))
    return torch.randperm(num_pages, generator=g).to(torch.int32)
