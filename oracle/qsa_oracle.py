"""CPU oracle for Qwen Sparse Attention (QSA) decode -- TEST INFRASTRUCTURE ONLY.

Plain, slow, obviously-correct numpy code in fp64 (fp32 only where the CUDA path
makes an integer-deciding rounding: the BF16 quantisation of the compressed
indexer key).  Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s
CPU-baseline / reference leg may import it; the product path never does, and it
shares no code, constants or helpers with the CUDA library.

Sources.  The method is stated in a few sentences on the pages:
  [DCP]  "Qwen 4 QSA krijgt decode-contextparallellisme: in vLLM's concept-PR voor
         Qwen3.8-Flash-Next" (orcarouter.ai, nl), section "Wat de pull request
         daadwerkelijk verandert": a lightweight indexer compresses keys into
         micro-blocks with compression ratio 4, scores them, keeps the best 512
         blocks (about 2,048 token positions); final softmax and value
         aggregation run on the uncompressed K and V; under decode context
         parallelism the split attention results are combined across ranks.
  [CANN] "Qwen4-Exp QSA komt naar Huawei's Ascend: binnen SGLang's opt-in CANN
         prefill-PR" (orcarouter.ai, nl):
           - "Wat de pull request daadwerkelijk toevoegt": the [K,V] / [Q,0]
             layout embedding, D256 scale kept; fully masked rows keep the
             zero-output convention;
           - "Negen tests die geslaagd zijn ...": causal tail remainders 0..3 at
             ratio 4; 2,051 selected slots per query in the long case;
           - "Waarom QSA het lastige onderdeel is, in cijfers": head dim 256,
             GQA, an MQA indexer of head dim 128, ratio 4.
  [BSS]  "Pengambilan sampel batch-sharded Qwen4Exp" (orcarouter.ai, id), section
         "Apa yang dikatakan oleh klaster patch di sekitarnya tentang Qwen4Exp":
         the indexer compresses keys by a factor of four and keeps a budget of
         2,048 positions.

Readings where the pages are silent (each is listed in the design notes):
  * compressed indexer key kc_j = sum of the 4 tokens' indexer keys, summed in
    fp32 in token order and stored as BF16 (round to nearest even);
  * block score s_j = sum_h w_h * ReLU(q_idx,h . kc_j), 8 indexer heads x 128;
  * top-K by (score descending, block index ascending), emitted sorted by block
    index ascending;
  * a query at absolute position p sees the nb = (p+1) // 4 complete
    micro-blocks; its t = (p+1) % 4 trailing tokens (the incomplete micro-block)
    are always attended on top of the K selected blocks;
  * softmax scale defaults to 1/sqrt(256) = 1/16;
  * the KV split: every (query, KV head) has K+1 "unit" slots (the K selection
    slots, then the tail micro-block); the slots of all (query, KV head) pairs,
    query-major, are cut into fixed chunks of C slots; a split is the part of
    one pair's slots that falls in one chunk; an empty split has o = 0 and
    lse = -inf;
  * combine: lse = log sum_s exp(lse_s), o = sum_s exp(lse_s - lse) o_s; every
    lse_s = -inf gives o = 0 exactly and lse = -inf;
  * the FP8 main K/V cache stores e4m3(K) and e4m3(V) of the BF16 rows (round
    to nearest even, saturated, no scale); attention runs on those values and
    the indexer side cache stays BF16;
  * DCP: page P = position // 64 of a sequence lives on rank (P // I) % N; a
    rank attends to the attended tokens it holds; the ranks' (o, lse) are
    merged by the same log-sum-exp combine as the splits.

Every function below is pinned by tests in ``tests/test_oracle_pins.py``
against closed forms, library routines or brute force; no function is
"parity unpinned".
"""
from __future__ import annotations

import numpy as np

RATIO = 4          # micro-block compression ratio ([DCP], [CANN], [BSS])
HEAD_DIM = 256     # attention head dim ([CANN] "Waarom QSA ...")
IDX_DIM = 128      # indexer head dim ([CANN] "Waarom QSA ...")
IDX_HEADS = 8      # indexer query heads (fixed reading; the pages give 4 or 1)


# ----------------------------------------------------------------------------
# BF16


def bf16_round(x) -> np.ndarray:
    """Round fp32 values to the nearest BF16 value (ties to even); returns fp32."""
    a = np.ascontiguousarray(np.asarray(x, dtype=np.float32))
    b = a.view(np.uint32).astype(np.uint64)
    lsb = (b >> 16) & 1
    r = ((b + 0x7FFF + lsb) & 0xFFFF0000).astype(np.uint32)
    out = r.view(np.float32).copy()
    nan = np.isnan(a)
    out[nan] = np.nan
    return out


# ----------------------------------------------------------------------------
# FP8 e4m3 (the optional FP8 main K/V cache)


E4M3_MAX = 448.0   # largest finite e4m3 value: 1.75 * 2^8


def e4m3_round(x) -> np.ndarray:
    """Round values to the nearest FP8 e4m3 value (ties to even), saturating
    finite values beyond +-448 to +-448; returns fp64.

    e4m3 ([BSS], section "Apa yang dikatakan oleh klaster patch di sekitarnya
    tentang Qwen4Exp": the FP8 e4m3 main KV cache) has a sign, 4 exponent bits
    with bias 7 and 3 mantissa bits: normal values (1 + m/8) * 2^(e-7) for
    e in 1..15 (the all-ones code is NaN, no infinities), subnormal values
    m * 2^-9.  Between 2^E and 2^(E+1) the grid step is 2^(E-3); below 2^-6 it
    is 2^-9.  The quantisation carries no scale factor (scale 1)."""
    a = np.asarray(x, dtype=np.float64)
    mag = np.abs(a)
    _, ex = np.frexp(mag)                     # mag = f * 2^ex, f in [0.5, 1)
    E = np.maximum(ex - 1, -6)                # floor(log2 mag), subnormal range below 2^-6
    step = np.ldexp(1.0, E - 3)
    q = np.rint(mag / step) * step            # np.rint: round half to even
    q = np.minimum(q, E4M3_MAX)
    out = np.copysign(q, a)
    out[np.isnan(a)] = np.nan
    return out


# ----------------------------------------------------------------------------
# indexer


def visible(p: int) -> tuple[int, int]:
    """(nb, t): complete micro-blocks and trailing tokens seen by a query at
    absolute position p (its own token included)."""
    return (p + 1) // RATIO, (p + 1) % RATIO


def compress_keys(kidx_seq) -> np.ndarray:
    """kc[j] = BF16(k_idx[4j] + k_idx[4j+1] + k_idx[4j+2] + k_idx[4j+3]) for every
    complete micro-block of one sequence (summed in fp32, token order)."""
    k = np.asarray(kidx_seq, dtype=np.float32)
    nb = k.shape[0] // RATIO
    blocks = k[: nb * RATIO].reshape(nb, RATIO, k.shape[1])
    acc = np.zeros((nb, k.shape[1]), dtype=np.float32)
    for i in range(RATIO):
        acc = acc + blocks[:, i]
    return bf16_round(acc)


def open_block_partial(kidx_seq) -> np.ndarray:
    """fp32 running sum of the tokens of the trailing incomplete micro-block."""
    k = np.asarray(kidx_seq, dtype=np.float32)
    L = k.shape[0]
    start = (L // RATIO) * RATIO
    acc = np.zeros(k.shape[1], dtype=np.float32)
    for i in range(start, L):
        acc = acc + k[i]
    return acc


def block_scores(q_idx, w, kc) -> np.ndarray:
    """s_j = sum_h w_h * max(0, q_idx[h] . kc[j]) in fp64, for every row j of kc."""
    q = np.asarray(q_idx, dtype=np.float64)          # [H_i][D_i]
    c = np.asarray(kc, dtype=np.float64)             # [nb][D_i]
    wt = np.asarray(w, dtype=np.float64)             # [H_i]
    dots = c @ q.T                                   # [nb][H_i]
    return np.maximum(dots, 0.0) @ wt


def select_blocks(scores, k: int) -> np.ndarray:
    """The first min(k, nb) block indices under (score desc, index asc), returned
    sorted by block index ascending."""
    s = np.asarray(scores, dtype=np.float64)
    nb = s.shape[0]
    idx = np.arange(nb)
    order = np.lexsort((idx, -s))    # primary: -score, secondary: index
    return np.sort(order[: min(k, nb)]).astype(np.int64)


def token_positions(sel, p: int) -> np.ndarray:
    """The attended token set of a query at position p: the 4 tokens of every
    selected block, then the trailing tokens 4*nb .. p."""
    nb, t = visible(p)
    sel = np.asarray(sel, dtype=np.int64)
    main = (sel[:, None] * RATIO + np.arange(RATIO)[None, :]).reshape(-1)
    tail = np.arange(nb * RATIO, nb * RATIO + t)
    return np.concatenate([main, tail]).astype(np.int64)


# ----------------------------------------------------------------------------
# attention


def attend(q, keys, vals, scale: float):
    """Softmax attention of G query rows over n tokens in fp64.
    q [G][d], keys [n][d], vals [n][dv] -> (o [G][dv], lse [G]) with natural-log
    lse.  n = 0 gives o = 0 and lse = -inf (zero-output convention)."""
    q = np.asarray(q, dtype=np.float64)
    K = np.asarray(keys, dtype=np.float64)
    V = np.asarray(vals, dtype=np.float64)
    G = q.shape[0]
    if K.shape[0] == 0:
        return np.zeros((G, V.shape[1])), np.full(G, -np.inf)
    z = scale * (q @ K.T)                      # [G][n]
    m = z.max(axis=1, keepdims=True)
    e = np.exp(z - m)
    l = e.sum(axis=1, keepdims=True)
    o = (e @ V) / l
    lse = (m + np.log(l))[:, 0]
    return o, lse


def attend_gqa(q_heads, K, V, scale: float):
    """All Q heads of one query over the same tokens.  q_heads [Hq][256],
    K/V [n][Hkv][256]; Q head h reads KV head h // (Hq / Hkv)."""
    q_heads = np.asarray(q_heads, dtype=np.float64)
    K = np.asarray(K, dtype=np.float64)
    V = np.asarray(V, dtype=np.float64)
    hq, hkv = q_heads.shape[0], K.shape[1]
    G = hq // hkv
    o = np.zeros((hq, V.shape[2]))
    lse = np.zeros(hq)
    for g in range(hkv):
        og, lg = attend(q_heads[g * G:(g + 1) * G], K[:, g], V[:, g], scale)
        o[g * G:(g + 1) * G] = og
        lse[g * G:(g + 1) * G] = lg
    return o, lse


# ----------------------------------------------------------------------------
# one query, end to end


def decode_query(q_heads, q_idx, w, p: int, kidx_seq, kv_rows, k: int, scale: float):
    """QSA for one query at absolute position p.
    kidx_seq: the sequence's indexer keys for positions 0..p (at least);
    kv_rows(positions) -> (K [n][Hkv][256], V [n][Hkv][256]).
    Returns dict(nb, t, scores, sel, positions, o [Hq][256], lse [Hq])."""
    nb, t = visible(p)
    kc = compress_keys(np.asarray(kidx_seq)[: nb * RATIO])
    s = block_scores(q_idx, w, kc)
    sel = select_blocks(s, k)
    pos = token_positions(sel, p)
    K, V = kv_rows(pos)
    o, lse = attend_gqa(q_heads, K, V, scale)
    return {"nb": nb, "t": t, "kc": kc, "scores": s, "sel": sel, "positions": pos, "o": o, "lse": lse}


# ----------------------------------------------------------------------------
# KV split and log-sum-exp combine


def max_splits(k: int, chunk: int) -> int:
    """Upper bound on the number of chunks one pair's K+1 unit slots can touch."""
    n = k + 1
    return (n + chunk - 2) // chunk + 1


def chunk_segments(qi: int, g: int, hkv: int, k: int, chunk: int):
    """[(split s, first slot, end slot)] of pair (query row qi, KV head g)."""
    n = k + 1
    a = (qi * hkv + g) * n
    b = a + n
    w0, w1 = a // chunk, (b - 1) // chunk
    return [(w - w0, max(a, w * chunk) - a, min(b, (w + 1) * chunk) - a) for w in range(w0, w1 + 1)]


def unit_positions(sel, p: int, k: int):
    """Token positions of each of the K+1 unit slots of one query: slot u < len(sel)
    holds selected block sel[u]; the remaining selection slots are empty; slot K
    holds the trailing tokens."""
    nb, t = visible(p)
    sel = np.asarray(sel, dtype=np.int64)
    units = []
    for u in range(k):
        if u < sel.shape[0]:
            units.append(sel[u] * RATIO + np.arange(RATIO))
        else:
            units.append(np.zeros(0, dtype=np.int64))
    units.append(np.arange(nb * RATIO, nb * RATIO + t))
    return units


def decode_partials(q_heads, qi: int, p: int, sel, kv_rows, k: int, scale: float, chunk: int, hkv: int):
    """Split partials of one query: (part_o [S][Hq][256], part_lse [S][Hq]) with
    S = max_splits(k, chunk); slots a pair does not use hold o = 0, lse = -inf."""
    q_heads = np.asarray(q_heads, dtype=np.float64)
    hq = q_heads.shape[0]
    G = hq // hkv
    S = max_splits(k, chunk)
    po = np.zeros((S, hq, HEAD_DIM))
    pl = np.full((S, hq), -np.inf)
    units = unit_positions(sel, p, k)
    for g in range(hkv):
        for s, u0, u1 in chunk_segments(qi, g, hkv, k, chunk):
            pos = np.concatenate([units[u] for u in range(u0, u1)]) if u1 > u0 else np.zeros(0, np.int64)
            K, V = kv_rows(pos)
            o, lse = attend(q_heads[g * G:(g + 1) * G], np.asarray(K)[:, g], np.asarray(V)[:, g], scale)
            po[s, g * G:(g + 1) * G] = o
            pl[s, g * G:(g + 1) * G] = lse
    return po, pl


def combine(part_o, part_lse):
    """Log-sum-exp merge over the split axis (axis 0)."""
    po = np.asarray(part_o, dtype=np.float64)
    pl = np.asarray(part_lse, dtype=np.float64)
    H = pl.shape[1]
    o = np.zeros(po.shape[1:])
    lse = np.full(H, -np.inf)
    for h in range(H):
        live = np.isfinite(pl[:, h])
        if not live.any():
            continue
        m = pl[live, h].max()
        wts = np.exp(pl[live, h] - m)
        L = wts.sum()
        lse[h] = m + np.log(L)
        o[h] = (wts[:, None] * po[live, h]).sum(axis=0) / L
    return o, lse


# ----------------------------------------------------------------------------
# decode context parallelism (DCP)
#
# [DCP] "Qwen 4 QSA krijgt decode-contextparallellisme ...", section "Wat de
# pull request daadwerkelijk verandert": the main KV is split by context over
# the ranks, each rank reads its own slice, the selection is the same on every
# rank (the selector is replicated), and the ranks' partial attention results
# are combined.  The shard rule is a reading (the pages give none): logical
# page P = position // 64 of a sequence lives on rank (P // I) % N.

PAGE_TOKENS = 64


def dcp_owner(position, nranks: int, interleave_pages: int = 1):
    """Rank holding the K/V of a token position (array or scalar)."""
    page = np.asarray(position, dtype=np.int64) // PAGE_TOKENS
    return (page // interleave_pages) % nranks


def dcp_rank_partial(q_heads, sel, p: int, kv_rows, scale: float, nranks: int, rank: int,
                     interleave_pages: int = 1):
    """One rank's share of a query: attention of every Q head over the attended
    tokens (selected blocks and trailing tokens) that the rank holds.
    Returns (o [Hq][256], lse [Hq]); a rank holding none of them gives o = 0,
    lse = -inf."""
    pos = token_positions(sel, p)
    mine = pos[dcp_owner(pos, nranks, interleave_pages) == rank]
    K, V = kv_rows(mine)
    return attend_gqa(q_heads, K, V, scale) if mine.shape[0] else (
        np.zeros((np.asarray(q_heads).shape[0], HEAD_DIM)), np.full(np.asarray(q_heads).shape[0], -np.inf))
