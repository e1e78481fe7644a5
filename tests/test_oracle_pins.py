"""Pins of the CPU oracle against facts that do not come from the oracle itself:
closed forms, library routines (torch's BF16 conversion and scaled-dot-product
attention), brute force on tiny inputs, the values the pages print, and the
invariants the pages fix (dense equivalence, the [Q,0]/[K,V] layout embedding,
split + log-sum-exp = unsplit).  CPU only."""
import json
import math
import os

import numpy as np
import pytest
import torch

from oracle import qsa_oracle as O

RNG = np.random.default_rng(1234)


# ---------------------------------------------------------------- BF16 rounding

def test_bf16_round_matches_torch_conversion():
    x = np.concatenate([
        RNG.standard_normal(20000).astype(np.float32) * np.float32(10.0) ** RNG.integers(-30, 30, 20000).astype(np.float32),
        np.array([0.0, -0.0, 1.0, 1.00390625, 1.01171875, 1.0078125 + 2 ** -24, 3.3895314e38, -3.3895314e38,
                  1e-40, -1e-42, 65504.0, np.inf, -np.inf], dtype=np.float32),
    ]).astype(np.float32)
    # exact ties: values halfway between two bf16 numbers
    ties = (np.arange(1, 2000, dtype=np.uint32) << 16 | 0x8000).view(np.float32)
    x = np.concatenate([x, ties, -ties])
    ref = torch.from_numpy(x).to(torch.bfloat16).to(torch.float32).numpy()
    got = O.bf16_round(x)
    fin = np.isfinite(x)
    assert np.array_equal(got[fin].view(np.uint32), ref[fin].view(np.uint32))
    assert np.array_equal(np.isinf(got), np.isinf(ref))


# ---------------------------------------------------------------- FP8 e4m3 rounding

def _e4m3_code_values():
    """The value of every non-NaN e4m3 code, decoded from its bit fields."""
    vals = []
    for code in range(256):
        s, e, m = code >> 7, (code >> 3) & 15, code & 7
        if e == 15 and m == 7:
            continue  # NaN
        v = (m / 8.0) * 2.0 ** -6 if e == 0 else (1 + m / 8.0) * 2.0 ** (e - 7)
        vals.append(-v if s else v)
    return np.array(vals)


def test_e4m3_round_matches_torch_float8_conversion():
    x = np.concatenate([
        RNG.standard_normal(30000) * np.exp(RNG.uniform(-16, 7, 30000)),
        RNG.uniform(-448, 448, 5000), [0.0, -0.0, 448.0, -448.0, 2.0 ** -9, 2.0 ** -10, 3 * 2.0 ** -10]])
    x = x[np.abs(x) <= 448].astype(np.float32)
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).to(torch.float64).numpy()
    assert np.array_equal(O.e4m3_round(x), ref)


def test_e4m3_every_code_is_a_fixed_point():
    v = _e4m3_code_values()
    assert np.array_equal(O.e4m3_round(v), v)
    u = np.unique(v)
    assert u.size == 253 and u.max() == 448.0 and np.min(u[u > 0]) == 2.0 ** -9


def test_e4m3_ties_to_even_and_saturation():
    u = np.unique(_e4m3_code_values())
    pos = u[u >= 0]
    mid = (pos[:-1] + pos[1:]) / 2          # exact midpoints of neighbouring codes
    got = O.e4m3_round(mid)
    # the code with an even mantissa wins: its value / (grid step) is even
    lo, hi = pos[:-1], pos[1:]
    step = hi - lo
    want = np.where(np.rint(lo / step) % 2 == 0, lo, hi)
    assert np.array_equal(got, want)
    assert np.array_equal(O.e4m3_round(-mid), -want)
    sat = O.e4m3_round(np.array([448.5, 464.0, 479.0, 1e6, -1e30]))
    assert np.array_equal(sat, [448.0, 448.0, 448.0, 448.0, -448.0])
    assert np.isnan(O.e4m3_round(np.array([np.nan])))[0]


# ---------------------------------------------------------------- compression

def test_compress_keys_integer_sum_is_exact():
    k = RNG.integers(-8, 9, size=(4 * 37 + 3, 128))
    kc = O.compress_keys(k.astype(np.float32))
    exact = k[: 4 * 37].reshape(37, 4, 128).sum(axis=1)
    assert kc.shape == (37, 128)
    assert np.array_equal(kc, exact.astype(np.float32))


def test_compress_keys_fp32_token_order_and_bf16_store():
    # 1 + 2^24 rounds to 2^24 in fp32 (tie to even); then -2^24 and +1 give 1,
    # whereas the exact sum is 2.  The fp32, token-order reading gives 1.
    k = np.zeros((4, 128), np.float32)
    k[:, 0] = [1.0, 2.0 ** 24, -(2.0 ** 24), 1.0]
    # 1 + 3*2^-9 = 1.005859375 in fp32; the nearest BF16 value is 1.0078125
    k[:, 1] = [1.0, 2.0 ** -9, 2.0 ** -9, 2.0 ** -9]
    kc = O.compress_keys(k)
    assert kc[0, 0] == 1.0
    assert kc[0, 1] == np.float32(1.0078125)
    assert np.all(kc[0, 2:] == 0.0)


def test_open_block_partial():
    k = RNG.integers(-8, 9, size=(4 * 5 + 3, 128)).astype(np.float32)
    assert np.array_equal(O.open_block_partial(k), k[20:23].sum(axis=0))
    assert np.array_equal(O.open_block_partial(k[:20]), np.zeros(128, np.float32))


# ---------------------------------------------------------------- visibility / token set

def test_visibility_and_slot_counts(golden_dir):
    g = json.load(open(os.path.join(golden_dir, "slot_counts.json")))
    R, K = g["ratio"], g["k_blocks"]
    assert R == O.RATIO
    assert O.visible(0) == (0, 1)
    assert O.visible(3) == (1, 0)
    assert O.visible(4) == (1, 1)
    # budget: K blocks x ratio positions
    assert K * R == g["budget_positions"]
    # the long case: 2,051 slots = K * R + 3, a query whose tail holds 3 tokens
    L = g["long_case_cache_tokens"]
    p = L + 2                       # p + 1 = L + 3 -> tail of 3
    nb, t = O.visible(p)
    assert t == 3 and nb >= K
    sel = np.arange(K) * 7 % nb
    sel = np.unique(sel)[:K]
    assert O.token_positions(sel, p).shape[0] == g["long_case_selected_slots"]
    for t_rem in g["tail_remainders"]:
        p = 4 * 600 + t_rem - 1
        assert O.visible(p)[1] == t_rem
        assert O.token_positions(np.arange(K), p).shape[0] == K * R + t_rem


def test_token_positions_layout():
    pos = O.token_positions(np.array([0, 5]), 4 * 9 + 1)   # nb=9, t=2
    assert list(pos) == [0, 1, 2, 3, 20, 21, 22, 23, 36, 37]


# ---------------------------------------------------------------- scores

def test_block_scores_per_head_coordinates():
    # q_idx[h] = e_h: head h reads coordinate h of kc; s_j = sum_h w_h max(0, kc[j][h])
    q = np.zeros((8, 128)); q[np.arange(8), np.arange(8)] = 1.0
    w = np.array([0.5, 1, 2, 0.5, 1, 2, 0.5, 1])
    kc = np.zeros((3, 128))
    kc[0, :8] = [1, -2, 3, -4, 5, -6, 7, -8]
    kc[1, :8] = [-1, -1, -1, -1, -1, -1, -1, -1]
    kc[2, 8:] = 5.0                                  # coordinates no head reads
    s = O.block_scores(q, w, kc)
    assert s[0] == 0.5 * 1 + 2 * 3 + 1 * 5 + 0.5 * 7
    assert s[1] == 0.0                               # every dot negative -> ReLU kills it
    assert s[2] == 0.0


def test_block_scores_closed_form_constant_vectors():
    # q_idx[h] = (h - 3) * ones, kc[j] = (j - 2) * ones: dot = 128 (h-3)(j-2)
    q = np.outer(np.arange(8) - 3.0, np.ones(128))
    w = np.array([1, 2, 0.5, 1, 2, 0.5, 1, 2])
    kc = np.outer(np.arange(6) - 2.0, np.ones(128))
    s = O.block_scores(q, w, kc)
    for j in range(6):
        a = j - 2
        want = sum(w[h] * 128 * (h - 3) * a for h in range(8) if (h - 3) * a > 0)
        assert s[j] == want


def test_block_scores_ignore_weight_of_inactive_heads():
    q = np.zeros((8, 128)); q[3, :] = 1.0
    kc = np.ones((1, 128))
    for w3 in (0.5, 1.0, 2.0):
        w = np.full(8, 100.0); w[3] = w3
        assert O.block_scores(q, w, kc)[0] == 128 * w3


# ---------------------------------------------------------------- top-k

def brute_topk(s, k):
    n = len(s)
    keep = [j for j in range(n) if sum(1 for i in range(n) if s[i] > s[j] or (s[i] == s[j] and i < j)) < k]
    return sorted(keep)


@pytest.mark.parametrize("n,k", [(1, 1), (5, 3), (17, 4), (40, 16), (64, 16), (33, 0), (10, 12)])
def test_select_blocks_brute_force(n, k):
    for trial in range(20):
        s = RNG.integers(0, 6, size=n).astype(np.float64) * 0.5
        assert list(O.select_blocks(s, k)) == brute_topk(list(s), k)


def test_select_blocks_ties_and_edges():
    assert list(O.select_blocks(np.full(100, 3.0), 7)) == list(range(7))
    assert list(O.select_blocks(np.arange(10.0), 20)) == list(range(10))
    assert O.select_blocks(np.arange(10.0), 0).shape == (0,)
    assert list(O.select_blocks(np.array([1.0, 5.0, 5.0, 2.0, 5.0]), 2)) == [1, 2]
    # -0 and +0 are the same score (IEEE equality): they tie and the lower index wins
    assert list(O.select_blocks(np.array([-1.0, -0.0, 0.0]), 1)) == [1]
    assert list(O.select_blocks(np.array([0.0, -1.0, -0.0, -0.0]), 2)) == [0, 2]


# ---------------------------------------------------------------- attention

def test_attend_single_token_and_uniform_and_empty():
    q = RNG.standard_normal((3, 256)); K = RNG.standard_normal((1, 256)); V = RNG.standard_normal((1, 256))
    o, lse = O.attend(q, K, V, 0.0625)
    assert np.allclose(o, np.repeat(V, 3, axis=0), atol=0, rtol=1e-15)
    assert np.allclose(lse, 0.0625 * (q @ K[0]), rtol=1e-14)
    K = RNG.standard_normal((9, 256)); V = RNG.standard_normal((9, 256))
    o, lse = O.attend(np.zeros((2, 256)), K, V, 0.0625)
    assert np.allclose(o, V.mean(axis=0)[None], rtol=1e-14, atol=1e-15)
    assert np.allclose(lse, math.log(9), rtol=1e-15)
    o, lse = O.attend(q, np.zeros((0, 256)), np.zeros((0, 256)), 0.0625)
    assert np.all(o == 0) and np.all(np.isneginf(lse))


def test_attend_matches_torch_sdpa():
    q = RNG.standard_normal((12, 256)); K = RNG.standard_normal((300, 256)); V = RNG.standard_normal((300, 256))
    o, lse = O.attend(q, K, V, 1 / 16)
    tq, tk, tv = (torch.from_numpy(a)[None, None] for a in (q, K, V))
    ref = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, scale=1 / 16)[0, 0].numpy()
    ref_lse = torch.logsumexp(torch.from_numpy(q @ K.T / 16), dim=1).numpy()
    assert np.allclose(o, ref, rtol=1e-12, atol=1e-13)
    assert np.allclose(lse, ref_lse, rtol=1e-13)


def test_layout_embedding_identity():
    """[CANN] layout embedding: Q' = [Q, 0], C = [K, V] used as keys and values:
    Q' C^T = Q K^T and softmax(s Q' C^T) C = [P K, P V]."""
    q = RNG.standard_normal((6, 256)); K = RNG.standard_normal((50, 256)); V = RNG.standard_normal((50, 256))
    qp = np.concatenate([q, np.zeros_like(q)], axis=1)
    C = np.concatenate([K, V], axis=1)
    o2, lse2 = O.attend(qp, C, C, 1 / 16)             # D256 scale kept
    oV, lseV = O.attend(q, K, V, 1 / 16)
    oK, _ = O.attend(q, K, K, 1 / 16)
    assert np.allclose(o2[:, 256:], oV, rtol=1e-12, atol=1e-13)
    assert np.allclose(o2[:, :256], oK, rtol=1e-12, atol=1e-13)
    assert np.allclose(lse2, lseV, rtol=1e-13)


# ---------------------------------------------------------------- end to end

def _toy(L, hq, hkv, seed=0):
    r = np.random.default_rng(seed)
    K = r.standard_normal((L, hkv, 256)); V = r.standard_normal((L, hkv, 256))
    kidx = r.integers(-8, 9, size=(L, 128)).astype(np.float32)
    q = r.standard_normal((hq, 256)); qi = r.integers(-8, 9, size=(8, 128)).astype(np.float64)
    w = r.choice([0.5, 1.0, 2.0], size=8)
    return K, V, kidx, q, qi, w


@pytest.mark.parametrize("L,hq,hkv", [(37, 16, 2), (64, 24, 2), (81, 12, 1), (130, 6, 1), (9, 3, 1)])
def test_dense_equivalence_when_budget_covers_context(L, hq, hkv):
    """With K >= visible blocks, QSA equals dense causal GQA attention (torch SDPA)."""
    K, V, kidx, q, qi, w = _toy(L, hq, hkv)
    p = L - 1
    r = O.decode_query(q, qi, w, p, kidx, lambda pos: (K[pos], V[pos]), k=1024, scale=1 / 16)
    assert len(r["positions"]) == L
    tq = torch.from_numpy(q)[None, :, None, :]                       # [1][Hq][1][D]
    tk = torch.from_numpy(K[: p + 1]).permute(1, 0, 2)[None]        # [1][Hkv][L][D]
    tv = torch.from_numpy(V[: p + 1]).permute(1, 0, 2)[None]
    G = hq // hkv
    tk = tk.repeat_interleave(G, dim=1); tv = tv.repeat_interleave(G, dim=1)
    ref = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, scale=1 / 16)[0, :, 0].numpy()
    assert np.allclose(r["o"], ref, rtol=1e-12, atol=1e-13)


def test_sparse_selection_excludes_low_blocks():
    # with K < nb, attention runs over exactly the chosen blocks plus the tail
    K, V, kidx, q, qi, w = _toy(4 * 50 + 2, 8, 2, seed=3)
    p = 4 * 50 + 1
    r = O.decode_query(q, qi, w, p, kidx, lambda pos: (K[pos], V[pos]), k=10, scale=0.1)
    assert len(r["sel"]) == 10 and r["t"] == 2
    s = r["scores"]
    assert s[r["sel"]].min() >= np.delete(s, r["sel"]).max()
    o_ref, _ = O.attend_gqa(q, K[r["positions"]], V[r["positions"]], 0.1)
    assert np.array_equal(r["o"], o_ref)


@pytest.mark.parametrize("chunk", [1, 2, 3, 7, 16, 64, 1000000])
def test_split_plus_lse_equals_unsplit(chunk):
    hq, hkv, k = 12, 2, 16
    K, V, kidx, q, qi, w = _toy(4 * 30 + 3, hq, hkv, seed=chunk)
    for p, qrow in ((4 * 30 + 2, 0), (4 * 30 + 2, 5), (4 * 3 + 0, 2), (2, 1)):   # incl. nb < k and nb = 0
        r = O.decode_query(q, qi, w, p, kidx, lambda pos: (K[pos], V[pos]), k=k, scale=1 / 16)
        po, pl = O.decode_partials(q, qrow, p, r["sel"], lambda pos: (K[pos], V[pos]), k, 1 / 16, chunk, hkv)
        assert po.shape[0] == O.max_splits(k, chunk)
        o, lse = O.combine(po, pl)
        assert np.allclose(o, r["o"], rtol=1e-12, atol=1e-12)
        assert np.allclose(lse, r["lse"], rtol=1e-12)


def test_chunk_segments_partition_and_bound():
    for k in (0, 1, 5, 16, 512):
        for chunk in (1, 2, 5, 17, 100, 513, 5000):
            S = O.max_splits(k, chunk)
            for qi in range(7):
                for hkv in (1, 2):
                    for g in range(hkv):
                        segs = O.chunk_segments(qi, g, hkv, k, chunk)
                        assert len(segs) <= S
                        assert [s for s, _, _ in segs] == list(range(len(segs)))
                        assert segs[0][1] == 0 and segs[-1][2] == k + 1
                        for (_, _, e), (_, b, _) in zip(segs, segs[1:]):
                            assert e == b
                        assert all(hi - lo <= chunk and hi > lo for _, lo, hi in segs)


def test_combine_all_empty_and_identity():
    po = RNG.standard_normal((3, 4, 256)); pl = np.full((3, 4), -np.inf)
    o, lse = O.combine(po, pl)
    assert np.all(o == 0) and np.all(np.isneginf(lse))
    pl = np.full((3, 4), -np.inf); pl[1] = 2.5
    o, lse = O.combine(po, pl)
    assert np.array_equal(o, po[1]) and np.all(lse == 2.5)


def test_fully_masked_row_is_zero():
    """[CANN] zero-output convention: an empty token set gives exactly 0."""
    K, V, kidx, q, qi, w = _toy(8, 4, 1)
    r = O.decode_query(q, qi, w, 3, kidx, lambda pos: (K[pos], V[pos]), k=0, scale=1 / 16)  # nb=1, t=0, K=0
    assert r["positions"].shape == (0,)
    assert np.all(r["o"] == 0) and np.all(np.isneginf(r["lse"]))


# ---------------------------------------------------------------- DCP (decode context parallelism)

def test_dcp_owner_follows_the_page_rule():
    pos = np.array([0, 63, 64, 127, 128, 191, 192, 255, 256, 320])
    # round robin by page over 2 ranks, and pairs of pages over 2 ranks
    assert O.dcp_owner(pos, 2, 1).tolist() == [0, 0, 1, 1, 0, 0, 1, 1, 0, 1]
    assert O.dcp_owner(pos, 2, 2).tolist() == [0, 0, 0, 0, 1, 1, 1, 1, 0, 0]
    assert O.dcp_owner(pos, 3, 1).tolist() == [0, 0, 1, 1, 2, 2, 0, 0, 1, 2]
    assert np.all(O.dcp_owner(pos, 1, 1) == 0)


@pytest.mark.parametrize("nranks,interleave", [(1, 1), (2, 1), (3, 1), (4, 1), (2, 2), (3, 2)])
def test_dcp_rank_partials_merge_to_the_unsharded_result(nranks, interleave):
    """The ranks' shares partition the attended tokens, so their log-sum-exp
    merge is the unsharded attention (fp64 rounding only), including ranks that
    hold nothing of a query and tails on any rank."""
    hq, hkv, k = 12, 2, 24
    L = 64 * 7 + 13
    K, V, kidx, q, qi, w = _toy(L, hq, hkv, seed=nranks * 10 + interleave)
    rows = lambda pos: (K[pos], V[pos])
    for p in (L - 1, 64 * 3 + 1, 64 * 5 - 1, 70, 2):
        r = O.decode_query(q, qi, w, p, kidx, rows, k=k, scale=1 / 16)
        parts = [O.dcp_rank_partial(q, r["sel"], p, rows, 1 / 16, nranks, rank, interleave) for rank in range(nranks)]
        po = np.stack([x[0] for x in parts])
        pl = np.stack([x[1] for x in parts])
        n_tok = sum(int(np.sum(O.dcp_owner(r["positions"], nranks, interleave) == rank)) for rank in range(nranks))
        assert n_tok == len(r["positions"])
        o, lse = O.combine(po, pl)
        assert np.allclose(o, r["o"], rtol=1e-12, atol=1e-12)
        assert np.allclose(lse, r["lse"], rtol=1e-12)
        for rank in range(nranks):   # a rank without tokens contributes o = 0, lse = -inf
            if not np.any(O.dcp_owner(r["positions"], nranks, interleave) == rank):
                assert np.all(parts[rank][0] == 0) and np.all(np.isneginf(parts[rank][1]))
