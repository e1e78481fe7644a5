"""Oracle expectations for workload queries, from inputs regenerated on the CPU.

Test-only helper: it calls ``oracle`` with rows produced by ``workloads.configs``
on the host, never with anything read back from the device."""
from __future__ import annotations

import numpy as np
import torch

from oracle import qsa_oracle as O
from workloads import configs as C

# |gpu - oracle| <= ATOL + RTOL * |oracle| (elementwise), the stated output tolerance
ATOL = 2e-3
RTOL = 1e-2


def query_inputs(wl: C.Workload, row: int) -> dict:
    qs = C.queries(wl, rows=[row])
    return {"q": qs["q"][0].float().numpy(), "q_idx": qs["q_idx"][0].float().numpy(),
            "w": qs["w"][0].numpy(), "seq": int(qs["q_seq"][0]), "p": int(qs["q_pos"][0])}


def kv_reader(wl: C.Workload, seq: int, prefix_from=None):
    """kv_rows(positions) for the oracle.  ``prefix_from=(seq0, P)`` makes
    positions < P read sequence seq0 (a shared-prefix mapping)."""
    def rows(pos):
        pos = np.asarray(pos, dtype=np.int64)
        K = np.zeros((pos.shape[0], wl.hkv, C.HEAD_DIM), np.float32)
        V = np.zeros_like(K)
        if pos.shape[0] == 0:
            return K, V
        src = np.full(pos.shape, seq)
        if prefix_from is not None:
            src[pos < prefix_from[1]] = prefix_from[0]
        for s in np.unique(src):
            m = src == s
            t = torch.from_numpy(pos[m])
            K[m] = C.k_rows(wl, int(s), t).float().numpy()
            V[m] = C.v_rows(wl, int(s), t).float().numpy()
        if wl.kv_fp8:  # the cache holds e4m3 of the BF16 rows
            K, V = O.e4m3_round(K), O.e4m3_round(V)
        return K, V
    return rows


def kidx_seq(wl: C.Workload, seq: int, upto: int, prefix_from=None) -> np.ndarray:
    pos = torch.arange(0, upto)
    k = C.kidx_rows(wl, seq, pos).float().numpy()
    if prefix_from is not None and prefix_from[1] > 0:
        P = min(prefix_from[1], upto)
        k[:P] = C.kidx_rows(wl, prefix_from[0], torch.arange(0, P)).float().numpy()
    return k


def expect_query(wl: C.Workload, row: int, k=None, scale=None, chunk=None, qi=None, prefix_from=None) -> dict:
    """Oracle result for query `row` of the workload (its own token included)."""
    d = query_inputs(wl, row)
    k = wl.k_top if k is None else k
    scale = wl.scale if scale is None else scale
    rows = kv_reader(wl, d["seq"], prefix_from)
    kid = kidx_seq(wl, d["seq"], d["p"] + 1, prefix_from)
    r = O.decode_query(d["q"], d["q_idx"], d["w"], d["p"], kid, rows, k, scale)
    if chunk is not None:
        qrow = row if qi is None else qi
        po, pl = O.decode_partials(d["q"], qrow, d["p"], r["sel"], rows, k, scale, chunk, wl.hkv)
        r["part_o"], r["part_lse"] = po, pl
    r.update(d)
    return r


def assert_close(gpu, ref, what: str, slack=None):
    gpu = np.asarray(gpu, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert gpu.shape == ref.shape, (what, gpu.shape, ref.shape)
    ninf_g, ninf_r = np.isneginf(gpu), np.isneginf(ref)
    assert np.array_equal(ninf_g, ninf_r), f"{what}: -inf pattern differs"
    fin = ~ninf_r
    err = np.abs(gpu[fin] - ref[fin])
    bound = ATOL + RTOL * np.abs(ref[fin])
    if slack is not None:
        bound = bound + np.broadcast_to(np.asarray(slack, dtype=np.float64), ref.shape)[fin]
    bad = err > bound
    if bad.any():
        i = int(np.argmax(err - bound))
        raise AssertionError(f"{what}: {int(bad.sum())}/{bad.size} elements out of tolerance; worst gpu="
                             f"{gpu[fin][i]!r} oracle={ref[fin][i]!r}")


def rel_l2(gpu, ref) -> float:
    g = np.asarray(gpu, np.float64).ravel()
    r = np.asarray(ref, np.float64).ravel()
    return float(np.linalg.norm(g - r) / max(np.linalg.norm(r), 1e-30))
