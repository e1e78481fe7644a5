"""Thin ctypes binding of libqsa (include/qsa.h).

Argument marshalling only: every step of the QSA decode path runs in the CUDA
kernels of libqsa.so.  PyTorch supplies device memory and the current stream.
The functions keep the C names; they take torch tensors, check dtype / device /
shape / contiguity, pass raw pointers, and raise :class:`QSAError` on a
non-zero status.  There is no fallback: if libqsa.so is missing, importing this
module raises.
"""
from __future__ import annotations

import ctypes
import math
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libqsa.so")

HEAD_DIM = 256
IDX_HEADS = 8
IDX_DIM = 128
RATIO = 4
PAGE_TOKENS = 64
BLOCKS_PER_PAGE = 16
MAX_TOPK = 2048
MAX_GROUP = 16

QSA_OK, QSA_ERR_INVALID_ARG, QSA_ERR_UNSUPPORTED, QSA_ERR_CUDA = 0, -1, -2, -3
DEV_BITS = {1: "BAD_PAGE", 2: "BAD_SEQ", 4: "BAD_POS", 8: "BAD_SEL", 16: "BAD_COUNT", 32: "BAD_ORDER",
            64: "TIMEOUT", 128: "SCORES_LD"}


class QSAError(RuntimeError):
    def __init__(self, fn: str, status: int):
        super().__init__(f"{fn} failed: {status_string(status)} ({status})")
        self.status = status


class qsa_cache_t(ctypes.Structure):
    _fields_ = [("kv_pages", ctypes.c_void_p), ("kc_pages", ctypes.c_void_p),
                ("kc_partial", ctypes.c_void_p), ("block_table", ctypes.c_void_p), ("num_pages", ctypes.c_int32),
                ("max_seqs", ctypes.c_int32), ("max_pages_per_seq", ctypes.c_int32),
                ("num_kv_heads", ctypes.c_int32), ("kv_dtype", ctypes.c_int32)]


KV_BF16 = 0
KV_FP8_E4M3 = 1
_KV_TORCH = {KV_BF16: torch.bfloat16, KV_FP8_E4M3: torch.float8_e4m3fn}


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"libqsa.so not built at {LIB_PATH}; run `python sparse_attention_decode_03_b200/build.py`")
    lib = ctypes.CDLL(LIB_PATH)
    P, I32, I64, F = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_float
    PC = ctypes.POINTER(qsa_cache_t)
    sig = {
        "qsa_status_string": (ctypes.c_char_p, [ctypes.c_int]),
        "qsa_abi_version": (ctypes.c_int, []),
        "qsa_append_kv": (ctypes.c_int, [PC, P, P, P, P, P, I32, P, P]),
        "qsa_index_scores": (ctypes.c_int, [PC, P, P, P, P, I32, P, I64, P, P]),
        "qsa_topk_blocks": (ctypes.c_int, [P, I64, P, I32, I32, P, P, P, P]),
        "qsa_index_topk": (ctypes.c_int, [PC, P, P, P, P, I32, I32, P, I64, P, P, P, P]),
        "qsa_index_topk_smem_bytes": (ctypes.c_int, [PC, I64]),
        "qsa_index_topk_resident_queries": (ctypes.c_int, [PC, I64]),
        "qsa_decode_plan": (ctypes.c_int, [I32, I32, I32, I32, ctypes.POINTER(I32), ctypes.POINTER(I32)]),
        "qsa_sparse_decode": (ctypes.c_int, [PC, P, I32, I32, P, P, P, P, I32, F, I32, I32, P, P, P, P]),
        "qsa_sparse_attention": (ctypes.c_int, [PC, P, I32, I32, P, P, P, P, I32, F, I32, I32, P, P, P, P, P, P, P]),
        "qsa_combine": (ctypes.c_int, [P, P, I32, I32, I32, P, P, P]),
        "qsa_combine_strided": (ctypes.c_int, [P, P, I32, I32, I32, I64, I64, I64, I64, P, I32, P, P]),
        "qsa_dcp_localize_tokens": (ctypes.c_int, [P, P, I32, I32, I32, I32, P, P, P]),
        "qsa_dcp_localize_selection": (ctypes.c_int, [P, P, P, I32, I32, I32, I32, I32, P, P, P, P, P]),
        "qsa_sparse_attention_noalloc": (ctypes.c_int, [PC, P, I32, I32, P, P, P, P, I32, F, I32, P, P, P, P]),
    }
    for name, (res, args) in sig.items():
        f = getattr(lib, name)
        f.restype = res
        f.argtypes = args
    return lib


LIB = _load()
ABI_VERSION = LIB.qsa_abi_version()


def status_string(status: int) -> str:
    return LIB.qsa_status_string(int(status)).decode()


def _check(fn: str, rc: int) -> None:
    if rc != QSA_OK:
        raise QSAError(fn, rc)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _req(t: torch.Tensor, name: str, dtype, shape=None):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name}: expected {dtype}, got {t.dtype}")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if shape is not None:
        if t.dim() != len(shape) or any(s is not None and a != s for a, s in zip(t.shape, shape)):
            raise ValueError(f"{name}: expected shape {shape}, got {tuple(t.shape)}")
    return t


# ----------------------------------------------------------------------------
# cache group


class PagedCache:
    """Device buffers of one cache group: main K/V pages and the compressed-indexer
    side cache, paged by the same page ids, plus the per-sequence open-block sum.

    kv_pages holds, per page and KV head, 16 micro-blocks of 4 tokens, each one
    contiguous run (one selected micro-block of one KV head is one copy):
    BF16 (kv_dtype KV_BF16): [page][Hkv][16][4 dim atoms][8 rows][64], rows 0-3
    the K rows and 4-7 the V rows, the 16-byte chunk c of row r at chunk
    position c ^ r (the tensor cores' 128-byte swizzled operand layout);
    FP8 e4m3 (KV_FP8_E4M3): [page][Hkv][16][2 (K, V)][4 rows][256].
    with_kv=False leaves out the main K/V (a selector-only group),
    with_kc=False the side cache (a K/V-only group, e.g. a DCP rank's shard)."""

    def __init__(self, num_pages: int, max_seqs: int, max_pages_per_seq: int, num_kv_heads: int,
                 block_table: torch.Tensor | None = None, device="cuda", kv_dtype: int = KV_BF16,
                 with_kv: bool = True, with_kc: bool = True):
        dev = torch.device(device)
        if kv_dtype not in _KV_TORCH:
            raise ValueError(f"kv_dtype must be KV_BF16 or KV_FP8_E4M3, got {kv_dtype}")
        self.num_pages, self.max_seqs, self.max_pages_per_seq, self.num_kv_heads = (
            int(num_pages), int(max_seqs), int(max_pages_per_seq), int(num_kv_heads))
        self.kv_dtype = int(kv_dtype)
        if not (with_kv or with_kc):
            raise ValueError("a cache group needs the main K/V, the side cache, or both")
        shape = ((num_pages, num_kv_heads, BLOCKS_PER_PAGE, 4, 2 * RATIO, HEAD_DIM // 4) if self.kv_dtype == KV_BF16
                 else (num_pages, num_kv_heads, BLOCKS_PER_PAGE, 2, RATIO, HEAD_DIM))
        self.kv_pages = torch.empty(shape, dtype=_KV_TORCH[self.kv_dtype], device=dev) if with_kv else None
        self.kc_pages = torch.empty((num_pages, BLOCKS_PER_PAGE, IDX_DIM), dtype=torch.bfloat16,
                                    device=dev) if with_kc else None
        self.kc_partial = torch.zeros((max_seqs, IDX_DIM), dtype=torch.float32, device=dev) if with_kc else None
        self.device = dev
        if block_table is None:
            block_table = torch.full((max_seqs, max_pages_per_seq), -1, dtype=torch.int32)
        self.block_table = block_table.to(device=dev, dtype=torch.int32).contiguous()
        assert tuple(self.block_table.shape) == (max_seqs, max_pages_per_seq)
        self._struct = None

    def struct(self) -> qsa_cache_t:
        if self._struct is None:
            dp = lambda t: None if t is None else t.data_ptr()
            self._struct = qsa_cache_t(dp(self.kv_pages), dp(self.kc_pages), dp(self.kc_partial),
                                       self.block_table.data_ptr(), self.num_pages, self.max_seqs,
                                       self.max_pages_per_seq, self.num_kv_heads, self.kv_dtype)
        return self._struct

    def _rows(self, kv: int) -> torch.Tensor:
        if self.kv_dtype != KV_BF16:
            return self.kv_pages[:, :, :, kv].reshape(self.num_pages, self.num_kv_heads, PAGE_TOKENS, HEAD_DIM)
        # [page][Hkv][blk][atom][row][chunk position][8]: row r's chunk c sits at position c ^ r
        x = self.kv_pages.view(self.num_pages, self.num_kv_heads, BLOCKS_PER_PAGE, 4, 2 * RATIO, 8, 8)
        r = torch.arange(2 * RATIO, device=x.device)
        pos = (torch.arange(8, device=x.device)[None, :] ^ r[:, None])      # [row][chunk] -> position
        x = torch.gather(x, 5, pos[None, None, None, None, :, :, None].expand(x.shape))
        x = x[:, :, :, :, kv * RATIO:(kv + 1) * RATIO]                       # [page][Hkv][blk][atom][4][8][8]
        return x.permute(0, 1, 2, 4, 3, 5, 6).reshape(self.num_pages, self.num_kv_heads, PAGE_TOKENS, HEAD_DIM)

    def k_view(self) -> torch.Tensor:
        """K as [page][Hkv][64][256] (a copy in logical order, for inspection)."""
        return self._rows(0)

    def v_view(self) -> torch.Tensor:
        """V as [page][Hkv][64][256] (a copy in logical order, for inspection)."""
        return self._rows(1)

    @property
    def capacity_tokens(self) -> int:
        return self.max_pages_per_seq * PAGE_TOKENS


# ----------------------------------------------------------------------------
# the five calls


def qsa_append_kv(cache: PagedCache, k_new, v_new, kidx_new, seq_id, pos, dev_status=None, stream=None):
    n = int(seq_id.shape[0]) if isinstance(seq_id, torch.Tensor) else -1
    hkv = cache.num_kv_heads
    _req(k_new, "k_new", torch.bfloat16, (n, hkv, HEAD_DIM))
    _req(v_new, "v_new", torch.bfloat16, (n, hkv, HEAD_DIM))
    _req(kidx_new, "kidx_new", torch.bfloat16, (n, IDX_DIM))
    _req(seq_id, "seq_id", torch.int32, (n,))
    _req(pos, "pos", torch.int32, (n,))
    if dev_status is not None:
        _req(dev_status, "dev_status", torch.int32, (1,))
    _check("qsa_append_kv", LIB.qsa_append_kv(ctypes.byref(cache.struct()), _ptr(k_new), _ptr(v_new), _ptr(kidx_new),
                                              _ptr(seq_id), _ptr(pos), n, _ptr(dev_status), _stream(stream)))


def qsa_index_scores(cache: PagedCache, q_idx, w, q_seq, q_pos, scores, dev_status=None, stream=None):
    nq = int(q_seq.shape[0])
    _req(q_idx, "q_idx", torch.bfloat16, (nq, IDX_HEADS, IDX_DIM))
    _req(w, "w", torch.float32, (nq, IDX_HEADS))
    _req(q_seq, "q_seq", torch.int32, (nq,))
    _req(q_pos, "q_pos", torch.int32, (nq,))
    _req(scores, "scores", torch.float32, (nq, None))
    if dev_status is not None:
        _req(dev_status, "dev_status", torch.int32, (1,))
    _check("qsa_index_scores", LIB.qsa_index_scores(ctypes.byref(cache.struct()), _ptr(q_idx), _ptr(w), _ptr(q_seq),
                                                    _ptr(q_pos), nq, _ptr(scores), int(scores.shape[1]),
                                                    _ptr(dev_status), _stream(stream)))


def qsa_topk_blocks(scores, q_pos, k: int, sel, count, dev_status=None, stream=None):
    nq = int(q_pos.shape[0])
    _req(scores, "scores", torch.float32, (nq, None))
    _req(q_pos, "q_pos", torch.int32, (nq,))
    _req(sel, "sel", torch.int32, (nq, k))
    _req(count, "count", torch.int32, (nq,))
    if dev_status is not None:
        _req(dev_status, "dev_status", torch.int32, (1,))
    _check("qsa_topk_blocks", LIB.qsa_topk_blocks(_ptr(scores), int(scores.shape[1]), _ptr(q_pos), nq, int(k),
                                                  _ptr(sel), _ptr(count), _ptr(dev_status), _stream(stream)))


def qsa_index_topk(cache: PagedCache, q_idx, w, q_seq, q_pos, k: int, scores, sel, count, dev_status=None,
                   stream=None):
    """qsa_index_scores + qsa_topk_blocks in one kernel (a cluster of 8 CTAs per
    query keeps the score row on chip while it selects from it)."""
    nq = int(q_seq.shape[0])
    _req(q_idx, "q_idx", torch.bfloat16, (nq, IDX_HEADS, IDX_DIM))
    _req(w, "w", torch.float32, (nq, IDX_HEADS))
    _req(q_seq, "q_seq", torch.int32, (nq,))
    _req(q_pos, "q_pos", torch.int32, (nq,))
    _req(scores, "scores", torch.float32, (nq, None))
    _req(sel, "sel", torch.int32, (nq, k))
    _req(count, "count", torch.int32, (nq,))
    if dev_status is not None:
        _req(dev_status, "dev_status", torch.int32, (1,))
    _check("qsa_index_topk", LIB.qsa_index_topk(ctypes.byref(cache.struct()), _ptr(q_idx), _ptr(w), _ptr(q_seq),
                                                _ptr(q_pos), nq, int(k), _ptr(scores), int(scores.shape[1]),
                                                _ptr(sel), _ptr(count), _ptr(dev_status), _stream(stream)))


def index_topk_smem_bytes(cache: PagedCache, scores_ld: int) -> int:
    r = LIB.qsa_index_topk_smem_bytes(ctypes.byref(cache.struct()), int(scores_ld))
    _check("qsa_index_topk_smem_bytes", r if r < 0 else QSA_OK)
    return r


def index_topk_resident_queries(cache: PagedCache, scores_ld: int) -> int:
    r = LIB.qsa_index_topk_resident_queries(ctypes.byref(cache.struct()), int(scores_ld))
    _check("qsa_index_topk_resident_queries", r if r < 0 else QSA_OK)
    return r


FUSED_CLUSTER_CTAS = 8  # CTAs per query of qsa_index_topk (one cluster)


def fused_selection_pays(nq: int, max_seqs: int, sms: int, resident: int) -> bool:
    """Whether a step of nq queries should run the fused indexer + selection:
    its clusters fill the GPU (nq * FUSED_CLUSTER_CTAS >= the SM count) and all
    fit at once (nq <= resident: with a second wave the longest rows start late
    and the two-call form, which spreads a row over many CTAs, is faster), and
    the call is decode-shaped (fewer than 8 queries per sequence on average;
    prefill calls take the tensor-core query-tiled indexer)."""
    return nq * FUSED_CLUSTER_CTAS >= sms and nq <= resident and nq < 8 * max_seqs


def fused_default(cache: PagedCache, scores_ld: int, nq: int, sms: int) -> bool:
    """The Decoder's default selection form for a step of up to nq queries.  A
    device that cannot place the fused kernel's clusters (the occupancy query
    fails, or the clusters do not fit) keeps the two calls; an invalid cache or
    scores_ld is the caller's error and raises QSAError."""
    if cache.kc_pages is None:
        return False
    try:
        resident = index_topk_resident_queries(cache, scores_ld)
    except QSAError as e:
        if e.status not in (QSA_ERR_UNSUPPORTED, QSA_ERR_CUDA):
            raise
        resident = 0
    return fused_selection_pays(nq, cache.max_seqs, sms, resident)


def qsa_decode_plan(nq: int, hkv: int, k: int, target_ctas: int) -> tuple[int, int]:
    c, s = ctypes.c_int32(), ctypes.c_int32()
    _check("qsa_decode_plan", LIB.qsa_decode_plan(int(nq), int(hkv), int(k), int(target_ctas), ctypes.byref(c),
                                                  ctypes.byref(s)))
    return c.value, s.value


def qsa_sparse_decode(cache: PagedCache, q, q_seq, q_pos, sel, count, k: int, scale: float, chunk_units: int,
                      max_splits: int, part_o, part_lse, dev_status=None, stream=None):
    nq = int(q_seq.shape[0])
    hq = int(q.shape[1]) if q.dim() == 3 else -1
    _req(q, "q", torch.bfloat16, (nq, hq, HEAD_DIM))
    _req(q_seq, "q_seq", torch.int32, (nq,))
    _req(q_pos, "q_pos", torch.int32, (nq,))
    _req(sel, "sel", torch.int32, (nq, k))
    _req(count, "count", torch.int32, (nq,))
    _req(part_o, "part_o", torch.float32, (nq, max_splits, hq, HEAD_DIM))
    _req(part_lse, "part_lse", torch.float32, (nq, max_splits, hq))
    if dev_status is not None:
        _req(dev_status, "dev_status", torch.int32, (1,))
    _check("qsa_sparse_decode", LIB.qsa_sparse_decode(
        ctypes.byref(cache.struct()), _ptr(q), nq, hq, _ptr(q_seq), _ptr(q_pos), _ptr(sel), _ptr(count), int(k),
        float(scale), int(chunk_units), int(max_splits), _ptr(part_o), _ptr(part_lse), _ptr(dev_status),
        _stream(stream)))


def qsa_sparse_attention(cache: PagedCache, q, q_seq, q_pos, sel, count, k: int, scale: float, chunk_units: int,
                         max_splits: int, part_o, part_lse, pair_done, out, lse, dev_status=None, stream=None):
    """qsa_sparse_decode + qsa_combine in one kernel: the CTA that writes a
    (query, KV head) pair's last split merges it.  pair_done (int32 [nq][Hkv])
    must be zero on entry and is zero again afterwards."""
    nq = int(q_seq.shape[0])
    hq = int(q.shape[1]) if q.dim() == 3 else -1
    _req(q, "q", torch.bfloat16, (nq, hq, HEAD_DIM))
    _req(q_seq, "q_seq", torch.int32, (nq,))
    _req(q_pos, "q_pos", torch.int32, (nq,))
    _req(sel, "sel", torch.int32, (nq, k))
    _req(count, "count", torch.int32, (nq,))
    _req(part_o, "part_o", torch.float32, (nq, max_splits, hq, HEAD_DIM))
    _req(part_lse, "part_lse", torch.float32, (nq, max_splits, hq))
    _req(pair_done, "pair_done", torch.int32, (nq * cache.num_kv_heads,))
    _req(out, "out", torch.bfloat16, (nq, hq, HEAD_DIM))
    _req(lse, "lse", torch.float32, (nq, hq))
    if dev_status is not None:
        _req(dev_status, "dev_status", torch.int32, (1,))
    _check("qsa_sparse_attention", LIB.qsa_sparse_attention(
        ctypes.byref(cache.struct()), _ptr(q), nq, hq, _ptr(q_seq), _ptr(q_pos), _ptr(sel), _ptr(count), int(k),
        float(scale), int(chunk_units), int(max_splits), _ptr(part_o), _ptr(part_lse), _ptr(pair_done), _ptr(out),
        _ptr(lse), _ptr(dev_status), _stream(stream)))


def qsa_combine(part_o, part_lse, out, lse, stream=None):
    nq, S, hq = (int(x) for x in part_lse.shape)
    _req(part_o, "part_o", torch.float32, (nq, S, hq, HEAD_DIM))
    _req(part_lse, "part_lse", torch.float32, (nq, S, hq))
    _req(out, "out", torch.bfloat16, (nq, hq, HEAD_DIM))
    _req(lse, "lse", torch.float32, (nq, hq))
    _check("qsa_combine", LIB.qsa_combine(_ptr(part_o), _ptr(part_lse), nq, S, hq, _ptr(out), _ptr(lse),
                                          _stream(stream)))


OUT_BF16 = 0
OUT_F32 = 1


def qsa_combine_ranks(part_o, part_lse, out, lse, stream=None):
    """Merge results laid out split-major: part_o [S][nq][hq][256] fp32 and
    part_lse [S][nq][hq] (e.g. one fp32 result per DCP rank, gathered rank-major).
    out: bf16 or fp32 [nq][hq][256]; lse fp32 [nq][hq]."""
    S, nq, hq = (int(x) for x in part_lse.shape)
    _req(part_o, "part_o", torch.float32, (S, nq, hq, HEAD_DIM))
    _req(part_lse, "part_lse", torch.float32, (S, nq, hq))
    if out.dtype not in (torch.bfloat16, torch.float32):
        raise ValueError("out must be bf16 or fp32")
    _req(out, "out", out.dtype, (nq, hq, HEAD_DIM))
    _req(lse, "lse", torch.float32, (nq, hq))
    od = OUT_F32 if out.dtype == torch.float32 else OUT_BF16
    _check("qsa_combine_strided", LIB.qsa_combine_strided(
        _ptr(part_o), _ptr(part_lse), nq, S, hq, hq * HEAD_DIM, nq * hq * HEAD_DIM, hq, nq * hq, _ptr(out), od,
        _ptr(lse), _stream(stream)))


def qsa_combine_f32(part_o, part_lse, out, lse, stream=None):
    """qsa_combine with an fp32 result (part_o [nq][S][hq][256]); the result can
    be one split of a later merge."""
    nq, S, hq = (int(x) for x in part_lse.shape)
    _req(part_o, "part_o", torch.float32, (nq, S, hq, HEAD_DIM))
    _req(part_lse, "part_lse", torch.float32, (nq, S, hq))
    _req(out, "out", torch.float32, (nq, hq, HEAD_DIM))
    _req(lse, "lse", torch.float32, (nq, hq))
    _check("qsa_combine_strided", LIB.qsa_combine_strided(
        _ptr(part_o), _ptr(part_lse), nq, S, hq, S * hq * HEAD_DIM, hq * HEAD_DIM, S * hq, hq, _ptr(out), OUT_F32,
        _ptr(lse), _stream(stream)))


def qsa_dcp_localize_tokens(seq_id, pos, nranks: int, rank: int, interleave_pages: int, seq_id_local, pos_local,
                            stream=None):
    n = int(seq_id.shape[0])
    for t, nm in ((seq_id, "seq_id"), (pos, "pos"), (seq_id_local, "seq_id_local"), (pos_local, "pos_local")):
        _req(t, nm, torch.int32, (n,))
    _check("qsa_dcp_localize_tokens", LIB.qsa_dcp_localize_tokens(
        _ptr(seq_id), _ptr(pos), n, int(nranks), int(rank), int(interleave_pages), _ptr(seq_id_local),
        _ptr(pos_local), _stream(stream)))


def qsa_dcp_localize_selection(sel, count, q_pos, k: int, nranks: int, rank: int, interleave_pages: int, sel_local,
                               count_local, q_pos_local, dev_status=None, stream=None):
    nq = int(q_pos.shape[0])
    _req(sel, "sel", torch.int32, (nq, k))
    _req(sel_local, "sel_local", torch.int32, (nq, k))
    for t, nm in ((count, "count"), (q_pos, "q_pos"), (count_local, "count_local"), (q_pos_local, "q_pos_local")):
        _req(t, nm, torch.int32, (nq,))
    if dev_status is not None:
        _req(dev_status, "dev_status", torch.int32, (1,))
    _check("qsa_dcp_localize_selection", LIB.qsa_dcp_localize_selection(
        _ptr(sel), _ptr(count), _ptr(q_pos), nq, int(k), int(nranks), int(rank), int(interleave_pages),
        _ptr(sel_local), _ptr(count_local), _ptr(q_pos_local), _ptr(dev_status), _stream(stream)))


NOALLOC_SCRATCH_BYTES = 16 << 20


def qsa_sparse_attention_noalloc(cache: PagedCache, q, q_seq, q_pos, sel, count, k: int, scale: float,
                                 chunk_units: int, out, lse, dev_status=None, stream=None):
    """qsa_sparse_decode + qsa_combine for callers that cannot allocate device
    memory: the split partials live in a fixed device array of
    NOALLOC_SCRATCH_BYTES inside libqsa.  Calls on one device share that array,
    so calls that can overlap on the GPU must be ordered (one stream).  The
    first call on each device looks up the array's address; make it before any
    stream capture."""
    nq = int(q_seq.shape[0])
    hq = int(q.shape[1]) if q.dim() == 3 else -1
    _req(q, "q", torch.bfloat16, (nq, hq, HEAD_DIM))
    _req(q_seq, "q_seq", torch.int32, (nq,))
    _req(q_pos, "q_pos", torch.int32, (nq,))
    _req(sel, "sel", torch.int32, (nq, k))
    _req(count, "count", torch.int32, (nq,))
    _req(out, "out", torch.bfloat16, (nq, hq, HEAD_DIM))
    _req(lse, "lse", torch.float32, (nq, hq))
    if dev_status is not None:
        _req(dev_status, "dev_status", torch.int32, (1,))
    _check("qsa_sparse_attention_noalloc", LIB.qsa_sparse_attention_noalloc(
        ctypes.byref(cache.struct()), _ptr(q), nq, hq, _ptr(q_seq), _ptr(q_pos), _ptr(sel), _ptr(count), int(k),
        float(scale), int(chunk_units), _ptr(out), _ptr(lse), _ptr(dev_status), _stream(stream)))


# ----------------------------------------------------------------------------
# pre-bound launches: validate once, then call the C entry point directly


class BoundCall:
    """A C entry point with its arguments marshalled once.  Calling it only
    enqueues the kernels (a few microseconds of host time), so a step of
    several launches keeps the GPU fed.  The tensors must stay alive and
    unchanged in shape while the call is used."""

    def __init__(self, name: str, args: tuple, keep: tuple):
        self.name = name
        self.fn = getattr(LIB, name)
        self.args = args
        self._keep = keep  # tensors / structs referenced by raw pointers

    def __call__(self):
        rc = self.fn(*self.args)
        if rc != QSA_OK:
            raise QSAError(self.name, rc)


def bind_append_kv(cache: PagedCache, k_new, v_new, kidx_new, seq_id, pos, dev_status=None, stream=None):
    n = int(seq_id.shape[0])
    hkv = cache.num_kv_heads
    _req(k_new, "k_new", torch.bfloat16, (n, hkv, HEAD_DIM))
    _req(v_new, "v_new", torch.bfloat16, (n, hkv, HEAD_DIM))
    _req(kidx_new, "kidx_new", torch.bfloat16, (n, IDX_DIM))
    _req(seq_id, "seq_id", torch.int32, (n,))
    _req(pos, "pos", torch.int32, (n,))
    st = cache.struct()
    return BoundCall("qsa_append_kv", (ctypes.byref(st), _ptr(k_new), _ptr(v_new), _ptr(kidx_new), _ptr(seq_id),
                                       _ptr(pos), n, _ptr(dev_status), _stream(stream)),
                     (cache, st, k_new, v_new, kidx_new, seq_id, pos, dev_status))


# ----------------------------------------------------------------------------
# a decode step: its calls on preallocated buffers


class Decoder:
    """Holds the per-step buffers (scores, selection, split partials, outputs) for
    up to `max_nq` queries and runs index_scores -> topk -> sparse_decode ->
    combine on the current stream, with no host synchronisation.

    ``fused=True`` runs the first two as the one fused call qsa_index_topk,
    ``fused=False`` as the two calls; the default chooses the fused call when
    fused_selection_pays(max_nq, ...).  ``merged=True`` runs the last two as
    the one call qsa_sparse_attention (the split kernel merges each pair's
    splits itself), the default ``merged=False`` as qsa_sparse_decode +
    qsa_combine (faster on B200: the merge's fences and L2 round trips in the
    split kernel cost more than the separate launch)."""

    def __init__(self, cache: PagedCache, hq: int, max_nq: int, k: int = 512, scale: float = 1.0 / 16.0,
                 target_ctas: int | None = None, chunk_units: int | None = None, scores_ld: int | None = None,
                 fused: bool | None = None, merged: bool = False):
        dev = cache.device
        self.cache, self.hq, self.k, self.scale, self.max_nq = cache, hq, k, scale, max_nq
        sms = torch.cuda.get_device_properties(dev).multi_processor_count
        if target_ctas is None:
            target_ctas = sms
        self.scores_ld = scores_ld or cache.max_pages_per_seq * BLOCKS_PER_PAGE
        if fused is None:
            fused = fused_default(cache, self.scores_ld, max_nq, sms)
        self.fused = bool(fused)
        if chunk_units is None:
            chunk_units, self.max_splits = qsa_decode_plan(max_nq, cache.num_kv_heads, k, target_ctas)
        else:
            self.max_splits = splits_bound(k, chunk_units)
        self.chunk_units = chunk_units
        self.scores = torch.empty((max_nq, self.scores_ld), dtype=torch.float32, device=dev)
        self.sel = torch.empty((max_nq, k), dtype=torch.int32, device=dev)
        self.count = torch.empty((max_nq,), dtype=torch.int32, device=dev)
        self.part_o = torch.empty((max_nq, self.max_splits, hq, HEAD_DIM), dtype=torch.float32, device=dev)
        self.part_lse = torch.empty((max_nq, self.max_splits, hq), dtype=torch.float32, device=dev)
        # out and lse share one allocation, so a full batch reads back in one copy
        out_bytes = max_nq * hq * HEAD_DIM * 2
        self._out_arena = torch.empty(_align(out_bytes) + max_nq * hq * 4, dtype=torch.uint8, device=dev)
        self.out = self._out_arena[:out_bytes].view(torch.bfloat16).view(max_nq, hq, HEAD_DIM)
        self.lse = self._out_arena[_align(out_bytes):].view(torch.float32).view(max_nq, hq)
        self.merged = bool(merged)
        self.pair_done = torch.zeros((max_nq * cache.num_kv_heads,), dtype=torch.int32, device=dev)
        self.dev_status = torch.zeros((1,), dtype=torch.int32, device=dev)

    def bind(self, q, q_idx, w, q_seq, q_pos, stream=None) -> list:
        """Validate the step inputs once and return the pre-bound launches for
        them: (index_scores, topk, sparse_decode, combine), or (index_topk,
        sparse_decode, combine) when fused."""
        nq = int(q_seq.shape[0])
        assert nq <= self.max_nq
        hq = self.hq
        _req(q_idx, "q_idx", torch.bfloat16, (nq, IDX_HEADS, IDX_DIM))
        _req(w, "w", torch.float32, (nq, IDX_HEADS))
        _req(q_seq, "q_seq", torch.int32, (nq,))
        _req(q_pos, "q_pos", torch.int32, (nq,))
        _req(q, "q", torch.bfloat16, (nq, hq, HEAD_DIM))
        sc, se, cn = self.scores[:nq], self.sel[:nq], self.count[:nq]
        po, pl = self.part_o[:nq], self.part_lse[:nq]
        out, lse = self.out[:nq], self.lse[:nq]
        st = self.cache.struct()
        ds, sp = _ptr(self.dev_status), _stream(stream)
        keep = (self.cache, st, q, q_idx, w, q_seq, q_pos, self.dev_status)
        if self.fused:
            select = [BoundCall("qsa_index_topk", (ctypes.byref(st), _ptr(q_idx), _ptr(w), _ptr(q_seq), _ptr(q_pos),
                                                   nq, self.k, _ptr(sc), int(sc.shape[1]), _ptr(se), _ptr(cn), ds,
                                                   sp), keep)]
        else:
            select = [
                BoundCall("qsa_index_scores", (ctypes.byref(st), _ptr(q_idx), _ptr(w), _ptr(q_seq), _ptr(q_pos), nq,
                                               _ptr(sc), int(sc.shape[1]), ds, sp), keep),
                BoundCall("qsa_topk_blocks", (_ptr(sc), int(sc.shape[1]), _ptr(q_pos), nq, self.k, _ptr(se),
                                              _ptr(cn), ds, sp), keep)]
        if self.merged:
            return select + [
                BoundCall("qsa_sparse_attention", (ctypes.byref(st), _ptr(q), nq, hq, _ptr(q_seq), _ptr(q_pos),
                                                   _ptr(se), _ptr(cn), self.k, float(self.scale), self.chunk_units,
                                                   self.max_splits, _ptr(po), _ptr(pl), _ptr(self.pair_done),
                                                   _ptr(out), _ptr(lse), ds, sp), keep + (self.pair_done,))]
        return select + [
            BoundCall("qsa_sparse_decode", (ctypes.byref(st), _ptr(q), nq, hq, _ptr(q_seq), _ptr(q_pos), _ptr(se),
                                            _ptr(cn), self.k, float(self.scale), self.chunk_units, self.max_splits,
                                            _ptr(po), _ptr(pl), ds, sp), keep),
            BoundCall("qsa_combine", (_ptr(po), _ptr(pl), nq, self.max_splits, hq, _ptr(out), _ptr(lse), sp), keep),
        ]

    def host_outputs(self):
        """Pinned host buffers laid out like the device outputs: (arena, out, lse)."""
        arena = torch.empty(self._out_arena.shape, dtype=torch.uint8).pin_memory()
        out = arena[:self.out.numel() * 2].view(torch.bfloat16).view(self.out.shape)
        lse = arena[self._out_arena.numel() - self.lse.numel() * 4:].view(torch.float32).view(self.lse.shape)
        return arena, out, lse

    def download(self, host, nq: int, stream=None) -> int:
        """Enqueue the device-to-host copy of out[:nq] and lse[:nq] into `host`
        (from host_outputs()): one copy for a full batch, two otherwise.
        Returns the bytes copied."""
        arena, out, lse = host
        s = stream or torch.cuda.current_stream()
        with torch.cuda.stream(s):
            if nq == self.max_nq:
                arena.copy_(self._out_arena, non_blocking=True)
                return arena.numel()
            out[:nq].copy_(self.out[:nq], non_blocking=True)
            lse[:nq].copy_(self.lse[:nq], non_blocking=True)
        return out[:nq].numel() * 2 + lse[:nq].numel() * 4

    def run(self, q, q_idx, w, q_seq, q_pos, stream=None):
        nq = int(q_seq.shape[0])
        assert nq <= self.max_nq
        sc, se, cn = self.scores[:nq], self.sel[:nq], self.count[:nq]
        po, pl = self.part_o[:nq], self.part_lse[:nq]
        if self.fused:
            qsa_index_topk(self.cache, q_idx, w, q_seq, q_pos, self.k, sc, se, cn, self.dev_status, stream)
        else:
            qsa_index_scores(self.cache, q_idx, w, q_seq, q_pos, sc, self.dev_status, stream)
            qsa_topk_blocks(sc, q_pos, self.k, se, cn, self.dev_status, stream)
        if self.merged:
            qsa_sparse_attention(self.cache, q, q_seq, q_pos, se, cn, self.k, self.scale, self.chunk_units,
                                 self.max_splits, po, pl, self.pair_done[:nq * self.cache.num_kv_heads],
                                 self.out[:nq], self.lse[:nq], self.dev_status, stream)
        else:
            qsa_sparse_decode(self.cache, q, q_seq, q_pos, se, cn, self.k, self.scale, self.chunk_units,
                              self.max_splits, po, pl, self.dev_status, stream)
            qsa_combine(po, pl, self.out[:nq], self.lse[:nq], stream)
        return self.out[:nq], self.lse[:nq]


def _align(n: int, a: int = 256) -> int:
    return (n + a - 1) // a * a


class StepIO:
    """The inputs of one step (the appended tokens and the queries) staged in one
    pinned host buffer and one device buffer, 256-byte aligned fields, so that
    sending a step's inputs is a single host-to-device copy.  `host[name]` and
    `dev[name]` are views of the same field; bind the step to the `dev` views,
    fill the `host` views, then upload()."""

    def __init__(self, n_new: int, nq: int, hq: int, hkv: int, device="cuda"):
        fields = [("k_new", torch.bfloat16, (n_new, hkv, HEAD_DIM)), ("v_new", torch.bfloat16, (n_new, hkv, HEAD_DIM)),
                  ("kidx_new", torch.bfloat16, (n_new, IDX_DIM)), ("seq_id", torch.int32, (n_new,)),
                  ("pos", torch.int32, (n_new,)), ("q", torch.bfloat16, (nq, hq, HEAD_DIM)),
                  ("q_idx", torch.bfloat16, (nq, IDX_HEADS, IDX_DIM)), ("w", torch.float32, (nq, IDX_HEADS)),
                  ("q_seq", torch.int32, (nq,)), ("q_pos", torch.int32, (nq,))]
        off, spans = 0, []
        for name, dt, shape in fields:
            nbytes = torch.Size(shape).numel() * torch.empty((), dtype=dt).element_size()
            spans.append((name, dt, shape, off, nbytes))
            off = _align(off + nbytes)
        self.nbytes = off
        self.host_buf = torch.empty(off, dtype=torch.uint8).pin_memory()
        self.dev_buf = torch.empty(off, dtype=torch.uint8, device=device)
        self.host, self.dev = {}, {}
        for name, dt, shape, o, nb in spans:
            self.host[name] = self.host_buf[o:o + nb].view(dt).view(shape)
            self.dev[name] = self.dev_buf[o:o + nb].view(dt).view(shape)

    def upload(self, stream=None):
        """Enqueue the single host-to-device copy of every field."""
        s = stream or torch.cuda.current_stream()
        with torch.cuda.stream(s):
            self.dev_buf.copy_(self.host_buf, non_blocking=True)


class StepGraph:
    """The pre-bound launches of one step captured once into a CUDA graph and
    replayed with a single launch, so a step costs no per-kernel host work.
    The library calls only enqueue kernels (no allocation, no host
    synchronisation), which is what lets them be captured.  The calls must have
    been bound to `stream` (a side stream, not the legacy default stream).

    With ``timing=True`` a timing event is captured before every call and
    after the last one; after a replay, :meth:`kernel_ms` gives each call's
    device time for that replay."""

    def __init__(self, calls, stream: torch.cuda.Stream, timing: bool = False):
        self.calls = list(calls)
        self.stream = stream
        self.events = ([torch.cuda.Event(enable_timing=True, external=True) for _ in range(len(self.calls) + 1)]
                       if timing else None)
        self.graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(self.graph, stream=stream):
            for k, c in enumerate(self.calls):
                if self.events:
                    self.events[k].record(stream)
                c()
            if self.events:
                self.events[-1].record(stream)

    def replay(self):
        """Enqueue one replay on the graph's stream (stream-ordered after the
        work already enqueued there)."""
        with torch.cuda.stream(self.stream):
            self.graph.replay()

    def kernel_ms(self) -> list:
        """Device time of each call in the last replay (synchronises on it)."""
        self.events[-1].synchronize()
        return [self.events[k].elapsed_time(self.events[k + 1]) for k in range(len(self.calls))]


class StepPipeline:
    """Serving-style double buffering of whole steps.  Two slots, each with its
    own staged inputs (a StepIO), Decoder, pinned host outputs and step graph;
    step i runs in slot i % 2.  The inputs of a step go up on one copy stream
    while the previous step computes, and its outputs come back on another
    while the next one computes.  Events order every reuse of a slot:
      upload(i)   after compute(i - 2) has read the slot's inputs,
      compute(i)  after upload(i) and after download(i - 2) has read the
                  slot's outputs,
      download(i) after compute(i).
    `calls[s]` are slot s's pre-bound launches (bound to `compute`, reading
    ios[s].dev and writing decs[s]'s buffers); `before(stream)`, if given,
    enqueues work on the compute stream ahead of every step's graph.  Nothing
    synchronises the host."""

    def __init__(self, ios, decs, calls, compute: torch.cuda.Stream, before=None, nq: int | None = None):
        assert len(ios) == len(decs) == len(calls) == 2
        self.ios, self.decs, self.compute, self.before = ios, decs, compute, before
        self.nq = decs[0].max_nq if nq is None else nq
        self.up_stream = torch.cuda.Stream(device=compute.device)
        self.down_stream = torch.cuda.Stream(device=compute.device)
        self.hosts = [d.host_outputs() for d in decs]
        self.graphs = [StepGraph(c, compute) for c in calls]
        self._up = [torch.cuda.Event() for _ in range(2)]
        self._done = [torch.cuda.Event() for _ in range(2)]
        self._down = [torch.cuda.Event() for _ in range(2)]
        self._used = [False, False]
        self.d2h_bytes = 0

    def step(self, i: int):
        """Enqueue step i (inputs already in ios[i % 2].host)."""
        s = i % 2
        if self._used[s]:
            self.up_stream.wait_event(self._done[s])
        self.ios[s].upload(self.up_stream)
        self._up[s].record(self.up_stream)
        self.compute.wait_event(self._up[s])
        if self._used[s]:
            self.compute.wait_event(self._down[s])
        if self.before is not None:
            self.before(self.compute)
        self.graphs[s].replay()
        self._done[s].record(self.compute)
        self.down_stream.wait_event(self._done[s])
        self.d2h_bytes = self.decs[s].download(self.hosts[s], self.nq, self.down_stream)
        self._down[s].record(self.down_stream)
        self._used[s] = True

    def uploaded(self, i: int) -> bool:
        """Whether step i's inputs have left ios[i % 2].host (the slot's host
        inputs may be refilled for step i + 2 only then)."""
        return self._up[i % 2].query()

    def wait_outputs(self, i: int):
        """Block the host until step i's outputs are in host memory; return them
        as (out, lse).  Step i + 2 reuses the slot's host outputs."""
        self._down[i % 2].synchronize()
        return self.outputs(i)

    def outputs(self, i: int):
        """Host (out, lse) of step i: valid once its download has completed."""
        _, out, lse = self.hosts[i % 2]
        return out, lse


def splits_bound(k: int, chunk_units: int) -> int:
    """Most KV chunks one (query, KV head) pair's k+1 unit slots can touch."""
    return (k + 1 + chunk_units - 2) // chunk_units + 1


def dev_status_names(v: int) -> list[str]:
    return [n for b, n in DEV_BITS.items() if v & b]


def pages_for(tokens: int) -> int:
    return math.ceil(tokens / PAGE_TOKENS)
