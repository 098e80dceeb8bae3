"""ctypes binding of ``libdsa.so`` (C ABI in ``include/dsa.h``).

Argument marshalling only: each function checks dtypes and shapes of the
torch tensors it is given, passes their device pointers and the current CUDA
stream to the C entry point of the same name, and raises ``DSAError`` on a
non-zero status.  Every arithmetic step runs in the library's CUDA kernels;
there is no other implementation behind these names, and a missing library
raises instead of falling back to anything.
"""
from __future__ import annotations

import ctypes
import math
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libdsa.so")
PAGE_SIZE = 64

_lib = None


class DSAError(RuntimeError):
    pass


_P, _I, _I64, _SZ, _F = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_size_t, ctypes.c_float

_SIGNATURES = {
    "dsa_status_string": ([_I], ctypes.c_char_p),
    "dsa_version": ([], _I),
    "dsa_last_error_string": ([], ctypes.c_char_p),
    "dsa_check_device_error": ([], _I),
    "dsa_set_wait_limit_ns": ([ctypes.c_ulonglong], _I),
    "dsa_row_stats_bytes": ([_I], _SZ),
    "dsa_indexer_scores": ([_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _P, _I64, _P, _P], _I),
    "dsa_topk_workspace_size": ([_I, _I, _I], _SZ),
    "dsa_topk": ([_P, _I64, _I, _I, _P, _I, _I, _P, _P, _P, _SZ, _P], _I),
    "dsa_indexer_topk_workspace_size": ([_I, _I, _I, _I, _I], _SZ),
    "dsa_indexer_topk": ([_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _P, _P, _SZ, _P, _P], _I),
    "dsa_indexer_topk_varlen": ([_P, _P, _P, _P, _P, _I, _I, _I, _P, _I, _I, _I, _I, _P, _P, _SZ, _P, _P], _I),
    "dsa_sparse_gqa_prefill_varlen": ([_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _F, _P, _P, _P], _I),
    "dsa_indexer_topk_threshold": ([_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _P, _P, _SZ, _P, _P], _I),
    "dsa_indexer_topk_candidates": ([_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _P, _P, _SZ, _P, _P], _I),
    "dsa_indexer_topk_select": ([_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _P, _P, _SZ, _P, _P], _I),
    "dsa_indexer_kl": ([_P, _I64, _I, _I, _P, _I, _I64, _P, _I, _P, _P, _P], _I),
    "dsa_sparse_gqa_prefill": ([_P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _F, _P, _P, _P], _I),
    "dsa_decode_workspace_size": ([_I, _I, _I, _I, _I, _I], _SZ),
    "dsa_sparse_gqa_decode": ([_P, _P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _P, _I,
                               _I, _I, _I, _I, _I, _I, _I, _F, _P, _SZ, _P, _P, _P], _I),
    "dsa_decode_indexer_scores": ([_P, _P, _P, _P, _P, _P, _I, _I, _P, _I, _I, _I, _I, _P, _I64, _P], _I),
    "dsa_decode_attention_workspace_size": ([_I, _I, _I, _I, _I], _SZ),
    "dsa_sparse_gqa_decode_attention": ([_P, _P, _P, _P, _I, _I, _P, _P, _I, _I, _I, _I, _I, _F,
                                         _P, _SZ, _P, _P, _P], _I),
    "dsa_decode_attention_fixed_scratch_bytes": ([], _SZ),
    "dsa_sparse_gqa_decode_attention_noalloc": ([_P, _P, _P, _P, _I, _I, _P, _P, _I, _I, _I, _I, _I, _F,
                                                 _P, _P, _P], _I),
    "dsa_read_probe": ([_P, _SZ, _I, _P, _P], _I),
}


def lib():
    """Open libdsa.so (once).  Raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise DSAError(f"{LIB_PATH} is missing; build it with `python -m sparse_long_context_03_b200.build`")
        handle = ctypes.CDLL(LIB_PATH)
        for name, (args, res) in _SIGNATURES.items():
            fn = getattr(handle, name)
            fn.argtypes = args
            fn.restype = res
        _lib = handle
    return _lib


def exported_symbols():
    return list(_SIGNATURES)


def version() -> int:
    return lib().dsa_version()


def status_string(code: int) -> str:
    return lib().dsa_status_string(int(code)).decode()


def check_device_error():
    """Synchronises; raises DSAError if a kernel's bounded wait expired."""
    _check(lib().dsa_check_device_error(), "dsa_check_device_error")


def device_error_status() -> int:
    """dsa_check_device_error's status code (0 = none), without raising."""
    return int(lib().dsa_check_device_error())


def set_wait_limit_ns(ns: int) -> None:
    """dsa_set_wait_limit_ns: bound of the prefill indexer's pipeline waits
    on the current device (0 restores the default).  For failure-path tests."""
    _check(lib().dsa_set_wait_limit_ns(int(ns)), "dsa_set_wait_limit_ns")


def _check(code: int, name: str):
    if code != 0:
        err = lib().dsa_last_error_string().decode()
        raise DSAError(f"{name}: {status_string(code)}" + (f" ({err})" if err else ""))


def _ptr(t):
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream):
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _need(t, dtype, ndim, name):
    if t.dtype != dtype:
        raise TypeError(f"{name}: expected {dtype}, got {t.dtype}")
    if t.dim() != ndim:
        raise ValueError(f"{name}: expected {ndim} dims, got shape {tuple(t.shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name}: must be contiguous")
    if not t.is_cuda:
        raise ValueError(f"{name}: must be a CUDA tensor")


# ---------------------------------------------------------------------------
# prefill
# ---------------------------------------------------------------------------

def row_stats_bytes(n_rows) -> int:
    return int(lib().dsa_row_stats_bytes(int(n_rows)))


def indexer_scores(q8, q_scale, w, k8, k_scale, row_begin, n_rows, scores, row_stats=None, stream=None):
    """dsa_indexer_scores: rows [row_begin, row_begin+n_rows) of the causal
    lightning-indexer score matrix into ``scores`` [n_rows, ld] float32;
    optionally the rows' value ranges into ``row_stats`` for dsa_topk."""
    _need(q8, torch.uint8, 3, "q8")
    _need(k8, torch.uint8, 2, "k8")
    _need(scores, torch.float32, 2, "scores")
    L, HI, dI = q8.shape
    _check(lib().dsa_indexer_scores(_ptr(q8), _ptr(q_scale), _ptr(w), _ptr(k8), _ptr(k_scale), L, HI, dI,
                                    int(row_begin), int(n_rows), _ptr(scores), scores.stride(0), _ptr(row_stats),
                                    _stream(stream)),
           "dsa_indexer_scores")


def topk_workspace_size(n_rows, max_len, k) -> int:
    return int(lib().dsa_topk_workspace_size(int(n_rows), int(max_len), int(k)))


def topk(scores, row_begin, n_rows, k, idx, row_len=None, max_len=None, ws=None, row_stats=None, stream=None):
    """dsa_topk: per-row top-k (ascending indices, -1 padded) into idx [n_rows, k]."""
    _need(scores, torch.float32, 2, "scores")
    _need(idx, torch.int32, 2, "idx")
    if max_len is None:
        max_len = scores.shape[1] if row_len is not None else row_begin + n_rows
    need = topk_workspace_size(n_rows, max_len, k)
    ws_bytes = 0
    if need:
        if ws is None:
            raise DSAError(f"dsa_topk needs a {need}-byte workspace")
        ws_bytes = ws.numel() * ws.element_size()
    _check(lib().dsa_topk(_ptr(scores), scores.stride(0), int(row_begin), int(n_rows), _ptr(row_len), int(max_len),
                          int(k), _ptr(idx), _ptr(row_stats), _ptr(ws), ws_bytes, _stream(stream)), "dsa_topk")


def indexer_topk_workspace_size(row_begin, n_rows, k, HI, dI) -> int:
    return int(lib().dsa_indexer_topk_workspace_size(int(row_begin), int(n_rows), int(k), int(HI), int(dI)))


_TOPK_STAGES = {None: "dsa_indexer_topk", "threshold": "dsa_indexer_topk_threshold",
                "candidates": "dsa_indexer_topk_candidates", "select": "dsa_indexer_topk_select"}


def indexer_topk(q8, q_scale, w, k8, k_scale, row_begin, n_rows, k, idx, ws, stats=None, stream=None,
                 stage=None):
    """dsa_indexer_topk: Omega_t of query rows [row_begin, row_begin+n_rows)
    (the top-k of their causal indexer scores, ascending, -1 padded) into
    idx [n_rows, k] int32, without writing the score matrix.  ``ws`` is a
    uint8 CUDA tensor of indexer_topk_workspace_size(...) bytes or more;
    ``stats`` (optional int64 CUDA tensor of 2) receives the number of rows
    scored again in full and the number of candidates kept.  ``stage`` = "threshold", "candidates" or "select"
    runs one stage only (dsa_indexer_topk_<stage>)."""
    _need(q8, torch.uint8, 3, "q8")
    _need(k8, torch.uint8, 2, "k8")
    _need(idx, torch.int32, 2, "idx")
    name = _TOPK_STAGES[stage]
    L, HI, dI = q8.shape
    _check(getattr(lib(), name)(_ptr(q8), _ptr(q_scale), _ptr(w), _ptr(k8), _ptr(k_scale), L, HI, dI,
                                int(row_begin), int(n_rows), int(k), _ptr(idx), _ptr(ws),
                                ws.numel() * ws.element_size(), _ptr(stats), _stream(stream)), name)


def indexer_kl(scores, row_begin, n_rows, p, loss_rows, idx=None, loss_total=None, stream=None):
    """dsa_indexer_kl: per-row indexer distillation loss
    sum_g KL(p[r,g,S] normalised || Softmax(I[t,S])) into loss_rows [n_rows]
    float64; S = [0, t] (idx None: dense warm-up) or the valid entries of idx
    row r (sparse adaptation).  scores [n_rows, ld] float32, p [n_rows, G,
    ld_p] float32; loss_total (optional, 1 float64) gets the sum."""
    _need(scores, torch.float32, 2, "scores")
    _need(p, torch.float32, 3, "p")
    _need(loss_rows, torch.float64, 1, "loss_rows")
    k = 0
    if idx is not None:
        _need(idx, torch.int32, 2, "idx")
        k = idx.shape[1]
    _check(lib().dsa_indexer_kl(_ptr(scores), scores.stride(0), int(row_begin), int(n_rows), _ptr(p), p.shape[1],
                                p.stride(1), _ptr(idx), k, _ptr(loss_rows), _ptr(loss_total), _stream(stream)),
           "dsa_indexer_kl")


def sparse_gqa_prefill(Q, K, V, idx, row_begin, n_rows, k, sm_scale, O, lse=None, stream=None):
    """dsa_sparse_gqa_prefill: attention of query rows [row_begin, row_begin+n_rows)
    over their selected keys.  Q/O [n_rows,Hq,D] bf16, K/V [L,Hkv,D] bf16."""
    for t, n in ((Q, "Q"), (K, "K"), (V, "V"), (O, "O")):
        _need(t, torch.bfloat16, 3, n)
    _need(idx, torch.int32, 2, "idx")
    Hq, D = Q.shape[1], Q.shape[2]
    Hkv = K.shape[1]
    _check(lib().dsa_sparse_gqa_prefill(_ptr(Q), _ptr(K), _ptr(V), _ptr(idx), int(row_begin), int(n_rows), Hq, Hkv,
                                        D, int(k), float(sm_scale), _ptr(O), _ptr(lse), _stream(stream)),
           "dsa_sparse_gqa_prefill")


def indexer_topk_varlen(q8, q_scale, w, k8, k_scale, cu_seqlens, row_begin, n_rows, k, idx, ws, stats=None,
                        stream=None):
    """dsa_indexer_topk_varlen: Omega_t of packed query rows [row_begin,
    row_begin+n_rows); cu_seqlens int32 CUDA tensor [nseq+1].  idx [n_rows,
    k] receives positions within each query's own sequence."""
    _need(q8, torch.uint8, 3, "q8")
    _need(k8, torch.uint8, 2, "k8")
    _need(idx, torch.int32, 2, "idx")
    _need(cu_seqlens, torch.int32, 1, "cu_seqlens")
    L, HI, dI = q8.shape
    _check(lib().dsa_indexer_topk_varlen(_ptr(q8), _ptr(q_scale), _ptr(w), _ptr(k8), _ptr(k_scale), L, HI, dI,
                                         _ptr(cu_seqlens), cu_seqlens.numel() - 1, int(row_begin), int(n_rows), int(k),
                                         _ptr(idx), _ptr(ws), ws.numel() * ws.element_size(), _ptr(stats),
                                         _stream(stream)), "dsa_indexer_topk_varlen")


def sparse_gqa_prefill_varlen(Q, K, V, idx, cu_seqlens, row_begin, n_rows, k, sm_scale, O, lse=None, stream=None):
    """dsa_sparse_gqa_prefill_varlen: attention of packed query rows over
    their selected positions (relative to each query's own sequence)."""
    for t, n in ((Q, "Q"), (K, "K"), (V, "V"), (O, "O")):
        _need(t, torch.bfloat16, 3, n)
    _need(idx, torch.int32, 2, "idx")
    _need(cu_seqlens, torch.int32, 1, "cu_seqlens")
    Hq, D = Q.shape[1], Q.shape[2]
    Hkv = K.shape[1]
    _check(lib().dsa_sparse_gqa_prefill_varlen(_ptr(Q), _ptr(K), _ptr(V), _ptr(idx), _ptr(cu_seqlens),
                                               cu_seqlens.numel() - 1, int(row_begin), int(n_rows), Hq, Hkv, D,
                                               int(k), float(sm_scale), _ptr(O), _ptr(lse), _stream(stream)),
           "dsa_sparse_gqa_prefill_varlen")


class PrefillPlan:
    """Buffers for a prefill of one sequence.

    fused=True (the default where the shape allows it): the fused indexer +
    top-k (dsa_indexer_topk), whose workspace holds sampled scores,
    thresholds and candidate lists instead of the score matrix; query rows
    are chunked only to keep that workspace within ``fused_budget_bytes``.
    fused=False: the score matrix of one chunk of query rows at a time
    ([chunk_rows, ld] float32, the chunked indexer of report section 5.2.1),
    then dsa_topk."""

    def __init__(self, L, HI, dI, Hq, Hkv, D, k, chunk_rows=None, device="cuda", score_budget_bytes=4 << 30,
                 fused=None, fused_budget_bytes=24 << 30):
        self.L, self.HI, self.dI, self.Hq, self.Hkv, self.D, self.k = L, HI, dI, Hq, Hkv, D, k
        self.ld = (L + 3) // 4 * 4
        if fused is None:
            fused = indexer_topk_workspace_size(0, 1, k, HI, dI) > 0
        self.fused = bool(fused)
        self.idx = torch.empty(L, k, dtype=torch.int32, device=device)
        if self.fused:
            if chunk_rows is None:
                chunk_rows = L
                while chunk_rows > 1 and self._fused_ws(chunk_rows) > fused_budget_bytes:
                    chunk_rows = (chunk_rows + 1) // 2
            self.chunk_rows = int(chunk_rows)
            self.scores = None
            self.row_stats = None
            self.ws = torch.empty(max(self._fused_ws(self.chunk_rows), 1), dtype=torch.uint8, device=device)
            self.stats = torch.zeros(2, dtype=torch.int64, device=device)
        else:
            if chunk_rows is None:
                chunk_rows = max(1, min(L, score_budget_bytes // (4 * self.ld)))
            self.chunk_rows = int(chunk_rows)
            self.scores = torch.empty(self.chunk_rows, self.ld, dtype=torch.float32, device=device)
            need = topk_workspace_size(self.chunk_rows, L, k)
            self.ws = torch.empty(max(need, 1), dtype=torch.uint8, device=device) if need else None
            self.row_stats = torch.empty(row_stats_bytes(self.chunk_rows), dtype=torch.uint8, device=device)
            self.stats = None

    def _fused_ws(self, chunk_rows):
        # the workspace grows with the chunk's last row, so the last chunk needs the most
        need = 0
        for r0 in range(0, self.L, chunk_rows):
            need = max(need, indexer_topk_workspace_size(r0, min(chunk_rows, self.L - r0), self.k, self.HI, self.dI))
        return need

    def chunks(self):
        for r0 in range(0, self.L, self.chunk_rows):
            yield r0, min(self.chunk_rows, self.L - r0)


def select_rows(plan: PrefillPlan, q8, sq, w, k8, sk, stream=None):
    """Omega_t of every query row into plan.idx [L, k]: the fused indexer +
    top-k, or the chunked score matrix followed by dsa_topk."""
    for r0, n in plan.chunks():
        if plan.fused:
            indexer_topk(q8, sq, w, k8, sk, r0, n, plan.k, plan.idx[r0:r0 + n], plan.ws, stream=stream)
        else:
            indexer_scores(q8, sq, w, k8, sk, r0, n, plan.scores[:n], row_stats=plan.row_stats, stream=stream)
            topk(plan.scores[:n], r0, n, plan.k, plan.idx[r0:r0 + n], max_len=r0 + n, ws=plan.ws,
                 row_stats=plan.row_stats, stream=stream)


def prefill_forward(plan: PrefillPlan, q8, sq, w, k8, sk, Q, K, V, O, sm_scale=None, lse=None, stream=None):
    """Whole DSA prefill of one sequence: Omega_t of every query row (the
    indexer and the top-k), then the sparse attention of every row.
    Writes plan.idx [L,k] and O [L,Hq,D] (lse [L,Hq] if given)."""
    if sm_scale is None:
        sm_scale = 1.0 / math.sqrt(plan.D)
    select_rows(plan, q8, sq, w, k8, sk, stream=stream)
    sparse_gqa_prefill(Q, K, V, plan.idx, 0, plan.L, plan.k, sm_scale, O, lse, stream=stream)


def prefill_forward_packed(plan: PrefillPlan, cu_seqlens, q8, sq, w, k8, sk, Q, K, V, O, sm_scale=None, lse=None,
                           idx_out=None, stream=None):
    """DSA prefill of several sequences packed along the token axis: sequence
    b holds tokens cu_seqlens[b] .. cu_seqlens[b+1]-1 and is its own causal
    prefill -- no query scores or attends a key of another sequence.  Every
    per-token tensor (q8, sq, w, k8, sk, Q, K, V, O, lse) is indexed by the
    packed token.  idx_out, if given, [total, k] int32, receives each token's
    selected positions within its own sequence.

    With the fused indexer + top-k (plan.fused; the plan sized for the
    packed total), every stage is one launch per chunk of packed rows over
    all sequences at once (dsa_indexer_topk_varlen,
    dsa_sparse_gqa_prefill_varlen; cu_seqlens as a host sequence or an int32
    CUDA tensor).  Otherwise (HI = 4) the score-matrix chain runs once per
    sequence on its slice (cu_seqlens host ints; the plan sized for the
    longest sequence)."""
    cu = [int(x) for x in (cu_seqlens.tolist() if isinstance(cu_seqlens, torch.Tensor) else cu_seqlens)]
    if any(b < a for a, b in zip(cu, cu[1:])) or (cu and cu[0] != 0):
        raise DSAError("cu_seqlens must start at 0 and be non-decreasing")
    if sm_scale is None:
        sm_scale = 1.0 / math.sqrt(plan.D)
    total = cu[-1] if cu else 0
    if plan.fused:
        if total > plan.L:
            raise DSAError("the packed tokens exceed the plan")
        cu_dev = cu_seqlens if isinstance(cu_seqlens, torch.Tensor) and cu_seqlens.is_cuda else \
            torch.tensor(cu, dtype=torch.int32, device=q8.device)
        idx = plan.idx[:total] if idx_out is None else idx_out
        for r0 in range(0, total, plan.chunk_rows):
            n = min(plan.chunk_rows, total - r0)
            indexer_topk_varlen(q8, sq, w, k8, sk, cu_dev, r0, n, plan.k, idx[r0:r0 + n], plan.ws, stream=stream)
        sparse_gqa_prefill_varlen(Q, K, V, idx, cu_dev, 0, total, plan.k, sm_scale, O, lse, stream=stream)
        return
    if max((b - a for a, b in zip(cu, cu[1:])), default=0) > plan.L:
        raise DSAError("a sequence is longer than the plan")
    for s0, s1 in zip(cu, cu[1:]):
        n_tok = s1 - s0
        if n_tok == 0:
            continue
        sl = slice(s0, s1)
        for r0 in range(0, n_tok, plan.chunk_rows):
            n = min(plan.chunk_rows, n_tok - r0)
            indexer_scores(q8[sl], sq[sl], w[sl], k8[sl], sk[sl], r0, n, plan.scores[:n], row_stats=plan.row_stats,
                           stream=stream)
            topk(plan.scores[:n], r0, n, plan.k, plan.idx[r0:r0 + n], max_len=r0 + n, ws=plan.ws,
                 row_stats=plan.row_stats, stream=stream)
        sparse_gqa_prefill(Q[sl], K[sl], V[sl], plan.idx[:n_tok], 0, n_tok, plan.k, sm_scale, O[sl],
                           None if lse is None else lse[sl], stream=stream)
        if idx_out is not None:
            idx_out[sl].copy_(plan.idx[:n_tok])


# ---------------------------------------------------------------------------
# decode
# ---------------------------------------------------------------------------

def decode_workspace_size(B, max_seq_len, Hq, Hkv, D, k) -> int:
    return int(lib().dsa_decode_workspace_size(int(B), int(max_seq_len), int(Hq), int(Hkv), int(D), int(k)))


def decode_attention_workspace_size(B, Hq, Hkv, D, k) -> int:
    return int(lib().dsa_decode_attention_workspace_size(int(B), int(Hq), int(Hkv), int(D), int(k)))


def decode_indexer_scores(q8, q_scale, w, k8_cache, k_scale_cache, block_table, seq_lens, max_seq_len, scores,
                          stream=None):
    _need(q8, torch.uint8, 3, "q8")
    _need(k8_cache, torch.uint8, 3, "k8_cache")
    _need(block_table, torch.int32, 2, "block_table")
    _need(scores, torch.float32, 2, "scores")
    B, HI, dI = q8.shape
    _check(lib().dsa_decode_indexer_scores(_ptr(q8), _ptr(q_scale), _ptr(w), _ptr(k8_cache), _ptr(k_scale_cache),
                                           _ptr(block_table), block_table.shape[1], k8_cache.shape[0],
                                           _ptr(seq_lens), int(max_seq_len), B, HI, dI, _ptr(scores),
                                           scores.stride(0), _stream(stream)), "dsa_decode_indexer_scores")


def sparse_gqa_decode_attention(q, k_cache, v_cache, block_table, seq_lens, idx, k, sm_scale, ws, out, lse=None,
                                stream=None):
    _need(q, torch.bfloat16, 3, "q")
    _need(k_cache, torch.bfloat16, 4, "k_cache")
    _need(v_cache, torch.bfloat16, 4, "v_cache")
    _need(out, torch.bfloat16, 3, "out")
    B, Hq, D = q.shape
    Hkv = k_cache.shape[2]
    _check(lib().dsa_sparse_gqa_decode_attention(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_table),
                                                 block_table.shape[1], k_cache.shape[0], _ptr(seq_lens), _ptr(idx),
                                                 B, Hq, Hkv, D, int(k), float(sm_scale), _ptr(ws),
                                                 ws.numel() * ws.element_size(), _ptr(out), _ptr(lse),
                                                 _stream(stream)), "dsa_sparse_gqa_decode_attention")


def sparse_gqa_decode(q, q8, q_scale, w, k8_cache, k_scale_cache, k_cache, v_cache, block_table, seq_lens,
                      max_seq_len, k, sm_scale, ws, out, idx_out=None, stream=None):
    """dsa_sparse_gqa_decode: indexer -> top-k -> attention for one new token per sequence."""
    _need(q, torch.bfloat16, 3, "q")
    _need(q8, torch.uint8, 3, "q8")
    _need(k_cache, torch.bfloat16, 4, "k_cache")
    _need(block_table, torch.int32, 2, "block_table")
    _need(out, torch.bfloat16, 3, "out")
    B, Hq, D = q.shape
    HI, dI = q8.shape[1], q8.shape[2]
    Hkv = k_cache.shape[2]
    _check(lib().dsa_sparse_gqa_decode(_ptr(q), _ptr(q8), _ptr(q_scale), _ptr(w), _ptr(k8_cache),
                                       _ptr(k_scale_cache), _ptr(k_cache), _ptr(v_cache), _ptr(block_table),
                                       block_table.shape[1], k_cache.shape[0], _ptr(seq_lens), int(max_seq_len), B,
                                       Hq, Hkv, D, HI, dI, int(k), float(sm_scale), _ptr(ws),
                                       ws.numel() * ws.element_size(), _ptr(out), _ptr(idx_out), _stream(stream)),
           "dsa_sparse_gqa_decode")


def decode_attention_fixed_scratch_bytes() -> int:
    return int(lib().dsa_decode_attention_fixed_scratch_bytes())


def sparse_gqa_decode_attention_noalloc(q, k_cache, v_cache, block_table, seq_lens, idx, k, sm_scale, out, lse=None,
                                        stream=None):
    """dsa_sparse_gqa_decode_attention_noalloc: the decode attention with no
    caller workspace (its scratch is a fixed array inside the library).  For
    callers that cannot allocate device memory; calls that overlap on one
    GPU race on that array."""
    _need(q, torch.bfloat16, 3, "q")
    _need(k_cache, torch.bfloat16, 4, "k_cache")
    _need(v_cache, torch.bfloat16, 4, "v_cache")
    _need(out, torch.bfloat16, 3, "out")
    B, Hq, D = q.shape
    Hkv = k_cache.shape[2]
    _check(lib().dsa_sparse_gqa_decode_attention_noalloc(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_table),
                                                         block_table.shape[1], k_cache.shape[0], _ptr(seq_lens),
                                                         _ptr(idx), B, Hq, Hkv, D, int(k), float(sm_scale),
                                                         _ptr(out), _ptr(lse), _stream(stream)),
           "dsa_sparse_gqa_decode_attention_noalloc")


# ---------------------------------------------------------------------------
# diagnostics
# ---------------------------------------------------------------------------

def read_probe(buf, reps, sink, stream=None):
    """dsa_read_probe: read ``buf`` (a contiguous CUDA tensor, 16-byte
    multiple) ``reps`` times with L2-only 16-byte loads.  For timing the
    memory system's read bandwidth; ``sink`` is a small CUDA tensor the kernel
    may write."""
    if not buf.is_cuda or not buf.is_contiguous():
        raise ValueError("buf must be a contiguous CUDA tensor")
    _check(lib().dsa_read_probe(_ptr(buf), buf.numel() * buf.element_size(), int(reps), _ptr(sink),
                                _stream(stream)), "dsa_read_probe")
