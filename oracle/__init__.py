"""fp64 CPU oracle for the GQA-adapted DeepSeek Sparse Attention layer.

TEST INFRASTRUCTURE ONLY.  The product path (the CUDA library and its
binding) never imports, links or runs anything here; only ``tests/``,
``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py`` do.  The
oracle and the CUDA path share no code: they meet only through the seeded
input tensors of ``sparse_long_context_03_b200.inputs``.

The arithmetic lives in ``dsa_oracle.c`` (plain C, fp64, OpenMP over rows);
this module compiles it with gcc and wraps it for numpy arrays.  Each function
states the passage of the pages it follows:

* indexer  -- "Kwai Keye-VL-2.0 Technical Report" review (xllm-io), 核心公式,
  lightning-indexer score; report translation section 2.3.1.
* topk     -- same formula block, the top-k set Omega_t; report sections 2.3.1,
  5.1.2 (rows below k keep all of [0, t]) and 5.2.1 (deterministic top-k).
* attention -- same formula block, GQA sparse aggregation u_{t,g}; report
  section 2.3.2 (one index set for every group).
* indexer_kl -- same formula block, the dense warm-up and sparse adaptation
  losses of the indexer; report section 2.3.3.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "dsa_oracle.c")
_LIB = os.path.join(_HERE, "libdsa_oracle.so")
_lib = None

PAGE_SIZE = 64


def build(force: bool = False) -> str:
    """Compile the oracle into ``oracle/libdsa_oracle.so`` (gcc, -O2, OpenMP).

    ``DSA_ORACLE_LIB`` names another build of the same source to load instead;
    the mutation test uses it to load copies with planted mistakes."""
    override = os.environ.get("DSA_ORACLE_LIB")
    if override:
        return override
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared",
                               "-fvisibility=hidden", "-Wall", "-Wextra", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        P = ctypes.c_void_p
        I = ctypes.c_int
        I64 = ctypes.c_int64
        D = ctypes.c_double
        lib.dsa_oracle_e4m3_to_double.argtypes = [ctypes.c_uint8]
        lib.dsa_oracle_e4m3_to_double.restype = D
        lib.dsa_oracle_bf16_to_double.argtypes = [ctypes.c_uint16]
        lib.dsa_oracle_bf16_to_double.restype = D
        lib.dsa_oracle_max_threads.restype = I
        lib.dsa_oracle_set_threads.argtypes = [I]
        lib.dsa_oracle_indexer.argtypes = [P, P, P, P, P, I, I, I, I, I, P, I64]
        lib.dsa_oracle_topk.argtypes = [P, I64, P, I, I, P]
        lib.dsa_oracle_sparse_attention.argtypes = [P, P, P, P, I, I, I, I, I, I, D, P, P]
        lib.dsa_oracle_decode_indexer.argtypes = [P, P, P, P, P, P, I, I, I, P, I, I, I, P, I64]
        lib.dsa_oracle_decode_attention.argtypes = [P, P, P, P, I, I, I, P, P, I, I, I, I, I, D, P, P]
        lib.dsa_oracle_indexer_kl.argtypes = [P, I64, I, I, P, I, I64, P, I, P, P]
        for f in ("dsa_oracle_indexer", "dsa_oracle_topk", "dsa_oracle_sparse_attention",
                  "dsa_oracle_decode_indexer", "dsa_oracle_decode_attention", "dsa_oracle_indexer_kl"):
            getattr(lib, f).restype = I
        _lib = lib
    return _lib


def _c(a, dtype):
    """Contiguous numpy array of exactly ``dtype`` (bit patterns kept)."""
    a = np.asarray(a)
    if a.dtype != dtype:
        if a.dtype.itemsize == np.dtype(dtype).itemsize and a.dtype.kind in "ui" and np.dtype(dtype).kind in "ui":
            a = a.view(dtype)
        else:
            a = a.astype(dtype)
    return np.ascontiguousarray(a)


def _p(a):
    return a.ctypes.data_as(ctypes.c_void_p)


def _check(rc, what):
    if rc != 0:
        raise ValueError(f"oracle {what}: invalid arguments")


def threads() -> int:
    return _load().dsa_oracle_max_threads()


def set_threads(n: int) -> None:
    _load().dsa_oracle_set_threads(int(n))


def e4m3_to_double(b: int) -> float:
    """OCP e4m3fn byte -> real value (NaN for S.1111.111)."""
    return _load().dsa_oracle_e4m3_to_double(int(b) & 0xFF)


def bf16_to_double(h: int) -> float:
    return _load().dsa_oracle_bf16_to_double(int(h) & 0xFFFF)


def indexer(q8, sq, w, k8, sk, row_begin: int = 0, n_rows: int | None = None) -> np.ndarray:
    """Lightning-indexer scores I[t, s] = sum_j w[t,j] ReLU(qI[t,j] . kI[s]).

    q8 [L,HI,dI] / k8 [L,dI] are e4m3 bytes, sq / sk per-token scales, w [L,HI].
    Returns float64 [n_rows, row_begin+n_rows]; entries with s > t are -inf.
    """
    q8 = _c(q8, np.uint8)
    k8 = _c(k8, np.uint8)
    sq = _c(sq, np.float32)
    sk = _c(sk, np.float32)
    w = _c(w, np.float32)
    L, HI, dI = q8.shape
    if n_rows is None:
        n_rows = L - row_begin
    ld = row_begin + n_rows
    out = np.empty((n_rows, ld), np.float64)
    _check(_load().dsa_oracle_indexer(_p(q8), _p(sq), _p(w), _p(k8), _p(sk), L, HI, dI,
                                      row_begin, n_rows, _p(out), ld), "indexer")
    return out


def topk(scores, row_len, k: int) -> np.ndarray:
    """Top-k per row: descending score, ties to the lower index, output
    ascending and padded with -1; rows with row_len <= k keep all of [0, row_len)."""
    scores = _c(scores, np.float64)
    if scores.ndim == 1:
        scores = scores[None, :]
    n_rows, ld = scores.shape
    row_len = _c(np.broadcast_to(np.asarray(row_len), (n_rows,)), np.int32)
    idx = np.empty((n_rows, k), np.int32)
    _check(_load().dsa_oracle_topk(_p(scores), ld, _p(row_len), n_rows, k, _p(idx)), "topk")
    return idx


def causal_topk(scores, row_begin: int, k: int) -> np.ndarray:
    """Top-k of prefill rows: row r is query t = row_begin + r with t+1 keys."""
    n_rows = np.asarray(scores).shape[0]
    return topk(scores, np.arange(row_begin + 1, row_begin + n_rows + 1), k)


def sparse_attention(Q, K, V, idx, row_begin: int, sm_scale: float):
    """O[t,h] = softmax over s in Omega_t of sm_scale*Q[t,h].K[s,g] times V[s,g].

    Q [n_rows,Hq,D], K/V [>=row_begin+n_rows,Hkv,D] as bf16 bit patterns
    (uint16 or int16 arrays), idx [n_rows,k].  Returns (O float64, lse float64).
    """
    Q = _c(Q, np.uint16)
    K = _c(K, np.uint16)
    V = _c(V, np.uint16)
    idx = _c(idx, np.int32)
    n_rows, Hq, D = Q.shape
    Hkv = K.shape[1]
    k = idx.shape[1]
    O = np.empty((n_rows, Hq, D), np.float64)
    lse = np.empty((n_rows, Hq), np.float64)
    _check(_load().dsa_oracle_sparse_attention(_p(Q), _p(K), _p(V), _p(idx), row_begin, n_rows,
                                               Hq, Hkv, D, k, float(sm_scale), _p(O), _p(lse)),
           "sparse_attention")
    return O, lse


def decode_indexer(q8, sq, w, k8_cache, sk_cache, block_table, seq_lens, ld: int | None = None):
    """Paged decode indexer; returns float64 [B, ld], -inf past each seq_len
    and for tokens whose page id is not a page of the cache."""
    q8 = _c(q8, np.uint8)
    sq = _c(sq, np.float32)
    w = _c(w, np.float32)
    k8_cache = _c(k8_cache, np.uint8)
    sk_cache = _c(sk_cache, np.float32)
    block_table = _c(block_table, np.int32)
    seq_lens = _c(seq_lens, np.int32)
    B, HI, dI = q8.shape
    page = k8_cache.shape[1]
    max_pages = block_table.shape[1]
    if ld is None:
        ld = int(seq_lens.max()) if B else 1
    out = np.empty((B, ld), np.float64)
    _check(_load().dsa_oracle_decode_indexer(_p(q8), _p(sq), _p(w), _p(k8_cache), _p(sk_cache),
                                             _p(block_table), max_pages, page, k8_cache.shape[0], _p(seq_lens),
                                             B, HI, dI,
                                             _p(out), ld), "decode_indexer")
    return out


def decode_attention(q, k_cache, v_cache, block_table, seq_lens, idx, sm_scale: float):
    """Paged decode attention; returns (out float64 [B,Hq,D], lse float64 [B,Hq])."""
    q = _c(q, np.uint16)
    k_cache = _c(k_cache, np.uint16)
    v_cache = _c(v_cache, np.uint16)
    block_table = _c(block_table, np.int32)
    seq_lens = _c(seq_lens, np.int32)
    idx = _c(idx, np.int32)
    B, Hq, D = q.shape
    page, Hkv = k_cache.shape[1], k_cache.shape[2]
    max_pages = block_table.shape[1]
    k = idx.shape[1]
    out = np.empty((B, Hq, D), np.float64)
    lse = np.empty((B, Hq), np.float64)
    _check(_load().dsa_oracle_decode_attention(_p(q), _p(k_cache), _p(v_cache), _p(block_table), max_pages,
                                               page, k_cache.shape[0], _p(seq_lens), _p(idx), B, Hq, Hkv, D, k,
                                               float(sm_scale), _p(out), _p(lse)), "decode_attention")
    return out, lse


def indexer_kl(I, p, row_begin: int = 0, idx=None):
    """Indexer distillation loss per query row ("Kwai Keye-VL-2.0 Technical
    Report" review, 核心公式, dense warm-up / sparse adaptation losses;
    report translation section 2.3.3):
        sum_g KL( p[t,S,g] / sum_S p[t,S,g]  ||  Softmax(I[t,S]) )
    with S = [0, t] (idx None: dense warm-up) or the valid entries of idx
    row r (sparse adaptation).  I [n_rows, >= row_begin+n_rows] scores,
    p [n_rows, G, >= row_begin+n_rows] non-negative target weights.
    Returns (loss per row float64 [n_rows], total)."""
    I = _c(I, np.float64)
    p = _c(p, np.float64)
    n_rows, ld_I = I.shape
    _, G, ld_p = p.shape
    k = 0
    if idx is not None:
        idx = _c(idx, np.int32)
        k = idx.shape[1]
    loss = np.empty(n_rows, np.float64)
    total = np.empty(1, np.float64)
    _check(_load().dsa_oracle_indexer_kl(_p(I), ld_I, row_begin, n_rows, _p(p), G, ld_p,
                                         None if idx is None else _p(idx), k, _p(loss), _p(total)), "indexer_kl")
    return loss, float(total[0])


def prefill(q8, sq, w, k8, sk, Q, K, V, k: int, sm_scale: float, rows=None):
    """The whole prefill chain on selected query rows (default: all rows).

    Returns (scores list per row, idx [n,k], O [n,Hq,D], lse [n,Hq]) for the
    rows in ``rows`` (absolute query positions)."""
    L = np.asarray(q8).shape[0]
    rows = list(range(L)) if rows is None else [int(r) for r in rows]
    idx = np.empty((len(rows), k), np.int32)
    Os, lses, scs = [], [], []
    Qn = _c(Q, np.uint16)
    for i, t in enumerate(rows):
        sc = indexer(q8, sq, w, k8, sk, row_begin=t, n_rows=1)
        scs.append(sc[0, : t + 1])
        idx[i] = topk(sc, [t + 1], k)[0]
        O, lse = sparse_attention(Qn[t: t + 1], K, V, idx[i: i + 1], t, sm_scale)
        Os.append(O[0])
        lses.append(lse[0])
    return scs, idx, np.stack(Os), np.stack(lses)
