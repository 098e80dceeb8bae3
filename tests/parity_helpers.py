"""Comparison helpers for the GPU parity tests.

Tolerances follow the correctness criteria of the layer (stated per check):
  * indexer scores: |gpu - oracle| <= 1e-3 * |oracle| + 1e-6 * max_s |oracle[t, s]|
    (the absolute floor covers scores that the ReLU makes exactly zero);
  * top-k on random inputs: identical sets except for indices whose oracle
    score lies within 1e-5 relative (plus 1e-7 * max |I| absolute) of the
    oracle's k-th score; bit-exact on exact-arithmetic inputs;
  * attention output (bf16) vs fp64: max-abs 2e-2; lse: 1e-3 absolute.
"""
import numpy as np

SCORE_RTOL = 1e-3
SCORE_ATOL_REL_MAX = 1e-6
TOPK_REL = 1e-5
TOPK_ABS_REL_MAX = 1e-7
ATTN_MAX_ABS = 2e-2
LSE_ATOL = 1e-3


def check_scores(gpu_row, oracle_row, what=""):
    gpu_row = np.asarray(gpu_row, np.float64)
    oracle_row = np.asarray(oracle_row, np.float64)
    assert gpu_row.shape == oracle_row.shape
    tol = SCORE_RTOL * np.abs(oracle_row) + SCORE_ATOL_REL_MAX * np.max(np.abs(oracle_row))
    bad = np.abs(gpu_row - oracle_row) > tol
    assert not bad.any(), f"{what}: {bad.sum()} scores out of tolerance, first at {np.argmax(bad)}"


def check_topk_structure(row, n, k):
    cnt = min(n, k)
    assert np.all(row[cnt:] == -1), "padding must be -1"
    sel = row[:cnt]
    assert np.all(sel >= 0) and np.all(sel < n), "indices outside [0, n)"
    assert np.all(np.diff(sel) > 0), "indices must be strictly ascending"


def check_topk_row(gpu_row, oracle_row, oracle_scores, n, k, what=""):
    """Structure, then set equality up to near-ties at the k-th score."""
    gpu_row = np.asarray(gpu_row)
    oracle_row = np.asarray(oracle_row)
    check_topk_structure(gpu_row, n, k)
    if n <= k:
        assert np.array_equal(gpu_row, oracle_row), f"{what}: short row must keep 0..n-1"
        return 0
    g = set(gpu_row[:k].tolist())
    o = set(oracle_row[:k].tolist())
    diff = g ^ o
    if not diff:
        return 0
    sc = np.asarray(oracle_scores[:n], np.float64)
    Ik = np.sort(sc)[::-1][k - 1]
    band = TOPK_REL * abs(Ik) + TOPK_ABS_REL_MAX * np.max(np.abs(sc))
    for s in diff:
        assert abs(sc[s] - Ik) <= band, f"{what}: index {s} (score {sc[s]!r}) differs and is not a near-tie of I_k={Ik!r}"
    return len(g - o)


def check_attention(gpu_o, oracle_o, gpu_lse=None, oracle_lse=None, what=""):
    err = np.max(np.abs(np.asarray(gpu_o, np.float64) - oracle_o))
    assert err <= ATTN_MAX_ABS, f"{what}: attention max-abs error {err}"
    if gpu_lse is not None:
        fin = np.isfinite(oracle_lse)
        assert np.array_equal(np.isfinite(gpu_lse), fin)
        lerr = np.max(np.abs(np.asarray(gpu_lse, np.float64)[fin] - oracle_lse[fin])) if fin.any() else 0.0
        assert lerr <= LSE_ATOL, f"{what}: lse error {lerr}"
    return err
