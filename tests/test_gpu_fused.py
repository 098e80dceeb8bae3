"""GPU parity of the fused lightning indexer + top-k (dsa_indexer_topk), which
never writes the score matrix, against the fp64 oracle and against the
unfused path (dsa_indexer_scores + dsa_topk).

What must hold (criteria of parity_helpers): bit-exact Omega_t on
exact-arithmetic inputs, whichever way a row is decided -- from the
candidates at or above its sampled threshold (rows with more than 6144
visible keys at k = 2048), from all of its keys (shorter rows), or by the full re-scoring
of a row the candidates cannot decide (massive exact ties); on random inputs
the near-tie criterion, and the same indices as the unfused path, which
computes the same fp32 scores.
"""
import numpy as np
import pytest
import torch

import oracle
from parity_helpers import check_topk_row, check_topk_structure
from sparse_long_context_03_b200 import dsa, inputs

pytestmark = pytest.mark.gpu

DEV = "cuda"
KEEP_ALL = 6144  # rows with at most this many keys keep every key as a candidate (k = 2048)


def H(t):
    return inputs.to_numpy_bits(t)


def fused(d, row_begin, n_rows, k):
    q8 = d["q8"].to(DEV)
    HI, dI = q8.shape[1], q8.shape[2]
    ws = torch.empty(dsa.indexer_topk_workspace_size(row_begin, n_rows, k, HI, dI), dtype=torch.uint8, device=DEV)
    idx = torch.full((n_rows, k), -7, dtype=torch.int32, device=DEV)
    stats = torch.full((2,), -1, dtype=torch.int64, device=DEV)
    dsa.indexer_topk(q8, d["sq"].to(DEV), d["w"].to(DEV), d["k8"].to(DEV), d["sk"].to(DEV), row_begin, n_rows, k,
                     idx, ws, stats=stats)
    torch.cuda.synchronize()
    return idx.cpu().numpy(), int(stats[0].item())


def oracle_rows(d, rows, k):
    h = {kk: H(d[kk]) for kk in ("q8", "sq", "w", "k8", "sk")}
    out = {}
    for t in rows:
        I = oracle.indexer(h["q8"], h["sq"], h["w"], h["k8"], h["sk"], row_begin=t, n_rows=1)[0]
        out[t] = (I, oracle.topk(I[None, :], [t + 1], k)[0])
    return out


@pytest.mark.parametrize("HI,dI,L,k", [(32, 64, 1200, 64), (32, 64, 1100, 2048), (8, 32, 700, 7),
                                       (16, 64, 900, 300), (64, 128, 520, 64), (32, 32, 800, 1)])
def test_fused_short_rows_bit_exact(HI, dI, L, k):
    # every row has at most KEEP_ALL keys: all of them are candidates
    d = inputs.exact_indexer_inputs(L, HI, dI, seed=200 + HI + dI + k)
    h = {kk: H(d[kk]) for kk in ("q8", "sq", "w", "k8", "sk")}
    I = oracle.indexer(h["q8"], h["sq"], h["w"], h["k8"], h["sk"])
    ref = oracle.causal_topk(I, 0, k)
    got, rep = fused(d, 0, L, k)
    assert np.array_equal(got, ref)
    assert rep == 0


def test_fused_chunk_offsets_bit_exact():
    # a chunk that starts inside the sequence, with rows below and above k
    HI, dI, L, k = 32, 64, 1000, 300
    d = inputs.exact_indexer_inputs(L, HI, dI, seed=77, key_pool=40)
    h = {kk: H(d[kk]) for kk in ("q8", "sq", "w", "k8", "sk")}
    r0, n = 250, 611
    I = oracle.indexer(h["q8"], h["sq"], h["w"], h["k8"], h["sk"], row_begin=r0, n_rows=n)
    ref = oracle.causal_topk(I, r0, k)
    got, _ = fused(d, r0, n, k)
    assert np.array_equal(got, ref)


def _long_rows(L, n_rand, seed):
    rng = np.random.default_rng(seed)
    rows = {KEEP_ALL - 1, KEEP_ALL, KEEP_ALL + 1, L - 1} | set(int(x) for x in rng.integers(KEEP_ALL, L, n_rand))
    return sorted(rows)


def test_fused_sampled_threshold_bit_exact():
    # rows beyond KEEP_ALL keys are decided from the candidates at or above
    # their sampled threshold; exact inputs make every score exact, so the
    # indices must equal the oracle's bit for bit
    HI, dI, L, k = 32, 64, 11000, 2048
    d = inputs.exact_indexer_inputs(L, HI, dI, seed=301)
    got, rep = fused(d, 0, L, k)
    rows = _long_rows(L, 20, seed=3)
    for t, (I, ref) in oracle_rows(d, rows, k).items():
        assert np.array_equal(got[t], ref), f"row {t}"
    for t in range(0, L, 97):
        check_topk_structure(got[t], t + 1, k)
    assert rep <= L // 100, f"{rep} rows had to be scored again"


def test_fused_repair_path_massive_ties_bit_exact():
    # every key is one of two distinct keys: a row holds two score values,
    # its threshold lands on one of them and the candidates overflow, so the
    # rows are scored again in full and selected by the exact whole-row path
    HI, dI, L, k = 32, 64, 9000, 2048
    d = inputs.exact_indexer_inputs(L, HI, dI, seed=302, key_pool=2)
    got, rep = fused(d, 0, L, k)
    assert rep > 0
    rows = _long_rows(L, 6, seed=4) + [k, k + 1, 5000]
    for t, (I, ref) in oracle_rows(d, sorted(set(rows)), k).items():
        assert np.array_equal(got[t], ref), f"row {t}"


def test_fused_random_inputs_near_tie_criterion():
    cfg = inputs.config(1)
    L = 12000
    d = inputs.prefill_inputs(cfg, L=L, seed=303)
    got, rep = fused(d, 0, L, cfg.k)
    assert rep == 0
    rows = _long_rows(L, 10, seed=5) + [0, cfg.k - 1, cfg.k, 4000]
    for t, (I, ref) in oracle_rows(d, sorted(set(rows)), cfg.k).items():
        check_topk_row(got[t], ref, I, t + 1, cfg.k, f"row {t}")


def test_fused_equals_unfused_every_row_32k():
    # both paths compute the same fp32 scores (same tensor-core kernel and
    # epilogue arithmetic), so every row's indices must be identical
    cfg = inputs.config(1)
    d = inputs.prefill_inputs(cfg, device=DEV)
    L = cfg.L
    pf = dsa.PrefillPlan(L, cfg.HI, cfg.dI, cfg.Hq, cfg.Hkv, cfg.D, cfg.k, fused=True, device=DEV)
    dsa.select_rows(pf, d["q8"], d["sq"], d["w"], d["k8"], d["sk"])
    rep = torch.zeros(2, dtype=torch.int64, device=DEV)
    # the last chunk again, for its repair count
    r0, n = list(pf.chunks())[-1]
    dsa.indexer_topk(d["q8"], d["sq"], d["w"], d["k8"], d["sk"], r0, n, cfg.k, pf.idx[r0:r0 + n], pf.ws,
                     stats=rep)
    fused_idx = pf.idx.clone()
    del pf
    pu = dsa.PrefillPlan(L, cfg.HI, cfg.dI, cfg.Hq, cfg.Hkv, cfg.D, cfg.k, fused=False, device=DEV)
    dsa.select_rows(pu, d["q8"], d["sq"], d["w"], d["k8"], d["sk"])
    torch.cuda.synchronize()
    assert int(rep[0].item()) == 0
    diff = (fused_idx != pu.idx).any(dim=1)
    assert int(diff.sum().item()) == 0, f"rows differing: {torch.nonzero(diff)[:10].flatten().tolist()}"


def test_fused_rejects_bad_arguments():
    d = {k: v.to(DEV) for k, v in inputs.exact_indexer_inputs(300, 32, 64, seed=1).items()}
    idx = torch.empty(300, 64, dtype=torch.int32, device=DEV)
    need = dsa.indexer_topk_workspace_size(0, 300, 64, 32, 64)
    small = torch.empty(need - 256, dtype=torch.uint8, device=DEV)
    with pytest.raises(dsa.DSAError, match="WORKSPACE"):
        dsa.indexer_topk(d["q8"], d["sq"], d["w"], d["k8"], d["sk"], 0, 300, 64, idx, small)
    ws = torch.empty(need, dtype=torch.uint8, device=DEV)
    with pytest.raises(dsa.DSAError, match="INVALID_ARG"):
        dsa.indexer_topk(d["q8"], d["sq"], d["w"], d["k8"], d["sk"], 200, 101, 64, idx, ws)
    # HI = 4 has no tensor-core indexer: the fused call is not offered
    assert dsa.indexer_topk_workspace_size(0, 300, 64, 4, 32) == 0
