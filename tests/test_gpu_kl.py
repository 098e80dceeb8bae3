"""GPU parity of the indexer distillation losses (dsa_indexer_kl) against the
fp64 oracle: dense warm-up KL over every causal key and sparse adaptation KL
over the selected set ("Kwai Keye-VL-2.0 Technical Report" review, 核心公式;
report translation section 2.3.3).

Both sides read the same float32 scores and targets; the library
accumulates in fp64 and rearranges the sum (KL = A/S - ln S - (B/S - ln sum
exp I)), so the criterion is |gpu - oracle| <= 1e-9 * (1 + |oracle|) per
row: far below any float32 effect, far above fp64 rounding of sums over up to
32K keys.
"""
import numpy as np
import pytest
import torch

import oracle
from conftest import read_golden
from sparse_long_context_03_b200 import dsa, inputs

pytestmark = pytest.mark.gpu

DEV = "cuda"
TOL = 1e-9


def H(t):
    return inputs.to_numpy_bits(t)


def gpu_kl(scores, r0, p, idx=None):
    n = scores.shape[0]
    loss = torch.full((n,), float("nan"), dtype=torch.float64, device=DEV)
    total = torch.full((1,), float("nan"), dtype=torch.float64, device=DEV)
    dsa.indexer_kl(scores, r0, n, p, loss, idx=idx, loss_total=total)
    torch.cuda.synchronize()
    return loss.cpu().numpy(), float(total.item())


def check(got, ref, what):
    err = np.abs(got - ref)
    bad = err > TOL * (1 + np.abs(ref))
    assert not bad.any(), f"{what}: {bad.sum()} rows out of tolerance, worst {err.max():.3e}"


def test_kl_hand_example_on_gpu():
    g = read_golden("indexer_kl_hand_example.txt")
    I = torch.tensor([g["dense_I"]], dtype=torch.float32, device=DEV)
    p = torch.tensor([[g["dense_p_g0"], g["dense_p_g1"]]], dtype=torch.float32, device=DEV)
    loss, total = gpu_kl(I, 1, p)
    # the float32 copy of ln 3 moves the result by ~1e-8
    assert loss[0] == pytest.approx(g["dense_loss"][0], rel=1e-7)
    I = torch.tensor([g["sparse_I"]], dtype=torch.float32, device=DEV)
    p = torch.tensor([[g["sparse_p"]]], dtype=torch.float32, device=DEV)
    idx = torch.tensor([[int(x) for x in g["sparse_idx"]]], dtype=torch.int32, device=DEV)
    loss, _ = gpu_kl(I, 2, p, idx)
    assert loss[0] == pytest.approx(g["sparse_loss"][0], rel=1e-7)


@pytest.mark.parametrize("G", [1, 4, 6])
def test_kl_dense_and_sparse_tiny_layer(G):
    # scores from the library's indexer on the tiny layer, targets synthetic
    cfg = inputs.config(0)
    d = {k: v.to(DEV) for k, v in inputs.prefill_inputs(cfg).items()}
    r0, n = 100, 412
    L = cfg.L
    scores = torch.full((n, L), float("nan"), dtype=torch.float32, device=DEV)
    dsa.indexer_scores(d["q8"], d["sq"], d["w"], d["k8"], d["sk"], r0, n, scores)
    idx = torch.empty(n, cfg.k, dtype=torch.int32, device=DEV)
    dsa.topk(scores, r0, n, cfg.k, idx, max_len=r0 + n)
    p = inputs.kl_targets(n, G, L, seed=50 + G, device=DEV)
    Ih = scores.cpu().numpy().astype(np.float64)
    Ih[~np.isfinite(Ih)] = 0.0  # columns right of the causal range are never read
    ph = p.cpu().numpy().astype(np.float64)
    ref, ref_total = oracle.indexer_kl(Ih, ph, row_begin=r0)
    got, total = gpu_kl(scores, r0, p)
    check(got, ref, f"dense G={G}")
    assert total == pytest.approx(ref_total, rel=1e-12)
    assert total == pytest.approx(got.sum(), rel=1e-13)
    ref_s, _ = oracle.indexer_kl(Ih, ph, row_begin=r0, idx=idx.cpu().numpy())
    got_s, _ = gpu_kl(scores, r0, p, idx)
    check(got_s, ref_s, f"sparse G={G}")
    assert np.all(got_s >= -1e-12) and np.all(got >= -1e-12)


def test_kl_edge_cases():
    rng = np.random.default_rng(9)
    n, L, r0 = 5, 64, 40
    I = torch.tensor(rng.normal(0, 4, (n, L)), dtype=torch.float32, device=DEV)
    p = inputs.kl_targets(n, 2, L, seed=3, device=DEV)
    p[1, 1] = 0.0                       # a group without target mass
    idx = torch.full((n, 8), -1, dtype=torch.int32, device=DEV)
    idx[0, :3] = torch.tensor([5, 0, 44], dtype=torch.int32)   # 44 > t = 40 is skipped
    idx[2, :2] = torch.tensor([-5, 1000], dtype=torch.int32)   # no valid entry: loss 0
    idx[3, 0] = 7                                              # one key: KL 0 whatever p is
    idx[4, :8] = torch.arange(8, dtype=torch.int32)
    got, _ = gpu_kl(I, r0, p, idx)
    ref, _ = oracle.indexer_kl(I.cpu().numpy().astype(np.float64), p.cpu().numpy().astype(np.float64),
                               row_begin=r0, idx=idx.cpu().numpy())
    check(got, ref, "edge cases")
    assert got[2] == 0.0 and abs(got[3]) < 1e-15
    dense, _ = gpu_kl(I, r0, p)
    dref, _ = oracle.indexer_kl(I.cpu().numpy().astype(np.float64), p.cpu().numpy().astype(np.float64), row_begin=r0)
    check(dense, dref, "dense with a massless group")


def test_kl_32k_chunk_matches_oracle_and_is_reproducible():
    cfg = inputs.config(1)
    d = inputs.prefill_inputs(cfg, device=DEV)
    L, G = cfg.L, cfg.Hkv
    r0, n = L - 256, 256
    scores = torch.empty(n, L, dtype=torch.float32, device=DEV)
    dsa.indexer_scores(d["q8"], d["sq"], d["w"], d["k8"], d["sk"], r0, n, scores)
    ws = None
    need = dsa.topk_workspace_size(n, L, cfg.k)
    if need:
        ws = torch.empty(need, dtype=torch.uint8, device=DEV)
    idx = torch.empty(n, cfg.k, dtype=torch.int32, device=DEV)
    dsa.topk(scores, r0, n, cfg.k, idx, max_len=L, ws=ws)
    p = inputs.kl_targets(n, G, L, seed=61, device=DEV)
    got, total = gpu_kl(scores, r0, p)
    got2, total2 = gpu_kl(scores, r0, p)
    assert np.array_equal(got, got2) and total == total2
    ref, _ = oracle.indexer_kl(scores.cpu().numpy().astype(np.float64), p.cpu().numpy().astype(np.float64),
                               row_begin=r0)
    check(got, ref, "dense 32K")
    got_s, _ = gpu_kl(scores, r0, p, idx)
    ref_s, _ = oracle.indexer_kl(scores.cpu().numpy().astype(np.float64), p.cpu().numpy().astype(np.float64),
                                 row_begin=r0, idx=idx.cpu().numpy())
    check(got_s, ref_s, "sparse 32K")
