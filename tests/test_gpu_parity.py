"""GPU parity: the CUDA library (through its C ABI) against the fp64 oracle.

Every case draws seeded inputs, runs the library on a B200 and the oracle on
the host on the same bytes, and compares with the criteria in
parity_helpers.  Small cases cover whole matrices (several tiles and a
ragged tail); the full-size workloads run in the benchmark's launch
configuration and are compared on sampled rows.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from parity_helpers import (check_attention, check_scores, check_topk_row, check_topk_structure)
from sparse_long_context_03_b200 import dsa, inputs

pytestmark = pytest.mark.gpu

DEV = "cuda"


def H(t):
    return inputs.to_numpy_bits(t)


def _gpu(d):
    return {k: (v.to(DEV) if isinstance(v, torch.Tensor) else v) for k, v in d.items()}


def gpu_scores(d, row_begin, n_rows, L):
    ld = (L + 3) // 4 * 4
    out = torch.full((n_rows, ld), float("nan"), dtype=torch.float32, device=DEV)
    dsa.indexer_scores(d["q8"], d["sq"], d["w"], d["k8"], d["sk"], row_begin, n_rows, out)
    torch.cuda.synchronize()
    return out.cpu().numpy()


# ----------------------------------------------------------------------------
# indexer
# ----------------------------------------------------------------------------

@pytest.mark.parametrize("row_begin,n_rows", [(0, 512), (200, 137), (511, 1)])
def test_indexer_tiny_matches_oracle(row_begin, n_rows):
    cfg = inputs.config(0)
    d = inputs.prefill_inputs(cfg)
    ref = oracle.indexer(*(H(d[k]) for k in ("q8", "sq", "w", "k8", "sk")), row_begin=row_begin, n_rows=n_rows)
    got = gpu_scores(_gpu(d), row_begin, n_rows, cfg.L)
    for r in range(n_rows):
        t = row_begin + r
        check_scores(got[r, : t + 1], ref[r, : t + 1], f"row {t}")


@pytest.mark.parametrize("HI,dI,L", [(32, 64, 700), (4, 32, 300), (64, 128, 260), (16, 64, 333), (8, 32, 129)])
def test_indexer_exact_inputs_bit_exact(HI, dI, L):
    d = inputs.exact_indexer_inputs(L, HI, dI, seed=100 + HI + dI)
    ref = oracle.indexer(*(H(d[k]) for k in ("q8", "sq", "w", "k8", "sk")))
    got = gpu_scores(_gpu(d), 0, L, L)
    tri = np.tril(np.ones((L, L), bool))
    assert np.array_equal(got[:, :L][tri].astype(np.float64), ref[tri])


def test_indexer_exact_inputs_bit_exact_8k_many_blocks_per_cta():
    # L = 8192 in one launch: 2048 query blocks over the persistent CTAs
    # (about 14 each) and up to 32 key steps per block, so the 8-stage key
    # ring wraps many times within and across blocks
    L, HI, dI = 8192, 32, 64
    d = inputs.exact_indexer_inputs(L, HI, dI, seed=808)
    got = gpu_scores(_gpu(d), 0, L, L)
    h = {k: H(d[k]) for k in ("q8", "sq", "w", "k8", "sk")}
    rng = np.random.default_rng(8)
    rows = sorted({0, 3, 255, 256, 511, 4095, 4096, 6000, L - 5, L - 1} | set(int(x) for x in rng.integers(0, L, 8)))
    for t in rows:
        ref = oracle.indexer(h["q8"], h["sq"], h["w"], h["k8"], h["sk"], row_begin=t, n_rows=1)[0]
        assert np.array_equal(got[t, : t + 1], ref[: t + 1]), f"row {t}"


def test_indexer_signed_weights():
    cfg = inputs.config(0)
    d = inputs.prefill_inputs(cfg, L=300, seed=44)
    g = torch.Generator().manual_seed(3)
    d["w"] = torch.randn(300, cfg.HI, generator=g)
    ref = oracle.indexer(*(H(d[k]) for k in ("q8", "sq", "w", "k8", "sk")))
    got = gpu_scores(_gpu(d), 0, 300, 300)
    assert (ref[np.tril(np.ones((300, 300), bool))] < 0).any()
    for t in range(300):
        check_scores(got[t, : t + 1], ref[t, : t + 1], f"row {t}")


# ----------------------------------------------------------------------------
# top-k
# ----------------------------------------------------------------------------

def gpu_topk(scores_np, k, row_begin=0, row_len=None, max_len=None):
    n_rows, w = scores_np.shape
    ld = (w + 3) // 4 * 4
    s = torch.zeros(n_rows, ld, dtype=torch.float32)
    s[:, :w] = torch.from_numpy(scores_np)
    s = s.to(DEV)
    idx = torch.full((n_rows, k), -7, dtype=torch.int32, device=DEV)
    rl = None if row_len is None else torch.as_tensor(row_len, dtype=torch.int32, device=DEV)
    if max_len is None:
        max_len = w if row_len is not None else row_begin + n_rows
    need = dsa.topk_workspace_size(n_rows, max_len, k)
    ws = torch.empty(max(need, 1), dtype=torch.uint8, device=DEV) if need else None
    dsa.topk(s, row_begin, n_rows, k, idx, row_len=rl, max_len=max_len, ws=ws)
    torch.cuda.synchronize()
    return idx.cpu().numpy()


@pytest.mark.parametrize("k", [1, 7, 64, 300])
def test_topk_causal_rows_bit_exact(k):
    n_rows = 600
    x = inputs.tie_heavy_scores(n_rows, n_rows, seed=10 + k).numpy()
    got = gpu_topk(x, k)
    ref = oracle.causal_topk(x.astype(np.float64), 0, k)
    assert np.array_equal(got, ref)


@pytest.mark.parametrize("k", [1, 64, 2048])
def test_topk_row_lengths_bit_exact(k):
    lens = [0, 1, 2, k - 1, k, k + 1, 2 * k + 3, 5000, 20000, 65537, 3, 100000]
    width = max(lens)
    x = inputs.tie_heavy_scores(len(lens), width, seed=77 + k).numpy()
    got = gpu_topk(x, k, row_len=lens)
    ref = oracle.topk(x.astype(np.float64), lens, k)
    assert np.array_equal(got, ref)


def test_topk_chunk_offset_and_determinism():
    x = inputs.tie_heavy_scores(97, 3000, seed=5).numpy()
    a = gpu_topk(x, 256, row_begin=2903, max_len=3000)
    b = gpu_topk(x, 256, row_begin=2903, max_len=3000)
    assert np.array_equal(a, b)
    ref = oracle.topk(x.astype(np.float64), np.arange(2904, 3001), 256)
    assert np.array_equal(a, ref)


def test_topk_fallback_massive_ties():
    # Three distinct values over 100000 entries: the threshold bucket holds
    # ~33K entries, more than shared memory stages, so the whole-row radix
    # path decides; the result must be the same deterministic set.
    rng = np.random.default_rng(3)
    x = rng.choice(np.array([0.5, 1.0, 2.0], np.float32), size=(3, 100000))
    x[2, :] = 1.0
    x[2, 77777] = 3.0
    got = gpu_topk(x, 2048, row_len=[100000, 99999, 100000])
    ref = oracle.topk(x.astype(np.float64), [100000, 99999, 100000], 2048)
    assert np.array_equal(got, ref)


def test_topk_clustered_near_ties():
    # Frame-like clusters: groups of 256 scores within 1e-6 relative of each
    # other, as the multimodal workload produces.
    rng = np.random.default_rng(11)
    n = 50000
    centers = rng.standard_normal(n // 256 + 1).astype(np.float32)
    x = (np.repeat(centers, 256)[:n] * (1 + 1e-6 * rng.standard_normal(n))).astype(np.float32)[None, :]
    for k in (64, 2048, 2047):
        got = gpu_topk(x, k, row_len=[n])
        assert np.array_equal(got, oracle.topk(x.astype(np.float64), [n], k))


def test_topk_many_long_rows_bit_exact():
    # At least one row per SM and rows past 16384 entries: the one-CTA-per-row
    # kernel with the bitmap collect (not the per-row cluster).
    rng = np.random.default_rng(21)
    lens = rng.integers(2000, 70000, 160).tolist()
    lens[:4] = [2049, 16384, 65537, 69999]
    x = inputs.tie_heavy_scores(len(lens), max(lens), seed=21).numpy()
    got = gpu_topk(x, 2048, row_len=lens)
    assert np.array_equal(got, oracle.topk(x.astype(np.float64), lens, 2048))


@pytest.mark.parametrize("k", [512, 2048])
@pytest.mark.parametrize("stats", [False, True])
def test_topk_cluster_rows_bit_exact(k, stats):
    # Fewer rows than SMs and rows past 16384 entries: one 8-CTA cluster per
    # row.  Slices of at most 32 k entries mark winners in per-slice bitmaps
    # and write the output from every CTA; longer slices gather ordered lists
    # on one CTA.  Both sides of that bound, with and without row statistics.
    rng = np.random.default_rng(41 + k)
    lens = [16385, 70001, 131072, 131073, 262144, 300001, 524288, 524289]
    x = rng.standard_normal((len(lens), max(lens))).astype(np.float32)
    if stats:
        got = _gpu_topk_with_stats(x, k, lens)
    else:
        got = gpu_topk(x, k, row_len=lens)
    assert np.array_equal(got, oracle.topk(x.astype(np.float64), lens, k))


def test_topk_cluster_threshold_ties_across_slices():
    # 1500 entries above and 200 entries exactly at the k-th value spread over
    # every slice of the cluster: the ties are taken lowest index first
    # across slices.
    rng = np.random.default_rng(43)
    n_rows, n = 6, 100000
    x = rng.random((n_rows, n), dtype=np.float32)
    for r in range(n_rows):
        pos = rng.permutation(n)
        x[r, pos[:1500]] = 5.0 + rng.random(1500, dtype=np.float32)
        x[r, pos[1500:1700]] = 3.0
    lens = [n - 3 * r for r in range(n_rows)]
    ref = oracle.topk(x.astype(np.float64), lens, 2048)
    assert np.array_equal(gpu_topk(x, 2048, row_len=lens), ref)
    assert np.array_equal(_gpu_topk_with_stats(x, 2048, lens), ref)


@pytest.mark.parametrize("k", [30000, 40000])
def test_topk_cluster_large_k(k):
    # k up to the ABI's bound on the per-row cluster path (few rows, long
    # row bound): random rows past k, one below it
    rng = np.random.default_rng(k)
    lens = [150000, 90001, k - 1]
    x = rng.standard_normal((len(lens), max(lens))).astype(np.float32)
    ref = oracle.topk(x.astype(np.float64), lens, k)
    assert np.array_equal(gpu_topk(x, k, row_len=lens), ref)
    assert np.array_equal(_gpu_topk_with_stats(x, k, lens), ref)


@pytest.mark.parametrize("n_tied", [300, 7000])
def test_topk_cluster_crowded_threshold_bucket(n_tied):
    # Few long rows (one cluster each) whose threshold bucket holds more
    # than 256 entries: 300 exact ties take the gathered ordered lists, 7000
    # (more than fit in shared memory) the whole-row radix select; both with
    # and without row statistics.
    rng = np.random.default_rng(44 + n_tied)
    n_rows, n = 4, 120000
    x = rng.random((n_rows, n), dtype=np.float32)
    for r in range(n_rows):
        pos = rng.permutation(n)
        x[r, pos[:1500]] = 5.0 + rng.random(1500, dtype=np.float32)
        x[r, pos[1500:1500 + n_tied]] = 3.0
    lens = [n - 5 * r for r in range(n_rows)]
    ref = oracle.topk(x.astype(np.float64), lens, 2048)
    assert np.array_equal(gpu_topk(x, 2048, row_len=lens), ref)
    assert np.array_equal(_gpu_topk_with_stats(x, 2048, lens), ref)


@pytest.mark.parametrize("n_tied", [300, 1000])
def test_topk_exact_ties_at_the_threshold(n_tied):
    # 1500 entries above, n_tied entries exactly equal at the k-th value and
    # the rest below it: the tied entries must be taken lowest index first.
    # 300 ties are ranked pairwise, 1000 take the whole-row radix path.
    rng = np.random.default_rng(n_tied)
    n_rows, n = 150, 20000
    x = rng.random((n_rows, n), dtype=np.float32)
    for r in range(n_rows):
        pos = rng.permutation(n)
        x[r, pos[:1500]] = 5.0 + rng.random(1500, dtype=np.float32)
        x[r, pos[1500:1500 + n_tied]] = 3.0
    got = gpu_topk(x, 2048, row_len=[n] * n_rows)
    assert np.array_equal(got, oracle.topk(x.astype(np.float64), [n] * n_rows, 2048))


def test_topk_rows_beyond_the_bitmap_limit():
    # A row bound past 557K entries selects the ordered-collect kernel; the
    # rows themselves are short, so only the bound differs.
    rng = np.random.default_rng(8)
    lens = rng.integers(3000, 9000, 150).tolist()
    x = inputs.tie_heavy_scores(150, max(lens), seed=8).numpy()
    n_rows, w = x.shape
    max_len = 600000
    s = torch.zeros(n_rows, max_len, dtype=torch.float32)
    s[:, :w] = torch.from_numpy(x)
    s = s.to(DEV)
    idx = torch.full((n_rows, 2048), -7, dtype=torch.int32, device=DEV)
    rl = torch.as_tensor(lens, dtype=torch.int32, device=DEV)
    dsa.topk(s, 0, n_rows, 2048, idx, row_len=rl, max_len=max_len)
    torch.cuda.synchronize()
    assert np.array_equal(idx.cpu().numpy(), oracle.topk(x.astype(np.float64), lens, 2048))


def _gpu_topk_with_stats(x, k, lens):
    """Top-k with the row statistics the indexer would give (each row's min
    and max, repeated over the four lane quarters)."""
    n_rows, w = x.shape
    ld = (w + 3) // 4 * 4
    s = torch.zeros(n_rows, ld, dtype=torch.float32)
    s[:, :w] = torch.from_numpy(x)
    st = np.zeros((n_rows, 8), np.float32)
    for r, n in enumerate(lens):
        st[r, 0::2] = x[r, :n].min()
        st[r, 1::2] = x[r, :n].max()
    idx = torch.full((n_rows, k), -7, dtype=torch.int32, device=DEV)
    dsa.topk(s.to(DEV), 0, n_rows, k, idx, row_len=torch.as_tensor(lens, dtype=torch.int32, device=DEV),
             max_len=w, row_stats=torch.from_numpy(st).to(DEV))
    torch.cuda.synchronize()
    return idx.cpu().numpy()


def test_topk_sampled_band_bit_exact():
    # With row statistics, rows of at least 16 k entries locate their
    # threshold band from a sample (shorter rows take the full histogram);
    # the selection must be exact either way.
    rng = np.random.default_rng(31)
    lens = rng.integers(16384, 70000, 200).tolist()
    lens[:3] = [16384, 16385, 69999]
    x = inputs.tie_heavy_scores(len(lens), max(lens), seed=31).numpy()
    got = _gpu_topk_with_stats(x, 2048, lens)
    assert np.array_equal(got, oracle.topk(x.astype(np.float64), lens, 2048))


def test_topk_sampled_band_miss_takes_the_exact_path():
    # The large entries sit only in pieces the sample skips (every eighth
    # 16-entry piece is sampled), so the band misses the k-th entry; the row
    # must fall back to the full histogram and give the same exact set.
    rng = np.random.default_rng(32)
    n_rows, n = 150, 40000
    x = rng.random((n_rows, n), dtype=np.float32)
    unsampled = np.array([i for i in range(n) if (i // 16) % 8 != 0])
    for r in range(n_rows):
        pos = rng.choice(unsampled, 3000, replace=False)
        x[r, pos] = 10.0 + rng.random(3000, dtype=np.float32)
    got = _gpu_topk_with_stats(x, 2048, [n] * n_rows)
    assert np.array_equal(got, oracle.topk(x.astype(np.float64), [n] * n_rows, 2048))


def test_topk_signed_zeros_and_all_equal():
    x = np.zeros((3, 100), np.float32)
    x[0, ::2] = -0.0
    x[1, :] = 0.5
    x[2, :] = -3.0
    x[2, 50] = -0.0
    got = gpu_topk(x, 10, row_len=[100, 100, 100])
    assert list(got[0]) == list(range(10))
    assert list(got[1]) == list(range(10))
    assert list(got[2]) == [0, 1, 2, 3, 4, 5, 6, 7, 8, 50]


# ----------------------------------------------------------------------------
# whole prefill chain, small
# ----------------------------------------------------------------------------

def run_prefill(cfg, d, chunk_rows=None, want_rows=(), lse=True, use_stats=True, fused=False):
    """Run the prefill exactly as the benchmark does (fused=True: the fused
    indexer + top-k; otherwise the chunked score matrix and dsa_topk); also
    return the indexer score rows listed in want_rows (the unfused path
    keeps them as each chunk is produced; the fused path never writes them,
    so they are scored alone)."""
    L = d["q8"].shape[0]
    plan = dsa.PrefillPlan(L, cfg.HI, cfg.dI, cfg.Hq, cfg.Hkv, cfg.D, cfg.k, chunk_rows=chunk_rows, fused=fused)
    O = torch.empty(L, cfg.Hq, cfg.D, dtype=torch.bfloat16, device=DEV)
    lse_t = torch.empty(L, cfg.Hq, dtype=torch.float32, device=DEV) if lse else None
    want = sorted(want_rows)
    rows = {}
    if fused:
        dsa.select_rows(plan, d["q8"], d["sq"], d["w"], d["k8"], d["sk"])
        ld = (L + 3) // 4 * 4
        one = torch.empty(1, ld, dtype=torch.float32, device=DEV)
        for t in want:
            dsa.indexer_scores(d["q8"], d["sq"], d["w"], d["k8"], d["sk"], t, 1, one)
            rows[t] = one[0, : t + 1].cpu().numpy()
    else:
        for r0, n in plan.chunks():
            dsa.indexer_scores(d["q8"], d["sq"], d["w"], d["k8"], d["sk"], r0, n, plan.scores[:n],
                               row_stats=plan.row_stats if use_stats else None)
            for t in want:
                if r0 <= t < r0 + n:
                    rows[t] = plan.scores[t - r0, : t + 1].cpu().numpy()
            dsa.topk(plan.scores[:n], r0, n, cfg.k, plan.idx[r0:r0 + n], max_len=r0 + n, ws=plan.ws,
                     row_stats=plan.row_stats if use_stats else None)
    dsa.sparse_gqa_prefill(d["Q"], d["K"], d["V"], plan.idx, 0, L, cfg.k, cfg.sm_scale, O, lse_t)
    torch.cuda.synchronize()
    return plan, O, lse_t, rows


@pytest.mark.parametrize("use_stats", [True, False])
def test_prefill_chain_tiny_full(use_stats):
    cfg = inputs.config(0)
    d = inputs.prefill_inputs(cfg)
    plan, O, lse, _ = run_prefill(cfg, _gpu(d), chunk_rows=200, use_stats=use_stats)
    h = {k: H(v) for k, v in d.items()}
    I = oracle.indexer(h["q8"], h["sq"], h["w"], h["k8"], h["sk"])
    ref_idx = oracle.causal_topk(I, 0, cfg.k)
    gidx = plan.idx.cpu().numpy()
    for t in range(cfg.L):
        check_topk_row(gidx[t], ref_idx[t], I[t], t + 1, cfg.k, f"row {t}")
    Oref, lref = oracle.sparse_attention(h["Q"], h["K"], h["V"], ref_idx, 0, cfg.sm_scale)
    same = np.all(gidx == ref_idx, axis=1)
    Og = O.float().cpu().numpy()
    check_attention(Og[same], Oref[same], lse.cpu().numpy()[same], lref[same], "chain")
    # the attention kernel alone on the oracle's index sets, every row
    O2 = torch.empty_like(O)
    l2 = torch.empty_like(lse)
    dsa.sparse_gqa_prefill(_gpu(d)["Q"], _gpu(d)["K"], _gpu(d)["V"], torch.from_numpy(ref_idx).to(DEV), 0, cfg.L,
                           cfg.k, cfg.sm_scale, O2, l2)
    torch.cuda.synchronize()
    check_attention(O2.float().cpu().numpy(), Oref, l2.cpu().numpy(), lref, "attention on oracle idx")


def test_packed_sequences_are_independent_prefills():
    # Several sequences packed along the token axis: each one is its own
    # causal prefill.  Compare every token with the oracle run on its own
    # sequence's slice (empty and one-token sequences included).
    cfg = inputs.config(0)
    lens = [300, 1, 0, 777, 64]
    cu = np.concatenate([[0], np.cumsum(lens)]).tolist()
    d = inputs.prefill_inputs(cfg, L=cu[-1], seed=41)
    g = _gpu(d)
    plan = dsa.PrefillPlan(max(lens), cfg.HI, cfg.dI, cfg.Hq, cfg.Hkv, cfg.D, cfg.k, chunk_rows=256, device=DEV)
    O = torch.full((cu[-1], cfg.Hq, cfg.D), float("nan"), dtype=torch.bfloat16, device=DEV)
    lse = torch.full((cu[-1], cfg.Hq), float("nan"), dtype=torch.float32, device=DEV)
    idx = torch.full((cu[-1], cfg.k), -7, dtype=torch.int32, device=DEV)
    dsa.prefill_forward_packed(plan, cu, g["q8"], g["sq"], g["w"], g["k8"], g["sk"], g["Q"], g["K"], g["V"], O,
                               cfg.sm_scale, lse=lse, idx_out=idx)
    torch.cuda.synchronize()
    h = {k: H(v) for k, v in d.items()}
    gidx, Og, lg = idx.cpu().numpy(), O.float().cpu().numpy(), lse.cpu().numpy()
    for s0, s1 in zip(cu, cu[1:]):
        if s1 == s0:
            continue
        sl = {k: v[s0:s1] for k, v in h.items()}
        I = oracle.indexer(sl["q8"], sl["sq"], sl["w"], sl["k8"], sl["sk"])
        ref_idx = oracle.causal_topk(I, 0, cfg.k)
        for t in range(s1 - s0):
            check_topk_row(gidx[s0 + t], ref_idx[t], I[t], t + 1, cfg.k, f"sequence at {s0}, row {t}")
        Oref, lref = oracle.sparse_attention(sl["Q"], sl["K"], sl["V"], ref_idx, 0, cfg.sm_scale)
        same = np.all(gidx[s0:s1] == ref_idx, axis=1)
        check_attention(Og[s0:s1][same], Oref[same], lg[s0:s1][same], lref[same], f"sequence at {s0}")


def test_prefill_bitwise_deterministic_and_stream_independent():
    # Same inputs, twice on the default stream and once on a side stream:
    # indices, outputs and lse must be identical bit for bit (no kernel of
    # the chain accumulates in a scheduling-dependent order).
    cfg = inputs.config(1)
    L = 4096
    d = _gpu(inputs.prefill_inputs(cfg, L=L, seed=43))
    runs = []
    side = torch.cuda.Stream()
    for stream in (None, None, side):
        plan = dsa.PrefillPlan(L, cfg.HI, cfg.dI, cfg.Hq, cfg.Hkv, cfg.D, cfg.k, chunk_rows=1500, device=DEV)
        O = torch.empty(L, cfg.Hq, cfg.D, dtype=torch.bfloat16, device=DEV)
        lse = torch.empty(L, cfg.Hq, dtype=torch.float32, device=DEV)
        torch.cuda.synchronize()
        dsa.prefill_forward(plan, d["q8"], d["sq"], d["w"], d["k8"], d["sk"], d["Q"], d["K"], d["V"], O,
                            cfg.sm_scale, lse=lse, stream=stream)
        torch.cuda.synchronize()
        runs.append((plan.idx.cpu().numpy(), H(O), lse.cpu().numpy()))
    for other in runs[1:]:
        for a, b in zip(runs[0], other):
            assert np.array_equal(a, b)


def test_prefill_chain_exact_inputs_bit_exact_indices():
    cfg = inputs.config(1, k=64)
    L = 900
    d = inputs.exact_indexer_inputs(L, cfg.HI, cfg.dI, seed=9, key_pool=24)
    g = torch.Generator().manual_seed(1)
    for name, Hh in (("Q", cfg.Hq), ("K", cfg.Hkv), ("V", cfg.Hkv)):
        d[name] = (torch.randn(L, Hh, cfg.D, generator=g) * 0.5).to(torch.bfloat16)
    h = {k: H(v) for k, v in d.items()}
    I = oracle.indexer(h["q8"], h["sq"], h["w"], h["k8"], h["sk"])
    ref_idx = oracle.causal_topk(I, 0, cfg.k)
    for use_stats in (True, False):
        plan, O, lse, _ = run_prefill(cfg, _gpu(d), chunk_rows=256, use_stats=use_stats)
        assert np.array_equal(plan.idx.cpu().numpy(), ref_idx)
    Oref, lref = oracle.sparse_attention(h["Q"], h["K"], h["V"], ref_idx, 0, cfg.sm_scale)
    check_attention(O.float().cpu().numpy(), Oref, lse.cpu().numpy(), lref, "exact chain")


# ----------------------------------------------------------------------------
# attention edge cases
# ----------------------------------------------------------------------------

def _dense_causal(Qd, Kd, Vd, sm):
    L, Hq, D = Qd.shape
    G = Hq // Kd.shape[1]
    O = np.zeros_like(Qd)
    for h in range(Hq):
        lg = sm * Qd[:, h] @ Kd[:, h // G].T
        lg[np.triu(np.ones((L, L), bool), 1)] = -np.inf
        lg -= lg.max(axis=1, keepdims=True)
        p = np.exp(lg)
        O[:, h] = (p / p.sum(axis=1, keepdims=True)) @ Vd[:, h // G]
    return O


@pytest.mark.parametrize("Hq,Hkv,D", [(8, 2, 64), (32, 4, 128), (8, 8, 64), (16, 2, 128)])
def test_attention_full_budget_equals_dense(Hq, Hkv, D):
    L, k = 150, 160
    g = torch.Generator().manual_seed(Hq + D)
    Q = torch.randn(L, Hq, D, generator=g).to(torch.bfloat16)
    K = torch.randn(L, Hkv, D, generator=g).to(torch.bfloat16)
    V = torch.randn(L, Hkv, D, generator=g).to(torch.bfloat16)
    idx = np.full((L, k), -1, np.int32)
    for t in range(L):
        idx[t, : t + 1] = np.arange(t + 1)
    O = torch.empty(L, Hq, D, dtype=torch.bfloat16, device=DEV)
    sm = 1 / math.sqrt(D)
    dsa.sparse_gqa_prefill(Q.to(DEV), K.to(DEV), V.to(DEV), torch.from_numpy(idx).to(DEV), 0, L, k, sm, O)
    torch.cuda.synchronize()
    ref = _dense_causal(Q.double().numpy(), K.double().numpy(), V.double().numpy(), sm)
    check_attention(O.float().cpu().numpy(), ref, what="dense")


def test_attention_skips_invalid_entries_and_empty_rows():
    L, Hq, Hkv, D, k = 40, 8, 2, 64, 16
    g = torch.Generator().manual_seed(8)
    Q = torch.randn(L, Hq, D, generator=g).to(torch.bfloat16)
    K = torch.randn(L, Hkv, D, generator=g).to(torch.bfloat16)
    V = torch.randn(L, Hkv, D, generator=g).to(torch.bfloat16)
    idx = np.full((L, k), -1, np.int32)
    for t in range(1, L):
        sel = np.arange(0, t + 1, 3)[:k]
        idx[t, : len(sel)] = sel
    idx[30, 5] = 35          # beyond t: must be skipped
    idx[31, 2] = 1 << 30     # far out of range: must be skipped
    idx[0, :] = -1           # no valid entry: O = 0, lse = -inf
    O = torch.empty(L, Hq, D, dtype=torch.bfloat16, device=DEV)
    lse = torch.empty(L, Hq, dtype=torch.float32, device=DEV)
    dsa.sparse_gqa_prefill(Q.to(DEV), K.to(DEV), V.to(DEV), torch.from_numpy(idx).to(DEV), 0, L, k, 0.125, O, lse)
    torch.cuda.synchronize()
    Oref, lref = oracle.sparse_attention(H(Q), H(K), H(V), idx, 0, 0.125)
    check_attention(O.float().cpu().numpy(), Oref, lse.cpu().numpy(), lref, "invalid entries")
    assert np.all(O[0].float().cpu().numpy() == 0) and np.all(np.isneginf(lse[0].cpu().numpy()))


# ----------------------------------------------------------------------------
# decode
# ----------------------------------------------------------------------------

def run_decode(cfg, d, k):
    B = d["q"].shape[0]
    need = dsa.decode_workspace_size(B, d["max_seq_len"], cfg.Hq, cfg.Hkv, cfg.D, k)
    ws = torch.empty(need, dtype=torch.uint8, device=DEV)
    out = torch.empty(B, cfg.Hq, cfg.D, dtype=torch.bfloat16, device=DEV)
    idx = torch.full((B, k), -7, dtype=torch.int32, device=DEV)
    dsa.sparse_gqa_decode(d["q"], d["q8"], d["sq"], d["w"], d["k8_cache"], d["sk_cache"], d["k_cache"],
                          d["v_cache"], d["block_table"], d["seq_lens"], d["max_seq_len"], k, cfg.sm_scale, ws,
                          out, idx_out=idx)
    torch.cuda.synchronize()
    return out.float().cpu().numpy(), idx.cpu().numpy()


def check_decode(cfg, dh, out, idx, k):
    h = {kk: (H(v) if isinstance(v, torch.Tensor) else v) for kk, v in dh.items()}
    I = oracle.decode_indexer(h["q8"], h["sq"], h["w"], h["k8_cache"], h["sk_cache"], h["block_table"],
                              h["seq_lens"])
    ref_idx = oracle.topk(I, h["seq_lens"], k)
    for b in range(len(h["seq_lens"])):
        check_topk_row(idx[b], ref_idx[b], I[b], int(h["seq_lens"][b]), k, f"seq {b}")
    Oref, _ = oracle.decode_attention(h["q"], h["k_cache"], h["v_cache"], h["block_table"], h["seq_lens"],
                                      ref_idx, cfg.sm_scale)
    same = np.all(idx == ref_idx, axis=1)
    check_attention(out[same], Oref[same], what="decode")
    if not same.all():
        # sequences whose set differs from the oracle's by near-ties: the
        # attention stage alone on the oracle's sets, so every sequence's
        # output is checked
        g = {kk: (v.to(DEV) if isinstance(v, torch.Tensor) else v) for kk, v in dh.items()}
        B = len(h["seq_lens"])
        ws = torch.empty(dsa.decode_attention_workspace_size(B, cfg.Hq, cfg.Hkv, cfg.D, k), dtype=torch.uint8,
                         device=DEV)
        o3 = torch.empty(B, cfg.Hq, cfg.D, dtype=torch.bfloat16, device=DEV)
        dsa.sparse_gqa_decode_attention(g["q"], g["k_cache"], g["v_cache"], g["block_table"], g["seq_lens"],
                                        torch.from_numpy(ref_idx).to(DEV), k, cfg.sm_scale, ws, o3)
        torch.cuda.synchronize()
        check_attention(o3.float().cpu().numpy()[~same], Oref[~same], what="decode (oracle index sets)")
    return I, ref_idx, Oref


@pytest.mark.parametrize("cfg_id,lens,k", [
    (0, [1, 63, 64, 65, 300, 1000], 64),
    (3, [1, 64, 2047, 2048, 2049, 5000, 70000], 2048),
])
def test_decode_small_matches_oracle(cfg_id, lens, k):
    cfg = inputs.config(cfg_id)
    d = inputs.decode_inputs(cfg, seq_lens=lens, seed=50 + cfg_id)
    out, idx = run_decode(cfg, _gpu(d), k)
    I, ref_idx, Oref = check_decode(cfg, d, out, idx, k)
    # stage 1 alone: scores through the block table
    g = _gpu(d)
    ld = (d["max_seq_len"] + 3) // 4 * 4
    sc = torch.zeros(len(lens), ld, dtype=torch.float32, device=DEV)
    dsa.decode_indexer_scores(g["q8"], g["sq"], g["w"], g["k8_cache"], g["sk_cache"], g["block_table"],
                              g["seq_lens"], d["max_seq_len"], sc)
    # stage 3 alone on the oracle's index sets
    ws = torch.empty(dsa.decode_attention_workspace_size(len(lens), cfg.Hq, cfg.Hkv, cfg.D, k), dtype=torch.uint8,
                     device=DEV)
    o3 = torch.empty(len(lens), cfg.Hq, cfg.D, dtype=torch.bfloat16, device=DEV)
    l3 = torch.empty(len(lens), cfg.Hq, dtype=torch.float32, device=DEV)
    dsa.sparse_gqa_decode_attention(g["q"], g["k_cache"], g["v_cache"], g["block_table"], g["seq_lens"],
                                    torch.from_numpy(ref_idx).to(DEV), k, cfg.sm_scale, ws, o3, l3)
    torch.cuda.synchronize()
    scn = sc.cpu().numpy()
    for b, n in enumerate(lens):
        check_scores(scn[b, :n], I[b, :n], f"decode scores seq {b}")
    h = {kk: (H(v) if isinstance(v, torch.Tensor) else v) for kk, v in d.items()}
    Oref2, lref2 = oracle.decode_attention(h["q"], h["k_cache"], h["v_cache"], h["block_table"], h["seq_lens"],
                                           ref_idx, cfg.sm_scale)
    check_attention(o3.float().cpu().numpy(), Oref2, l3.cpu().numpy(), lref2, "decode attention stage")


def _paged_exact(HI, dI, lens, seed, unmapped=()):
    """Exact-arithmetic keys (see inputs.exact_indexer_inputs) dealt to cache
    pages in a random order and shared by every sequence; sequence b's query
    is the exact query row of position lens[b] - 1.  `unmapped` lists
    (sequence, logical page, page id) entries written into the block table."""
    L = max(lens)
    P = (L + 63) // 64
    d = {k: v.numpy() for k, v in inputs.exact_indexer_inputs(L, HI, dI, seed=seed).items()}
    rng = np.random.default_rng(seed)
    n_pages = P + 2
    perm = rng.permutation(n_pages).astype(np.int32)
    k8c = np.zeros((n_pages, 64, dI), np.uint8)
    skc = np.ones((n_pages, 64), np.float32)
    for j in range(P):
        lo, hi = j * 64, min(L, j * 64 + 64)
        k8c[perm[j], : hi - lo] = d["k8"][lo:hi]
        skc[perm[j], : hi - lo] = d["sk"][lo:hi]
    B = len(lens)
    bt = np.tile(perm[:P], (B, 1)).astype(np.int32)
    for b, j, v in unmapped:
        bt[b, j] = v
    t = np.array(lens) - 1
    return dict(q8=d["q8"][t].copy(), sq=d["sq"][t].copy(), w=d["w"][t].copy(), k8_cache=k8c, sk_cache=skc,
                block_table=bt, seq_lens=np.array(lens, np.int32), max_seq_len=L, num_pages=n_pages)


def _decode_scores_gpu(h):
    g = {k: (torch.from_numpy(v).to(DEV) if isinstance(v, np.ndarray) else v) for k, v in h.items()}
    B = len(h["seq_lens"])
    ld = (h["max_seq_len"] + 3) // 4 * 4
    sc = torch.full((B, ld), float("nan"), dtype=torch.float32, device=DEV)
    dsa.decode_indexer_scores(g["q8"], g["sq"], g["w"], g["k8_cache"], g["sk_cache"], g["block_table"],
                              g["seq_lens"], h["max_seq_len"], sc)
    torch.cuda.synchronize()
    return sc.cpu().numpy()


@pytest.mark.parametrize("HI,dI", [(4, 32), (8, 64), (16, 128), (32, 64), (64, 128), (32, 32), (64, 64)])
def test_decode_indexer_exact_inputs_bit_exact(HI, dI):
    # lengths around page and 128-key item boundaries, one long sequence;
    # unmapped entries: past the cache, negative, and a whole odd last page
    lens = [1, 63, 64, 65, 127, 128, 129, 700, 1000, 257]
    P = (max(lens) + 63) // 64
    n_pages = P + 2
    unmapped = [(7, 3, n_pages), (8, 10, -3), (8, 0, n_pages + 100), (9, 4, -1), (2, 1, 2 ** 31 - 1)]
    h = _paged_exact(HI, dI, lens, seed=300 + HI + dI, unmapped=unmapped)
    ref = oracle.decode_indexer(h["q8"], h["sq"], h["w"], h["k8_cache"], h["sk_cache"], h["block_table"],
                                h["seq_lens"])
    got = _decode_scores_gpu(h)
    for b, n in enumerate(lens):
        assert np.array_equal(got[b, :n], ref[b, :n]), f"sequence {b}"
    assert np.isneginf(ref[7, 3 * 64]) and np.isneginf(ref[8, 0]) and np.isneginf(ref[9, 256])


@pytest.mark.parametrize("B", [4096, 4100])
def test_decode_indexer_large_batches(B):
    # 4096 sequences is the tensor-core path's largest batch; 4100 takes the
    # other path.  Both must give the same scores.
    cfg = inputs.config(0)
    lens = np.random.default_rng(B).integers(1, 300, B).tolist()
    d = inputs.decode_inputs(cfg, seq_lens=lens, seed=B)
    h = {k: (H(v) if isinstance(v, torch.Tensor) else v) for k, v in d.items()}
    ref = oracle.decode_indexer(h["q8"], h["sq"], h["w"], h["k8_cache"], h["sk_cache"], h["block_table"],
                                h["seq_lens"])
    got = _decode_scores_gpu(h)
    for b, n in enumerate(lens):
        check_scores(got[b, :n], ref[b, :n], f"sequence {b}")


# ----------------------------------------------------------------------------
# full-size workloads, sampled rows, benchmark launch configuration
# ----------------------------------------------------------------------------

def _sample_rows(L, k, extra, seed):
    rng = np.random.default_rng(seed)
    rows = {0, k - 2, k - 1, k, k + 1, L // 2 + 3, L - 1} | set(int(x) for x in rng.integers(0, L, 3)) | set(extra)
    return sorted(r for r in rows if 0 <= r < L)


@pytest.mark.parametrize("cfg_id", [1, 2, 4])
def test_full_size_prefill_sampled_rows(cfg_id):
    cfg = inputs.config(cfg_id)
    d = inputs.prefill_inputs(cfg, device=DEV)
    extra = []
    if cfg.multimodal:  # frame / text boundaries
        P = inputs.PERIOD
        extra = [P * 7 + 4095, P * 7 + 4096, P * 7 + 4159, P * 20 + 256]
    rows = _sample_rows(cfg.L, cfg.k, extra, seed=cfg_id)
    plan, O, lse, got_rows = run_prefill(cfg, d, want_rows=rows, fused=True)
    h = {kk: H(d[kk]) for kk in ("q8", "sq", "w", "k8", "sk")}
    Kh, Vh = H(d["K"]), H(d["V"])
    sel = torch.tensor(rows, device=DEV)
    gidx = plan.idx[sel].cpu().numpy()
    Og, lg = O[sel].float().cpu().numpy(), lse[sel].cpu().numpy()
    Qh = H(d["Q"][sel])
    for i, t in enumerate(rows):
        I = oracle.indexer(h["q8"], h["sq"], h["w"], h["k8"], h["sk"], row_begin=t, n_rows=1)[0]
        check_scores(got_rows[t], I, f"cfg{cfg_id} row {t}")
        ref_idx = oracle.topk(I[None, :], [t + 1], cfg.k)
        check_topk_row(gidx[i], ref_idx[0], I, t + 1, cfg.k, f"cfg{cfg_id} row {t}")
        Oref, lref = oracle.sparse_attention(Qh[i:i + 1], Kh, Vh, ref_idx, t, cfg.sm_scale)
        if np.array_equal(gidx[i], ref_idx[0]):
            check_attention(Og[i:i + 1], Oref, lg[i:i + 1], lref, f"cfg{cfg_id} row {t}")
        else:
            O1 = torch.empty(1, cfg.Hq, cfg.D, dtype=torch.bfloat16, device=DEV)
            dsa.sparse_gqa_prefill(d["Q"][t:t + 1], d["K"], d["V"], torch.from_numpy(ref_idx).to(DEV), t, 1, cfg.k,
                                   cfg.sm_scale, O1)
            torch.cuda.synchronize()
            check_attention(O1.float().cpu().numpy(), Oref, what=f"cfg{cfg_id} row {t} (oracle idx)")
    check_index_structure_on_device(plan.idx, 0, cfg.k)


def check_index_structure_on_device(idx, row_begin, k, row_len=None, step=8192):
    """Every row: count = min(k, n), ascending, within [0, n), -1 padded."""
    L = idx.shape[0]
    ar = torch.arange(k, device=idx.device)
    for r0 in range(0, L, step):
        blk = idx[r0:r0 + step]
        r = torch.arange(r0, r0 + blk.shape[0], device=idx.device)
        n = (row_begin + r + 1) if row_len is None else row_len[r0:r0 + step]
        cnt = torch.clamp(n, max=k)
        valid = blk >= 0
        assert torch.equal(valid, ar[None, :] < cnt[:, None]), "count / padding"
        assert bool(((blk[:, 1:] > blk[:, :-1]) | ~valid[:, 1:]).all()), "ascending"
        assert bool((torch.where(valid, blk, -1) < n[:, None]).all()), "range"
        assert bool((blk[~valid] == -1).all()), "padding value"


def test_full_size_decode_all_sequences():
    cfg = inputs.config(3)
    d = inputs.decode_inputs(cfg, device=DEV)
    out, idx = run_decode(cfg, d, cfg.k)
    check_decode(cfg, d, out, idx, cfg.k)
