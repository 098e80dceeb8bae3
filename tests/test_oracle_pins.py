"""Pins of the fp64 oracle against what the pages and mathematics fix.

Each test ties one part of the oracle to something other than itself: a
hand-worked or closed-form example (tests/golden), a library routine (torch's
e4m3 / bf16 conversions, numpy's sort and argmax, scipy's logsumexp), a
separately written dense formulation, or an invariant of the definitions in
"Kwai Keye-VL-2.0 Technical Report" review (xllm-io), 核心公式 (indexer score,
top-k set, GQA sparse aggregation) and report translation sections 2.3.1,
2.3.2, 5.1.2 and 5.2.1.
"""
import math

import numpy as np
import pytest
import torch
from scipy.special import logsumexp

from conftest import read_golden
from sparse_long_context_03_b200 import inputs


def _e4m3_np(b):
    """Library decoding of e4m3fn bytes (torch), independent of the oracle."""
    t = torch.from_numpy(np.ascontiguousarray(b).astype(np.uint8))
    return t.view(torch.float8_e4m3fn).to(torch.float64).numpy()


def _bf16_np(h):
    t = torch.from_numpy(np.ascontiguousarray(h).astype(np.uint16).view(np.int16))
    return t.view(torch.bfloat16).to(torch.float64).numpy()


def _np(t):
    return inputs.to_numpy_bits(t)


# ----------------------------------------------------------------------------
# number formats
# ----------------------------------------------------------------------------

def test_e4m3_closed_forms(oracle_mod):
    o = oracle_mod
    assert o.e4m3_to_double(0x38) == 1.0
    assert o.e4m3_to_double(0x7E) == 448.0           # largest finite
    assert o.e4m3_to_double(0x01) == 2.0 ** -9       # smallest subnormal
    assert o.e4m3_to_double(0x07) == 7 * 2.0 ** -9   # largest subnormal
    assert o.e4m3_to_double(0x08) == 2.0 ** -6       # smallest normal
    assert o.e4m3_to_double(0x44) == 3.0
    assert o.e4m3_to_double(0xB8) == -1.0
    z = o.e4m3_to_double(0x80)
    assert z == 0.0 and math.copysign(1.0, z) < 0
    assert math.isnan(o.e4m3_to_double(0x7F)) and math.isnan(o.e4m3_to_double(0xFF))


def test_e4m3_all_codes_match_torch(oracle_mod):
    codes = np.arange(256, dtype=np.uint8)
    ref = _e4m3_np(codes)
    got = np.array([oracle_mod.e4m3_to_double(int(c)) for c in codes])
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], ref[~nan])


def test_bf16_matches_torch(oracle_mod):
    rng = np.random.default_rng(5)
    h = rng.integers(0, 1 << 16, 4000).astype(np.uint16)
    h = h[(h & 0x7F80) != 0x7F80]  # finite patterns only
    ref = _bf16_np(h)
    got = np.array([oracle_mod.bf16_to_double(int(v)) for v in h])
    assert np.array_equal(got, ref)


# ----------------------------------------------------------------------------
# indexer
# ----------------------------------------------------------------------------

def _golden_indexer():
    g = read_golden("indexer_hand_example.txt")
    q8 = np.array(g["q8"], np.uint8).reshape(3, 2, 2)
    k8 = np.array(g["k8"], np.uint8).reshape(3, 2)
    sq = np.array(g["sq"], np.float32)
    sk = np.array(g["sk"], np.float32)
    w = np.array(g["w"], np.float32).reshape(3, 2)
    return g, q8, sq, w, k8, sk


def test_indexer_hand_example(oracle_mod):
    g, q8, sq, w, k8, sk = _golden_indexer()
    I = oracle_mod.indexer(q8, sq, w, k8, sk)
    for t in range(3):
        assert np.array_equal(I[t, : t + 1], np.array(g[f"I{t}"]))
        assert np.all(np.isneginf(I[t, t + 1:]))
    assert np.array_equal(oracle_mod.causal_topk(I, 0, 1).ravel(), np.array(g["topk1"], np.int32))
    assert np.array_equal(oracle_mod.causal_topk(I, 0, 2).ravel(), np.array(g["topk2"], np.int32))


def test_indexer_chunk_rows_match_full(oracle_mod):
    g, q8, sq, w, k8, sk = _golden_indexer()
    full = oracle_mod.indexer(q8, sq, w, k8, sk)
    part = oracle_mod.indexer(q8, sq, w, k8, sk, row_begin=1, n_rows=2)
    assert np.array_equal(part, full[1:3])


def test_indexer_single_head_unit_weight_is_relu_dot(oracle_mod):
    # H^I = 1, w = 1: the score is the plain ReLU of a dot product.
    cfg = inputs.config(0, HI=1)
    d = inputs.prefill_inputs(cfg, L=64, seed=7)
    w = np.ones((64, 1), np.float32)
    I = oracle_mod.indexer(_np(d["q8"]), _np(d["sq"]), w, _np(d["k8"]), _np(d["sk"]))
    q = _e4m3_np(_np(d["q8"]))[:, 0, :] * _np(d["sq"]).astype(np.float64)[:, None]
    k = _e4m3_np(_np(d["k8"])) * _np(d["sk"]).astype(np.float64)[:, None]
    dots = q @ k.T
    ref = np.maximum(dots, 0.0)
    tri = np.tril(np.ones((64, 64), bool))
    assert (dots[tri] < 0).sum() > 100  # the ReLU is exercised
    np.testing.assert_allclose(I[tri], ref[tri], rtol=1e-12, atol=1e-12)


def _dense_indexer_numpy(q8, sq, w, k8, sk):
    """Separately written vectorised indexer (library matmul) for brute-force checks."""
    q = _e4m3_np(q8) * sq.astype(np.float64)[:, None, None]
    k = _e4m3_np(k8) * sk.astype(np.float64)[:, None]
    dots = np.einsum("tjc,sc->tjs", q, k)
    return np.einsum("tj,tjs->ts", w.astype(np.float64), np.maximum(dots, 0.0))


def test_indexer_brute_force_tiny(oracle_mod):
    cfg = inputs.config(0)
    d = inputs.prefill_inputs(cfg, L=160, seed=11)
    args = [_np(d[k]) for k in ("q8", "sq", "w", "k8", "sk")]
    I = oracle_mod.indexer(*args)
    ref = _dense_indexer_numpy(*args)
    tri = np.tril(np.ones(I.shape, bool))
    np.testing.assert_allclose(I[tri], ref[tri], rtol=1e-12, atol=1e-12)
    assert np.all(np.isneginf(I[~tri]))
    assert np.all(I[tri] >= 0.0)  # w >= 0 here


def test_indexer_signed_weights_and_linearity(oracle_mod):
    cfg = inputs.config(0)
    d = inputs.prefill_inputs(cfg, L=48, seed=12)
    q8, sq, k8, sk = (_np(d[k]) for k in ("q8", "sq", "k8", "sk"))
    rng = np.random.default_rng(3)
    w1 = rng.standard_normal((48, cfg.HI)).astype(np.float32)
    w2 = rng.standard_normal((48, cfg.HI)).astype(np.float32)
    I1 = oracle_mod.indexer(q8, sq, w1, k8, sk)
    I2 = oracle_mod.indexer(q8, sq, w2, k8, sk)
    I12 = oracle_mod.indexer(q8, sq, (w1.astype(np.float64) + w2).astype(np.float32), k8, sk)
    tri = np.tril(np.ones(I1.shape, bool))
    assert (I1[tri] < 0).any()  # negative w can give negative scores
    w12 = w1.astype(np.float64) + w2
    exact = np.array_equal(w12.astype(np.float32).astype(np.float64), w12)
    if exact:
        np.testing.assert_allclose(I12[tri], (I1 + I2)[tri], rtol=1e-12, atol=1e-12)
    # Positive homogeneity in the key scale: doubling sk doubles the row.
    I2k = oracle_mod.indexer(q8, sq, w1, k8, sk * 2)
    np.testing.assert_allclose(I2k[tri], 2 * I1[tri], rtol=1e-13, atol=0)


def test_indexer_is_causal(oracle_mod):
    cfg = inputs.config(0)
    d = inputs.prefill_inputs(cfg, L=64, seed=13)
    q8, sq, w, k8, sk = (_np(d[k]).copy() for k in ("q8", "sq", "w", "k8", "sk"))
    I = oracle_mod.indexer(q8, sq, w, k8, sk)
    k8b = k8.copy()
    k8b[40:] = np.uint8(0x38)
    Ib = oracle_mod.indexer(q8, sq, w, k8b, sk)
    assert np.array_equal(I[:40], Ib[:40])
    assert not np.array_equal(I[40:], Ib[40:])


def test_exact_inputs_are_fp32_exact(oracle_mod):
    d = inputs.exact_indexer_inputs(96, 32, 64, seed=21)
    I = oracle_mod.indexer(*(_np(d[k]) for k in ("q8", "sq", "w", "k8", "sk")))
    tri = np.tril(np.ones(I.shape, bool))
    vals = I[tri]
    assert np.array_equal(vals.astype(np.float32).astype(np.float64), vals)
    # with a key pool, rows hold many exact ties
    d = inputs.exact_indexer_inputs(96, 32, 64, seed=22, key_pool=6)
    I = oracle_mod.indexer(*(_np(d[k]) for k in ("q8", "sq", "w", "k8", "sk")))
    vals = I[tri]
    assert np.array_equal(vals.astype(np.float32).astype(np.float64), vals)
    assert len(I[95]) - len(np.unique(I[95])) >= 90


# ----------------------------------------------------------------------------
# top-k
# ----------------------------------------------------------------------------

def _topk_by_sort(row, k):
    order = sorted(range(len(row)), key=lambda s: (-row[s], s))
    sel = sorted(order[:k])
    return sel + [-1] * (k - len(sel))


def test_topk_matches_sorted_definition(oracle_mod):
    x = inputs.tie_heavy_scores(12, 300, seed=4).numpy().astype(np.float64)
    lens = np.array([300, 299, 257, 256, 255, 100, 64, 63, 10, 1, 0, 150], np.int32)
    for k in (1, 5, 64, 256, 299):
        got = oracle_mod.topk(x, lens, k)
        for r in range(len(lens)):
            assert list(got[r]) == _topk_by_sort(list(x[r, : lens[r]]), k)


def test_topk_k1_is_first_argmax(oracle_mod):
    x = inputs.tie_heavy_scores(20, 77, seed=8).numpy().astype(np.float64)
    got = oracle_mod.topk(x, 77, 1)
    assert np.array_equal(got[:, 0], np.argmax(x, axis=1).astype(np.int32))


def test_topk_short_rows_keep_everything(oracle_mod):
    x = np.random.default_rng(1).standard_normal((4, 50))
    got = oracle_mod.topk(x, [50, 49, 3, 1], 50)
    for r, n in enumerate([50, 49, 3, 1]):
        assert list(got[r]) == list(range(n)) + [-1] * (50 - n)


def test_topk_all_equal_and_signed_zero(oracle_mod):
    x = np.full((1, 40), 0.5)
    assert list(oracle_mod.topk(x, 40, 7)[0]) == list(range(7))
    z = np.array([[-0.0, 0.0, -0.0, 0.0, -1.0]])
    assert list(oracle_mod.topk(z, 5, 2)[0]) == [0, 1]
    z2 = np.array([[-1.0, -0.0, -2.0, 0.0]])
    assert list(oracle_mod.topk(z2, 4, 1)[0]) == [1]


# ----------------------------------------------------------------------------
# sparse GQA attention
# ----------------------------------------------------------------------------

def _dense_causal_gqa_numpy(Q, K, V, sm_scale):
    """Separately written dense causal GQA attention (scipy logsumexp)."""
    Qd, Kd, Vd = _bf16_np(Q), _bf16_np(K), _bf16_np(V)
    L, Hq, D = Qd.shape
    Hkv = Kd.shape[1]
    G = Hq // Hkv
    O = np.zeros_like(Qd)
    lse = np.zeros((L, Hq))
    for h in range(Hq):
        g = h // G
        logits = sm_scale * Qd[:, h, :] @ Kd[:, g, :].T
        logits[np.triu(np.ones((L, L), bool), 1)] = -np.inf
        lse[:, h] = logsumexp(logits, axis=1)
        P = np.exp(logits - lse[:, h:h + 1])
        O[:, h, :] = P @ Vd[:, g, :]
    return O, lse


def _attn_inputs(L, Hq=8, Hkv=2, D=16, seed=3):
    g = torch.Generator().manual_seed(seed)
    Q = (torch.randn(L, Hq, D, generator=g)).to(torch.bfloat16)
    K = (torch.randn(L, Hkv, D, generator=g)).to(torch.bfloat16)
    V = (torch.randn(L, Hkv, D, generator=g)).to(torch.bfloat16)
    return _np(Q), _np(K), _np(V)


def test_attention_closed_form(oracle_mod):
    g = read_golden("attention_closed_form.txt")
    bf = lambda v: _np(torch.tensor(v, dtype=torch.float32).to(torch.bfloat16))
    Q = bf(g["q"]).reshape(1, 1, 2)
    K = bf(g["K"]).reshape(2, 1, 2)
    V = bf(g["V"]).reshape(2, 1, 2)
    for idx in ([[0, 1]], [[1, 0]], [[1, 0, -1]]):
        O, lse = oracle_mod.sparse_attention(Q, K, V, np.array(idx, np.int32), 1, 1.0)
        np.testing.assert_allclose(O[0, 0], g["O"], rtol=1e-15)
        np.testing.assert_allclose(lse[0, 0], g["lse"][0], rtol=1e-15)


def test_attention_full_budget_equals_dense(oracle_mod):
    # k >= L selects every causal key: sparse attention must equal dense.
    L = 40
    Q, K, V = _attn_inputs(L)
    sm = 1 / math.sqrt(16)
    idx = np.full((L, L + 3), -1, np.int32)
    for t in range(L):
        idx[t, : t + 1] = np.arange(t + 1)
    O, lse = oracle_mod.sparse_attention(Q, K, V, idx, 0, sm)
    Od, lsed = _dense_causal_gqa_numpy(Q, K, V, sm)
    np.testing.assert_allclose(O, Od, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(lse, lsed, rtol=1e-12, atol=1e-12)


def test_attention_special_cases(oracle_mod):
    L = 24
    Q, K, V = _attn_inputs(L, seed=9)
    sm = 0.25
    # t = 0 attends only to itself: O = V[0, g]
    O, _ = oracle_mod.sparse_attention(Q[:1], K, V, np.array([[0, -1, -1]], np.int32), 0, sm)
    Vd = _bf16_np(V)
    for h in range(8):
        np.testing.assert_array_equal(O[0, h], Vd[0, h // 4])
    # constant V rows: O equals that row whatever the weights
    Vc = np.tile(V[5:6], (L, 1, 1))
    idx = np.array([[3, 9, 17, 20]], np.int32)
    O, _ = oracle_mod.sparse_attention(Q[20:21], K, Vc, idx, 20, sm)
    for h in range(8):
        np.testing.assert_allclose(O[0, h], _bf16_np(Vc)[0, h // 4], rtol=1e-14)
    # permuting Omega leaves the output unchanged
    O1, l1 = oracle_mod.sparse_attention(Q[20:21], K, V, idx, 20, sm)
    O2, l2 = oracle_mod.sparse_attention(Q[20:21], K, V, idx[:, ::-1].copy(), 20, sm)
    np.testing.assert_allclose(O1, O2, rtol=1e-14, atol=1e-15)
    np.testing.assert_allclose(l1, l2, rtol=1e-14)


def test_attention_one_index_set_for_every_group(oracle_mod):
    # Distinct K/V per group; each head must read its own group's rows at the
    # same positions Omega_t (report translation 2.3.2).
    L, Hq, Hkv, D = 30, 8, 4, 16
    Q, K, V = _attn_inputs(L, Hq, Hkv, D, seed=15)
    sm = 0.3
    idx = np.array([[2, 7, 11, 29, -1]], np.int32)
    O, lse = oracle_mod.sparse_attention(Q[29:30], K, V, idx, 29, sm)
    Qd, Kd, Vd = _bf16_np(Q), _bf16_np(K), _bf16_np(V)
    sel = [2, 7, 11, 29]
    for h in range(Hq):
        g = h // (Hq // Hkv)
        logits = sm * Kd[sel, g, :] @ Qd[29, h, :]
        p = np.exp(logits - logsumexp(logits))
        np.testing.assert_allclose(O[0, h], p @ Vd[sel, g, :], rtol=1e-12, atol=1e-14)
        np.testing.assert_allclose(lse[0, h], logsumexp(logits), rtol=1e-13)


# ----------------------------------------------------------------------------
# paged decode
# ----------------------------------------------------------------------------

def _contiguous_from_pages(cache, bt_row, n):
    pages = cache[bt_row[: (n + 63) // 64]]
    return pages.reshape((-1,) + cache.shape[2:])[:n]


def test_decode_paged_equals_contiguous(oracle_mod):
    cfg = inputs.config(0)
    d = inputs.decode_inputs(cfg, B=3, seq_lens=[130, 64, 77], seed=5)
    n = {k: (_np(v) if isinstance(v, torch.Tensor) else v) for k, v in d.items()}
    I = oracle_mod.decode_indexer(n["q8"], n["sq"], n["w"], n["k8_cache"], n["sk_cache"],
                                  n["block_table"], n["seq_lens"], ld=130)
    k = 16
    idx = np.full((3, k), -1, np.int32)
    for b in range(3):
        sl = int(n["seq_lens"][b])
        t = sl - 1
        k8 = _contiguous_from_pages(n["k8_cache"], n["block_table"][b], sl)
        sk = _contiguous_from_pages(n["sk_cache"], n["block_table"][b], sl)
        q8 = np.zeros((sl, cfg.HI, cfg.dI), np.uint8)
        q8[t] = n["q8"][b]
        sq = np.ones(sl, np.float32)
        sq[t] = n["sq"][b]
        w = np.zeros((sl, cfg.HI), np.float32)
        w[t] = n["w"][b]
        ref = oracle_mod.indexer(q8, sq, w, k8, sk, row_begin=t, n_rows=1)
        assert np.array_equal(I[b, :sl], ref[0])
        assert np.all(np.isneginf(I[b, sl:]))
        idx[b] = oracle_mod.topk(I[b:b + 1], sl, k)[0]
        # attention through the pages equals contiguous attention at t
        Kc = _contiguous_from_pages(n["k_cache"], n["block_table"][b], sl)
        Vc = _contiguous_from_pages(n["v_cache"], n["block_table"][b], sl)
        Oc, lc = oracle_mod.sparse_attention(n["q"][b:b + 1], Kc, Vc, idx[b:b + 1], t, cfg.sm_scale)
        Od, ld_ = oracle_mod.decode_attention(n["q"][b:b + 1], n["k_cache"], n["v_cache"],
                                              n["block_table"][b:b + 1], n["seq_lens"][b:b + 1],
                                              idx[b:b + 1], cfg.sm_scale)
        np.testing.assert_array_equal(Od, Oc)
        np.testing.assert_array_equal(ld_, lc)


def test_decode_unmapped_pages_have_no_keys(oracle_mod):
    # Library convention, not from the pages: a block-table entry outside the
    # cache's pages maps no key.  Its tokens score -inf, the others keep the
    # scores of the fully mapped table, and attention over an index set that
    # names them equals contiguous attention over the set without them.
    cfg = inputs.config(0)
    d = inputs.decode_inputs(cfg, seq_lens=[200], seed=6)
    n = {k: (_np(v) if isinstance(v, torch.Tensor) else v) for k, v in d.items()}
    full = oracle_mod.decode_indexer(n["q8"], n["sq"], n["w"], n["k8_cache"], n["sk_cache"],
                                     n["block_table"], n["seq_lens"])
    bt = n["block_table"].copy()
    P = n["k8_cache"].shape[0]
    bt[0, 1] = P       # tokens 64..127
    bt[0, 3] = -5      # tokens 192..199
    I = oracle_mod.decode_indexer(n["q8"], n["sq"], n["w"], n["k8_cache"], n["sk_cache"], bt, n["seq_lens"])
    gone = np.zeros(200, bool)
    gone[64:128] = True
    gone[192:200] = True
    assert np.all(np.isneginf(I[0, gone]))
    np.testing.assert_array_equal(I[0, ~gone], full[0, ~gone])
    idx = np.array([[3, 70, 130, 195, 199, 10, 127, 64]], np.int32)
    Od, lse_d = oracle_mod.decode_attention(n["q"], n["k_cache"], n["v_cache"], bt, n["seq_lens"], idx,
                                            cfg.sm_scale)
    keep = np.array([[3, 130, 10, -1, -1, -1, -1, -1]], np.int32)
    Kc = _contiguous_from_pages(n["k_cache"], n["block_table"][0], 200)
    Vc = _contiguous_from_pages(n["v_cache"], n["block_table"][0], 200)
    Oc, lc = oracle_mod.sparse_attention(n["q"], Kc, Vc, keep, 199, cfg.sm_scale)
    np.testing.assert_array_equal(Od, Oc)
    np.testing.assert_array_equal(lse_d, lc)


def test_oracle_results_do_not_depend_on_thread_count(oracle_mod):
    cfg = inputs.config(0)
    d = inputs.prefill_inputs(cfg, L=96, seed=31)
    args = [_np(d[k]) for k in ("q8", "sq", "w", "k8", "sk")]
    n0 = oracle_mod.threads()
    try:
        oracle_mod.set_threads(1)
        a = oracle_mod.indexer(*args)
        oracle_mod.set_threads(max(2, n0))
        b = oracle_mod.indexer(*args)
    finally:
        oracle_mod.set_threads(n0)
    assert np.array_equal(a, b)


# ----------------------------------------------------------------------------
# indexer distillation losses (dense warm-up, sparse adaptation)
# ----------------------------------------------------------------------------

def test_indexer_kl_hand_example(oracle_mod):
    g = read_golden("indexer_kl_hand_example.txt")
    I = np.array([g["dense_I"]])                      # row t = 1
    p = np.array([[g["dense_p_g0"], g["dense_p_g1"]]])
    loss, total = oracle_mod.indexer_kl(I, p, row_begin=1)
    assert loss[0] == pytest.approx(g["dense_loss"][0], rel=1e-14)
    assert total == pytest.approx(g["dense_loss"][0], rel=1e-14)
    I = np.array([g["sparse_I"]])                     # row t = 2
    p = np.array([[g["sparse_p"]]])
    idx = np.array([[int(x) for x in g["sparse_idx"]]], np.int32)
    loss, _ = oracle_mod.indexer_kl(I, p, row_begin=2, idx=idx)
    assert loss[0] == pytest.approx(g["sparse_loss"][0], rel=1e-14)


def _kl_case(seed, n_rows=6, L=40, G=3, zeros=True):
    rng = np.random.default_rng(seed)
    I = rng.normal(0, 3, (n_rows, L))
    p = rng.random((n_rows, G, L)) ** 3
    if zeros:
        p[rng.random(p.shape) < 0.3] = 0.0
    return I, p


def test_indexer_kl_matches_scipy_entropy(oracle_mod):
    # scipy.stats.entropy(pk, qk) normalises pk and qk and returns KL(pk || qk)
    from scipy.special import softmax
    from scipy.stats import entropy
    I, p = _kl_case(1)
    r0 = 30
    loss, total = oracle_mod.indexer_kl(I, p, row_begin=r0)
    for r in range(I.shape[0]):
        t = r0 + r
        q = softmax(I[r, : t + 1])
        ref = sum(entropy(p[r, g, : t + 1], q) for g in range(p.shape[1]))
        assert loss[r] == pytest.approx(ref, rel=1e-12, abs=1e-14)
    assert total == pytest.approx(loss.sum(), rel=1e-14)


def test_indexer_kl_zero_when_target_is_the_indexer_softmax(oracle_mod):
    from scipy.special import softmax
    rng = np.random.default_rng(2)
    L, r0 = 20, 14
    I = rng.normal(0, 2, (6, L))
    p = np.zeros((6, 2, L))
    for r in range(6):
        t = r0 + r
        for g, c in enumerate((1.0, 7.5)):   # any positive multiple of the softmax
            p[r, g, : t + 1] = softmax(I[r, : t + 1]) * c
    loss, _ = oracle_mod.indexer_kl(I, p, row_begin=r0)
    assert np.all(np.abs(loss) < 1e-12)


def test_indexer_kl_invariances_and_sign(oracle_mod):
    I, p = _kl_case(3)
    r0 = 34
    base, _ = oracle_mod.indexer_kl(I, p, row_begin=r0)
    assert np.all(base > 0)                                        # Gibbs: KL >= 0
    shifted, _ = oracle_mod.indexer_kl(I + 11.25, p, row_begin=r0)  # softmax is shift invariant
    np.testing.assert_allclose(shifted, base, rtol=1e-11)
    scaled, _ = oracle_mod.indexer_kl(I, p * 3.5, row_begin=r0)     # the target is normalised
    np.testing.assert_allclose(scaled, base, rtol=1e-12)
    # entries right of the causal range take no part
    I2, p2 = I.copy(), p.copy()
    for r in range(I.shape[0]):
        I2[r, r0 + r + 1:] = 1e3
        p2[r, :, r0 + r + 1:] = 5.0
    np.testing.assert_allclose(oracle_mod.indexer_kl(I2, p2, row_begin=r0)[0], base, rtol=1e-14)


def test_indexer_kl_sparse_over_every_causal_key_is_dense(oracle_mod):
    I, p = _kl_case(4)
    r0 = 34
    dense, _ = oracle_mod.indexer_kl(I, p, row_begin=r0)
    k = 48
    rng = np.random.default_rng(5)
    idx = np.full((I.shape[0], k), -1, np.int32)
    for r in range(I.shape[0]):
        idx[r, : r0 + r + 1] = rng.permutation(r0 + r + 1)
    sparse, _ = oracle_mod.indexer_kl(I, p, row_begin=r0, idx=idx)
    np.testing.assert_allclose(sparse, dense, rtol=1e-12)


def test_indexer_kl_sparse_is_dense_on_the_truncated_row(oracle_mod):
    # the sparse loss over S equals the dense loss of a row that holds only
    # the keys of S (the target renormalised over S, the softmax over S)
    from scipy.special import softmax
    from scipy.stats import entropy
    I, p = _kl_case(6, n_rows=4, L=40, G=2)
    r0 = 36
    rng = np.random.default_rng(7)
    idx = np.full((4, 9), -1, np.int32)
    for r in range(4):
        idx[r, :7] = rng.choice(r0 + r + 1, 7, replace=False)
    sparse, _ = oracle_mod.indexer_kl(I, p, row_begin=r0, idx=idx)
    for r in range(4):
        S = idx[r, :7]
        ref = sum(entropy(p[r, g, S], softmax(I[r, S])) if p[r, g, S].sum() > 0 else 0.0 for g in range(2))
        assert sparse[r] == pytest.approx(ref, rel=1e-12, abs=1e-14)


def test_indexer_kl_group_without_mass_contributes_nothing(oracle_mod):
    I, p = _kl_case(8, n_rows=3, L=12, G=2, zeros=False)
    r0 = 9
    base, _ = oracle_mod.indexer_kl(I, p[:, :1], row_begin=r0)
    p[:, 1] = 0.0
    both, _ = oracle_mod.indexer_kl(I, p, row_begin=r0)
    np.testing.assert_allclose(both, base, rtol=1e-15)
