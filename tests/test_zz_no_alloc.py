"""The decode attention entry point that allocates nothing.

Some callers cannot allocate device memory: a plugin or serving hook that is
handed only its input and output buffers, or a latency-critical loop where
cudaMalloc is not allowed.  dsa_sparse_gqa_decode_attention_noalloc serves
them by keeping its split-K partials in a fixed array inside the library.
These tests call it through the C ABI and compare it with the workspace
entry point, dsa_sparse_gqa_decode_attention, on two calls in a row (the
second call reuses the array the first one left behind), within the
attention tolerance the parity tests use.  The file is named so that pytest
collects it last; it also passes on its own in a fresh process.
"""
import numpy as np
import pytest
import torch

from parity_helpers import ATTN_MAX_ABS, LSE_ATOL
from sparse_long_context_03_b200 import dsa, inputs

DEV = "cuda"


def _decode_case(cfg_id, lens, k, seed):
    cfg = inputs.config(cfg_id)
    g = inputs.decode_inputs(cfg, seq_lens=lens, seed=seed, device=DEV)
    d = g
    B = len(lens)
    # index rows from the library's own decode chain: any valid rows will do
    ws = torch.empty(dsa.decode_workspace_size(B, d["max_seq_len"], cfg.Hq, cfg.Hkv, cfg.D, k), dtype=torch.uint8,
                     device=DEV)
    out = torch.empty(B, cfg.Hq, cfg.D, dtype=torch.bfloat16, device=DEV)
    idx = torch.empty(B, k, dtype=torch.int32, device=DEV)
    dsa.sparse_gqa_decode(g["q"], g["q8"], g["sq"], g["w"], g["k8_cache"], g["sk_cache"], g["k_cache"],
                          g["v_cache"], g["block_table"], g["seq_lens"], d["max_seq_len"], k, cfg.sm_scale, ws, out,
                          idx_out=idx)
    return cfg, g, idx


def _with_workspace(cfg, g, idx, k):
    B = idx.shape[0]
    ws = torch.empty(dsa.decode_attention_workspace_size(B, cfg.Hq, cfg.Hkv, cfg.D, k), dtype=torch.uint8,
                     device=DEV)
    out = torch.empty(B, cfg.Hq, cfg.D, dtype=torch.bfloat16, device=DEV)
    lse = torch.empty(B, cfg.Hq, dtype=torch.float32, device=DEV)
    dsa.sparse_gqa_decode_attention(g["q"], g["k_cache"], g["v_cache"], g["block_table"], g["seq_lens"], idx, k,
                                    cfg.sm_scale, ws, out, lse)
    return out, lse


def _no_alloc(cfg, g, idx, k):
    B = idx.shape[0]
    out = torch.full((B, cfg.Hq, cfg.D), float("nan"), dtype=torch.bfloat16, device=DEV)
    lse = torch.full((B, cfg.Hq), float("nan"), dtype=torch.float32, device=DEV)
    dsa.sparse_gqa_decode_attention_noalloc(g["q"], g["k_cache"], g["v_cache"], g["block_table"], g["seq_lens"],
                                            idx, k, cfg.sm_scale, out, lse)
    return out, lse


def _compare(a, b):
    (oa, la), (ob, lb) = a, b
    err = (oa.float() - ob.float()).abs().max().item()
    assert err <= ATTN_MAX_ABS, f"output differs by {err}"
    la, lb = la.cpu().numpy(), lb.cpu().numpy()
    assert np.array_equal(np.isfinite(la), np.isfinite(lb))
    fin = np.isfinite(lb)
    assert np.max(np.abs(la[fin] - lb[fin])) <= LSE_ATOL


@pytest.mark.gpu
def test_no_alloc_decode_matches_workspace_entry_two_calls():
    # first call: the batch-32 layer shape; second call: a different, smaller
    # case reusing whatever the first call left in the fixed array
    k = 2048
    cfg, g, idx = _decode_case(3, [2049, 64, 70000, 1, 5000, 131072] * 5 + [40000, 2048], k, seed=71)
    _compare(_no_alloc(cfg, g, idx, k), _with_workspace(cfg, g, idx, k))
    cfg2, g2, idx2 = _decode_case(0, [1, 63, 300, 1000], 64, seed=72)
    _compare(_no_alloc(cfg2, g2, idx2, 64), _with_workspace(cfg2, g2, idx2, 64))
    # and the first case once more, after the second overwrote the array
    _compare(_no_alloc(cfg, g, idx, k), _with_workspace(cfg, g, idx, k))
    torch.cuda.synchronize()


@pytest.mark.gpu
def test_no_alloc_rejects_batches_beyond_its_scratch():
    assert dsa.decode_attention_fixed_scratch_bytes() == 8 << 20
    lib = dsa.lib()
    bogus = 0x1000  # never dereferenced: the size check comes before any launch
    B = 505  # 505 * 4 * 8 * 130 * 4 bytes > 8 MiB
    rc = lib.dsa_sparse_gqa_decode_attention_noalloc(*([bogus] * 4), 16, 100, bogus, bogus, B, 32, 4, 128, 2048,
                                                     0.1, bogus, None, None)
    assert rc == 3  # DSA_ERR_WORKSPACE
    assert b"fixed decode scratch" in lib.dsa_last_error_string()


@pytest.mark.gpu
@pytest.mark.parametrize("cfg_id,B", [(3, 504), (0, 1985)])
def test_no_alloc_largest_accepted_batch(cfg_id, B):
    # the largest batch whose partials fit the fixed array (B * Hkv * 8 *
    # (D + 2) * 4 bytes <= 8 MiB): one split per (sequence, group), the
    # partials reaching the end of the array
    cfg = inputs.config(cfg_id)
    assert B * cfg.Hkv * 8 * (cfg.D + 2) * 4 <= dsa.decode_attention_fixed_scratch_bytes()
    assert (B + 1) * cfg.Hkv * 8 * (cfg.D + 2) * 4 > dsa.decode_attention_fixed_scratch_bytes()
    rng = np.random.default_rng(B)
    lens = [int(x) for x in rng.integers(1, 400, B)]
    k = cfg.k
    cfg, g, idx = _decode_case(cfg_id, lens, k, seed=80 + cfg_id)
    _compare(_no_alloc(cfg, g, idx, k), _with_workspace(cfg, g, idx, k))
    _compare(_no_alloc(cfg, g, idx, k), _with_workspace(cfg, g, idx, k))
    torch.cuda.synchronize()
