"""GPU parity of packed (varlen) prefill: several sequences along one token
axis, each its own causal prefill, one launch per stage for all of them
(dsa_indexer_topk_varlen, dsa_sparse_gqa_prefill_varlen; report translation
section 5.1.2, per-sample causal regions).

Each sequence is checked against the oracle run on its own slice (bit-exact
indices on exact-arithmetic inputs, attention within the criterion), and the
packed result must equal, bit for bit, the same library calls made on each
sequence alone: a query scores the same keys with the same arithmetic
either way.
"""
import numpy as np
import pytest
import torch

import oracle
from parity_helpers import check_attention
from sparse_long_context_03_b200 import dsa, inputs

pytestmark = pytest.mark.gpu

DEV = "cuda"


def H(t):
    return inputs.to_numpy_bits(t)


def packed_run(cfg, d, lens, chunk_rows=None):
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    total = int(cu[-1])
    plan = dsa.PrefillPlan(total, cfg.HI, cfg.dI, cfg.Hq, cfg.Hkv, cfg.D, cfg.k, chunk_rows=chunk_rows, device=DEV,
                           fused=True)
    O = torch.full((total, cfg.Hq, cfg.D), float("nan"), dtype=torch.bfloat16, device=DEV)
    lse = torch.full((total, cfg.Hq), float("nan"), dtype=torch.float32, device=DEV)
    idx = torch.full((total, cfg.k), -7, dtype=torch.int32, device=DEV)
    dsa.prefill_forward_packed(plan, torch.from_numpy(cu).to(DEV), d["q8"], d["sq"], d["w"], d["k8"], d["sk"],
                               d["Q"], d["K"], d["V"], O, cfg.sm_scale, lse=lse, idx_out=idx)
    torch.cuda.synchronize()
    return cu, idx, O, lse


def attention_inputs(cfg, total, seed):
    d = inputs.prefill_inputs(cfg, L=total, seed=seed)
    return d["Q"], d["K"], d["V"]


@pytest.mark.parametrize("chunk_rows", [None, 333])
def test_packed_exact_inputs_match_the_oracle_per_sequence(chunk_rows):
    cfg = inputs.config(1, k=64)
    lens = [300, 1, 0, 777, 64, 65, 1000]
    total = sum(lens)
    d = inputs.exact_indexer_inputs(total, cfg.HI, cfg.dI, seed=501, key_pool=50)
    d["Q"], d["K"], d["V"] = attention_inputs(cfg, total, 502)
    g = {k: v.to(DEV) for k, v in d.items()}
    cu, idx, O, lse = packed_run(cfg, g, lens, chunk_rows)
    h = {k: H(v) for k, v in d.items()}
    gidx, Og, lg = idx.cpu().numpy(), O.float().cpu().numpy(), lse.cpu().numpy()
    for s0, s1 in zip(cu, cu[1:]):
        if s1 == s0:
            continue
        sl = {k: v[s0:s1] for k, v in h.items()}
        I = oracle.indexer(sl["q8"], sl["sq"], sl["w"], sl["k8"], sl["sk"])
        ref = oracle.causal_topk(I, 0, cfg.k)
        assert np.array_equal(gidx[s0:s1], ref), f"sequence at {s0}"
        Oref, lref = oracle.sparse_attention(sl["Q"], sl["K"], sl["V"], ref, 0, cfg.sm_scale)
        check_attention(Og[s0:s1], Oref, lg[s0:s1], lref, f"sequence at {s0}")


def test_packed_equals_each_sequence_alone_bitwise():
    # sequences long enough for the sampled threshold (more than 8192 keys),
    # starting at offsets that are not multiples of 32 or 256
    cfg = inputs.config(1)
    lens = [9000, 37, 10001, 3, 2500]
    total = sum(lens)
    d = {k: v.to(DEV) for k, v in inputs.prefill_inputs(cfg, L=total, seed=503).items()}
    cu, idx, O, lse = packed_run(cfg, d, lens, chunk_rows=7000)
    for s0, s1 in zip(cu, cu[1:]):
        n = int(s1 - s0)
        sl = slice(int(s0), int(s1))
        ws = torch.empty(dsa.indexer_topk_workspace_size(0, n, cfg.k, cfg.HI, cfg.dI), dtype=torch.uint8,
                         device=DEV)
        one = torch.empty(n, cfg.k, dtype=torch.int32, device=DEV)
        dsa.indexer_topk(d["q8"][sl], d["sq"][sl], d["w"][sl], d["k8"][sl], d["sk"][sl], 0, n, cfg.k, one, ws)
        O1 = torch.empty(n, cfg.Hq, cfg.D, dtype=torch.bfloat16, device=DEV)
        l1 = torch.empty(n, cfg.Hq, dtype=torch.float32, device=DEV)
        dsa.sparse_gqa_prefill(d["Q"][sl], d["K"][sl], d["V"][sl], one, 0, n, cfg.k, cfg.sm_scale, O1, l1)
        torch.cuda.synchronize()
        assert torch.equal(one, idx[sl]), f"indices of the sequence at {s0}"
        assert torch.equal(O1.view(torch.int16), O[sl].view(torch.int16)), f"output of the sequence at {s0}"
        assert torch.equal(l1, lse[sl]), f"lse of the sequence at {s0}"


def test_packed_rejects_missing_offsets():
    cfg = inputs.config(1, k=64)
    d = {k: v.to(DEV) for k, v in inputs.exact_indexer_inputs(100, cfg.HI, cfg.dI, seed=1).items()}
    lib = dsa.lib()
    ws = torch.empty(dsa.indexer_topk_workspace_size(0, 100, 64, cfg.HI, cfg.dI), dtype=torch.uint8, device=DEV)
    idx = torch.empty(100, 64, dtype=torch.int32, device=DEV)
    rc = lib.dsa_indexer_topk_varlen(d["q8"].data_ptr(), d["sq"].data_ptr(), d["w"].data_ptr(), d["k8"].data_ptr(),
                                     d["sk"].data_ptr(), 100, cfg.HI, cfg.dI, None, 1, 0, 100, 64, idx.data_ptr(),
                                     ws.data_ptr(), ws.numel(), None, None)
    assert rc == 1  # DSA_ERR_INVALID_ARG
