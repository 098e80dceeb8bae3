"""Failure detection on the GPU without a fault: a bounded on-chip wait that
gives up.

The prefill indexer's pipeline waits (TMA producer <-> tensor-core issuer <->
epilogue) are bounded; a test lowers the bound to 1 ns so that waits give up
during a launch.  The kernel must then set the flag that
dsa_check_device_error reports as DSA_ERR_TIMEOUT, unwind every role (drain
its copies in flight, free its tensor memory) and leave the context usable:
after the bound is restored, the next call must be complete and exact.
Nothing here traps, faults or hangs the GPU.
"""
import numpy as np
import pytest
import torch

import oracle
from sparse_long_context_03_b200 import dsa, inputs

pytestmark = pytest.mark.gpu

DEV = "cuda"
DSA_ERR_TIMEOUT = 5


def H(t):
    return inputs.to_numpy_bits(t)


def test_expired_pipeline_wait_reports_timeout_and_the_next_call_is_exact():
    L, HI, dI = 4096, 32, 64
    d = {k: v.to(DEV) for k, v in inputs.exact_indexer_inputs(L, HI, dI, seed=404).items()}
    assert dsa.device_error_status() == 0
    scores = torch.zeros(L, L, dtype=torch.float32, device=DEV)
    dsa.set_wait_limit_ns(1)
    try:
        for _ in range(3):
            dsa.indexer_scores(d["q8"], d["sq"], d["w"], d["k8"], d["sk"], 0, L, scores)
        torch.cuda.synchronize()
        code = dsa.device_error_status()
    finally:
        dsa.set_wait_limit_ns(0)
    assert code == DSA_ERR_TIMEOUT
    assert dsa.device_error_status() == 0  # the flag was cleared
    # the context is usable and the kernel is whole again
    scores.fill_(float("nan"))
    dsa.indexer_scores(d["q8"], d["sq"], d["w"], d["k8"], d["sk"], 0, L, scores)
    torch.cuda.synchronize()
    assert dsa.device_error_status() == 0
    h = {k: H(v) for k, v in d.items()}
    for t in (0, 1, 255, 256, 2047, 3000, L - 1):
        ref = oracle.indexer(h["q8"], h["sq"], h["w"], h["k8"], h["sk"], row_begin=t, n_rows=1)[0]
        got = scores[t, : t + 1].cpu().numpy().astype(np.float64)
        assert np.array_equal(got, ref[: t + 1]), f"row {t}"
