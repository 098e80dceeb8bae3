"""Multi-rank host logic on CPU (gloo, world size 2).

The benchmark shards the workload as independent sequences (one per rank, no
collective on the data path); the only collectives are the barrier and the
max over ranks of each rank's device-timed duration.  These tests run that
logic with the gloo backend on CPU: distinct per-rank inputs, the max over
ranks, the whole-job throughput formula, and that a rank's oracle result
depends only on its own inputs.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from conftest import ROOT


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out_dir):
    import sys
    sys.path.insert(0, ROOT)
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        import oracle
        from sparse_long_context_03_b200 import inputs
        cfg = inputs.config(0)
        seed = bench.rank_seed(cfg, rank)
        d = inputs.prefill_inputs(cfg, L=96, seed=seed)
        h = {k: inputs.to_numpy_bits(v) for k, v in d.items()}
        I = oracle.indexer(h["q8"], h["sq"], h["w"], h["k8"], h["sk"], row_begin=90, n_rows=6)
        my_ms = 10.0 + 7.5 * rank
        ms_max = bench.max_over_ranks(my_ms, world, device="cpu")
        value = bench.aggregate_tok_per_s(world, cfg.L, 3, ms_max)
        bench.barrier(world)
        np.savez(os.path.join(out_dir, f"rank{rank}.npz"), I=I, seed=seed, ms_max=ms_max, value=value,
                 q8=h["q8"][:4])
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(300)
def test_two_ranks_weak_scaling_logic(tmp_path):
    world = 2
    mp.spawn(_worker, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True)
    r = [np.load(tmp_path / f"rank{i}.npz") for i in range(world)]
    # each rank drew its own independent sequence
    assert int(r[0]["seed"]) != int(r[1]["seed"])
    assert not np.array_equal(r[0]["q8"], r[1]["q8"])
    # the time is the slowest rank's, identical on every rank
    assert float(r[0]["ms_max"]) == float(r[1]["ms_max"]) == 17.5
    # whole-job throughput: tokens of all ranks over the slowest time
    assert float(r[0]["value"]) == pytest.approx(2 * 512 * 3 / 0.0175)
    # a rank's result depends only on its own inputs: recompute rank 1 alone
    import oracle
    from sparse_long_context_03_b200 import inputs
    import bench
    cfg = inputs.config(0)
    d = inputs.prefill_inputs(cfg, L=96, seed=bench.rank_seed(cfg, 1))
    h = {k: inputs.to_numpy_bits(v) for k, v in d.items()}
    I1 = oracle.indexer(h["q8"], h["sq"], h["w"], h["k8"], h["sk"], row_begin=90, n_rows=6)
    assert np.array_equal(I1, r[1]["I"])
