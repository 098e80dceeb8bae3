#!/usr/bin/env python
"""Benchmark of the B200 DSA layer: 128K-token prefill throughput and
decode-step latency, with roofline fractions and the fp64 oracle timed on the
host cores beside it.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config 2] [--impl reference]

One step = one whole prefill of a 131072-token sequence (chunked lightning
indexer -> per-row top-k -> sparse GQA attention) on synthetic inputs
already resident in HBM.  Prints ONE JSON line on rank 0.  Under torchrun
(N > 1) every rank prefills its own independent sequence (weak scaling, no
collective on the data path); the time is the max over ranks.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import torch  # noqa: E402

METRIC = "GQA-DSA prefill tok/s @128K & decode step µs; % of HBM / FP8 tensor roofline"
UNIT = "tok/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
FP8_PER_BF16 = 2.0  # nominal dense ratio, 4.5 / 2.25 PFLOP/s (used only if the FP8 measurement fails)


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def _best_ms(fn, reps, stream):
    """Best of `reps` CUDA-event timings of fn() on `stream` (after one warm-up call)."""
    fn()
    torch.cuda.synchronize()
    best = float("inf")
    for _ in range(reps):
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record(stream)
        fn()
        b.record(stream)
        b.synchronize()
        best = min(best, a.elapsed_time(b))
    return best


def measure_fp8_peak(gpu_index, n=8192, sustain_s=2.0):
    """Dense FP8 e4m3 GEMM throughput on this GPU: torch._scaled_mm n^3
    (2 n^3 FLOP), best of 10 (burst) and back to back for ~sustain_s seconds
    (sustained, under the power cap), with the SM clock sampled meanwhile."""
    try:
        a = torch.randn(n, n, device="cuda").to(torch.float8_e4m3fn)
        b = torch.randn(n, n, device="cuda").to(torch.float8_e4m3fn).t()  # column-major operand
        one = torch.ones((), device="cuda", dtype=torch.float32)
        stream = torch.cuda.current_stream()

        def mm():
            return torch._scaled_mm(a, b, scale_a=one, scale_b=one, out_dtype=torch.bfloat16)

        burst_ms = _best_ms(mm, 10, stream)
        with ClockSampler(gpu_index) as clk:
            iters = max(10, int(sustain_s / (burst_ms / 1e3)))
            s = torch.cuda.Event(enable_timing=True)
            e = torch.cuda.Event(enable_timing=True)
            s.record(stream)
            for _ in range(iters):
                mm()
            e.record(stream)
            torch.cuda.synchronize()
        sus_ms = s.elapsed_time(e) / iters
        flop = 2.0 * n ** 3
        del a, b
        return {"fp8_tflops": flop / (burst_ms / 1e3) / 1e12, "fp8_tflops_sustained": flop / (sus_ms / 1e3) / 1e12,
                "how": f"torch._scaled_mm e4m3 x e4m3 -> bf16, {n}^3, best of 10 (burst) and {iters} back to back "
                       f"(sustained), CUDA events", "clocks_sustained": clk.summary()}
    except (RuntimeError, TypeError) as exc:  # no FP8 GEMM in this torch build
        return {"error": str(exc).splitlines()[0][:200]}


def measure_read_peaks(dsa):
    """Read bandwidth of the memory system with the library's read probe
    (16-byte L2-only loads on every SM): a buffer that fits in L2, read many
    times (best over a few sizes), and one pass over a 4 GiB buffer (HBM)."""
    stream = torch.cuda.current_stream()
    sink = torch.zeros(4, dtype=torch.int32, device="cuda")
    l2 = {}
    for mb in (8, 16, 24, 32, 48, 64):
        buf = torch.ones(mb << 18, dtype=torch.int32, device="cuda")
        reps = max(64, 2048 // mb)
        ms = _best_ms(lambda: dsa.read_probe(buf, reps, sink), 10, stream)
        l2[mb] = reps * buf.numel() * 4 / (ms / 1e3) / 1e9
        del buf
    big = torch.ones(1 << 30, dtype=torch.int32, device="cuda")
    ms = _best_ms(lambda: dsa.read_probe(big, 1, sink), 5, stream)
    hbm_read = big.numel() * 4 / (ms / 1e3) / 1e9
    del big
    best_mb = max(l2, key=l2.get)
    return {"l2_read_gbs": l2[best_mb], "l2_read_gbs_by_mb": l2, "hbm_read_gbs": hbm_read,
            "how": f"dsa_read_probe: {best_mb} MiB buffer read repeatedly (best of 8-64 MiB buffers, best of 10); "
                   f"HBM: one pass over 4 GiB, best of 5; CUDA events"}


def _avg_back_to_back_ms(fn, n=20):
    """Mean time of one fn() call over n back-to-back calls between two CUDA
    events (after three warm-up calls): the GPU never waits for the host, so
    the figure is the kernels' time.  For buffers well beyond L2, a pass does
    not find the previous pass's data in L2: the previous pass's tail is
    evicted before this pass reaches it."""
    stream = torch.cuda.current_stream()
    for _ in range(3):
        fn()
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(n):
        fn()
    b.record(stream)
    b.synchronize()
    return a.elapsed_time(b) / n


def measure_single_pass_read(dsa, n_bytes):
    """Read bandwidth of one pass over a buffer of n_bytes (beyond L2) with
    the library's read probe, averaged over back-to-back passes: what a
    kernel that reads that many bytes once can reach, ramp-up and tail
    included."""
    sink = torch.zeros(4, dtype=torch.int32, device="cuda")
    buf = torch.ones((n_bytes + 15) // 16 * 4, dtype=torch.int32, device="cuda")
    ms = _avg_back_to_back_ms(lambda: dsa.read_probe(buf, 1, sink))
    gbs = buf.numel() * 4 / (ms / 1e3) / 1e9
    del buf
    return gbs


# ----------------------------------------------------------------------------
# distributed plumbing
# ----------------------------------------------------------------------------

def dist_setup(n_gpus):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        torch.cuda.set_device(local)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                             device_id=torch.device("cuda", local))
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    return rank, world, local


def barrier(world):
    if world > 1:
        torch.distributed.barrier()


def max_over_ranks(x: float, world: int, device="cuda") -> float:
    """The slowest rank's time: every rank contributes its own device-timed value."""
    if world == 1:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def rank_seed(cfg, rank: int) -> int:
    """Each rank prefills its own independent sequence (weak scaling)."""
    return cfg.seed + 7919 * rank


def aggregate_tok_per_s(world: int, tokens_per_rank: int, steps: int, ms_max: float) -> float:
    """Whole-job throughput: tokens of all ranks over the slowest rank's time."""
    return world * tokens_per_rank * steps / (ms_max / 1e3)


# ----------------------------------------------------------------------------
# clocks
# ----------------------------------------------------------------------------

class ClockSampler:
    """nvidia-smi sampling of SM clock and throttle reasons during the timed region."""
    FIELDS = ["index", "clocks.sm", "clocks.max.sm", "power.draw", "clocks_event_reasons.active",
              "clocks_event_reasons.hw_slowdown", "clocks_event_reasons.hw_thermal_slowdown",
              "clocks_event_reasons.sw_thermal_slowdown", "clocks_event_reasons.sw_power_cap"]

    def __init__(self, gpu_index):
        self.gpu_index = gpu_index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={','.join(self.FIELDS)}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        return self

    def __exit__(self, *a):
        self.lines = []
        if self.proc is not None:
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                out, _ = self.proc.communicate()
            self.lines = out.splitlines()

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in getattr(self, "lines", []):
            f = [x.strip() for x in ln.split(",")]
            if len(f) < len(self.FIELDS) or f[0] != str(self.gpu_index):
                continue
            try:
                sm.append(float(f[1]))
                mx = float(f[2])
            except ValueError:
                continue
            for name, val in zip(names, f[5:9]):
                if val.lower() == "active":
                    reasons.add(name)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# ----------------------------------------------------------------------------
# workloads
# ----------------------------------------------------------------------------

def causal_pairs(r0, n):
    """Number of (t, s) pairs with s <= t for t in [r0, r0+n)."""
    return n * r0 + n * (n + 1) // 2


class PrefillBench:
    def __init__(self, cfg, seed, device, chunk_rows=None, fused=None):
        from sparse_long_context_03_b200 import dsa, inputs
        self.dsa = dsa
        self.cfg = cfg
        self.d = inputs.prefill_inputs(cfg, device=device, seed=seed)
        self.plan = dsa.PrefillPlan(cfg.L, cfg.HI, cfg.dI, cfg.Hq, cfg.Hkv, cfg.D, cfg.k, chunk_rows=chunk_rows,
                                    device=device, fused=fused)
        self.O = torch.empty(cfg.L, cfg.Hq, cfg.D, dtype=torch.bfloat16, device=device)
        self.stream = torch.cuda.current_stream()
        self.chunks = list(self.plan.chunks())
        self.stats = torch.zeros(len(self.chunks), 2, dtype=torch.int64, device=device) if self.plan.fused else None

    def stage_names(self):
        return ["threshold", "indexer", "select", "attention"] if self.plan.fused else ["indexer", "topk", "attention"]

    def step(self, ev=None):
        """One whole prefill.  With ev (a dict of lists), brackets every
        library call with CUDA events on the launching stream."""
        d, p, c, dsa = self.d, self.plan, self.cfg, self.dsa

        def mark():
            if ev is None:
                return None
            e = torch.cuda.Event(enable_timing=True)
            e.record(self.stream)
            return e

        a = mark()
        for ci, (r0, n) in enumerate(self.chunks):
            if p.fused:
                for stage, name in (("threshold", "threshold"), ("candidates", "indexer"), ("select", "select")):
                    dsa.indexer_topk(d["q8"], d["sq"], d["w"], d["k8"], d["sk"], r0, n, c.k, p.idx[r0:r0 + n], p.ws,
                                     stats=self.stats[ci] if stage == "select" else None, stage=stage)
                    b = mark()
                    if ev is not None:
                        ev[name].append((a, b, (r0, n)))
                    a = b
            else:
                dsa.indexer_scores(d["q8"], d["sq"], d["w"], d["k8"], d["sk"], r0, n, p.scores[:n],
                                   row_stats=p.row_stats)
                b = mark()
                dsa.topk(p.scores[:n], r0, n, c.k, p.idx[r0:r0 + n], max_len=r0 + n, ws=p.ws, row_stats=p.row_stats)
                e = mark()
                if ev is not None:
                    ev["indexer"].append((a, b, (r0, n)))
                    ev["topk"].append((b, e, (r0, n)))
                a = e
        dsa.sparse_gqa_prefill(d["Q"], d["K"], d["V"], p.idx, 0, c.L, c.k, c.sm_scale, self.O)
        b = mark()
        if ev is not None:
            ev["attention"].append((a, b, (0, c.L)))

    # algorithmic work of one call of each stage
    def flops_indexer(self, r0, n):
        """4096 FLOP per causal (t, s) pair of the rows that need scores:
        every row on the unfused path; rows with t + 1 > k on the fused path
        (a row with t + 1 <= k selects all of 0..t without scoring)."""
        c = self.cfg
        if self.plan.fused:
            lo = max(r0, c.k)
            return 2 * c.HI * c.dI * (causal_pairs(lo, r0 + n - lo) if lo < r0 + n else 0)
        return 2 * c.HI * c.dI * causal_pairs(r0, n)

    def flops_threshold(self, r0, n):
        """The sampled scores: every 32nd key of the rows scored from candidates."""
        c = self.cfg
        keep_all = 4 * max(3 * c.k // 4, 1024)  # rows with more keys than this are sampled
        lo = max(r0, keep_all)
        return 2 * c.HI * c.dI * sum(t // 32 + 1 for t in range(lo, r0 + n))

    def bytes_topk(self, r0, n):
        return 4 * causal_pairs(r0, n) + 4 * self.cfg.k * n

    def bytes_select(self, ci, r0, n, cand):
        """Candidates read (8 B each, counted on the device), 16 B of counts
        per row, index rows written."""
        return 8 * cand + 16 * n + 4 * self.cfg.k * n

    def bytes_attention(self, r0, n):
        c = self.cfg
        t = torch.arange(r0, r0 + n, dtype=torch.float64)
        rows = torch.clamp(t + 1, max=c.k).sum().item()
        gather = rows * c.Hkv * 2 * c.D * 2          # each selected K and V row once per KV head
        qo = n * c.Hq * c.D * 2 * 2                   # Q read, O written
        return gather + qo + 4 * c.k * n              # + index rows


TRAFFIC_FILE = os.path.join(os.path.dirname(os.path.abspath(__file__)), "profiles", "dram_traffic.txt")
STAGE_KERNEL = {"attention": ("sparse_prefill_kernel", "attention.cu"),
                "indexer": ("indexer_tc_kernel", "indexer_tc.cu"),
                "topk": ("topk_rows_bitmap_kernel", "topk.cu"),
                "select": ("cand_select_kernel", "topk_fused.cu"),
                "threshold": ("sample_threshold_kernel", "topk_fused.cu")}


def measured_traffic(stage, workload):
    """DRAM bytes (read + write) per launch of a stage's kernel on this
    workload, from the ncu capture recorded in profiles/dram_traffic.txt --
    only if that capture was taken on the kernel's current source (its
    sha256 is recorded beside the figure); None otherwise."""
    import hashlib
    kernel, src = STAGE_KERNEL[stage]
    try:
        from sparse_long_context_03_b200 import build
        digest = hashlib.sha256(open(os.path.join(build.CSRC, src), "rb").read()).hexdigest()
        with open(TRAFFIC_FILE) as f:
            for line in f:
                parts = line.split()
                if len(parts) >= 5 and not line.startswith("#") and parts[0] == kernel and parts[1] == workload \
                        and parts[4] == digest:
                    return int(parts[2]) + int(parts[3])
    except OSError:
        return None
    return None


def run_prefill_timed(pb, steps, warmup, world, gpu_index):
    for _ in range(warmup):
        pb.step()
    torch.cuda.synchronize()
    ev = {name: [] for name in pb.stage_names()}
    barrier(world)
    torch.cuda.synchronize()
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    with ClockSampler(gpu_index) as clk:
        start.record(pb.stream)
        for _ in range(steps):
            pb.step(ev)
        end.record(pb.stream)
        torch.cuda.synchronize()
    barrier(world)
    pb.dsa.check_device_error()  # a kernel that gave up a bounded wait voids the run
    ms = start.elapsed_time(end)
    per = {}
    for name, lst in ev.items():
        per[name] = [(a.elapsed_time(b), rn) for a, b, rn in lst]
    return ms, per, clk.summary()


def run_prefill_e2e(pb, steps, warmup):
    """Same prefill through the public API, from pinned HOST buffers: every
    step copies its inputs host->device, runs, and copies O back.  Copies
    run on their own streams, double-buffered: the inputs of step i+1 go up
    and the output of step i-1 comes down while step i computes, as a serving
    loop would; every byte of every step is inside the timed region."""
    names = ["q8", "sq", "w", "k8", "sk", "Q", "K", "V"]
    host = {k: pb.d[k].cpu().pin_memory() for k in names}
    dev = [{k: torch.empty_like(pb.d[k]) for k in names} for _ in range(2)]
    outs = [torch.empty_like(pb.O) for _ in range(2)]
    out_host = [torch.empty(pb.O.shape, dtype=pb.O.dtype).pin_memory() for _ in range(2)]
    h2d_bytes = sum(v.numel() * v.element_size() for v in host.values())
    d2h_bytes = out_host[0].numel() * out_host[0].element_size()
    c, p, dsa = pb.cfg, pb.plan, pb.dsa
    comp = pb.stream
    up, down = torch.cuda.Stream(), torch.cuda.Stream()
    ev = lambda: torch.cuda.Event()  # noqa: E731
    in_ready, in_free, out_ready, out_free = ([ev(), ev()] for _ in range(4))

    def run(n):
        used = [False, False]
        done = [False, False]

        def upload(i):
            b = i % 2
            with torch.cuda.stream(up):
                if used[b]:
                    up.wait_event(in_free[b])
                for k in names:
                    dev[b][k].copy_(host[k], non_blocking=True)
                in_ready[b].record(up)

        upload(0)
        for i in range(n):
            b = i % 2
            if i + 1 < n:
                upload(i + 1)
            comp.wait_event(in_ready[b])
            if done[b]:
                comp.wait_event(out_free[b])
            d = dev[b]
            dsa.prefill_forward(p, d["q8"], d["sq"], d["w"], d["k8"], d["sk"], d["Q"], d["K"], d["V"], outs[b],
                                c.sm_scale, stream=comp)
            in_free[b].record(comp)
            out_ready[b].record(comp)
            used[b] = True
            with torch.cuda.stream(down):
                down.wait_event(out_ready[b])
                out_host[b].copy_(outs[b], non_blocking=True)
                out_free[b].record(down)
            done[b] = True
        for b in range(2):
            if done[b]:
                comp.wait_event(out_free[b])

    run(warmup)
    torch.cuda.synchronize()
    s = torch.cuda.Event(enable_timing=True)
    e = torch.cuda.Event(enable_timing=True)
    s.record(comp)
    up.wait_event(s)
    down.wait_event(s)
    run(steps)
    e.record(comp)
    torch.cuda.synchronize()
    dsa.check_device_error()
    ms = s.elapsed_time(e)
    del dev, host, outs
    return ms, h2d_bytes, d2h_bytes


def run_kl_timed(dsa, inputs, pk, reps=5, n_rows=4096, G=4):
    """The indexer's distillation losses (dense warm-up over every causal key,
    sparse adaptation over Omega_t) on the last n_rows query rows of the
    32K layer, against HBM: algorithmic bytes are the scores and G target
    weights of every key visited (plus the index rows for the sparse loss)."""
    cfg = inputs.config(1)
    d = inputs.prefill_inputs(cfg, device="cuda")
    L, k = cfg.L, cfg.k
    r0 = L - n_rows
    scores = torch.empty(n_rows, L, dtype=torch.float32, device="cuda")
    dsa.indexer_scores(d["q8"], d["sq"], d["w"], d["k8"], d["sk"], r0, n_rows, scores)
    need = dsa.topk_workspace_size(n_rows, L, k)
    ws = torch.empty(need, dtype=torch.uint8, device="cuda") if need else None
    idx = torch.empty(n_rows, k, dtype=torch.int32, device="cuda")
    dsa.topk(scores, r0, n_rows, k, idx, max_len=L, ws=ws)
    del d
    p = inputs.kl_targets(n_rows, G, L, seed=77, device="cuda")
    loss = torch.empty(n_rows, dtype=torch.float64, device="cuda")
    total = torch.empty(1, dtype=torch.float64, device="cuda")
    stream = torch.cuda.current_stream()
    out = {"workload": f"prefill-32k rows {r0}..{L - 1} ({n_rows} rows), G={G} target groups, k={k}"}
    keys = sum(t + 1 for t in range(r0, L))
    for name, ix, byts in (("dense", None, keys * (4 + 4 * G)), ("sparse", idx, n_rows * k * (4 + 4 + 4 * G))):
        ms = _best_ms(lambda: dsa.indexer_kl(scores, r0, n_rows, p, loss, idx=ix, loss_total=total), reps, stream)
        gbs = byts / (ms / 1e3) / 1e9
        out[name] = {"ms": ms, "bound": "hbm", "achieved": gbs, "peak": pk["hbm_gbs"], "unit": "GB/s",
                     "frac": gbs / pk["hbm_gbs"], "algorithmic_bytes": byts}
    dsa.check_device_error()
    return out


def run_packed_timed(dsa, inputs, steps, warmup, lens=None):
    """Packed (varlen) prefill: 64 sequences of 2K tokens and 4 of 32K in one
    token axis, every stage one launch over all of them
    (dsa_indexer_topk_varlen, dsa_sparse_gqa_prefill_varlen).  Returns
    tokens/s and the stage times, CUDA events on the launch stream."""
    cfg = inputs.config(1)
    lens = lens or [2048] * 64 + [32768] * 4
    cu = torch.tensor([0] + list(torch.tensor(lens).cumsum(0).tolist()), dtype=torch.int32, device="cuda")
    total = int(cu[-1].item())
    d = inputs.prefill_inputs(cfg, device="cuda", L=total, seed=cfg.seed + 17)
    plan = dsa.PrefillPlan(total, cfg.HI, cfg.dI, cfg.Hq, cfg.Hkv, cfg.D, cfg.k, device="cuda", fused=True)
    O = torch.empty(total, cfg.Hq, cfg.D, dtype=torch.bfloat16, device="cuda")
    stream = torch.cuda.current_stream()

    def step(ev=None):
        a = torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for r0, n in plan.chunks():
            dsa.indexer_topk_varlen(d["q8"], d["sq"], d["w"], d["k8"], d["sk"], cu, r0, n, cfg.k,
                                    plan.idx[r0:r0 + n], plan.ws)
        b = torch.cuda.Event(enable_timing=True)
        b.record(stream)
        dsa.sparse_gqa_prefill_varlen(d["Q"], d["K"], d["V"], plan.idx, cu, 0, total, cfg.k, cfg.sm_scale, O)
        c = torch.cuda.Event(enable_timing=True)
        c.record(stream)
        if ev is not None:
            ev.append((a, b, c))

    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    ev = []
    for _ in range(steps):
        step(ev)
    torch.cuda.synchronize()
    dsa.check_device_error()
    sel = sum(a.elapsed_time(b) for a, b, _ in ev) / steps
    att = sum(b.elapsed_time(c) for _, b, c in ev) / steps
    ms = sel + att
    pairs = sum(n * (n + 1) // 2 for n in lens)
    return {"workload": f"packed prefill: {len(lens)} sequences ({lens.count(2048)} x 2048 + "
                        f"{lens.count(32768)} x 32768 tokens, {total} in all), layer as prefill-32k",
            "value": total / (ms / 1e3), "unit": "tok/s", "ms_per_step": ms, "steps": steps,
            "stages_ms": {"indexer_topk_varlen": sel, "attention_varlen": att},
            "indexer_tflops": 2 * cfg.HI * cfg.dI * pairs / (sel / 1e3) / 1e12,
            "launches_per_step": 5 * len(list(plan.chunks())) + 1}


class DecodeBench:
    def __init__(self, cfg, seed, device, batch=None):
        from sparse_long_context_03_b200 import dsa, inputs
        self.dsa = dsa
        self.cfg = cfg
        self.d = inputs.decode_inputs(cfg, device=device, seed=seed, B=batch)
        B = self.d["q"].shape[0]
        self.B = B
        self.ws = torch.empty(dsa.decode_workspace_size(B, self.d["max_seq_len"], cfg.Hq, cfg.Hkv, cfg.D, cfg.k),
                              dtype=torch.uint8, device=device)
        self.out = torch.empty(B, cfg.Hq, cfg.D, dtype=torch.bfloat16, device=device)
        self.stream = torch.cuda.current_stream()
        self.lens = [int(x) for x in self.d["seq_lens"].cpu()]

    def step(self):
        d, c = self.d, self.cfg
        self.dsa.sparse_gqa_decode(d["q"], d["q8"], d["sq"], d["w"], d["k8_cache"], d["sk_cache"], d["k_cache"],
                                   d["v_cache"], d["block_table"], d["seq_lens"], d["max_seq_len"], c.k, c.sm_scale,
                                   self.ws, self.out)

    def algorithmic_bytes(self):
        c = self.cfg
        n = sum(self.lens)
        idx_rows = sum(min(c.k, x) for x in self.lens)
        indexer = n * (c.dI + 4)                        # FP8 key + its scale, every cached token
        scores = n * 4 * 2                               # score row written, read by the top-k
        gather = idx_rows * c.Hkv * 2 * c.D * 2          # selected K and V rows once per KV head
        small = self.B * (c.Hq * c.D * 2 * 2 + c.HI * c.dI + c.HI * 4 + 4 * c.k * 2)
        return indexer + scores + gather + small


def run_decode_timed(db, steps, warmup, gpu_index, min_seconds=0.6):
    """Decode steps back to back: `steps` of them, or more so that the timed
    region lasts about min_seconds (long enough for the clock sampler)."""
    for _ in range(warmup):
        db.step()
    torch.cuda.synchronize()
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    a.record(db.stream)
    db.step()
    b.record(db.stream)
    torch.cuda.synchronize()
    steps = max(steps, int(min_seconds * 1e3 / max(a.elapsed_time(b), 1e-3)))
    s = torch.cuda.Event(enable_timing=True)
    e = torch.cuda.Event(enable_timing=True)
    with ClockSampler(gpu_index) as clk:
        s.record(db.stream)
        for _ in range(steps):
            db.step()
        e.record(db.stream)
        torch.cuda.synchronize()
    db.dsa.check_device_error()
    return s.elapsed_time(e) / steps, clk.summary()


def decode_host_inputs(db):
    """Host copies of the decode inputs for the oracle, or None when the host
    has not got twice their size free."""
    from sparse_long_context_03_b200 import inputs
    need = sum(v.numel() * v.element_size() for v in db.d.values() if isinstance(v, torch.Tensor))
    try:
        import psutil
        if psutil.virtual_memory().available < 2 * need:
            return None
    except ImportError:
        pass
    return {k: (inputs.to_numpy_bits(v) if isinstance(v, torch.Tensor) else v) for k, v in db.d.items()}


# ----------------------------------------------------------------------------
# CPU baseline: the fp64 oracle on a bounded sample of the same workload
# ----------------------------------------------------------------------------

def sample_rows(cfg, n_total, seed):
    """Query rows for the oracle: the boundary rows t in {0, k-2, k-1, k,
    L-1} (plus, on the multimodal workload, the first and last token of a
    text segment and of the frame after it), then rows drawn uniformly at
    random without replacement up to n_total."""
    import numpy as np
    from sparse_long_context_03_b200 import inputs
    L, k = cfg.L, cfg.k
    fixed = {0, k - 2, k - 1, k, L - 1}
    if cfg.multimodal:
        t0 = inputs.FRAME_TOKENS * inputs.FRAMES_PER_GROUP
        fixed |= {t0 - 1, t0, t0 + inputs.TEXT_TOKENS - 1, t0 + inputs.TEXT_TOKENS}
    fixed = sorted(t for t in fixed if 0 <= t < L)
    rng = np.random.default_rng(seed)
    pool = np.setdiff1d(np.arange(L), np.asarray(fixed))
    n_rand = max(0, min(len(pool), n_total - len(fixed)))
    return sorted(fixed + [int(t) for t in rng.choice(pool, size=n_rand, replace=False)])


def oracle_rows_seconds(cfg, h, rows, threads):
    """Wall time of the oracle's whole chain (indexer row, top-k, attention)
    for each query row in `rows`, `threads` rows at a time on the host cores
    (one oracle thread per row; ctypes releases the GIL during the C call)."""
    import oracle
    from concurrent.futures import ThreadPoolExecutor

    def one(t):
        oracle.set_threads(1)
        I = oracle.indexer(h["q8"], h["sq"], h["w"], h["k8"], h["sk"], row_begin=t, n_rows=1)
        idx = oracle.causal_topk(I, t, cfg.k)
        oracle.sparse_attention(h["Q"][t:t + 1], h["K"], h["V"], idx, t, cfg.sm_scale)

    t0 = time.perf_counter()
    with ThreadPoolExecutor(max_workers=threads) as ex:
        list(ex.map(one, rows))
    return time.perf_counter() - t0


def extrapolate_tok_per_s(cfg, rows, seconds):
    """A row's cost grows with its t+1 visible keys: the whole prefill takes
    seconds * sum_{t<L}(t+1) / sum_{t in rows}(t+1).  Returns (tok/s, full s)."""
    units = sum(t + 1 for t in rows)
    full = seconds * (cfg.L * (cfg.L + 1) / 2) / units
    return cfg.L / full, full


def host_prefill(d):
    from sparse_long_context_03_b200 import inputs
    return {k: inputs.to_numpy_bits(d[k]) for k in ("q8", "sq", "w", "k8", "sk", "Q", "K", "V")}


def host_cores():
    return len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else (os.cpu_count() or 1)


def cpu_baseline(cfg, d, n_rows=256, n_rows_1core=8, decode_host=None, dcfg=None):
    """The oracle, as it stands, on the host cores: the prefill chain on
    n_rows sampled rows with every core, and on n_rows_1core of them with one
    core, each extrapolated to the whole sequence; the decode layer (every
    sequence, in full) when its host inputs are given."""
    import oracle
    oracle.build()
    h = host_prefill(d)
    cores = host_cores()
    rows = sample_rows(cfg, n_rows, seed=cfg.seed)
    sec = oracle_rows_seconds(cfg, h, rows, cores)
    value, full = extrapolate_tok_per_s(cfg, rows, sec)
    # one core: rows spread evenly over the sample
    sub = rows[:: max(1, len(rows) // n_rows_1core)][:n_rows_1core]
    sec1 = oracle_rows_seconds(cfg, h, sub, 1)
    v1, full1 = extrapolate_tok_per_s(cfg, sub, sec1)
    out = {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
           "sample": f"{len(rows)} query rows of the {cfg.L}-token prefill (t in {{0, k-2, k-1, k, L-1}} and "
                     f"uniform random rows), whole chain per row (fp64 indexer row, top-k, attention), measured "
                     f"{sec:.1f} s on {cores} cores; extrapolated to the whole sequence by the per-row cost "
                     f"sum(t+1): {full:.0f} s",
           "measured_s": sec, "extrapolated_full_s": full, "rows": len(rows),
           "one_core": {"value": v1, "unit": UNIT, "cores": 1, "rows": len(sub), "measured_s": sec1,
                        "extrapolated_full_s": full1}}
    if decode_host is not None:
        hd = decode_host
        oracle.set_threads(cores)
        t0 = time.perf_counter()
        Id = oracle.decode_indexer(hd["q8"], hd["sq"], hd["w"], hd["k8_cache"], hd["sk_cache"], hd["block_table"],
                                   hd["seq_lens"])
        idx = oracle.topk(Id, hd["seq_lens"], dcfg.k)
        oracle.decode_attention(hd["q"], hd["k_cache"], hd["v_cache"], hd["block_table"], hd["seq_lens"], idx,
                                dcfg.sm_scale)
        dsec = time.perf_counter() - t0
        out["decode"] = {"step_us": dsec * 1e6, "cores": cores, "higher_is_better": False,
                         "sample": f"the whole decode step (B={len(hd['seq_lens'])}, every cached token), "
                                   f"measured, not extrapolated"}
    return out


# ----------------------------------------------------------------------------
# reference arm: the oracle, as it stands, on the host cores
# ----------------------------------------------------------------------------

def run_reference(args, rank, world):
    if rank != 0:
        return 0
    import oracle
    from sparse_long_context_03_b200 import inputs
    oracle.build()
    cfg = inputs.config(args.config)
    d = inputs.prefill_inputs(cfg, device="cpu", seed=cfg.seed)
    h = host_prefill(d)
    cores = host_cores()
    per_step = max(cores, 16)
    for i in range(args.warmup):
        oracle_rows_seconds(cfg, h, sample_rows(cfg, per_step, seed=cfg.seed + 1 + i), cores)
    secs, units = 0.0, 0
    for i in range(args.steps):
        rows = sample_rows(cfg, per_step, seed=cfg.seed + 1000 + i)
        secs += oracle_rows_seconds(cfg, h, rows, cores)
        units += sum(t + 1 for t in rows)
    full = secs * (cfg.L * (cfg.L + 1) / 2) / units * args.steps  # whole-sequence time of all steps
    value = args.steps * cfg.L / full
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1000 * full / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": f"{cfg.name}: DSA prefill L={cfg.L}, Hq={cfg.Hq}, Hkv={cfg.Hkv}, D={cfg.D}, "
                               f"HI={cfg.HI}, dI={cfg.dI}, k={cfg.k}", "seq_len": cfg.L},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                         "sample": f"each step: {per_step} query rows (t in {{0, k-2, k-1, k, L-1}} and uniform "
                                   f"random rows; fp64 indexer row, top-k, attention), measured {secs:.1f} s in "
                                   f"all, extrapolated to whole sequences by the per-row cost sum(t+1)"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ----------------------------------------------------------------------------

def stage_roofline(per, pb, pk, src, fp8, reads):
    """Per-stage achieved work / time against the stage's own roofline:
    the indexer against the measured FP8 dense peak, the top-k against the
    HBM copy peak, the prefill attention against the measured L2 read
    bandwidth (its gathers are served from L2; its DRAM traffic is far below
    its algorithmic bytes)."""
    hbm = pk["hbm_gbs"]
    if "fp8_tflops" in fp8:
        fp8_peak, fp8_note = fp8["fp8_tflops"], f"measured FP8 dense (burst): {fp8['how']}"
    else:
        fp8_peak = pk["bf16_tflops"] * FP8_PER_BF16
        fp8_note = f"FP8 measurement failed ({fp8.get('error')}); bf16 burst ({src}) x {FP8_PER_BF16} nominal ratio"
    out = {}
    for name, lst in per.items():
        if not lst:
            continue
        tot_ms = sum(ms for ms, _ in lst)
        if name == "indexer":
            work = sum(pb.flops_indexer(*rn) for _, rn in lst)
            ach = work / (tot_ms / 1e3) / 1e12
            out[name] = {"bound": "tensor", "achieved": ach, "peak": fp8_peak, "unit": "TFLOP/s",
                         "frac": ach / fp8_peak, "ms_total": tot_ms, "launches": len(lst), "peak_note": fp8_note}
            if "fp8_tflops_sustained" in fp8:
                out[name]["frac_of_sustained"] = ach / fp8["fp8_tflops_sustained"]
        elif name == "threshold":
            work = sum(pb.flops_threshold(*rn) for _, rn in lst)
            ach = work / (tot_ms / 1e3) / 1e12
            out[name] = {"bound": "tensor", "achieved": ach, "peak": fp8_peak, "unit": "TFLOP/s",
                         "frac": ach / fp8_peak, "ms_total": tot_ms, "launches": len(lst), "peak_note": fp8_note,
                         "note": "sampled scores (every 32nd key) plus the per-row threshold select over them"}
        elif name == "select":
            cand = pb.stats[:, 1].tolist() if pb.stats is not None else [0] * len(lst)
            steps = max(1, len(lst) // max(1, len(pb.chunks)))
            work = sum(pb.bytes_select(i % len(pb.chunks), *rn, cand[i % len(pb.chunks)]) for i, (_, rn) in
                       enumerate(lst))
            ach = work / (tot_ms / 1e3) / 1e9
            out[name] = {"bound": "hbm", "achieved": ach, "peak": hbm, "unit": "GB/s", "frac": ach / hbm,
                         "ms_total": tot_ms, "launches": len(lst), "peak_note": f"HBM copy ({src})",
                         "candidates_per_row": sum(cand) / pb.cfg.L, "rows_rescored": int(pb.stats[:, 0].sum()),
                         "note": f"exact top-k of the candidate lists (8 B per candidate read, index rows written); "
                                 f"{steps} steps"}
        elif name == "attention":
            work = sum(pb.bytes_attention(*rn) for _, rn in lst)
            ach = work / (tot_ms / 1e3) / 1e9
            l2 = reads["l2_read_gbs"]
            out[name] = {"bound": "l2", "achieved": ach, "peak": l2, "unit": "GB/s", "frac": ach / l2,
                         "ms_total": tot_ms, "launches": len(lst),
                         "peak_note": f"measured L2 read bandwidth ({reads['how']})",
                         "note": "achieved = algorithmic gather bytes (each selected K/V row once per query and KV "
                                 "group, plus Q, O and the index rows) / time; the gathers are L2 reads, so the "
                                 "bound is L2 bandwidth (DRAM traffic per launch is in profiles/)",
                         "effective_gather_gbs_vs_hbm": ach / hbm}
        else:
            work = sum(pb.bytes_topk(*rn) for _, rn in lst)
            ach = work / (tot_ms / 1e3) / 1e9
            out[name] = {"bound": "hbm", "achieved": ach, "peak": hbm, "unit": "GB/s", "frac": ach / hbm,
                         "ms_total": tot_ms, "launches": len(lst), "peak_note": f"HBM copy ({src})"}
    return out


# ----------------------------------------------------------------------------
# untimed cases for profiler captures (no JSON bench line)
# ----------------------------------------------------------------------------

def omega_union(plan, L, k, width=16, fracs=(0.125, 0.25, 0.5, 0.75, 0.99), samples=32):
    """Distinct key positions selected by `width` adjacent queries (the Top-KV
    dedup's potential), at `samples` starting rows near each fraction of L."""
    res = {}
    for frac in fracs:
        sizes = []
        for j in range(samples):
            t0 = min(int(L * frac) + 4096 * j, L - width) // width * width
            blk = plan.idx[t0:t0 + width].flatten()
            sizes.append(int(torch.unique(blk[blk >= 0]).numel()))
        res[f"t~{int(L * frac)}"] = {"mean_union": sum(sizes) / len(sizes), "min": min(sizes), "max": max(sizes),
                                     "of_width_k": sum(sizes) / len(sizes) / (width * k)}
    return res


def run_profile_case(args):
    """One GPU, no timing: `fused` runs the fused indexer + top-k of the
    workload twice, `attention` selects once and runs the prefill attention
    twice, `decode-indexer` runs the decode indexer of a decode workload
    twice with only its FP8 key cache on the device (the second launch of
    each is the one to capture); `omega-union` prints the union of Omega
    over 16 adjacent queries as JSON."""
    from sparse_long_context_03_b200 import build, dsa, inputs
    build.build()
    cfg = inputs.config(args.config)
    if args.profile_case in ("decode-indexer", "decode-topk"):
        if cfg.B <= 0:
            raise SystemExit(f"--profile-case {args.profile_case} needs a decode workload (--config 3)")
        g = inputs.decode_inputs(cfg, device="cuda", B=args.decode_batch)
        for key in ("k_cache", "v_cache", "q"):
            del g[key]
        torch.cuda.empty_cache()
        B, L = g["q8"].shape[0], g["max_seq_len"]
        scores = torch.empty(B, (L + 3) // 4 * 4, dtype=torch.float32, device="cuda")
        for _ in range(2 if args.profile_case == "decode-indexer" else 1):
            dsa.decode_indexer_scores(g["q8"], g["sq"], g["w"], g["k8_cache"], g["sk_cache"], g["block_table"],
                                      g["seq_lens"], L, scores)
        if args.profile_case == "decode-topk":
            # the top-k of the decode rows with each row's range given (the
            # same path as the decode chain, where the indexer records it)
            valid = torch.arange(scores.shape[1], device="cuda")[None, :] < g["seq_lens"][:, None].long()
            lo = torch.where(valid, scores, torch.full_like(scores, float("inf"))).amin(1)
            hi = torch.where(valid, scores, torch.full_like(scores, float("-inf"))).amax(1)
            stats = torch.stack([lo, hi], 1).repeat(1, 4).contiguous()
            idx = torch.empty(B, cfg.k, dtype=torch.int32, device="cuda")
            for _ in range(2):
                dsa.topk(scores, 0, B, cfg.k, idx, row_len=g["seq_lens"], max_len=L, row_stats=stats)
        torch.cuda.synchronize()
        line = {"workload": cfg.name, "profile_case": args.profile_case, "B": B,
                "device_bytes": torch.cuda.memory_allocated(), "status": "ok"}
        if args.profile_case == "decode-indexer":
            # the indexer reads the key cache and its scales once: what one
            # read pass over that many bytes reaches, and the indexer's time
            n_bytes = g["k8_cache"].numel() + g["sk_cache"].numel() * 4
            line["single_pass_read_gbs"] = measure_single_pass_read(dsa, n_bytes)
            line["cache_bytes"] = n_bytes
            ms = _avg_back_to_back_ms(lambda: dsa.decode_indexer_scores(g["q8"], g["sq"], g["w"], g["k8_cache"],
                                                                        g["sk_cache"], g["block_table"],
                                                                        g["seq_lens"], L, scores))
            line["indexer_us"] = ms * 1e3
            line["indexer_gbs"] = n_bytes / (ms / 1e3) / 1e9
        print(json.dumps(line))
        return 0
    d = inputs.prefill_inputs(cfg, device="cuda")
    plan = dsa.PrefillPlan(cfg.L, cfg.HI, cfg.dI, cfg.Hq, cfg.Hkv, cfg.D, cfg.k, chunk_rows=args.chunk_rows,
                           device="cuda", fused=False if args.unfused else True)
    case = args.profile_case
    for _ in range(2 if case == "fused" else 1):
        dsa.select_rows(plan, d["q8"], d["sq"], d["w"], d["k8"], d["sk"])
    if case == "attention":
        O = torch.empty(cfg.L, cfg.Hq, cfg.D, dtype=torch.bfloat16, device="cuda")
        for _ in range(2):
            dsa.sparse_gqa_prefill(d["Q"], d["K"], d["V"], plan.idx, 0, cfg.L, cfg.k, cfg.sm_scale, O)
    torch.cuda.synchronize()
    if case == "omega-union":
        print(json.dumps({"workload": cfg.name, "omega_union_16": omega_union(plan, cfg.L, cfg.k)}))
    else:
        print(json.dumps({"workload": cfg.name, "profile_case": case, "status": "ok"}))
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--config", type=int, default=2, help="prefill workload id (see inputs.CONFIGS)")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--chunk-rows", type=int, default=None,
                    help="query rows per indexer/top-k chunk (default: a 4 GiB score block)")
    ap.add_argument("--no-kl", action="store_true", help="skip the indexer distillation-loss leg")
    ap.add_argument("--no-packed", action="store_true", help="skip the packed (varlen) prefill leg")
    ap.add_argument("--unfused", action="store_true",
                    help="materialise the score matrix per chunk and run dsa_topk (instead of dsa_indexer_topk)")
    ap.add_argument("--decode-batch", type=int, default=None,
                    help="sequences in the decode workload (default: the decode-b32 layer's 32)")
    ap.add_argument("--profile-case", default=None, choices=["fused", "attention", "omega-union", "decode-indexer",
                                                               "decode-topk"],
                    help="run one untimed case on one GPU for a profiler capture (no bench line)")
    args = ap.parse_args()

    if args.profile_case is not None:
        return run_profile_case(args)
    if args.impl == "reference":
        rank = int(os.environ.get("RANK", "0"))
        world = int(os.environ.get("WORLD_SIZE", "1"))
        return run_reference(args, rank, world)

    rank, world, local = dist_setup(args.gpus)
    from sparse_long_context_03_b200 import build, inputs
    if rank == 0:
        build.build()
    barrier(world)

    pk, src = peaks()
    from sparse_long_context_03_b200 import dsa as _dsa
    fp8, reads = {}, {}
    if rank == 0:
        fp8 = measure_fp8_peak(local)
        reads = measure_read_peaks(_dsa)
        torch.cuda.empty_cache()
    cfg = inputs.config(args.config)
    pb = PrefillBench(cfg, seed=rank_seed(cfg, rank), device="cuda", chunk_rows=args.chunk_rows,
                      fused=False if args.unfused else None)
    chunk_rows = pb.plan.chunk_rows
    pb_fused = pb.plan.fused
    ms, per, clocks = run_prefill_timed(pb, args.steps, args.warmup, world, local)
    ms_max = max_over_ranks(ms, world)
    value = aggregate_tok_per_s(world, cfg.L, args.steps, ms_max)
    stages, dom_line = {}, None
    if rank == 0:
        stages = stage_roofline(per, pb, pk, src, fp8, reads)
        dominant = max(stages, key=lambda k: stages[k]["ms_total"])
        dom = dict(stages[dominant])
        dom_line = {"kernel": dominant, "bound": dom["bound"], "achieved": dom["achieved"], "peak": dom["peak"],
                    "unit": dom["unit"], "frac": dom["frac"], "traffic": measured_traffic(dominant, cfg.name),
                    "peak_source": dom["peak_note"]}
        if "note" in dom:
            dom_line["note"] = dom["note"]

    e2e = None
    if not args.no_e2e:
        n_e2e = max(1, args.steps)
        with ClockSampler(local) as eclk:
            ems, h2d, d2h = run_prefill_e2e(pb, n_e2e, 1)
        ems = max_over_ranks(ems, world)
        e2e = {"value": aggregate_tok_per_s(world, cfg.L, n_e2e, ems), "unit": UNIT, "h2d_bytes_per_step": h2d,
               "d2h_bytes_per_step": d2h, "ms_per_step": ems / n_e2e,
               "copies": "pinned host buffers; step i+1's inputs up and step i-1's output down during step i",
               "clocks": eclk.summary()}

    decode, decode_host = None, None
    if not args.no_decode:
        del pb
        torch.cuda.empty_cache()
        dcfg = inputs.config(3)
        db = DecodeBench(dcfg, seed=rank_seed(dcfg, rank), device="cuda", batch=args.decode_batch)
        dms, dclk = run_decode_timed(db, max(args.steps, 20), max(args.warmup, 3), local)
        us = 1e3 * max_over_ranks(dms, world)
        byts = db.algorithmic_bytes()
        decode = {"workload": f"{dcfg.name}: B={db.B}, cached lengths U[{dcfg.len_lo},{dcfg.len_hi}] "
                              f"(mean {statistics.mean(db.lens):.0f}), page 64, k={dcfg.k}",
                  "step_us": us, "higher_is_better": False,
                  "roofline": {"bound": "hbm", "achieved": byts / (us / 1e6) / 1e9, "peak": pk["hbm_gbs"],
                               "unit": "GB/s", "frac": byts / (us / 1e6) / 1e9 / pk["hbm_gbs"],
                               "algorithmic_bytes": byts},
                  "gpu_launches_per_step": 4, "clocks": dclk}
        if rank == 0:
            # a step this short cannot reach the multi-GB copy figure: beside
            # it, one read pass over the step's own bytes, measured here
            sp = measure_single_pass_read(_dsa, byts)
            decode["roofline"].update({
                "single_pass_read_gbs": sp, "frac_of_single_pass": byts / (us / 1e6) / 1e9 / sp,
                "single_pass_note": "dsa_read_probe, one pass over a buffer of the step's algorithmic bytes, "
                                    "mean of 20 back-to-back passes"})
        if rank == 0 and world == 1 and not args.no_cpu_baseline:
            decode_host = decode_host_inputs(db)
        del db
        torch.cuda.empty_cache()
        pb = None

    packed = None
    if rank == 0 and not args.no_packed:
        from sparse_long_context_03_b200 import dsa as _dsa_pk
        packed = run_packed_timed(_dsa_pk, inputs, max(args.steps, 3), max(args.warmup, 1))
        torch.cuda.empty_cache()

    kl = None
    if rank == 0 and not args.no_kl:
        from sparse_long_context_03_b200 import dsa as _dsa_kl
        kl = run_kl_timed(_dsa_kl, inputs, pk)
        torch.cuda.empty_cache()

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        d_cpu = inputs.prefill_inputs(cfg, device="cuda", seed=cfg.seed)
        cpu = cpu_baseline(cfg, d_cpu, decode_host=decode_host, dcfg=inputs.config(3))
        del d_cpu

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_max / args.steps, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "fp8-e4m3 indexer / bf16 attention (fp32 accumulate)",
            "data": "synthetic (seeded; shapes and distributions of the 128K prefill workload)",
            "config": {"workload": f"{cfg.name}: DSA prefill L={cfg.L}, batch 1 per GPU, Hq={cfg.Hq}, Hkv={cfg.Hkv}, "
                                   f"D={cfg.D}, HI={cfg.HI}, dI={cfg.dI}, k={cfg.k}, "
                                   + (f"fused indexer + top-k (no score matrix), query chunks of {chunk_rows} rows"
                                      if pb_fused else f"score matrix in query chunks of {chunk_rows} rows"),
                       "global_batch": world, "seq_len": cfg.L, "parallelism": f"independent sequences x{world}",
                       "l2": "inputs larger than L2 between launches (1 GiB Q and O, 1 GiB of index rows, "
                             "candidate lists or 4 GiB score chunks)"},
            "roofline": dom_line, "stages": stages, "clocks": clocks, "gpu_launches": None,
            "peaks_measured_here": {"fp8": fp8, "reads": reads},
            "e2e": e2e, "decode": decode, "packed": packed, "indexer_kl": kl, "cpu_baseline": cpu,
        }
        # kernels per library call: the fused threshold stage runs the sampled indexer and the threshold
        # select, the select stage the candidate select, the repair kernel and the stats copy
        per_call = {"threshold": 2, "indexer": 1, "select": 3, "topk": 1, "attention": 1}
        line["gpu_launches"] = sum(per_call[k] * len(v) for k, v in per.items())
        print(json.dumps(line), flush=True)
    if world > 1:
        torch.distributed.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
