#!/usr/bin/env python
"""Benchmark of one MoBA causal-prefill attention layer on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config 1m] [--impl ours|reference]

One step = one full layer: block mean-pool, gate (scores, causal top-k, index
build) and block-sparse attention with the merge, through the C ABI, on inputs
already resident in HBM.  The metric is effective TFLOP/s on the algorithmic
attention FLOPs (4 * head_dim per attended (query, key) pair), with ms per
layer beside it.  With N > 1 (torchrun) every rank runs its own replica: the
path has no exchange step, so there is no collective on the data path.

Prints one JSON line on rank 0.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import torch  # noqa: E402

import moba_synth as S  # noqa: E402

METRIC = "MoBA prefill attn ms/layer & effective TFLOP/s (frac of bf16 TC peak) at 1M"
FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def algorithmic_pairs(cfg) -> int:
    """Attended (query, key) pairs: sum over (b, h, t) of min(topk-1, c)*B + (t - cB + 1)."""
    total = 0
    for c in range((cfg.seqlen + cfg.block - 1) // cfg.block):
        L = min(cfg.seqlen, (c + 1) * cfg.block) - c * cfg.block
        total += min(cfg.topk - 1, c) * cfg.block * L + L * (L + 1) // 2
    return total * cfg.batch * cfg.hq


def attn_flops(cfg) -> float:
    return 4.0 * cfg.head_dim * algorithmic_pairs(cfg)


def routed_flops(cfg, routed_pairs: int) -> float:
    """Algorithmic FLOPs of a layer whose gate routed `routed_pairs` (row,
    earlier block) pairs (offsets[last]): B keys per pair plus the causal part
    of every row's own block.  Earlier blocks are always full ones."""
    cur = 0
    for c in range(cfg.nblocks):
        L = min(cfg.seqlen, (c + 1) * cfg.block) - c * cfg.block
        cur += L * (L + 1) // 2
    return 4.0 * cfg.head_dim * (routed_pairs * cfg.block + cur * cfg.batch * cfg.hq)


ATTN_SOURCES = ("attn_tc.cu", "attn_pair_tc.cu")


def attention_source_sha() -> str:
    """sha256 of the attention kernels' sources (csrc/attn_tc.cu, then
    csrc/attn_pair_tc.cu), which the traffic record is tied to."""
    import hashlib
    h = hashlib.sha256()
    for name in ATTN_SOURCES:
        with open(os.path.join(ROOT, "long_context_prefill_moba_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def recorded_traffic(rows_per_layer: int):
    """DRAM bytes of one attention step (moba_attn_fwd) from the committed ncu
    capture (profiles/attn_traffic.json), scaled by the rows the gate routes
    (the partial results and the gathered q rows dominate and grow with them).
    None when the attention kernels changed since the capture."""
    p = os.path.join(ROOT, "profiles", "attn_traffic.json")
    if not os.path.exists(p):
        return None, "no capture"
    with open(p) as f:
        d = json.load(f)
    if attention_source_sha() != d.get("kernel_source_sha256"):
        return None, "kernel changed since the capture"
    return d["dram_bytes_per_row"] * rows_per_layer, (
        f"ncu capture of the {d['config']} layer ({d['dram_bytes_per_layer'] / 1e9:.2f} GB), "
        f"scaled by routed rows")


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK), "fallback"


class ClockSampler:
    """nvidia-smi clock/throttle sampling during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            with open(self.path, "w") as sink:   # the child keeps its own descriptor
                self.proc = subprocess.Popen(
                    ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.FIELDS}",
                     "--format=csv,noheader,nounits", "-lms", "200"],
                    stdout=sink, stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        with open(self.path) as f:
            lines = f.readlines()
        os.unlink(self.path)
        return self.summarize(lines)

    @staticmethod
    def summarize(lines):
        """Median SM clock of the samples under load (above half the maximum
        clock), the maximum clock, and every throttle reason seen active."""
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in lines:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx = float(parts[2])
            except ValueError:
                continue
            for nm, val in zip(names, parts[5:9]):
                if val.lower().startswith("active"):
                    reasons.add(nm)
        loaded = [x for x in sm if mx is None or x > 0.5 * mx] or sm
        return {"sm_mhz": statistics.median(loaded) if loaded else None, "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples": len(sm)}


def dist_setup():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=600),
                                device_id=torch.device("cuda", local))
    return world, rank, local


def max_over_ranks(x: float, world: int, device: str = "cuda") -> float:
    """Max of a per-rank timing over all ranks (the job's time is its slowest rank)."""
    if world == 1:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(per_rank_units: float, per_rank_ms: float, world: int, device: str = "cuda") -> float:
    """Whole-job throughput: units of all ranks (every replica runs the same
    work) divided by the slowest rank's time."""
    ms = max_over_ranks(per_rank_ms, world, device)
    return world * per_rank_units / (ms * 1e-3)


def barrier(world: int):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


# ---------------------------------------------------------------------------
# CPU oracle (the reference arm and the cpu_baseline leg)
# ---------------------------------------------------------------------------
class OracleSample:
    """The fp64 oracle on sampled query rows of the workload (one kv head)."""

    def __init__(self, cfg, seed=0):
        import numpy as np
        import oracle as O
        self.O, self.np, self.cfg = O, np, cfg
        self.K = S.gen_head_rows(cfg, "k", 0, 0)
        self.V = S.gen_head_rows(cfg, "v", 0, 0)
        t0 = time.perf_counter()
        self.kbar = O.mean_pool(self.K, cfg.block)
        self.t_pool = time.perf_counter() - t0
        self.rng = np.random.default_rng(seed)
        self.Kd = None

    def rows(self, n):
        """Run n random rows; returns (seconds, attended pairs)."""
        cfg, O, np = self.cfg, self.O, self.np
        ts = self.rng.integers(0, cfg.seqlen, size=n)
        hs = self.rng.integers(0, cfg.group, size=n)
        qrows = [S.gen_rows(cfg, "q", 0, int(t), int(t) + 1, int(h))[0] for t, h in zip(ts, hs)]
        pairs = 0
        t0 = time.perf_counter()
        for t, q in zip(ts, qrows):
            out, lse, sel, gap = O.moba_row(q, self.K, self.V, self.kbar, int(t), cfg.block, cfg.topk,
                                            cfg.softmax_scale)
            pairs += len(O.key_positions(sel, int(t), cfg.block, cfg.seqlen))
        return time.perf_counter() - t0, pairs


def cpu_baseline_pooled(cfg, extra, budget_s=15.0):
    """The pooled-gate variant's oracle (oracle/moba_pooled_gate.py) on sampled
    rows of one kv head: seconds per row, the pools' time, attended pairs."""
    from oracle import moba_pooled_gate as P
    smp = OracleSample(cfg)
    O, np = smp.O, smp.np
    t0 = time.perf_counter()
    kmax, kmin = P.max_pool(smp.K, cfg.block), P.min_pool(smp.K, cfg.block)
    t_pools = smp.t_pool + time.perf_counter() - t0
    secs, pairs, nrows = 0.0, 0, 0
    while secs < budget_s and nrows < 20000:
        ts = smp.rng.integers(0, cfg.seqlen, size=16)
        hs = smp.rng.integers(0, cfg.group, size=16)
        qrows = [S.gen_rows(cfg, "q", 0, int(t), int(t) + 1, int(h))[0] for t, h in zip(ts, hs)]
        t1 = time.perf_counter()
        for t, q in zip(ts, qrows):
            sel = P.select_blocks_pooled(q, smp.kbar, kmax, kmin, int(t), cfg.block, cfg.topk, extra)
            pos = O.key_positions(sel, int(t), cfg.block, cfg.seqlen)
            O.attend_row(q, smp.K[pos], smp.V[pos], cfg.softmax_scale)
            pairs += len(pos)
        secs += time.perf_counter() - t1
        nrows += 16
    full_s = secs / nrows * cfg.batch * cfg.seqlen * cfg.hq + t_pools * cfg.batch * cfg.hkv
    return {"cores": blas_threads(), "kind": "oracle", "extrapolated_full_layer_s": full_s,
            "sample_tflops": 4.0 * cfg.head_dim * pairs / secs / 1e12,
            "sample": (f"{nrows} random query rows of the {cfg.name} layer (fp64 pooled-gate oracle, "
                       f"{secs:.1f} s) plus the three pools of one kv head ({t_pools:.1f} s), "
                       f"extrapolated to the full layer")}


def blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [p.get("num_threads", 0) for p in threadpool_info()]
        return max(n) if n else 1
    except Exception:
        return 1


def cpu_baseline(cfg, budget_s=15.0):
    smp = OracleSample(cfg)
    secs, pairs, nrows = 0.0, 0, 0
    while secs < budget_s and nrows < 20000:
        s, p = smp.rows(16)
        secs += s
        pairs += p
        nrows += 16
    per_row = secs / nrows
    total_rows = cfg.batch * cfg.seqlen * cfg.hq
    full_s = per_row * total_rows + smp.t_pool * cfg.batch * cfg.hkv
    return {
        "value": attn_flops(cfg) / full_s / 1e12, "unit": "TFLOP/s",
        "cores": blas_threads(), "kind": "oracle",
        "sample": (f"{nrows} random query rows of the {cfg.name} layer (fp64 gather oracle, "
                   f"{secs:.1f} s) plus the mean-pool of one kv head ({smp.t_pool:.1f} s), "
                   f"extrapolated to the full layer"),
        "extrapolated_full_layer_s": full_s, "sample_tflops": 4.0 * cfg.head_dim * pairs / secs / 1e12,
    }


def run_reference(args, cfg):
    smp = OracleSample(cfg)
    n = args.ref_rows
    for _ in range(args.warmup):
        smp.rows(n)
    secs, pairs = 0.0, 0
    for _ in range(args.steps):
        s, p = smp.rows(n)
        secs += s
        pairs += p
    value = 4.0 * cfg.head_dim * pairs / secs / 1e12
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * secs / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": config_of(cfg, args),
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": blas_threads(), "kind": "oracle",
                         "sample": f"{n} random query rows of the {cfg.name} layer per step"},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def config_of(cfg, args):
    return {"workload": cfg.name, "batch": cfg.batch, "seqlen": cfg.seqlen, "hq": cfg.hq,
            "hkv": cfg.hkv, "head_dim": cfg.head_dim, "block": cfg.block, "topk": cfg.topk,
            "sparsity": 1.0 - algorithmic_pairs(cfg) / (cfg.batch * cfg.hq * cfg.seqlen *
                                                       (cfg.seqlen + 1) / 2),
            "parallelism": f"replicas{args.gpus}" if args.gpus > 1 else "single",
            "l2": "inputs larger than L2 (q alone 8.6 GB at 1M); no flush"}


# ---------------------------------------------------------------------------
# Other modes: the backward, the pooled-gate variant, and the speed-up curve
# (MoBA layer vs dense causal attention at growing lengths: the comparison of
# the paper's Figure 2a, on this GPU)
# ---------------------------------------------------------------------------
def backward_bench(cfg, steps, warmup):
    """One JSON line: the attention backward (moba_attn_bwd: dq, dk, dv given a
    seeded dout, the gate's selection of the forward held fixed) on `cfg`,
    inputs resident in HBM, CUDA events on the stream.  Algorithmic FLOPs are
    2.5x the forward's (5 matrix products per attended pair: the score
    recompute, dP, dV, dK, dQ); the tensor-core path also recomputes S and dP
    once more for dQ, which is not counted."""
    import long_context_prefill_moba_b200 as M
    M.load_library()
    dev = torch.device("cuda", 0)
    q, k, v = S.gen_q(cfg, dev), S.gen_k(cfg, dev), S.gen_v(cfg, dev)
    dout = S.gen_dout(cfg, dev)
    layer = M.MobaLayer.from_config(cfg, dev)
    out = torch.empty_like(q)
    lse = torch.empty(cfg.batch, cfg.hq, cfg.seqlen, dtype=torch.float32, device=dev)
    layer.forward(q, k, v, out, lse)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    for _ in range(warmup):
        layer.backward(q, k, v, out, lse, dout, dq, dk, dv)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(steps):
        layer.backward(q, k, v, out, lse, dout, dq, dk, dv)
    e1.record()
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / steps
    status = layer.bwd_ws[:4].view(torch.int32).item()
    flops = 2.5 * attn_flops(cfg)
    peaks, _ = load_peaks()
    peak = peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"])
    print(json.dumps({"mode": "backward", "workload": cfg.name, "seqlen": cfg.seqlen, "ms_per_layer": ms,
                      "tflops": flops / ms / 1e9, "frac_of_sustained_peak": flops / ms / 1e9 / peak,
                      "steps": steps, "warmup": warmup, "gpu_launches_per_step": layer.launches,
                      "device_status": status}), flush=True)


def pooled_gate_bench(cfg, extra, steps, warmup, cpu_budget=None):
    """One JSON line: the layer with the gate variant that also routes the top
    `extra` blocks by max- and min-pooled keys (mean-pool, max/min-pool, the
    three-ranking gate, attention at width topk + 2 extra) beside the plain
    layer on the same inputs, inputs resident in HBM, CUDA events on the
    stream.  Algorithmic FLOPs count the pairs the variant's gate routed:
    4 d (B x routed (row, earlier block) pairs + the causal current blocks)."""
    import long_context_prefill_moba_b200 as M
    M.load_library()
    dev = torch.device("cuda", 0)
    q, k, v = S.gen_q(cfg, dev), S.gen_k(cfg, dev), S.gen_v(cfg, dev)
    out = torch.empty_like(q)
    pooled = M.MobaPooledLayer.from_config(cfg, extra, dev)
    plain = M.MobaLayer.from_config(cfg, dev)

    def timed(layer):
        for _ in range(warmup):
            layer.forward(q, k, v, out)
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(steps):
            layer.forward(q, k, v, out)
        e1.record()
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / steps

    ms_plain = timed(plain)
    ms_pooled = timed(pooled)
    # the variant's stages, once more with events between the calls
    sh, x = pooled.shape, pooled.extra
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(5)]
    ev[0].record()
    M.moba_block_meanpool(sh, k, pooled.meank)
    ev[1].record()
    M.moba_block_maxminpool(sh, k, pooled.maxk, pooled.mink)
    ev[2].record()
    M.moba_gate_pooled(sh, x, q, pooled.meank, pooled.maxk, pooled.mink, pooled.sel, pooled.offsets,
                       pooled.rows, pooled.gate_ws)
    ev[3].record()
    M.moba_attn_fwd_pooled(sh, x, q, k, v, pooled.sel, pooled.offsets, pooled.rows, out, None,
                           pooled.attn_ws)
    ev[4].record()
    torch.cuda.synchronize()
    stages = {n: ev[i].elapsed_time(ev[i + 1]) for i, n in enumerate(("meanpool", "maxminpool", "gate",
                                                                      "attention"))}
    routed = int(pooled.offsets[-1].item())
    flops = routed_flops(cfg, routed)
    peaks, _ = load_peaks()
    peak = peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"])
    cpu = None
    if cpu_budget:
        cpu = cpu_baseline_pooled(cfg, extra, cpu_budget)
        cpu.update(value=flops / cpu["extrapolated_full_layer_s"] / 1e12, unit="TFLOP/s")
    print(json.dumps({"mode": "pooled_gate", "workload": cfg.name, "seqlen": cfg.seqlen, "topk": cfg.topk,
                      "extra": extra, "width": cfg.topk + 2 * extra, "ms_per_layer": ms_pooled,
                      "ms_per_layer_plain_gate": ms_plain, "stage_ms": stages,
                      "routed_pairs": routed, "routed_pairs_plain_gate": M.moba_rows_elems(plain.shape),
                      "tflops": flops / ms_pooled / 1e9, "frac_of_sustained_peak": flops / ms_pooled / 1e9 / peak,
                      "steps": steps, "warmup": warmup, "gpu_launches_per_step": pooled.launches,
                      "device_status": list(pooled.device_status()), "cpu_baseline": cpu}), flush=True)


def speedup_curve(seqlens, reps=2):
    """One JSON line per sequence length: the MoBA layer (mean-pool + gate +
    attention through the C ABI) against dense causal attention on the same
    q, k, v computed by torch's scaled_dot_product_attention (a library
    FlashAttention-class kernel; cuDNN when available) and by this library's
    own kernels (MoBA with a single block B = N and topk = 1, which is dense
    causal attention)."""
    import long_context_prefill_moba_b200 as M
    from torch.nn.attention import SDPBackend, sdpa_kernel
    M.load_library()
    dev = torch.device("cuda", 0)
    base = S.get_config("1m")
    for N in seqlens:
        cfg = base.replace(name=f"llama8b_{N // 1024}k", seqlen=N)
        q, k, v = S.gen_q(cfg, dev), S.gen_k(cfg, dev), S.gen_v(cfg, dev)
        out = torch.empty_like(q)

        def timed(fn):
            fn()
            torch.cuda.synchronize()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            for _ in range(reps):
                fn()
            e1.record()
            torch.cuda.synchronize()
            return e0.elapsed_time(e1) / reps

        layer = M.MobaLayer.from_config(cfg, dev)
        moba_ms = timed(lambda: layer.forward(q, k, v, out))
        del layer
        # dense causal attention through this library's own kernels: MoBA with
        # one block (B = N) and topk = 1 attends every earlier key; the
        # current-block kernel runs it with its causal window starting at key 0,
        # with no index and no partial results
        dcfg = cfg.replace(block=N, topk=1)
        dl = M.MobaLayer.from_config(dcfg, dev)
        dense_self = timed(lambda: dl.forward(q, k, v, out))
        del dl
        qt, kt, vt = (x.transpose(1, 2).contiguous() for x in (q, k, v))
        backend = None
        dense_ms = None
        for be in (SDPBackend.CUDNN_ATTENTION, SDPBackend.FLASH_ATTENTION, SDPBackend.EFFICIENT_ATTENTION):
            try:
                with sdpa_kernel([be]):
                    dense_ms = timed(lambda: torch.nn.functional.scaled_dot_product_attention(
                        qt, kt, vt, is_causal=True, scale=cfg.softmax_scale, enable_gqa=True))
                backend = str(be).split(".")[-1]
                break
            except Exception:   # backend not available for this shape or build
                continue
        dense_flops = 4.0 * cfg.head_dim * cfg.batch * cfg.hq * N * (N + 1) / 2
        print(json.dumps({
            "mode": "speedup_curve", "seqlen": N, "hq": cfg.hq, "hkv": cfg.hkv, "block": cfg.block,
            "topk": cfg.topk, "moba_ms": moba_ms, "moba_tflops": attn_flops(cfg) / moba_ms / 1e9,
            "dense_ms": dense_ms, "dense_backend": backend,
            "dense_tflops": None if dense_ms is None else dense_flops / dense_ms / 1e9,
            "speedup_vs_dense": None if dense_ms is None else dense_ms / moba_ms,
            "dense_via_moba_kernels_ms": dense_self,
            "dense_via_moba_kernels_tflops": dense_flops / dense_self / 1e9,
            "speedup_vs_dense_via_moba_kernels": dense_self / moba_ms}), flush=True)
        del q, k, v, out, qt, kt, vt
        torch.cuda.empty_cache()


# ---------------------------------------------------------------------------
# GPU arm
# ---------------------------------------------------------------------------
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--config", default="1m", choices=sorted(S.CONFIGS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--e2e-steps", type=int, default=2)
    ap.add_argument("--backward", action="store_true",
                    help="time the attention backward (moba_attn_bwd) instead; prints its own JSON line")
    ap.add_argument("--pooled-gate", type=int, default=None, metavar="EXTRA",
                    help="time the gate variant that adds the top EXTRA blocks by max- and "
                         "min-pooled keys, beside the plain layer")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-budget", type=float, default=15.0)
    ap.add_argument("--ref-rows", type=int, default=32)
    ap.add_argument("--speedup-curve", action="store_true",
                    help="MoBA vs dense causal attention at growing lengths (one line per length)")
    ap.add_argument("--curve-seqlens", default="32768,131072,262144,524288,1048576")
    args = ap.parse_args()
    if args.speedup_curve:
        speedup_curve([int(x) for x in args.curve_seqlens.split(",")])
        return
    if args.pooled_gate is not None:
        pooled_gate_bench(S.get_config(args.config), args.pooled_gate, args.steps, args.warmup,
                          None if args.no_cpu_baseline else args.cpu_budget)
        return
    if args.backward:
        backward_bench(S.get_config(args.config), args.steps, args.warmup)
        return
    cfg = S.get_config(args.config)

    if args.impl == "reference":
        # the CPU oracle needs no process group: under torchrun rank 0 runs it and
        # the other ranks exit at once
        if int(os.environ.get("RANK", "0")) == 0:
            run_reference(args, cfg)
        return

    world, rank, local = dist_setup()

    import long_context_prefill_moba_b200 as M
    M.load_library()
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    q, k, v = S.gen_q(cfg, dev), S.gen_k(cfg, dev), S.gen_v(cfg, dev)
    out = torch.empty_like(q)
    layer = M.MobaLayer.from_config(cfg, dev)
    sh = layer.shape
    stream = torch.cuda.current_stream()

    def step(ev=None):
        if ev is not None:
            ev[0].record(stream)
        M.moba_block_meanpool(sh, k, layer.meank)
        n = M.moba_last_launch_count()
        if ev is not None:
            ev[1].record(stream)
        M.moba_gate_topk(sh, q, layer.meank, layer.sel, layer.offsets, layer.rows, layer.gate_ws)
        n += M.moba_last_launch_count()
        if ev is not None:
            ev[2].record(stream)
        M.moba_attn_fwd(sh, q, k, v, layer.sel, layer.offsets, layer.rows, out, None, layer.attn_ws)
        n += M.moba_last_launch_count()
        if ev is not None:
            ev[3].record(stream)
        return n

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(local)
    barrier(world)
    torch.cuda.synchronize()
    clocks.start()
    start.record(stream)
    launches = 0
    for i in range(args.steps):
        launches += step(evs[i])
    end.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    clk = clocks.stop()
    ms_rank = start.elapsed_time(end) / args.steps
    pool_ms = statistics.mean(e[0].elapsed_time(e[1]) for e in evs)
    gate_ms = statistics.mean(e[1].elapsed_time(e[2]) for e in evs)
    attn_ms = statistics.mean(e[2].elapsed_time(e[3]) for e in evs)

    flops = attn_flops(cfg)
    ms = max_over_ranks(ms_rank, world)
    value = job_throughput(flops, ms_rank, world) / 1e12
    peaks, peak_kind = load_peaks()
    peak = peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"])
    attn_tf = flops / (attn_ms * 1e-3) / 1e12
    esz = 2 if cfg.dtype == "bf16" else 4
    kbytes = cfg.batch * cfg.seqlen * cfg.hkv * cfg.head_dim * esz
    qbytes = cfg.batch * cfg.seqlen * cfg.hq * cfg.head_dim * esz
    pool_bytes = kbytes + layer.meank.numel() * 4
    gate_bytes = qbytes + layer.sel.numel() * 4 * 2 + layer.rows.numel() * 4
    traffic, traffic_note = recorded_traffic(M.moba_rows_elems(sh))

    # end to end through the C ABI from host buffers (pinned): moba_prefill_host
    # copies k/v in, streams q in and out one query pass at a time and overlaps
    # those copies with the kernels; every copy is inside the timed region
    e2e = None
    if not args.no_e2e:
        hq_, hk_, hv_ = (x.cpu().pin_memory() for x in (q, k, v))
        ho = torch.empty(out.shape, dtype=out.dtype, pin_memory=True)
        del layer, q, k, v, out          # the host-buffer layer keeps its own device copies
        torch.cuda.empty_cache()
        host_layer = M.MobaHostLayer.from_config(cfg, dev)
        host_layer.forward(hq_, hk_, hv_, ho)          # warm-up (also checks the status words)
        if host_layer.device_status() != (0, 0):
            raise RuntimeError(f"moba_prefill_host: device status {host_layer.device_status()}")
        barrier(world)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(args.e2e_steps):
            host_layer.forward(hq_, hk_, hv_, ho)
        e1.record(stream)
        torch.cuda.synchronize()
        barrier(world)
        e2e_rank = e0.elapsed_time(e1) / args.e2e_steps
        e2e_ms = max_over_ranks(e2e_rank, world)
        e2e = {"value": job_throughput(flops, e2e_rank, world) / 1e12, "unit": "TFLOP/s", "ms_per_step": e2e_ms,
               "h2d_bytes_per_step": 2 * kbytes + qbytes, "d2h_bytes_per_step": qbytes,
               "api": "moba_prefill_host (copies overlapped with the kernels, pass by pass)",
               "gpu_launches_per_step": host_layer.launches}
        del hq_, hk_, hv_, ho, host_layer

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(cfg, args.cpu_budget)

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": cfg.dtype, "data": "synthetic",
            "config": config_of(cfg, args),
            "ms_per_layer": ms,
            "kernels_ms": {"meanpool": pool_ms, "gate": gate_ms, "attn": attn_ms},
            "roofline": {"bound": "tensor", "kernel": "moba_attn_fwd (attention + merge)",
                         "achieved": attn_tf, "peak": peak, "unit": "TFLOP/s", "frac": attn_tf / peak,
                         "peak_kind": f"{peak_kind} bf16 sustained", "peak_burst": peaks["bf16_tflops"],
                         "frac_of_burst": attn_tf / peaks["bf16_tflops"],
                         "peak_sustained_sm_mhz": peaks.get("clocks_under_load", {}).get("sm_mhz_median"),
                         "traffic": traffic,
                         "traffic_note": traffic_note},
            "hbm_kernels": {
                "meanpool": {"achieved": pool_bytes / (pool_ms * 1e-3) / 1e9, "unit": "GB/s",
                             "peak": peaks["hbm_gbs"]},
                "gate": {"achieved": gate_bytes / (gate_ms * 1e-3) / 1e9, "unit": "GB/s",
                         "peak": peaks["hbm_gbs"]}},
            "whole_step_frac_of_peak": (flops / (ms * 1e-3) / 1e12) / peaks["bf16_tflops"],
            "gpu_launches": launches,
            "clocks": clk,
            "e2e": e2e,
            "cpu_baseline": cpu,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
