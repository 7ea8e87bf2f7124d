"""Benchmark of the SeerAttention prefill hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]

A step is one pass of the inference hot path over one synthetic Llama-3.1-8B
attention layer at 128k tokens: the AttnGate (pooling, projections, block
scores, top-k at 10% density = 90% block sparsity) and the block-sparse
causal attention over the selected blocks.  The gate's ground-truth path
(the max-pooled attention map) is timed in the same run on its own workload
(B=1, 32k tokens) and reported as an extra object.

value = active-block attention TFLOP/s of the whole step (gate included), all
ranks together; each rank runs its own independent layer (weak scaling, no
data-path collective).  Inputs (1.5 GB) are larger than L2, so no flush is
needed between steps.  With --impl reference the fp64 CPU oracle is timed on
the host cores instead, on a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = ("sparse prefill attn ms & active-block TFLOP/s (% BF16 peak) at 128k, 90% sparsity")
WORKLOAD = "layer128k"
DENSITY = 0.1
BMAX_WORKLOAD = "bmax32k"
DECODE_WORKLOAD = "decode128k"
# packed variable-length prefill: sequence lengths inside the 128k layer buffer
VARLEN_LENS = [61477, 30000, 16384, 9000, 8191, 4000, 1500, 129]


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="seer", choices=["seer", "reference"])
    ap.add_argument("--workload", default=WORKLOAD)
    ap.add_argument("--density", type=float, default=DENSITY)
    ap.add_argument("--no-blockmax", action="store_true")
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--no-varlen", action="store_true")
    ap.add_argument("--no-tf32", action="store_true")
    ap.add_argument("--no-context", action="store_true", help="skip the dense-attention comparison")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-sweep", action="store_true", help="skip the 50-95%% sparsity sweep at 128k")
    ap.add_argument("--no-configs", action="store_true", help="skip the 8k / 32k / 4x4k per-workload figures")
    return ap.parse_args()


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d, "measured"
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}, "fallback"


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled during the timed region.

    The sampler is started (and its first line awaited) before the region, so
    that the process start-up of nvidia-smi falls outside it; each line is
    stamped on arrival and only lines that arrive inside [mark_start,
    mark_end] are used (if the region is shorter than the sampling period, the
    first line after it, which covers its last 50 ms, is used instead)."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.lines = []
        self.t0 = self.t1 = None

    def start(self, wait_s: float = 5.0):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.Q}", "--format=csv,noheader,nounits",
                 "-lms", "50"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except Exception:
            self.proc = None
            return
        t = time.time()
        while not self.lines and time.time() - t < wait_s and self.proc.poll() is None:
            time.sleep(0.02)

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append((time.time(), line.strip()))

    def mark_start(self):
        self.t0 = time.time()

    def mark_end(self):
        self.t1 = time.time()

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        t = time.time()
        while self.t1 is not None and not any(ts > self.t1 for ts, _ in self.lines) and time.time() - t < 1.0:
            time.sleep(0.02)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        inside = [ln for ts, ln in self.lines if self.t0 is not None and self.t0 <= ts <= self.t1]
        window = "inside the timed region"
        if not inside:
            after = [ln for ts, ln in self.lines if self.t1 is not None and ts > self.t1]
            inside = after[:1]
            window = "first sample after the timed region (region shorter than the 200 ms period)"
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in inside:
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                smax = float(f[2])
            except ValueError:
                continue
            for nm, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(nm)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": smax,
                "reasons": sorted(reasons), "samples": len(sm), "window": window}


# ------------------------------------------------------------ multi-rank --
# One process per GPU, each running its own independent layer (weak
# scaling); the only cross-rank traffic is these scalar reductions.
def rank_workload(base, rank: int):
    """The rank's own layer: the workload's shapes with seed + 1000 * rank."""
    from learned_block_sparse_seer_b200 import synth
    return synth.Workload(base.name, base.B, base.Hq, base.Hkv, base.n, base.d, base.h, base.dtype,
                          base.structure, base.seed + 1000 * rank)


def reduce_over_ranks(x: float, dev, op: str = "max") -> float:
    """x reduced over all ranks ("max" or "sum"); x itself with one rank."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX if op == "max" else dist.ReduceOp.SUM)
    return float(t.item())


def whole_job_tflops(flops_all_ranks: float, ms: float) -> float:
    """Whole-job throughput: the FLOPs of every rank over the slowest rank's
    time."""
    return flops_all_ranks / (ms * 1e-3) / 1e12


def attn_flops(counts, indices, d):
    """Algorithmic FLOPs of the active blocks: 4*d per (query, key) pair, a
    diagonal block counts its 64*65/2 causal pairs."""
    import torch
    nb = counts.shape[-1]
    total_blocks = counts.long().sum().item()
    cap = indices.shape[-1]
    i = torch.arange(nb, device=counts.device).view(1, 1, nb)
    pos = torch.arange(cap, device=counts.device).view(1, 1, 1, cap)
    valid = pos < counts.unsqueeze(-1)
    diag = ((indices == i.unsqueeze(-1)) & valid).sum().item()
    pairs = (total_blocks - diag) * 64 * 64 + diag * (64 * 65 // 2)
    causal = counts.shape[0] * counts.shape[1] * (nb * (nb + 1) // 2)
    return 4.0 * d * pairs, total_blocks, diag, 1.0 - total_blocks / causal


def launches_per_step(w) -> int:
    """This library's kernel launches in one timed step (gate, then sparse
    attention), as the host code issues them for workload w (no RoPE).

    Gate with h and d multiples of 32: Q and K pooling, already split into
    tf32 parts, and the tf32 split of Wq and Wk, in one launch (1); the two projections,
    whose epilogues write q~ and k~ split (2); the causal logits (1 when
    h <= 128 and nb % 4 == 0: the row-resident kernel; else the split of q~
    and k~ and the tile kernel, 3); the softmax and selection (2 launches,
    short and long rows, when nb % 4 == 0 and there are at least 8 rows per
    SM; else 1).  Otherwise the SIMT path: pooling (2), projections (2),
    logits (1), selection (1).
    Attention, bf16: the all-ones check (1), the K^T re-layout (1), the
    empty-row writer (1), the sparse kernel and its exact fallback (2), the
    dense kernel and its fallback (2; the pair not chosen returns at once).
    fp32: the conversion of Q and V (2), re-layout, empty rows, kernel and
    fallback (4).
    """
    nb = w.n // 64
    rows = w.B * w.Hq * nb
    if w.h % 32 == 0 and w.d % 32 == 0:
        logits = 1 if (w.h <= 128 and nb % 4 == 0) else 3
        select = 2 if (nb % 4 == 0 and rows >= 8 * 148) else 1
        gate = 1 + 2 + logits + select
    else:
        gate = 2 + 2 + 1 + 1
    attn = 7 if w.dtype == "bf16" else 6
    return gate + attn


def source_hash(names):
    h = hashlib.sha256()
    for n in names:
        h.update(open(os.path.join(ROOT, "learned_block_sparse_seer_b200", "csrc", n), "rb").read())
    return h.hexdigest()[:16]


def profiled_traffic(kernel, workload, src):
    """DRAM bytes per launch from the committed ncu summary, if it was taken
    on the current kernel source."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    try:
        d = json.load(open(p)).get(kernel, {})
    except Exception:
        return None
    if d.get("source_hash") != src or d.get("workload") != workload:
        return None
    return d.get("dram_bytes_per_launch")


# ------------------------------------------------------------------ oracle --
class OracleSampler:
    """Times the fp64 CPU oracle (as it stands) on a bounded sample of the
    workload and extrapolates to the whole layer.

    The oracle's work splits into a part per KV head (K max/min/avg pooling
    and its projection over all blocks) and a part per unit (Q pooling and
    projection of one block, its Eq. 1 score row, top-k selection, block-sparse
    attention of its 64 rows).  Full-layer time = (#KV heads) x mean per-head
    time + (#units) x mean per-unit time; value = the layer's active-block
    attention FLOPs / that time."""

    def __init__(self, w, Q, K, V, Wq, Wk, density, seed=0):
        import numpy as np

        import oracle
        self.np, self.oracle = np, oracle
        oracle.build()
        self.w, self.density = w, density
        # the oracle's input format: fp32 arrays holding the bf16 values exactly
        self.Qf = Q.float().numpy()
        self.Kf = K.float().numpy()
        self.Vf = V.float().numpy()
        self.Wq = Wq.numpy()
        self.Wk = Wk.numpy()
        self.rng = np.random.default_rng(seed)
        self.t_head, self.t_unit, self.flops = [], [], []

    def _units(self, b, g, hq, blocks, kt):
        """Gate rows, selection and attention for query blocks `blocks` of
        head hq, batched into single oracle calls (its OpenMP loops run over
        the units)."""
        np, oracle, w = self.np, self.oracle, self.w
        nb = w.nb
        cap = int(math.ceil(self.density * nb)) + 1
        rows = np.concatenate([np.arange(i * 64, (i + 1) * 64) for i in blocks])
        qb = oracle.pool_q(np.ascontiguousarray(self.Qf[b:b + 1, hq:hq + 1, rows]))
        qrow = oracle.project(qb, self.Wq[hq:hq + 1])
        qt = np.zeros((1, 1, nb, w.h))
        qt[0, 0, blocks] = qrow[0, 0]
        srows = oracle.gate_scores_units(qt, kt, w.d, blocks)
        c1, i1 = oracle.select_rows(srows, blocks, oracle.MODE_TOPK_DENSITY, density=self.density,
                                    cap=cap)
        counts = np.zeros((1, 1, nb), np.int32)
        idx = np.full((1, 1, nb, cap), -1, np.int32)
        counts[0, 0, blocks] = c1
        idx[0, 0, blocks] = i1
        oracle.sparse_attn_units(self.Qf[b:b + 1, hq:hq + 1], self.Kf[b:b + 1, g:g + 1],
                                 self.Vf[b:b + 1, g:g + 1], counts, idx, blocks)
        return int(c1.sum())

    def step(self, budget_s):
        """One KV head's fixed part plus a batch of random units of one of its
        query heads, sized to take about budget_s."""
        np, oracle, w = self.np, self.oracle, self.w
        b = int(self.rng.integers(w.B))
        g = int(self.rng.integers(w.Hkv))
        hq = g * w.G + int(self.rng.integers(w.G))
        nb = w.nb
        t0 = time.perf_counter()
        kt = oracle.project(oracle.pool_k(self.Kf[b:b + 1, g:g + 1]), self.Wk[g:g + 1])
        self.t_head.append(time.perf_counter() - t0)
        n = 8
        while True:
            blocks = np.sort(self.rng.choice(nb, size=min(n, nb), replace=False))
            t0 = time.perf_counter()
            nblk = self._units(b, g, hq, blocks, kt)
            dt = time.perf_counter() - t0
            self.t_unit.extend([dt / len(blocks)] * len(blocks))
            self.flops.append(4.0 * w.d * 64 * 64 * nblk)
            budget_s -= dt
            if budget_s <= 0:
                break
            n = int(min(nb, max(n * 2, len(blocks) * budget_s / max(dt, 1e-3))))

    def rate(self, layer_flops):
        """Extrapolated whole-layer TFLOP/s and layer time (s)."""
        w = self.w
        t_layer = (w.B * w.Hkv * (sum(self.t_head) / len(self.t_head))
                   + w.B * w.Hq * w.nb * (sum(self.t_unit) / len(self.t_unit)))
        return layer_flops / t_layer / 1e12, t_layer

    def describe(self):
        return (f"{len(self.t_head)} KV head(s) pooled+projected and {len(self.t_unit)} random units "
                f"(query head x 64-row block: Q pooling, Eq.1 row, top-k, attention), fp64, "
                f"{sum(self.t_head) + sum(self.t_unit):.1f} s; extrapolated to the whole layer")


def layer_flops_expected(w, density):
    """Active-block FLOPs of the layer under density top-k (diagonal counted
    in full), for the reference arm that has no GPU lists."""
    import oracle
    tot = 0
    for i in range(w.nb):
        tot += oracle.topk_count(i, oracle.MODE_TOPK_DENSITY, density=density)
    return 4.0 * w.d * 64 * 64 * tot * w.B * w.Hq


# -------------------------------------------------------------------- main --
def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    from learned_block_sparse_seer_b200 import synth
    w = synth.WORKLOADS[args.workload]
    Q, K, V = synth.make_qkv(w)
    Wq, Wk = synth.make_gate_weights(w)
    smp = OracleSampler(w, Q, K, V, Wq, Wk, args.density)
    lf = layer_flops_expected(w, args.density)
    per_step = max(3.0, 100.0 / max(1, args.steps + args.warmup))
    rates, times = [], []
    for step in range(args.warmup + args.steps):
        n0h, n0u = len(smp.t_head), len(smp.t_unit)
        smp.step(per_step)
        if step >= args.warmup:
            r, t_layer = smp.rate(lf)
            rates.append(r)
            times.append(t_layer)
    value, t_layer = smp.rate(lf)
    cores = smp.oracle.num_threads()
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": t_layer * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": f"{args.workload}: B={w.B} Hq={w.Hq} Hkv={w.Hkv} n={w.n} d={w.d} "
                               f"gate h={w.h}, top-k density {args.density}"},
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                         "sample": smp.describe()},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def context_bench(seer, dev, stream, w, Qd, Kd, Vd, O, lse, gate_ms, attn_ms):
    """Context for the sparse step: dense causal attention of the same layer
    by torch's scaled_dot_product_attention (its fastest backend on this GPU,
    GQA native) and by this library's kernel with every causal block listed
    (the all-ones mask), and the sparse step's speedup over the dense one."""
    import torch
    import torch.nn.functional as F

    def timed(fn, reps=2):
        fn()
        torch.cuda.synchronize(dev)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(reps):
            fn()
        b.record(stream)
        torch.cuda.synchronize(dev)
        return a.elapsed_time(b) / reps

    sdpa_ms = timed(lambda: F.scaled_dot_product_attention(Qd, Kd, Vd, is_causal=True, enable_gqa=True))
    nb = w.nb
    counts = (torch.arange(nb, device=dev, dtype=torch.int32) + 1).repeat(w.B, w.Hq, 1).contiguous()
    idx = torch.arange(nb, device=dev, dtype=torch.int32).repeat(w.B, w.Hq, nb, 1).contiguous()
    ws = torch.empty(seer.sparse_attn_workspace_size(w.B, w.Hq, w.Hkv, w.n, w.d), dtype=torch.uint8, device=dev)
    ones_ms = timed(lambda: seer.seer_sparse_attn(Qd, Kd, Vd, counts, idx, workspace=ws, out=(O, lse)))
    del idx, counts, ws
    dense_flops = 4.0 * w.d * w.B * w.Hq * (w.n * (w.n + 1) / 2)
    return {"workload": f"{w.name}: dense causal attention, same shapes",
            "sdpa_dense_ms": sdpa_ms, "sdpa_tflops": dense_flops / (sdpa_ms * 1e-3) / 1e12,
            "all_ones_mask_ms": ones_ms, "all_ones_tflops": dense_flops / (ones_ms * 1e-3) / 1e12,
            "speedup_sparse_attn_vs_sdpa": sdpa_ms / attn_ms,
            "speedup_gate_plus_sparse_attn_vs_sdpa": sdpa_ms / (gate_ms + attn_ms)}


def configs_bench(seer, synth, dev, stream, pk):
    """The other workloads' figures, each on its own seeded layer:
    layer8k (threshold T = 5e-4): gate and attention ms; layer32k (top-k at
    density 0.1): gate and attention ms, active-block TFLOP/s, and the
    all-ones mask against torch's dense causal SDPA on the same shapes;
    bmax4k (B = 4, 4k tokens): the max-pooled map."""
    import torch
    import torch.nn.functional as F

    def timed(fn, reps=5, warm=2):
        for _ in range(warm):
            fn()
        torch.cuda.synchronize(dev)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(reps):
            fn()
        b.record(stream)
        torch.cuda.synchronize(dev)
        return a.elapsed_time(b) / reps

    out = {}
    for name, mode, kw in (("layer8k", "threshold", {"T": 5e-4}), ("layer32k", "density", {"density": 0.1})):
        w = synth.WORKLOADS[name]
        Q, K, V = (t.to(dev) for t in synth.make_qkv(w))
        Wq, Wk = (t.to(dev) for t in synth.make_gate_weights(w))
        cap = seer.gate_required_cap(w.B, w.Hq, w.Hkv, w.n, w.d, mode, **{k: v for k, v in kw.items() if k != "T"})
        counts = torch.empty(w.B, w.Hq, w.nb, dtype=torch.int32, device=dev)
        idx = torch.empty(w.B, w.Hq, w.nb, cap, dtype=torch.int32, device=dev)
        O = torch.empty_like(Q)
        lse = torch.empty(w.B, w.Hq, w.n, dtype=torch.float32, device=dev)
        gws = torch.empty(seer.gate_workspace_size(w.B, w.Hq, w.Hkv, w.n, w.d, w.h), dtype=torch.uint8, device=dev)
        aws = torch.empty(seer.sparse_attn_workspace_size(w.B, w.Hq, w.Hkv, w.n, w.d), dtype=torch.uint8,
                          device=dev)
        gate = lambda: seer.seer_gate(Q, K, Wq, Wk, mode, cap=cap, workspace=gws, out=(counts, idx, None), **kw)
        attn = lambda: seer.seer_sparse_attn(Q, K, V, counts, idx, workspace=aws, out=(O, lse))
        g_ms = timed(gate)
        a_ms = timed(attn)
        f, nbk, _, sp = attn_flops(counts, idx, w.d)
        r = {"workload": f"{name}: B={w.B} Hq={w.Hq} Hkv={w.Hkv} n={w.n} d={w.d}, {mode} "
                         + ", ".join(f"{k}={v}" for k, v in kw.items()),
             "achieved_sparsity": sp, "active_blocks": nbk, "gate_ms": g_ms, "attn_ms": a_ms,
             "attn_tflops": f / (a_ms * 1e-3) / 1e12, "attn_frac_bf16_burst": f / (a_ms * 1e-3) / 1e12 / pk["bf16_tflops"],
             "gate_plus_attn_ms": g_ms + a_ms, "status": seer.seer_workspace_status(aws)}
        if name == "layer32k":
            sdpa_ms = timed(lambda: F.scaled_dot_product_attention(Q, K, V, is_causal=True, enable_gqa=True), reps=3)
            ones_c = (torch.arange(w.nb, device=dev, dtype=torch.int32) + 1).repeat(w.B, w.Hq, 1).contiguous()
            ones_i = torch.arange(w.nb, device=dev, dtype=torch.int32).repeat(w.B, w.Hq, w.nb, 1).contiguous()
            ones_ms = timed(lambda: seer.seer_sparse_attn(Q, K, V, ones_c, ones_i, workspace=aws, out=(O, lse)), reps=3)
            dense_flops = 4.0 * w.d * w.B * w.Hq * (w.n * (w.n + 1) / 2)
            r.update({"sdpa_dense_ms": sdpa_ms, "sdpa_tflops": dense_flops / (sdpa_ms * 1e-3) / 1e12,
                      "all_ones_mask_ms": ones_ms, "all_ones_tflops": dense_flops / (ones_ms * 1e-3) / 1e12,
                      "speedup_sparse_attn_vs_sdpa": sdpa_ms / a_ms})
            del ones_c, ones_i
        out[name] = r
        del Q, K, V, Wq, Wk, counts, idx, O, lse, gws, aws
    bw = synth.WORKLOADS["bmax4k"]
    bQ, bK, _ = (t.to(dev) for t in synth.make_qkv(bw))
    bws = torch.empty(seer.blockmax_workspace_size(bw.B, bw.Hq, bw.Hkv, bw.n, bw.d), dtype=torch.uint8, device=dev)
    M = torch.empty(bw.B, bw.Hq, bw.nb, bw.nb, dtype=torch.float32, device=dev)
    bl = torch.empty(bw.B, bw.Hq, bw.n, dtype=torch.float32, device=dev)
    bms = timed(lambda: seer.seer_attn_blockmax(bQ, bK, workspace=bws, out=(M, bl)))
    pairs = bw.B * bw.Hq * (bw.n * (bw.n + 1) // 2)
    out["bmax4k"] = {"workload": f"bmax4k: B={bw.B} Hq={bw.Hq} Hkv={bw.Hkv} n={bw.n} d={bw.d}", "ms": bms,
                     "qk_tflops": 2.0 * bw.d * pairs / (bms * 1e-3) / 1e12,
                     "frac_bf16_burst": 2.0 * bw.d * pairs / (bms * 1e-3) / 1e12 / pk["bf16_tflops"],
                     "exp_per_s": pairs / (bms * 1e-3), "status": seer.seer_workspace_status(bws)}
    return out


def tf32_bench(seer, dev, stream, w, Qd, Kd, Vd, counts, indices, flops, pk):
    """The fp32 path on the tf32 tensor cores: the 128k layer's tensors held
    in fp32 (the bf16 values, exact), the same density lists.  Peak: the
    measured bf16 peaks times the nominal dense tf32 / bf16 ratio (1.1 / 2.25
    PFLOP/s)."""
    import torch
    Qf, Kf, Vf = Qd.float(), Kd.float(), Vd.float()
    ws = torch.empty(seer.sparse_attn_tf32_workspace_size(w.B, w.Hq, w.Hkv, w.n, w.d), dtype=torch.uint8, device=dev)
    O = torch.empty_like(Qf)
    lse = torch.empty(w.B, w.Hq, w.n, dtype=torch.float32, device=dev)
    for _ in range(2):
        seer.seer_sparse_attn_tf32(Qf, Kf, Vf, counts, indices, workspace=ws, out=(O, lse))
    torch.cuda.synchronize(dev)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    reps = 3
    a.record(stream)
    for _ in range(reps):
        seer.seer_sparse_attn_tf32(Qf, Kf, Vf, counts, indices, workspace=ws, out=(O, lse))
    b.record(stream)
    torch.cuda.synchronize(dev)
    ms = a.elapsed_time(b) / reps
    ratio = 1.1 / 2.25
    tfl = flops / (ms * 1e-3) / 1e12
    res = {"workload": f"{w.name} in fp32, same lists", "ms": ms, "tflops": tfl,
           "peak_tf32_tflops": {"burst": pk["bf16_tflops"] * ratio,
                                "sustained": pk.get("bf16_tflops_sustained", pk["bf16_tflops"]) * ratio},
           "frac_of_tf32_peak": tfl / (pk["bf16_tflops"] * ratio),
           "status": seer.seer_workspace_status(ws)}
    del Qf, Kf, Vf, O, lse, ws
    return res


def varlen_bench(seer, synth, dev, stream, w, Qd, Kd, Vd, Wqd, Wkd, density, pk):
    """Packed variable-length prefill on the 128k layer's buffers: the
    sequences of VARLEN_LENS placed at 64-token boundaries, gate (top-k
    density) and sparse attention on the packed tensors.  Tokens outside the
    sequences keep the layer's finite values (the gate skips them, attention
    masks them).  FLOPs as attn_flops (a sequence's last, partial block is
    counted as a full tile)."""
    import torch
    starts, n = synth.varlen_layout(VARLEN_LENS)
    assert n <= w.n
    st = torch.tensor(starts, dtype=torch.int32, device=dev)
    ln = torch.tensor(VARLEN_LENS, dtype=torch.int32, device=dev)
    nb = w.nb
    cap = seer.gate_required_cap(1, w.Hq, w.Hkv, w.n, w.d, "density", density=density)
    counts = torch.empty(1, w.Hq, nb, dtype=torch.int32, device=dev)
    idx = torch.empty(1, w.Hq, nb, cap, dtype=torch.int32, device=dev)
    gws = torch.empty(seer.gate_varlen_workspace_size(w.Hq, w.Hkv, w.n, w.d, w.h), dtype=torch.uint8, device=dev)
    aws = torch.empty(seer.sparse_attn_workspace_size(1, w.Hq, w.Hkv, w.n, w.d), dtype=torch.uint8, device=dev)
    O = torch.empty_like(Qd)
    lse = torch.empty(1, w.Hq, w.n, dtype=torch.float32, device=dev)

    def gate():
        seer.seer_gate_varlen(Qd, Kd, Wqd, Wkd, st, ln, "density", density=density, cap=cap, workspace=gws,
                              out=(counts, idx, None))

    def attn():
        seer.seer_sparse_attn(Qd, Kd, Vd, counts, idx, workspace=aws, out=(O, lse))

    def timed(fn, reps=5):
        for _ in range(2):
            fn()
        torch.cuda.synchronize(dev)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(reps):
            fn()
        b.record(stream)
        torch.cuda.synchronize(dev)
        return a.elapsed_time(b) / reps

    gms = timed(gate)
    ams = timed(attn)
    flops, nblk, _, _ = attn_flops(counts, idx, w.d)
    causal = sum(((l + 63) // 64) * ((l + 63) // 64 + 1) // 2 for l in VARLEN_LENS) * w.Hq
    return {"workload": f"{len(VARLEN_LENS)} sequences {VARLEN_LENS} packed at 64-token boundaries into the "
                        f"{w.name} buffers (Hq={w.Hq} Hkv={w.Hkv} d={w.d}), top-k density {density}",
            "gate_ms": gms, "attn_ms": ams, "attn_tflops": flops / (ams * 1e-3) / 1e12,
            "active_blocks": nblk, "achieved_sparsity": 1.0 - nblk / causal,
            "gate_status": seer.seer_workspace_status(gws), "attn_status": seer.seer_workspace_status(aws)}


def decode_bench(seer, synth, dev, stream, density, pk):
    """The decode stage on a 128k-token cache: the compressed K cache built
    once for every complete block, then per token the gate (top-k density)
    and the block-sparse attention, and the 1D ground truth.  The L2 is
    flushed before every timed launch by reading a 512 MB buffer (a read leaves
    no dirty lines whose write-back would compete with the timed kernel), so
    each launch reads HBM."""
    import torch
    w = synth.WORKLOADS[DECODE_WORKLOAD]
    seq_len = synth.decode_seq_len(w)
    c = (seq_len - 1) // 64
    q, Kc, Vc = synth.make_decode(w, seq_len)
    _, Wk = synth.make_gate_weights(w)
    qd, Kd, Vd, Wkd = (t.to(dev) for t in (q, Kc, Vc, Wk))
    del q, Kc, Vc
    flush = torch.ones(128 << 20, dtype=torch.float32, device=dev)
    kt = torch.zeros(w.B, w.Hkv, w.nb, w.d, dtype=torch.float32, device=dev)
    cap = max(1, seer.decode_gate_required_cap(w.B, w.Hq, w.Hkv, w.n, w.d, seq_len, "density", density=density))
    counts = torch.empty(w.B, w.Hq, dtype=torch.int32, device=dev)
    idx = torch.empty(w.B, w.Hq, cap, dtype=torch.int32, device=dev)
    gws = torch.empty(seer.decode_gate_workspace_size(w.B, w.Hq, w.Hkv, w.n, w.d), dtype=torch.uint8, device=dev)
    aws = torch.empty(seer.sparse_decode_attn_workspace_size(w.B, w.Hq, w.Hkv, w.n, w.d), dtype=torch.uint8,
                      device=dev)
    O = torch.empty_like(qd)
    lse = torch.empty(w.B, w.Hq, dtype=torch.float32, device=dev)
    gt = torch.empty(w.B, w.Hq, c + 1, dtype=torch.float32, device=dev)
    glse = torch.empty(w.B, w.Hq, dtype=torch.float32, device=dev)

    def timed(fn, reps=10, warm=3):
        for _ in range(warm):
            fn()
        tot = 0.0
        for _ in range(reps):
            flush.sum()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            fn()
            b.record(stream)
            torch.cuda.synchronize(dev)
            tot += a.elapsed_time(b)
        return tot / reps

    kc_ms = timed(lambda: seer.seer_decode_kcache_update(Kd, Wkd, 0, c, kt))
    gate_ms = timed(lambda: seer.seer_decode_gate(qd, kt, w.n, seq_len, "density", density=density, cap=cap,
                                                  workspace=gws, out=(counts, idx, None)))
    attn_ms = timed(lambda: seer.seer_sparse_decode_attn(qd, Kd, Vd, seq_len, counts, idx, workspace=aws,
                                                         out=(O, lse)))
    step_ms = timed(lambda: (seer.seer_decode_gate(qd, kt, w.n, seq_len, "density", density=density, cap=cap,
                                                   workspace=gws, out=(counts, idx, None)),
                             seer.seer_sparse_decode_attn(qd, Kd, Vd, seq_len, counts, idx, workspace=aws,
                                                          out=(O, lse))))
    gt_ms = timed(lambda: seer.seer_decode_blockmax(qd, Kd, seq_len, out=(gt, glse)))
    # algorithmic bytes: each distinct (b, g, block) that some query head of
    # the group selects, plus the token's own block, read once for K and V
    cn = counts.cpu().numpy()
    ix = idx.cpu().numpy()
    G = w.G
    uniq = 0
    per_row = 0
    for b in range(w.B):
        for g in range(w.Hkv):
            sel = set()
            for hq in range(g * G, (g + 1) * G):
                sel.update(int(j) for j in ix[b, hq, :cn[b, hq]])
                per_row += int(cn[b, hq])
            uniq += len(sel)
    tail = seq_len - 64 * c
    kv_row = 64 * w.d * 2 * 2
    attn_bytes = (uniq * kv_row + w.B * w.Hkv * tail * w.d * 2 * 2 + qd.numel() * 2 * 2 + counts.numel() * 4
                  + cn.sum() * 4)
    gate_bytes = w.B * w.Hkv * c * w.d * 4 + qd.numel() * 2 + counts.numel() * 4 + cn.sum() * 4
    kc_bytes = w.B * w.Hkv * c * 64 * w.d * 2 + w.B * w.Hkv * c * w.d * 4
    gt_bytes = w.B * w.Hkv * seq_len * w.d * 2 + w.B * w.Hq * (c + 1) * 4
    hbm = pk["hbm_gbs"]

    def gbs(nbytes, ms):
        return nbytes / (ms * 1e-3) / 1e9

    return {"workload": f"{DECODE_WORKLOAD}: B={w.B} Hq={w.Hq} Hkv={w.Hkv} cache n={w.n} d={w.d} "
                        f"seq_len={seq_len}, top-k density {density}",
            "l2": "flushed (512 MB read) before every timed launch",
            "candidates": c, "selected_per_row": float(cn.mean()), "distinct_blocks_per_kv_head":
                uniq / (w.B * w.Hkv),
            "kcache_build": {"ms": kc_ms, "gb_s": gbs(kc_bytes, kc_ms), "frac_hbm": gbs(kc_bytes, kc_ms) / hbm},
            "gate": {"us": gate_ms * 1e3, "gb_s": gbs(gate_bytes, gate_ms)},
            "attn": {"us": attn_ms * 1e3, "gb_s": gbs(attn_bytes, attn_ms),
                     "frac_hbm": gbs(attn_bytes, attn_ms) / hbm, "algorithmic_bytes": int(attn_bytes),
                     "status": seer.seer_workspace_status(aws)},
            "token_step_us": step_ms * 1e3,
            "ground_truth": {"us": gt_ms * 1e3, "gb_s": gbs(gt_bytes, gt_ms), "frac_hbm": gbs(gt_bytes, gt_ms) / hbm},
            "hbm_peak_gbs": hbm}


def main():
    args = parse()
    if args.impl == "reference":
        return run_reference(args)

    import torch
    import torch.distributed as dist

    import learned_block_sparse_seer_b200 as seer
    from learned_block_sparse_seer_b200 import synth

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=__import__("datetime").timedelta(seconds=600))
    dev = torch.device("cuda", local if world > 1 else 0)
    torch.cuda.set_device(dev)
    seer.lib()

    base = synth.WORKLOADS[args.workload]
    w = rank_workload(base, rank)
    Q, K, V = synth.make_qkv(w)
    Wq, Wk = synth.make_gate_weights(w)
    Qd, Kd, Vd, Wqd, Wkd = (t.to(dev) for t in (Q, K, V, Wq, Wk))
    nb = w.nb
    cap = seer.gate_required_cap(w.B, w.Hq, w.Hkv, w.n, w.d, "density", density=args.density)
    counts = torch.empty(w.B, w.Hq, nb, dtype=torch.int32, device=dev)
    indices = torch.empty(w.B, w.Hq, nb, cap, dtype=torch.int32, device=dev)
    O = torch.empty_like(Qd)
    lse = torch.empty(w.B, w.Hq, w.n, dtype=torch.float32, device=dev)
    gws = torch.empty(seer.gate_workspace_size(w.B, w.Hq, w.Hkv, w.n, w.d, w.h), dtype=torch.uint8, device=dev)
    aws = torch.empty(seer.sparse_attn_workspace_size(w.B, w.Hq, w.Hkv, w.n, w.d), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    def gate():
        seer.seer_gate(Qd, Kd, Wqd, Wkd, "density", density=args.density, cap=cap, workspace=gws,
                       out=(counts, indices, None))

    def attn():
        seer.seer_sparse_attn(Qd, Kd, Vd, counts, indices, workspace=aws, out=(O, lse))

    for _ in range(args.warmup):
        gate()
        attn()
    torch.cuda.synchronize(dev)
    assert seer.seer_workspace_status(aws) == 0, "device status after warm-up"
    flops, nblocks, ndiag, sparsity = attn_flops(counts, indices, w.d)

    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True),
           torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    clocks = ClockSampler(dev.index if dev.index is not None else 0)
    clocks.start()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    clocks.mark_start()
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    t_start.record(stream)
    for s in range(args.steps):
        ev[s][0].record(stream)
        gate()
        ev[s][1].record(stream)
        attn()
        ev[s][2].record(stream)
    t_end.record(stream)
    torch.cuda.synchronize(dev)
    clocks.mark_end()
    clk = clocks.stop()
    if world > 1:
        dist.barrier()
    total_ms = t_start.elapsed_time(t_end)
    gate_ms = [a.elapsed_time(b) for a, b, _ in ev]
    attn_ms = [b.elapsed_time(c) for _, b, c in ev]
    total_ms = reduce_over_ranks(total_ms, dev, "max")
    flops_all = reduce_over_ranks(flops, dev, "sum")
    ms_per_step = total_ms / args.steps
    attn_avg = sum(attn_ms) / len(attn_ms)
    gate_avg = sum(gate_ms) / len(gate_ms)
    value = whole_job_tflops(flops_all, ms_per_step)
    attn_tflops = flops / (attn_avg * 1e-3) / 1e12
    pk, pk_kind = peaks()
    peak = pk["bf16_tflops"]  # burst: the kernel is timed in launches of ~20 ms, not a seconds-long loop
    gate_bytes = (Q.numel() + K.numel()) * 2 + counts.numel() * 4 + nblocks * 4
    src = source_hash(["attn.cu", "ptx.cuh"])
    traffic = profiled_traffic("sparse_attn_kernel", args.workload, src)

    # ------------------------------------------ end to end with host buffers --
    e2e = None
    if not args.no_e2e:
        # the public host-memory call: Q/K/V in page-locked host memory, O and
        # LSE back in host memory; every copy is inside the timed region
        hQ, hK, hV = (t.pin_memory() for t in (Q, K, V))
        hO = torch.empty(O.shape, dtype=O.dtype).pin_memory()
        hl = torch.empty(lse.shape, dtype=lse.dtype).pin_memory()
        hbuf = torch.empty(seer.prefill_host_buffer_size(w.B, w.Hq, w.Hkv, w.n, w.d, w.h, "density",
                                                         density=args.density), dtype=torch.uint8, device=dev)

        def e2e_step():
            seer.seer_prefill_host(hQ, hK, hV, Wqd, Wkd, "density", density=args.density, out=(hO, hl), buffer=hbuf)

        e2e_step()  # warm-up (the call returns with the outputs in host memory)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        n_e2e = max(2, min(args.steps, 5))
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize(dev)
        e0.record(stream)
        for _ in range(n_e2e):
            e2e_step()
        e1.record(stream)
        torch.cuda.synchronize(dev)
        e2e_ms = e0.elapsed_time(e1) / n_e2e
        e2e_ms = reduce_over_ranks(e2e_ms, dev, "max")
        assert torch.equal(hO, O.cpu()), "host-memory path differs from the device path"
        e2e = {"value": whole_job_tflops(flops_all, e2e_ms), "unit": "TFLOP/s",
               "ms_per_step": e2e_ms, "call": "seer_prefill_host (copies overlapped with the compute, per chunk of query heads sharing a KV head)",
               "h2d_bytes_per_step": (Q.numel() + K.numel() + V.numel()) * Q.element_size(),
               "d2h_bytes_per_step": O.numel() * O.element_size() + lse.numel() * lse.element_size()}

    # --------------------------------------------------------- blockmax path --
    bmax = None
    if not args.no_blockmax and rank == 0:
        bw = synth.WORKLOADS[BMAX_WORKLOAD]
        bQ, bK, _ = synth.make_qkv(bw)
        bQd, bKd = bQ.to(dev), bK.to(dev)
        bws = torch.empty(seer.blockmax_workspace_size(bw.B, bw.Hq, bw.Hkv, bw.n, bw.d), dtype=torch.uint8,
                          device=dev)
        M = torch.empty(bw.B, bw.Hq, bw.nb, bw.nb, dtype=torch.float32, device=dev)
        bl = torch.empty(bw.B, bw.Hq, bw.n, dtype=torch.float32, device=dev)
        for _ in range(2):
            seer.seer_attn_blockmax(bQd, bKd, workspace=bws, out=(M, bl))
        torch.cuda.synchronize(dev)
        b0, b1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        nrep = 5
        b0.record(stream)
        for _ in range(nrep):
            seer.seer_attn_blockmax(bQd, bKd, workspace=bws, out=(M, bl))
        b1.record(stream)
        torch.cuda.synchronize(dev)
        bms = b0.elapsed_time(b1) / nrep
        pairs = bw.B * bw.Hq * (bw.n * (bw.n + 1) // 2)
        bflops = 2.0 * bw.d * pairs
        bmax = {"workload": f"{BMAX_WORKLOAD}: B={bw.B} Hq={bw.Hq} Hkv={bw.Hkv} n={bw.n} d={bw.d}",
                "ms": bms, "qk_tflops": bflops / (bms * 1e-3) / 1e12,
                "frac_of_peak": bflops / (bms * 1e-3) / 1e12 / pk["bf16_tflops"],
                "exp_per_s": pairs / (bms * 1e-3),
                "status": seer.seer_workspace_status(bws)}
        # the gate's distillation step on that map: KL(gt || score) and the
        # gradients of Wq, Wk (the map just produced serves as gt)
        bWq, bWk = (t.to(dev) for t in synth.make_gate_weights(bw))
        tws = torch.empty(seer.gate_kl_backward_workspace_size(bw.B, bw.Hq, bw.Hkv, bw.n, bw.d, bw.h),
                          dtype=torch.uint8, device=dev)
        kout = (torch.empty(1, dtype=torch.float32, device=dev), torch.empty_like(bWq), torch.empty_like(bWk))
        for _ in range(2):
            seer.seer_gate_kl_backward(bQd, bKd, bWq, bWk, M, workspace=tws, out=kout)
        torch.cuda.synchronize(dev)
        b0.record(stream)
        for _ in range(nrep):
            seer.seer_gate_kl_backward(bQd, bKd, bWq, bWk, M, workspace=tws, out=kout)
        b1.record(stream)
        torch.cuda.synchronize(dev)
        kms = b0.elapsed_time(b1) / nrep
        # algorithmic bytes: Q and K read once (pooling), gt read, the logits
        # written and read back as dz, the small pooled/projected tensors
        kbytes = (bQd.numel() + bKd.numel()) * 2 + 3 * M.numel() * 4
        bmax["gate_kl_step"] = {"ms": kms, "loss": float(kout[0].item()), "gb_s": kbytes / (kms * 1e-3) / 1e9,
                                "algorithmic_bytes": kbytes}
        # the training forward (O, LSE and the map) on the same layer
        bV = synth.make_qkv(bw)[2].to(dev)
        fws = torch.empty(seer.attn_forward_map_workspace_size(bw.B, bw.Hq, bw.Hkv, bw.n, bw.d),
                          dtype=torch.uint8, device=dev)
        fout = (torch.empty_like(bQd), torch.empty(bw.B, bw.Hq, bw.n, dtype=torch.float32, device=dev),
                torch.empty(bw.B, bw.Hq, bw.nb, bw.nb, dtype=torch.float32, device=dev))
        for _ in range(2):
            seer.seer_attn_forward_map(bQd, bKd, bV, workspace=fws, out=fout)
        torch.cuda.synchronize(dev)
        b0.record(stream)
        for _ in range(nrep):
            seer.seer_attn_forward_map(bQd, bKd, bV, workspace=fws, out=fout)
        b1.record(stream)
        torch.cuda.synchronize(dev)
        fms = b0.elapsed_time(b1) / nrep
        # one pass: QK^T (shared by the map) and PV, 4 d per causal pair
        fflops = 4.0 * bw.d * pairs
        bmax["forward_map"] = {"ms": fms, "tflops": fflops / (fms * 1e-3) / 1e12,
                               "flops": fflops, "status": seer.seer_workspace_status(fws)}
        del bV, fws, fout
        del bQd, bKd, bws, M, bl, tws, kout

    # ----------------------------------------------------------- decode path --
    dec = None
    if not args.no_decode and rank == 0:
        dec = decode_bench(seer, synth, dev, stream, args.density, pk)

    # ------------------------------------------------------- varlen packing --
    vl = None
    if not args.no_varlen and rank == 0:
        vl = varlen_bench(seer, synth, dev, stream, w, Qd, Kd, Vd, Wqd, Wkd, args.density, pk)

    # ------------------------------------------------------------ tf32 path --
    tf = None
    if not args.no_tf32 and rank == 0:
        tf = tf32_bench(seer, dev, stream, w, Qd, Kd, Vd, counts, indices, flops, pk)

    # ------------------------------------------------- dense-attention context --
    ctx = None
    if not args.no_context and rank == 0:
        ctx = context_bench(seer, dev, stream, w, Qd, Kd, Vd, O, lse, gate_avg, attn_avg)

    # ------------------------------------------- the other workloads' figures --
    cfgs = None
    if not args.no_configs and rank == 0:
        cfgs = configs_bench(seer, synth, dev, stream, pk)

    # ------------------------------------------------------ density sweep ----
    sweep = None
    if not args.no_sweep and rank == 0:
        sweep = []
        # top-k density sweep (50..95 % block sparsity), then threshold mode
        cases = [("density", rho) for rho in (0.5, 0.3, 0.2, 0.1, 0.05)] + \
                [("threshold", t) for t in (1e-4, 5e-4, 2e-3)]
        for mode, val in cases:
            if mode == "density":
                c2 = seer.gate_required_cap(w.B, w.Hq, w.Hkv, w.n, w.d, "density", density=val)
            else:
                c2 = seer.gate_required_cap(w.B, w.Hq, w.Hkv, w.n, w.d, "threshold")
            cc = torch.empty(w.B, w.Hq, nb, dtype=torch.int32, device=dev)
            ii = torch.empty(w.B, w.Hq, nb, c2, dtype=torch.int32, device=dev)
            kw = {"density": val} if mode == "density" else {"T": val}

            def sw_gate():
                seer.seer_gate(Qd, Kd, Wqd, Wkd, mode, cap=c2, workspace=gws, out=(cc, ii, None), **kw)

            def sw_attn():
                seer.seer_sparse_attn(Qd, Kd, Vd, cc, ii, workspace=aws, out=(O, lse))

            sw_gate()
            for _ in range(2):
                sw_attn()
            torch.cuda.synchronize(dev)
            a, b, c = (torch.cuda.Event(enable_timing=True) for _ in range(3))
            a.record(stream)
            for _ in range(3):
                sw_gate()
            b.record(stream)
            for _ in range(3):
                sw_attn()
            c.record(stream)
            torch.cuda.synchronize(dev)
            gms = a.elapsed_time(b) / 3
            ms = b.elapsed_time(c) / 3
            f, nbk, _, sp = attn_flops(cc, ii, w.d)
            sweep.append({mode: val, "sparsity": sp, "active_blocks": nbk, "attn_ms": ms, "gate_ms": gms,
                          "gate_plus_attn_ms": gms + ms, "tflops": f / (ms * 1e-3) / 1e12,
                          "frac_bf16_burst": f / (ms * 1e-3) / 1e12 / pk["bf16_tflops"],
                          "status": seer.seer_workspace_status(aws)})
            del cc, ii
        # time against active tiles over the density sweep: least-squares line and R^2
        pts = [(e["active_blocks"], e["attn_ms"]) for e in sweep if "density" in e]
        xs = np.array([x for x, _ in pts], dtype=np.float64)
        ys = np.array([y for _, y in pts], dtype=np.float64)
        slope, icpt = np.polyfit(xs, ys, 1)
        resid = ys - (slope * xs + icpt)
        r2 = 1.0 - float((resid ** 2).sum() / max(((ys - ys.mean()) ** 2).sum(), 1e-30))
        sweep.append({"fit": "attn_ms = a * active_blocks + b over the density sweep",
                      "a_ms_per_block": float(slope), "b_ms": float(icpt), "r2": r2})

    # ------------------------------------------------------ oracle baseline --
    cpu = None
    if not args.no_cpu_baseline and rank == 0 and world == 1:
        smp = OracleSampler(w, Q, K, V, Wq, Wk, args.density)
        for _ in range(3):
            smp.step(4.0)
        rate, _ = smp.rate(flops)
        cpu = {"value": rate, "unit": "TFLOP/s", "cores": smp.oracle.num_threads(), "kind": "oracle",
               "sample": smp.describe()}

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": f"{args.workload}: B={w.B} Hq={w.Hq} Hkv={w.Hkv} n={w.n} d={w.d} "
                                   f"gate h={w.h}, top-k density {args.density}",
                       "achieved_sparsity": sparsity, "active_blocks": nblocks,
                       "l2": "inputs larger than L2 (Q+K+V = 1.5 GB), no flush",
                       "parallelism": f"replica per GPU (independent layer per rank), {world} GPU(s)"},
            "attn_ms": attn_avg, "gate_ms": gate_avg, "attn_tflops": attn_tflops,
            "attn_pct_bf16_peak": {"burst": attn_tflops / pk["bf16_tflops"],
                                   "sustained": attn_tflops / pk.get("bf16_tflops_sustained", pk["bf16_tflops"]),
                                   "peaks": pk_kind},
            "gate_gbs": gate_bytes / (gate_avg * 1e-3) / 1e9,
            "roofline": {"bound": "tensor", "achieved": attn_tflops, "peak": peak, "unit": "TFLOP/s",
                         "frac": attn_tflops / peak, "traffic": traffic,
                         "kernel": "sparse_attn_kernel", "peak_kind": f"bf16 burst ({pk_kind})",
                         "frac_of_sustained": attn_tflops / pk.get("bf16_tflops_sustained", peak),
                         "algorithmic_flops_per_launch": flops},
            "cpu_baseline": cpu, "e2e": e2e, "clocks": clk,
            "gpu_launches": launches_per_step(w) * args.steps,
            "blockmax": bmax, "decode": dec, "varlen": vl, "tf32": tf, "dense_context": ctx, "sweep": sweep,
            "configs": cfgs,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
