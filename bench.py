#!/usr/bin/env python
"""Benchmark: forward + backward alpha-entmax attention on B200.

One step = entmax_attn_fwd + entmax_attn_bwd (the whole hot path) over one
batch of the workload, inputs resident in HBM.  Prints ONE JSON line (rank 0).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

Workloads (seeded synthetic data, see differentiable_sparse_attention_b200/workloads.py):
  long_sweep      B=1 H=8 D=128 t=4, alpha in {1.5, 2}, N in {65536, 131072}
                  (the default: the long-context sweep whose points span block
                  sparsity from about 0.2 to above 0.6, the regime the metric
                  is about)
  alpha15_4k      B=2 H=16 N=4096 D=64 alpha=1.5 causal, q temperature t in {1, 2, 4}
  sparsemax_16k   B=1 H=16 N=16384 D=128 alpha=2 t=3
  planted_32k     B=1 H=8 N=32768 D=128 alpha=1.5, 32 planted key blocks per head
  dash_router_16k DashAttention stage-0/1 router: B=1, 32 query heads over 8 KV heads,
                  N=16384 D=128, chunks of 64 (256 chunks), gamma=16, alpha=1.5

Multi-GPU (torchrun): every rank runs its own replica of the workload (the
(batch, head) problems are independent: weak scaling, no collective on the
data path); the timed region is bracketed by barriers and the time is the
max over ranks.
"""

from __future__ import annotations

import argparse
import json
import os
import resource
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from differentiable_sparse_attention_b200 import workloads as W  # noqa: E402

# DRAM bytes (read + write) per launch of a kernel from one ncu capture, keyed
# by (sweep point, kernel) and valid only for the kernel code they were taken
# on (hash of the package's csrc/ with comments and white space removed); any
# other code reports traffic as null.  Each figure is dram__bytes_read.sum +
# dram__bytes_write.sum of the timed step's forward launch of that point's own
# workload at full size (a one-pass capture, after the L2 flush).
_TRAFFIC_SRC = "52624589d9a02622"
TRAFFIC = {
    ("long_n65536_alpha1.5_t4", "fwd"): {"bytes": 971897088 + 932220672, "src": _TRAFFIC_SRC},
    ("long_n131072_alpha1.5_t4", "fwd"): {"bytes": 3933710592 + 3003946752, "src": _TRAFFIC_SRC},
    ("long_n65536_alpha2.0_t4", "fwd"): {"bytes": 917617664 + 927312896, "src": _TRAFFIC_SRC},
    ("long_n131072_alpha2.0_t4", "fwd"): {"bytes": 3161120768 + 2982609664, "src": _TRAFFIC_SRC},
    ("alpha1.5_n4096_d64", "fwd"): {"bytes": 51134720 + 16934912, "src": _TRAFFIC_SRC},
}


def _code_only(text: str) -> str:
    """C++ source without comments and blank space: what the compiler sees."""
    import re
    text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
    text = re.sub(r"//[^\n]*", " ", text)
    return " ".join(text.split())


def kernel_source_hash() -> str:
    import glob
    import hashlib
    h = hashlib.sha256()
    for f in sorted(glob.glob(os.path.join(ROOT, "differentiable_sparse_attention_b200", "csrc", "*"))):
        h.update(os.path.basename(f).encode())
        with open(f, encoding="utf-8") as fh:
            h.update(_code_only(fh.read()).encode())
    return h.hexdigest()[:16]


# The two workloads' metrics; every line of an arm, its cpu_baseline and its e2e
# object use the same unit.
METRIC = "fwd+bwd alpha-entmax attn ms/step & effective TFLOP/s vs block sparsity, 1 B200"
UNIT = "effective TFLOP/s (dense-equivalent causal 7*B*H*N^2*D per fwd+bwd step)"
ROUTER_METRIC = "DashAttention stage-1 entmax router ms/call & logit TFLOP/s, 1 B200"
ROUTER_UNIT = "logit TFLOP/s (2*B*Hq*N*C*D per call)"

PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
                  "sm_max_mhz": 1965.0}


# Algorithmic ALU work per score of the forward's passes (lane-ops): running max
# and binning in the histogram pass, the sums of a refinement pass, t, p and the
# packing of the P.V pass.
ALU_OPS_HIST, ALU_OPS_REFINE, ALU_OPS_PV = 8, 6, 3


def max_over_ranks(x: float, device=None) -> float:
    """The maximum of x over the ranks of the default process group (x itself
    without one); the tensor lives on `device` (a CUDA device under NCCL)."""
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_tflops(eff_flop_per_step_per_rank: float, steps: int, world: int,
                     ms_total_max: float) -> float:
    """Weak scaling: every rank runs the full workload, so the job processed
    world x the per-rank work in the slowest rank's time."""
    return eff_flop_per_step_per_rank * steps * world / (ms_total_max * 1e-3) / 1e12


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            return json.load(f), "measured"
    return dict(PEAKS_FALLBACK), "fallback"


def workload_points(name: str):
    if name == "alpha15_4k":
        return [W.ALPHA15_4K.with_(temperature=t) for t in W.ALPHA15_4K_TEMPERATURES]
    if name == "sparsemax_16k":
        return [W.SPARSEMAX_16K]
    if name == "planted_32k":
        return [W.PLANTED_32K]
    if name == "long_sweep":
        return [W.long_sweep_point(n, a) for n, a in W.LONG_SWEEP_POINTS]
    if name.startswith("long_n"):
        n, a = name[len("long_n"):].split("_a")
        return [W.long_sweep_point(int(n), float(a))]
    raise SystemExit(f"unknown workload {name}")


def effective_flops(w) -> float:
    """Dense-equivalent FLOPs of fwd + bwd (FlashAttention convention): forward
    4 N^2 D per head (2 for causal), backward 2.5x the forward."""
    per_head = (7.0 if w.causal else 14.0) * w.N * w.N * w.D
    return per_head * w.B * w.H


def block_sparsity(mask: torch.Tensor, n: int, block: int, causal: bool) -> float:
    """1 - |active blocks| / |visible blocks| (causal: blocks i >= j)."""
    words = mask.to(torch.int64).cpu().numpy() & 0xFFFFFFFF
    tb = (n + block - 1) // block
    active = 0
    for j in range(tb):
        active += int(((words[..., j // 32] >> (j % 32)) & 1).sum())
    per_head = tb * (tb + 1) // 2 if causal else tb * tb
    total = per_head * mask.shape[0] * mask.shape[1]
    return 1.0 - active / total


def visible_blocks(w) -> int:
    """Blocks of the mask a query block can see: B*H*T(T+1)/2 causal, B*H*T^2 not."""
    tb = (w.N + w.block - 1) // w.block
    return w.B * w.H * (tb * (tb + 1) // 2 if w.causal else tb * tb)


def active_blocks(w, sparsity: float) -> int:
    return int(round((1.0 - sparsity) * visible_blocks(w)))


def active_block_fit(rows):
    """Least-squares fit of ms/step = a * visible blocks + b * active blocks over
    the sweep points: a is the time per block of the dense tau passes (every
    visible block), b per active block of the sparse passes (P.V and the
    backward).  None unless the points determine both (two points whose
    active fraction differs)."""
    if len(rows) < 2:
        return None
    A = np.array([[r["visible_blocks"], r["active_blocks"]] for r in rows], dtype=np.float64)
    y = np.array([r["ms_per_step"] for r in rows], dtype=np.float64)
    if (A.max(axis=0) <= 0).any() or np.linalg.matrix_rank(A / A.max(axis=0), tol=1e-3) < 2:
        return None
    (a, b), *_ = np.linalg.lstsq(A, y, rcond=None)
    resid = np.abs(A @ np.array([a, b]) - y) / y
    return {"model": "ms/step = a * visible blocks + b * active blocks",
            "a_us_per_visible_block": round(float(a) * 1e3, 6),
            "b_us_per_active_block": round(float(b) * 1e3, 6),
            "max_rel_residual": round(float(resid.max()), 4), "points": len(rows)}


class ClockSampler:
    """nvidia-smi clocks/throttle reasons sampled every 200 ms while running."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int, out_dir: str = ""):
        self.idx = device_index
        self.proc = None
        self.f = None
        out_dir = (out_dir or os.environ.get("BENCH_CLOCKS_DIR")
                   or os.path.join(ROOT, "bench_clocks"))
        self.path = os.path.join(out_dir, f"clocks_rank{device_index}.csv")

    def __enter__(self):
        try:
            os.makedirs(os.path.dirname(self.path), exist_ok=True)
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.idx), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"], stdout=self.f,
                stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
            if self.f is not None:
                self.f.close()
                self.f = None
            return self
        # wait (up to 3 s) for the first sample so the timed region is covered
        t0 = time.time()
        while time.time() - t0 < 3.0 and os.path.getsize(self.path) == 0:
            time.sleep(0.02)
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            time.sleep(0.25)  # one more sample at the end of the timed region
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            self.f.close()

    def summary(self):
        if self.proc is None or not os.path.exists(self.path):
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax = float(parts[2])
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        return {"sm_mhz": float(np.median(sm)) if sm else None, "sm_max_mhz": smax,
                "samples": len(sm), "reasons": sorted(reasons)}


def run_ours(args, points, rank, world, device):
    import differentiable_sparse_attention_b200 as dsa

    peaks, peaks_kind = load_peaks()
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=device)  # > 126 MB L2
    results = []
    total_eff = 0.0
    total_ms = 0.0
    phase_tot = {n: 0.0 for n in dsa.PHASE_NAMES}
    counters_acc = {}
    e2e_ms = 0.0
    h2d = d2h = 0
    kernel_launches = 0

    for w in points:
        x = W.make_inputs(w, device="cpu")
        dev = {k: v.to(device) for k, v in x.items()}
        B, H, N, D = w.B, w.H, w.N, w.D
        ws = dsa.alloc_workspace(B, H, N, D, w.block, w.causal, device)
        out = torch.empty_like(dev["q"])
        tau = torch.empty((B, H, N), dtype=torch.float32, device=device)
        mask = torch.empty((B, H, (N + w.block - 1) // w.block, dsa.mask_words(N, w.block)),
                           dtype=torch.int32, device=device)
        dq, dk, dv = (torch.empty_like(dev["q"]) for _ in range(3))

        def step(q, k, v, do):
            dsa.entmax_attn_fwd(q, k, v, w.alpha, w.causal, w.block, out=out, tau=tau, mask=mask,
                                workspace=ws)
            dsa.entmax_attn_bwd(q, k, v, do, tau, mask, w.alpha, w.causal, w.block, dq=dq, dk=dk,
                                dv=dv, workspace=ws)

        for _ in range(max(3, args.warmup)):
            step(dev["q"], dev["k"], dev["v"], dev["dout"])
        torch.cuda.synchronize(device)
        st = dsa.status(ws)
        cnt = dsa.counters(ws)
        sparsity = block_sparsity(mask, N, w.block, w.causal)

        # ---- timed region: device-resident inputs, L2 flushed before each step
        dsa.profile(True)
        ev0 = torch.cuda.Event(enable_timing=True)
        ev1 = torch.cuda.Event(enable_timing=True)
        if world > 1:
            torch.distributed.barrier()
        torch.cuda.synchronize(device)
        ms_steps = []
        phases = {n: 0.0 for n in dsa.PHASE_NAMES}
        with ClockSampler(device.index) as clk:
            for _ in range(args.steps):
                flush.zero_()
                ev0.record()
                step(dev["q"], dev["k"], dev["v"], dev["dout"])
                ev1.record()
                ev1.synchronize()
                ms_steps.append(ev0.elapsed_time(ev1))
                for n, v in dsa.profile_read().items():
                    phases[n] += v
        torch.cuda.synchronize(device)
        dsa.profile(False)
        ms_sum = max_over_ranks(sum(ms_steps), device)
        ms_step = ms_sum / args.steps
        eff = effective_flops(w)
        total_eff += eff * args.steps * world
        total_ms += ms_sum
        for n in phases:
            phase_tot[n] += phases[n]
        for n, v in cnt.items():
            counters_acc[n] = counters_acc.get(n, 0) + v
        # our kernels per step: forward (fp16 copy of v + kernel); backward (fp16 copies
        # of q, k, dout + 2 tile-mask kernels + row + column)
        kernel_launches += args.steps * (2 + 3 + 2 + 2)

        # ---- end to end through the public API: pinned host buffers in and out.
        # Every step copies its inputs host -> device and its results device ->
        # host inside the timed region; the copies of neighbouring steps overlap
        # the compute on two copy streams, over two complete buffer sets (inputs,
        # outputs, workspace: their working set exceeds L2).
        e2e = None
        if not args.no_e2e:
            names = ("q", "k", "v", "dout")
            host_in = {k: v.pin_memory() for k, v in x.items()}
            host_out = [torch.empty_like(x["q"]).pin_memory() for _ in range(4)]
            in_bytes = sum(host_in[k].numel() * host_in[k].element_size() for k in names)
            out_bytes = sum(t.numel() * t.element_size() for t in host_out)
            sets = []
            for _ in range(2):
                st_ = {k: torch.empty_like(dev[k]) for k in names}
                st_["out"] = torch.empty_like(dev["q"])
                st_["tau"] = torch.empty((B, H, N), dtype=torch.float32, device=device)
                st_["mask"] = torch.empty_like(mask)
                st_["ws"] = dsa.alloc_workspace(B, H, N, D, w.block, w.causal, device)
                for g_ in ("dq", "dk", "dv"):
                    st_[g_] = torch.empty_like(dev["q"])
                sets.append(st_)

            def run_set(st_):
                dsa.entmax_attn_fwd(st_["q"], st_["k"], st_["v"], w.alpha, w.causal, w.block,
                                    out=st_["out"], tau=st_["tau"], mask=st_["mask"],
                                    workspace=st_["ws"])
                dsa.entmax_attn_bwd(st_["q"], st_["k"], st_["v"], st_["dout"], st_["tau"],
                                    st_["mask"], w.alpha, w.causal, w.block, dq=st_["dq"],
                                    dk=st_["dk"], dv=st_["dv"], workspace=st_["ws"])

            comp = torch.cuda.current_stream(device)
            h2d_s = torch.cuda.Stream(device)
            d2h_s = torch.cuda.Stream(device)
            ev_in = [torch.cuda.Event() for _ in range(2)]
            ev_done = [torch.cuda.Event() for _ in range(2)]
            ev_out = [torch.cuda.Event() for _ in range(2)]
            ev_last = torch.cuda.Event()
            run_set(sets[0])
            run_set(sets[1])
            flush.zero_()
            torch.cuda.synchronize(device)
            if world > 1:
                torch.distributed.barrier()
            ev0.record(comp)
            h2d_s.wait_event(ev0)
            with torch.cuda.stream(h2d_s):
                for kname in names:
                    sets[0][kname].copy_(host_in[kname], non_blocking=True)
                ev_in[0].record(h2d_s)
            for s_ in range(args.steps):
                b = s_ % 2
                if s_ + 1 < args.steps:
                    nb = 1 - b
                    with torch.cuda.stream(h2d_s):
                        if s_ >= 1:
                            h2d_s.wait_event(ev_done[nb])   # step s - 1 is done with set nb
                        for kname in names:
                            sets[nb][kname].copy_(host_in[kname], non_blocking=True)
                        ev_in[nb].record(h2d_s)
                comp.wait_event(ev_in[b])
                if s_ >= 2:
                    comp.wait_event(ev_out[b])   # step s - 2's results have left set b
                run_set(sets[b])
                ev_done[b].record(comp)
                with torch.cuda.stream(d2h_s):
                    d2h_s.wait_event(ev_done[b])
                    for hb, g_ in zip(host_out, ("out", "dq", "dk", "dv")):
                        hb.copy_(sets[b][g_], non_blocking=True)
                    ev_out[b].record(d2h_s)
            ev_last.record(d2h_s)
            comp.wait_event(ev_last)
            ev1.record(comp)
            ev1.synchronize()
            e_sum = max_over_ranks(ev0.elapsed_time(ev1), device)
            e2e_ms += e_sum
            h2d += in_bytes
            d2h += out_bytes
            e2e = e_sum / args.steps
            del sets

        results.append({
            "point": w.name, "temperature": w.temperature, "alpha": w.alpha, "N": N,
            "block": w.block, "block_sparsity": round(sparsity, 4),
            "visible_blocks": visible_blocks(w), "active_blocks": active_blocks(w, sparsity),
            "ms_per_step": round(ms_step, 4),
            "eff_tflops": round(eff / (ms_step * 1e-3) / 1e12 * world, 2),
            "phases_ms": {n: round(v / args.steps, 4) for n, v in phases.items()},
            "counters": cnt, "status": st, "clocks": clk.summary(),
            "e2e_ms_per_step": None if e2e is None else round(e2e, 4)})
        del dev, ws, out, tau, mask, dq, dk, dv
        torch.cuda.empty_cache()

    value = total_eff / (total_ms * 1e-3) / 1e12
    n_steps_all = args.steps * len(points)

    # ---- roofline of the dominant kernel (by total event time)
    dom = max(phase_tot, key=phase_tot.get)
    dom_ms = phase_tot[dom] / n_steps_all
    roof = roofline_for(dom, dom_ms, points, results, peaks, peaks_kind, args.steps)
    src = kernel_source_hash()

    def traffic(point_name, kernel):
        tr = TRAFFIC.get((point_name, kernel))
        if tr is None or args.heads or args.alpha or args.block or tr["src"] != src:
            return None
        return tr["bytes"]

    per_point_traffic = [traffic(r["point"], dom) for r in results]
    if all(t is not None for t in per_point_traffic):
        roof["traffic"] = int(round(sum(per_point_traffic) / len(per_point_traffic)))
    # the same roofline for each sweep point on its own
    for w, r in zip(points, results):
        pk = max(r["phases_ms"], key=r["phases_ms"].get)
        r["roofline"] = roofline_for(pk, r["phases_ms"][pk], [w], [r], peaks, peaks_kind,
                                     args.steps)
        r["roofline"]["traffic"] = traffic(r["point"], pk)

    # the forward's tau passes are bound by the plain ALU pipes, not the tensor
    # cores: the same kernel against 128 lanes x 148 SMs x the clock
    roof_alu = None
    if "fwd" in phase_tot:
        fwd_ms = phase_tot["fwd"] / n_steps_all
        ops = 0.0
        for w, r in zip(points, results):
            c = r["counters"]
            scores = 128.0 * 128.0
            ops += (ALU_OPS_HIST * c["fwd_hist_tiles"] + ALU_OPS_REFINE * c["fwd_refine_tiles"]
                    + ALU_OPS_PV * c["fwd_pv_tiles"]) * scores
        ops /= len(points)
        sm_mhz = peaks.get("sm_max_mhz", 1965.0)
        alu_peak = 128 * 148 * sm_mhz * 1e6 / 1e12     # T lane-ops/s
        achieved = ops / (fwd_ms * 1e-3) / 1e12
        roof_alu = {"bound": "alu", "kernel": "fwd", "achieved": round(achieved, 3),
                    "peak": round(alu_peak, 2), "unit": "T lane-ops/s",
                    "frac": round(achieved / alu_peak, 4),
                    "note": f"{ALU_OPS_HIST} ops per histogram score, {ALU_OPS_REFINE} per "
                            f"refinement score, {ALU_OPS_PV} per P.V score over the tiles the "
                            f"counters report; peak = 128 lanes x 148 SMs x {sm_mhz:g} MHz"}

    line = {
        "metric": METRIC,
        "value": round(value, 3),
        "unit": UNIT,
        "n_gpus": world, "steps": args.steps, "warmup": max(3, args.warmup),
        "ms_per_step": round(total_ms / n_steps_all, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16", "data": "synthetic (seeded N(0,1), see workloads.py)",
        "config": {"workload": args.workload_desc, "l2": "flushed (256 MB write) before every step",
                   "e2e": "host copies of each step overlap the neighbouring steps' compute "
                          "(two copy streams, two buffer sets larger than L2)",
                   "points": [p["point"] for p in results], "parallelism": f"replica x{world}"},
        "sweep": results,
        "kernels_ms_per_step": {n: round(v / n_steps_all, 4) for n, v in phase_tot.items()},
        "roofline": roof,
        "roofline_fwd_alu": roof_alu,
        "gpu_launches": kernel_launches,
        "clocks": merge_clocks([r["clocks"] for r in results]),
    }
    fit = active_block_fit(results)
    if fit is not None:
        line["fit"] = fit
    if not args.no_e2e:
        line["e2e"] = {"value": round(total_eff / (e2e_ms * 1e-3) / 1e12, 3),
                       "unit": line["unit"], "h2d_bytes_per_step": h2d // len(points),
                       "d2h_bytes_per_step": d2h // len(points)}
    return line


def dense_context(args, points, results, device):
    """Dense causal softmax attention, forward + backward, on the same shapes:
    torch's scaled_dot_product_attention (whichever backend it dispatches to) and,
    if it runs on this GPU, the flash_attn package (FlashAttention-2), each timed
    like our step (CUDA events, L2 flushed before each step).  Context for the
    pages' comparison with FlashAttention-2 at high block sparsity: a different
    function (softmax, not entmax), never a parity or speed-up claim."""
    import torch.nn.functional as F
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=device)
    out = []
    for w, r in zip(points, results):
        x = W.make_inputs(w, device="cpu")
        q, k, v, do = (x[n].to(device) for n in ("q", "k", "v", "dout"))
        entry = {"point": w.name, "block_sparsity": r["block_sparsity"],
                 "entmax_ms_per_step": r["ms_per_step"]}

        def timed(fn):
            for _ in range(max(3, args.warmup)):
                fn()
            torch.cuda.synchronize(device)
            ev0 = torch.cuda.Event(enable_timing=True)
            ev1 = torch.cuda.Event(enable_timing=True)
            tot = 0.0
            for _ in range(args.steps):
                flush.zero_()
                ev0.record()
                fn()
                ev1.record()
                ev1.synchronize()
                tot += ev0.elapsed_time(ev1)
            return round(tot / args.steps, 4)

        qs, ks, vs = (t.detach().clone().requires_grad_(True) for t in (q, k, v))

        def sdpa_step():
            o = F.scaled_dot_product_attention(qs, ks, vs, is_causal=True)
            o.backward(do)
        try:
            entry["sdpa_ms_per_step"] = timed(sdpa_step)
        except Exception as e:  # noqa: BLE001 - context only
            entry["sdpa_ms_per_step"] = None
            entry["sdpa_error"] = str(e).splitlines()[0][:200]
        del qs, ks, vs
        try:
            from flash_attn import flash_attn_func
            qf, kf, vf = (t.transpose(1, 2).contiguous().requires_grad_(True) for t in (q, k, v))
            dof = do.transpose(1, 2).contiguous()

            def fa2_step():
                o = flash_attn_func(qf, kf, vf, causal=True)
                o.backward(dof)
            entry["flash_attn2_ms_per_step"] = timed(fa2_step)
            del qf, kf, vf, dof
        except Exception as e:  # noqa: BLE001 - context only
            entry["flash_attn2_ms_per_step"] = None
            entry["flash_attn2_error"] = str(e).splitlines()[0][:200]
        out.append(entry)
        del q, k, v, do
        torch.cuda.empty_cache()
    return {"note": "dense causal softmax attention fwd+bwd on the same shapes (bf16): a "
                    "different function, timed as context for the pages' comparison only",
            "points": out}


def merge_clocks(cl):
    sm = [c["sm_mhz"] for c in cl if c.get("sm_mhz")]
    reasons = sorted({r for c in cl for r in c.get("reasons", [])})
    smax = next((c["sm_max_mhz"] for c in cl if c.get("sm_max_mhz")), None)
    return {"sm_mhz": float(np.median(sm)) if sm else None, "sm_max_mhz": smax, "reasons": reasons}


def roofline_for(kernel, ms, points, results, peaks, peaks_kind, steps):
    """Achieved vs peak for the dominant kernel.  Tensor-bound kernels count the
    MMA FLOPs their tile lists imply (128 x 128 tiles):
      forward:   (hist + refine tiles) * 2*128*128*D + pv tiles * 3 * 2*128*128*D
                 (S, P.V, G.V)
      bwd row:   row tiles * 3 * 2*128*128*D                    (S, dP, dQ)
      bwd col:   col tiles * 5 * 2*128*128*D      (S^T, dP^T, dV, and dK from the
                 hi and the lo fp16 part of dS^T)
    """
    fl = 0.0
    for w, r in zip(points, results):
        c = r["counters"]
        unit = 2.0 * 128 * 128 * w.D
        if kernel == "fwd":
            fl += ((c["fwd_hist_tiles"] + c["fwd_refine_tiles"]) + 3 * c["fwd_pv_tiles"]) * unit
        elif kernel == "bwd_row":
            fl += c["bwd_row_tiles"] * 3 * unit
        elif kernel == "bwd_col":
            fl += c["bwd_col_tiles"] * 5 * unit
    fl /= len(points)
    if fl == 0.0:
        return {"bound": "hbm", "kernel": kernel, "achieved": None, "peak": peaks["hbm_gbs"],
                "unit": "GB/s", "frac": None, "traffic": None,
                "note": f"peak {peaks_kind}"}
    achieved = fl / (ms * 1e-3) / 1e12
    peak = peaks["bf16_tflops"]
    return {"bound": "tensor", "kernel": kernel, "achieved": round(achieved, 2),
            "peak": peak, "unit": "TFLOP/s", "frac": round(achieved / peak, 4), "traffic": None,
            "ms_per_launch": round(ms, 4),
            "note": f"executed MMA FLOPs per launch / CUDA-event duration; peak = {peaks_kind} "
                    "dense bf16 burst (fp16 runs at the same rate)"}


# ---------------------------------------------------------------- oracle legs
def oracle_rows(n: int, budget: int) -> int:
    """Query rows of a bounded oracle sample: about ``budget`` scores in all
    (rows x keys), at least 32 rows and at most n."""
    return int(min(n, max(32, budget // n)))


def blas_threads():
    """Threads of the BLAS library numpy calls into (None if unknown)."""
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads") for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else None
    except Exception:  # noqa: BLE001 - optional diagnostics only
        return None


def oracle_sample(w, n_rows: int):
    """Time the float64 oracle on n_rows query rows, spread evenly over
    (batch 0, head 0) of workload w: forward for those rows, then their
    backward (dQ rows and their dK/dV contributions) reusing the forward's tau.
    Returns (effective FLOP of the sample, wall seconds, measured parallelism
    = CPU seconds / wall seconds, rows).  A causal row sees on average N/2
    keys, so the sample's dense-equivalent work is the head's 7 N^2 D scaled by
    n_rows / N."""
    import oracle as O

    x = W.make_inputs(w.with_(B=1, H=1), device="cpu")
    q, k, v, do = (W.head_slice(x[n], 0, 0) for n in ("q", "k", "v", "dout"))
    n_rows = min(n_rows, w.N)
    rows = np.unique(np.linspace(0, w.N - 1, n_rows).round().astype(np.int64))
    r0 = resource.getrusage(resource.RUSAGE_SELF)
    t0 = time.perf_counter()
    f = O.attention_forward(q, k, v, w.alpha, w.causal, w.block, rows=rows)
    O.attention_backward(q, k, v, do, w.alpha, w.causal, rows=rows, tau=f["tau"])
    wall = time.perf_counter() - t0
    r1 = resource.getrusage(resource.RUSAGE_SELF)
    cpu = (r1.ru_utime - r0.ru_utime) + (r1.ru_stime - r0.ru_stime)
    eff = effective_flops(w.with_(B=1, H=1)) * rows.size / w.N
    return eff, wall, round(cpu / max(wall, 1e-9), 2), rows.size


def cpu_baseline(points):
    w = points[0]
    eff, wall, par, nr = oracle_sample(w, oracle_rows(w.N, 1 << 26))
    return {"value": round(eff / wall / 1e12, 8), "unit": UNIT, "cores": os.cpu_count(),
            "blas_threads": blas_threads(), "parallelism_measured": par,
            "kind": "oracle", "sample": f"{w.name} t={w.temperature}: {nr} of {w.N} query rows "
            f"(evenly spread) of batch 0 head 0 (1 of {w.B * w.H} heads), fwd+bwd in float64 "
            f"NumPy, {wall:.1f} s wall; cores = os.cpu_count() of the host, BLAS threads as "
            f"numpy reports them, parallelism = CPU seconds / wall seconds"}


def run_reference(args, points, rank, world):
    """The oracle as it stands, timed on the host cores: every step is a bounded
    sample (about 2^24 scores: 256 evenly spread query rows of batch 0 head 0
    up to N = 65536, 128 at 131072) of one sweep point, cycling through the
    points."""
    if rank != 0:
        return None
    total_eff = 0.0
    total_s = 0.0
    par = 1.0
    samples = []
    for i in range(args.steps):
        w = points[i % len(points)]
        eff, wall, par, nr = oracle_sample(w, min(256, oracle_rows(w.N, 1 << 24)))
        total_eff += eff
        total_s += wall
        samples.append(f"{w.name} t={w.temperature} ({nr} rows)")
    value = total_eff / total_s / 1e12
    return {
        "impl": "reference",
        "metric": METRIC,
        "value": round(value, 8),
        "unit": UNIT,
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(total_s * 1e3 / args.steps, 2), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": args.workload_desc,
                   "sample": "each step = up to 256 evenly spread query rows (about 2^24 "
                             "scores) of batch 0 head 0 of one sweep point, fwd+bwd through "
                             "the float64 oracle on host cores"},
        "cpu_baseline": {"value": round(value, 8), "unit": UNIT, "cores": os.cpu_count(),
                         "blas_threads": blas_threads(), "parallelism_measured": par,
                         "kind": "oracle", "sample": "; ".join(samples)},
        "e2e": {"value": round(value, 8), "unit": UNIT, "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


ROUTER = dict(B=1, Hq=32, Hkv=8, N=16384, D=128, chunk=64, gamma=16.0, alpha=1.5, seed=0)


def run_router(args, rank, world, device):
    """One step = dash_route on seeded N(0,1) bf16 q and k of the router
    workload.  value = logit FLOPs (2 B Hq N C D, one GEMM) per second; the
    roofline counts the MMAs the kernel issues (two fp16 parts of the chunk
    summaries over 128-row and 128-chunk tiles) against the call's event time,
    which also covers the fp16 copy of q and the chunk means."""
    import differentiable_sparse_attention_b200 as dsa

    w = dict(ROUTER)
    if args.alpha:
        w["alpha"] = args.alpha
    peaks, peaks_kind = load_peaks()
    g = torch.Generator().manual_seed(w["seed"])
    qh = torch.randn((w["B"], w["Hq"], w["N"], w["D"]), generator=g).to(torch.bfloat16)
    kh = torch.randn((w["B"], w["Hkv"], w["N"], w["D"]), generator=g).to(torch.bfloat16)
    q, k = qh.to(device), kh.to(device)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=device)
    step = lambda: dsa.dash_route(q, k, w["chunk"], w["gamma"], w["alpha"])
    for _ in range(max(3, args.warmup)):
        res = step()
    torch.cuda.synchronize(device)
    st = dsa.status(res.workspace)
    C = w["N"] // w["chunk"]
    active = res.wbar > 0
    density = float(active[..., w["chunk"]:, :].float().mean().item())
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize(device)
    ms = []
    with ClockSampler(device.index) as clk:
        for _ in range(args.steps):
            flush.zero_()
            ev0.record()
            res = step()
            ev1.record()
            ev1.synchronize()
            ms.append(ev0.elapsed_time(ev1))
    ms_sum = max_over_ranks(sum(ms), device)
    ms_step = ms_sum / args.steps
    logit_flop = 2.0 * w["B"] * w["Hq"] * w["N"] * C * w["D"]
    value = logit_flop * world / (ms_step * 1e-3) / 1e12
    tr = (w["N"] + 127) // 128
    cp = (C + 127) // 128 * 128
    mma_flop = 2 * 2.0 * w["B"] * w["Hq"] * tr * 128 * cp * w["D"]
    achieved = mma_flop / (ms_step * 1e-3) / 1e12
    line = {
        "metric": ROUTER_METRIC,
        "value": round(value, 3), "unit": ROUTER_UNIT,
        "n_gpus": world, "steps": args.steps, "warmup": max(3, args.warmup),
        "ms_per_step": round(ms_step, 4), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded N(0,1) q, k)",
        "config": {"workload": "dash_router_16k: " + ", ".join(f"{a}={b}" for a, b in w.items()),
                   "l2": "flushed (256 MB write) before every step",
                   "parallelism": f"replica x{world}"},
        "chunk_density": round(density, 4), "status": st,
        "roofline": {"bound": "tensor", "kernel": "dash_route (whole call)",
                     "achieved": round(achieved, 2), "peak": peaks["bf16_tflops"],
                     "unit": "TFLOP/s", "frac": round(achieved / peaks["bf16_tflops"], 4),
                     "traffic": None,
                     "note": f"issued MMA FLOPs / call time (fp16 copy of q and chunk means "
                             f"included); peak = {peaks_kind} dense bf16 burst"},
        "gpu_launches": 3 * args.steps,
        "clocks": clk.summary(),
    }
    return line


def run_router_reference(args, world):
    """The router oracle on the host cores: each step routes 128 evenly spread
    query rows of KV head 0 (its 4 query heads) of the router workload."""
    from oracle import dash_router as R

    w = dict(ROUTER)
    if args.alpha:
        w["alpha"] = args.alpha
    g = torch.Generator().manual_seed(w["seed"])
    qh = torch.randn((w["B"], w["Hq"], w["N"], w["D"]), generator=g).to(torch.bfloat16)
    kh = torch.randn((w["B"], w["Hkv"], w["N"], w["D"]), generator=g).to(torch.bfloat16)
    G = w["Hq"] // w["Hkv"]
    q64 = qh[0, :G].double().numpy()
    k64 = kh[0, :1].double().numpy()
    rows = np.unique(np.linspace(0, w["N"] - 1, 128).round().astype(np.int64))
    C = w["N"] // w["chunk"]
    r0 = resource.getrusage(resource.RUSAGE_SELF)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        R.route(q64, k64, w["alpha"], w["gamma"], w["chunk"], rows=rows)
    wall = time.perf_counter() - t0
    r1 = resource.getrusage(resource.RUSAGE_SELF)
    par = round(((r1.ru_utime - r0.ru_utime) + (r1.ru_stime - r0.ru_stime)) / wall, 2)
    flop = 2.0 * G * rows.size * C * w["D"] * args.steps
    value = flop / wall / 1e12
    sample = (f"{rows.size} evenly spread rows x {G} query heads of KV head 0 per step "
              f"({args.steps} steps, {wall:.1f} s)")
    return {"impl": "reference",
            "metric": ROUTER_METRIC,
            "value": round(value, 8), "unit": ROUTER_UNIT,
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(wall * 1e3 / args.steps, 2), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": "dash_router_16k (oracle sample)", "sample": sample},
            "cpu_baseline": {"value": round(value, 8), "unit": ROUTER_UNIT,
                             "cores": os.cpu_count(), "blas_threads": blas_threads(),
                             "parallelism_measured": par, "kind": "oracle", "sample": sample},
            "e2e": {"value": round(value, 8), "unit": ROUTER_UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", default="long_sweep")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--heads", type=int, default=0,
                    help="override H (small cases for profiler captures)")
    ap.add_argument("--alpha", type=float, default=0.0,
                    help="override alpha (any value in [1.05, 3]; 1.5 and 2 have closed forms)")
    ap.add_argument("--block", type=int, default=0, choices=[0, 64, 128],
                    help="override the mask block size (the sparsity is then reported at it)")
    ap.add_argument("--dense-context", action="store_true",
                    help="also time dense causal softmax attention (torch SDPA, flash_attn) "
                         "on the same shapes, as context")
    args = ap.parse_args()
    if args.workload == "dash_router_16k":
        world = int(os.environ.get("WORLD_SIZE", "1"))
        rank = int(os.environ.get("RANK", "0"))
        if args.impl == "reference":
            if rank == 0:
                print(json.dumps(run_router_reference(args, world)))
            return
        device = torch.device("cuda", int(os.environ.get("LOCAL_RANK", "0")))
        torch.cuda.set_device(device)
        if world > 1:
            import datetime
            torch.distributed.init_process_group("nccl", device_id=device,
                                                 timeout=datetime.timedelta(seconds=120))
        line = run_router(args, rank, world, device)
        if rank == 0:
            print(json.dumps(line))
        if world > 1:
            torch.distributed.barrier()
            torch.distributed.destroy_process_group()
        return
    points = workload_points(args.workload)
    if args.heads:
        points = [p.with_(H=args.heads) for p in points]
    if args.alpha:
        points = [p.with_(alpha=args.alpha, name=f"{p.name}_as_alpha{args.alpha:g}") for p in points]
    if args.block:
        points = [p.with_(block=args.block) for p in points]
    args.workload_desc = (f"{args.workload}: " + ", ".join(
        f"B={p.B} H={p.H} N={p.N} D={p.D} alpha={p.alpha} t={p.temperature}"
        + (f" planted={p.planted_blocks}" if p.planted_blocks else "") for p in points)
        + f"; causal, block {points[0].block}, bf16")

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        line = run_reference(args, points, rank, world)
        if line is not None:
            print(json.dumps(line))
        return

    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    if world > 1:
        import datetime
        torch.distributed.init_process_group("nccl", device_id=device,
                                             timeout=datetime.timedelta(seconds=120))
    line = run_ours(args, points, rank, world, device)
    if rank == 0:
        if args.dense_context and world == 1:
            line["dense_context"] = dense_context(args, points, line["sweep"], device)
        if not args.no_cpu_baseline and world == 1:
            line["cpu_baseline"] = cpu_baseline(points)
        print(json.dumps(line))
    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
