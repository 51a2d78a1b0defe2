"""bench.py's host-side arithmetic and the reference arm's JSON line, on CPU, and a
static check of the code that only runs on a GPU.

These cover what the numbers in bench.py's line are made of:
- the dense-equivalent FLOP convention;
- block sparsity read from the bit-packed mask;
- the MMA FLOPs that the tile counters imply for each kernel's roofline;
- the comment-insensitive hash that keys the measured DRAM traffic;
- the fields of the reference arm (the oracle on the host cores);
- the clock summary whose throttle reasons decide whether a run is kept.
"""

import os
import sys

import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from differentiable_sparse_attention_b200 import workloads as W  # noqa: E402


def test_effective_flops_convention():
    # forward 4 N^2 D per head (halved when causal), backward 2.5 x the forward
    w = W.ALPHA15_4K
    assert bench.effective_flops(w) == 7.0 * 2 * 16 * 4096 * 4096 * 64
    assert bench.effective_flops(w.with_(causal=False)) == 2 * bench.effective_flops(w)


def _mask(B, H, tb, rows):
    """int32 mask words [B, H, tb, ceil(tb / 32)] with the given (i, j) bits set
    in every head."""
    words = (tb + 31) // 32
    m = torch.zeros((B, H, tb, words), dtype=torch.int64)
    for i, j in rows:
        m[..., i, j // 32] |= 1 << (j % 32)
    # the library stores uint32 bit patterns in int32 tensors
    return torch.where(m >= 2**31, m - 2**32, m).to(torch.int32)


def test_block_sparsity_causal_counts_lower_triangle():
    tb = 32                                   # N = 4096, block 128: one word per row
    full = [(i, j) for i in range(tb) for j in range(i + 1)]
    assert bench.block_sparsity(_mask(1, 2, tb, full), 4096, 128, True) == 0.0
    # only the diagonal: tb active of tb (tb + 1) / 2 visible blocks
    diag = [(i, i) for i in range(tb)]
    got = bench.block_sparsity(_mask(1, 2, tb, diag), 4096, 128, True)
    assert got == pytest.approx(1.0 - tb / (tb * (tb + 1) / 2))


def test_block_sparsity_reads_bit_31_and_second_word():
    # block 31 sits in the sign bit of word 0; block 32 opens word 1
    tb = 40
    m = _mask(1, 1, tb, [(39, 31), (39, 32)])
    assert int(m[0, 0, 39, 0]) < 0
    got = bench.block_sparsity(m, 40 * 64, 64, False)
    assert got == pytest.approx(1.0 - 2 / (tb * tb))


def _result(**counters):
    base = dict(fwd_hist_tiles=0, fwd_refine_tiles=0, fwd_pv_tiles=0,
                bwd_row_tiles=0, bwd_col_tiles=0)
    base.update(counters)
    return {"counters": base}


def test_roofline_counts_the_mma_flops_of_each_kernel():
    peaks = {"bf16_tflops": 1000.0, "hbm_gbs": 7000.0}
    w = W.ALPHA15_4K                                  # D = 64
    unit = 2.0 * 128 * 128 * 64
    r = _result(fwd_hist_tiles=10, fwd_refine_tiles=2, fwd_pv_tiles=5,
                bwd_row_tiles=7, bwd_col_tiles=9)
    # forward: S per histogram or refinement tile; S, P.V and G.V per P.V tile
    f = bench.roofline_for("fwd", 1.0, [w], [r], peaks, "measured", 1)
    assert f["bound"] == "tensor"
    assert f["achieved"] == pytest.approx(round((12 + 3 * 5) * unit / 1e-3 / 1e12, 2))
    assert f["frac"] == pytest.approx(round(f["achieved"] / 1000.0, 4), abs=1e-4)
    # backward: 3 MMAs per row tile (S, dP, dQ), 5 per column tile (S^T, dP^T, dV and
    # dK from the two fp16 parts of dS^T)
    b = bench.roofline_for("bwd_row", 2.0, [w], [r], peaks, "measured", 1)
    assert b["achieved"] == pytest.approx(round(7 * 3 * unit / 2e-3 / 1e12, 2))
    c = bench.roofline_for("bwd_col", 2.0, [w], [r], peaks, "measured", 1)
    assert c["achieved"] == pytest.approx(round(9 * 5 * unit / 2e-3 / 1e12, 2))
    # points are averaged: two identical points give the same per-launch figure
    f2 = bench.roofline_for("fwd", 1.0, [w, w], [r, r], peaks, "measured", 1)
    assert f2["achieved"] == f["achieved"]


def test_roofline_without_mma_work_is_memory_bound():
    peaks = {"bf16_tflops": 1000.0, "hbm_gbs": 7000.0}
    h = bench.roofline_for("bwd_fp16_copies", 0.03, [W.ALPHA15_4K], [_result()], peaks,
                           "fallback", 1)
    assert h["bound"] == "hbm" and h["peak"] == 7000.0 and h["achieved"] is None


def test_source_hash_ignores_comments_only():
    a = "int f(int x) {  // the answer\n  return x + 1; /* add one */ }\n"
    b = "int f(int x) {\n/* a longer\n   comment */ return x + 1; }  // trailing\n"
    c = "int f(int x) { return x + 2; }"
    assert bench._code_only(a) == bench._code_only(b) == "int f(int x) { return x + 1; }"
    assert bench._code_only(c) != bench._code_only(a)
    h = bench.kernel_source_hash()
    assert len(h) == 16 and int(h, 16) >= 0


def test_reference_arm_line():
    class A:
        steps = 2
        warmup = 3
        workload_desc = "tiny"
    line = bench.run_reference(A, [W.TINY_FP32.with_(N=96)], 0, 1)
    assert line["impl"] == "reference" and line["dtype"] == "f64"
    assert line["value"] > 0 and line["higher_is_better"] is True
    cb = line["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == line["value"]
    assert "rows" in cb["sample"]
    e2e = line["e2e"]
    assert e2e["value"] == line["value"]
    assert e2e["h2d_bytes_per_step"] == 0 and e2e["d2h_bytes_per_step"] == 0
    # one metric and one unit for the line, its cpu_baseline and its e2e, the same
    # as the GPU arm's
    assert line["metric"] == bench.METRIC
    assert line["unit"] == cb["unit"] == e2e["unit"] == bench.UNIT
    assert line["config"]["workload"] == "tiny"
    # the other ranks do no work
    assert bench.run_reference(A, [W.TINY_FP32.with_(N=96)], 1, 2) is None


def test_clock_summary_median_and_throttle_reasons(tmp_path):
    cs = bench.ClockSampler(0, out_dir=str(tmp_path))
    rows = [
        "0, 1965, 1965, 700.1, 0x0000000000000000, Not Active, Not Active, Not Active, Not Active",
        "0, 1900, 1965, 990.0, 0x0000000000000004, Not Active, Not Active, Not Active, Active",
        "0, 1950, 1965, 800.0, 0x0000000000000000, Not Active, Not Active, Not Active, Not Active",
        "0, [N/A], 1965, [N/A], [N/A], [N/A], [N/A], [N/A], [N/A]",
    ]
    with open(cs.path, "w") as f:
        f.write("\n".join(rows) + "\n")
    cs.proc = object()     # as if nvidia-smi had run
    s = cs.summary()
    assert s["sm_mhz"] == 1950.0 and s["sm_max_mhz"] == 1965.0 and s["samples"] == 3
    assert s["reasons"] == ["sw_power_cap"]


def test_clock_sampler_without_nvidia_smi(tmp_path, monkeypatch):
    monkeypatch.setenv("PATH", str(tmp_path))          # no nvidia-smi on the path
    with bench.ClockSampler(0, out_dir=str(tmp_path / "clocks")) as cs:
        pass
    assert cs.proc is None and cs.f is None
    assert cs.summary()["reasons"] == ["nvidia-smi unavailable"]


def test_reference_arm_as_the_driver_runs_it():
    import json
    import subprocess
    run = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                          "--steps", "1", "--warmup", "3"],
                         capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert run.returncode == 0, run.stderr[-2000:]
    lines = [ln for ln in run.stdout.splitlines() if ln.strip()]
    assert len(lines) == 1
    line = json.loads(lines[0])
    assert line["impl"] == "reference" and line["steps"] == 1 and line["warmup"] == 3
    assert line["metric"] == bench.METRIC and line["unit"] == bench.UNIT
    assert line["config"]["workload"].startswith("long_sweep")
    cb = line["cpu_baseline"]
    assert cb["cores"] == os.cpu_count() and cb["parallelism_measured"] > 0


def test_cpu_baseline_of_the_gpu_arm_uses_the_line_unit():
    cb = bench.cpu_baseline([W.TINY_FP32.with_(N=96)])
    assert cb["unit"] == bench.UNIT and cb["kind"] == "oracle" and cb["value"] > 0
    assert cb["cores"] == os.cpu_count() and cb["parallelism_measured"] > 0


def test_oracle_sample_rows_are_bounded():
    # about 2^26 scores for the GPU arm's baseline, never more rows than N
    assert bench.oracle_rows(4096, 1 << 26) == 4096
    assert bench.oracle_rows(65536, 1 << 26) == 1024
    assert bench.oracle_rows(131072, 1 << 26) == 512
    assert bench.oracle_rows(131072, 1 << 24) == 128
    assert bench.oracle_rows(96, 1 << 26) == 96


def _gpu_only_sources():
    import glob
    files = [os.path.join(ROOT, "bench.py"), os.path.join(ROOT, "__graft_entry__.py"),
             os.path.join(ROOT, "differentiable_sparse_attention_b200", "__init__.py")]
    files += sorted(glob.glob(os.path.join(ROOT, "tests", "test_*_gpu.py")))
    files += [os.path.join(ROOT, "tests", "parity.py")]
    return files


@pytest.mark.parametrize("path", _gpu_only_sources(), ids=os.path.basename)
def test_every_global_name_resolves(path):
    """Parts of these files run only on a GPU (bench.py's timed legs, smoke(),
    the binding's CUDA calls, the GPU tests); check statically that every
    global name their functions read is defined at module level or built in,
    so that a misspelt name cannot first show up there."""
    import builtins
    import symtable

    with open(path) as f:
        top = symtable.symtable(f.read(), path, "exec")
    defined = {s.get_name() for s in top.get_symbols()
               if s.is_assigned() or s.is_imported() or s.is_namespace()}

    def scopes(t):
        yield t
        for c in t.get_children():
            yield from scopes(c)

    missing = set()
    for t in scopes(top):
        if str(t.get_type()).lower().split(".")[-1] != "function":
            continue
        for sym in t.get_symbols():
            if sym.is_global() and sym.is_referenced():
                name = sym.get_name()
                if name not in defined and not hasattr(builtins, name):
                    missing.add((t.get_name(), name))
    assert missing == set()


def test_block_counts_of_a_point():
    w = W.ALPHA15_4K                                    # 32 x 32 blocks of 128, causal
    assert bench.visible_blocks(w) == 2 * 16 * 32 * 33 // 2
    assert bench.visible_blocks(w.with_(causal=False)) == 2 * 16 * 32 * 32
    assert bench.active_blocks(w, 0.0) == bench.visible_blocks(w)
    assert bench.active_blocks(w, 0.25) == round(0.75 * bench.visible_blocks(w))


def test_active_block_fit():
    def row(w, sparsity, a_us, b_us):
        vis, act = bench.visible_blocks(w), bench.active_blocks(w, sparsity)
        return {"visible_blocks": vis, "active_blocks": act,
                "ms_per_step": (a_us * vis + b_us * act) * 1e-3}
    long64 = W.long_sweep_point(65536, 1.5)
    long128 = W.long_sweep_point(131072, 1.5)
    rows = [row(long64, 0.19, 0.02, 0.05), row(long128, 0.55, 0.02, 0.05),
            row(W.PLANTED_32K, 0.876, 0.02, 0.05)]
    fit = bench.active_block_fit(rows)
    assert fit["a_us_per_visible_block"] == pytest.approx(0.02, rel=1e-4)
    assert fit["b_us_per_active_block"] == pytest.approx(0.05, rel=1e-4)
    assert fit["max_rel_residual"] < 1e-4 and fit["points"] == 3
    # every point at the same active fraction (the 4K sweep at sparsity 0): a and
    # b cannot be told apart
    w = W.ALPHA15_4K
    assert bench.active_block_fit([row(w, 0.0, 0.02, 0.05)] * 3) is None
    assert bench.active_block_fit([row(long64, 0.19, 0.02, 0.05)]) is None
