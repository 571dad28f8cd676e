"""Host-side pieces of bench.py: the traffic models and the link to the committed ncu summaries (CPU only)."""

import os
import sys

import numpy as np

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
import bench  # noqa: E402
from synth import GDN_B256, MAMBA2_120B, SPEC_MAMBA2_B512  # noqa: E402


def test_step_traffic_model_window():
    """Over a window, the checkpoint is read every step and written once; records are read count times."""
    wl = MAMBA2_120B
    L, state = wl.window, wl.batch * wl.nheads * wl.headdim * wl.dstate * 4
    parts = [bench.traffic_model(wl, c) for c in range(L)]
    assert sum(p["state_read"] for p in parts) == L * state
    assert sum(p["state_write"] for p in parts) == state
    rec = parts[1]["ring_read"]
    assert sum(p["ring_read"] for p in parts) == rec * L * (L - 1) // 2


def test_verify_traffic_no_fold_and_fold():
    """With T + count <= L nothing folds: every round reads the checkpoint once.  Accepting T every round
    with L = 2T makes every second round pre-fold (one extra state write per sequence)."""
    wl = SPEC_MAMBA2_B512.replace(batch=4, nheads=2, ngroups=1, window=8)
    state = wl.nheads * wl.headdim * wl.dstate * 4
    zero = [np.zeros(wl.batch, np.int32)] * 3
    base = bench.verify_traffic(wl, 4, zero)
    full = [np.full(wl.batch, 4, np.int32)] * 4
    folded = bench.verify_traffic(wl, 4, full)
    esz = 2
    rec = wl.nheads * wl.headdim * esz + wl.ngroups * wl.dstate * esz + wl.nheads * 4
    per_round_fixed = wl.batch * state + wl.batch * 4 * (
        (wl.nheads * wl.headdim * esz + 2 * wl.ngroups * wl.dstate * esz + wl.nheads * esz) + rec + wl.nheads * wl.headdim * 4)
    assert base == 3 * per_round_fixed
    # counts before the rounds: 0, 4, 8 (pre-fold: 8 + 4 > 8), 4 -> one fold; buffered reads 0 + 4 + 8 + 4
    assert folded == 4 * per_round_fixed + wl.batch * state + wl.batch * rec * (0 + 4 + 8 + 4)


def test_gdn_traffic_model_window():
    wl = GDN_B256
    state = wl.batch * wl.nheads * wl.dv * wl.dk * 4
    tot = sum(bench.gdn_traffic(wl, c) for c in range(wl.window))
    assert tot > (wl.window + 1) * state
    assert tot < (wl.window + 1) * state * 1.2


def test_gdn_traffic_by_format():
    """Plain steps read the checkpoint in its own format, or the NVFP4 copy; a fold reads the checkpoint and
    writes it and the copy.  E4M3 is a quarter of fp32 plus one fp32 scale per 64 x 128 tile."""
    wl = GDN_B256
    elems = wl.batch * wl.nheads * wl.dv * wl.dk
    rest = bench.gdn_traffic(wl, 3) - elems * 4
    assert bench.gdn_traffic(wl, 3, "f8sr", "same") == rest + elems + elems // (64 * 128) * 4
    assert bench.gdn_traffic(wl, 3, "f16sr", "nvfp4") == rest + elems * (0.5 + 1 / 16) + elems // (64 * 128) * 4
    fold = wl.window - 1
    rest_f = bench.gdn_traffic(wl, fold) - 2 * elems * 4
    f8 = elems + elems // (64 * 128) * 4
    fp4 = elems * (0.5 + 1 / 16) + elems // (64 * 128) * 4
    assert bench.gdn_traffic(wl, fold, "f8sr", "nvfp4") == rest_f + 2 * f8 + fp4
    assert bench.gdn_traffic(wl, fold, "f32", "shared_nvfp4") == rest_f + 2 * fp4


def test_committed_profile_matches_kernel_source():
    """The committed ncu summary of the headline kernel was taken on the present kernel code, so the bench
    line reports its measured DRAM traffic (a kernel change without a new capture fails here)."""
    t = bench.profiled_traffic("m2_replay_kernel__mamba2_b256_L16.md", ("mamba2.cu", "common.cuh", "kernels.h"))
    assert t is not None
    model = sum(sum(bench.traffic_model(MAMBA2_120B, c).values()) for c in range(MAMBA2_120B.window)) / 16
    assert 0.9 * model < t < 1.1 * model


def test_both_arms_report_the_same_layer_shape():
    """The GPU arm and the oracle reference arm time the same layer shape; the reference arm's config says how
    many of the sequences it samples, and carries no replica or batch fields of the GPU arm."""
    one, four = bench.arm_config(1), bench.arm_config(4)
    assert one["global_batch"] == 256 and four["global_batch"] == 1024
    ref = bench.reference_config(12)
    shape = ("nheads", "headdim", "dstate", "ngroups", "window")
    assert {k: ref[k] for k in shape} == {k: one[k] for k in shape} == {k: four[k] for k in shape}
    assert ref["sampled_sequences"] == 12 and "12 of the 256 sequences" in ref["workload"]
    assert not {"parallelism", "global_batch", "batch_per_gpu"} & set(ref)


def test_clock_window_uses_neighbouring_samples():
    """A timed region shorter than the sampling period is described by the samples just before and after it."""
    c = bench.ClockSampler("0")
    line = "0, {sm}, 1965, 700, 0x0, Not Active, Not Active, Not Active, {cap}"
    c.samples = [(1.0, line.format(sm=1800, cap="Not Active")), (2.0, line.format(sm=1900, cap="Active")),
                 (3.0, line.format(sm=1950, cap="Not Active")), (4.0, line.format(sm=1000, cap="Not Active"))]
    c.t0, c.t1 = 2.2, 2.3
    s = c.summary()
    assert s["samples"] == 2 and s["sm_mhz"] == 1925 and s["reasons"] == ["sw_power_cap"]
    c.t0, c.t1 = 0.5, 0.6                      # region before the first sample: the first sample stands for it
    assert bench.ClockSampler.summary(c)["samples"] == 1


def test_host_workers_bounds():
    assert bench.host_workers(1) == 1
    assert 1 <= bench.host_workers(1000) <= 32
