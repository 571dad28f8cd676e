"""Benchmark: ReplaySSM Mamba-2 decode on B200, batch 256, L = 16 (the 120B-class layer).

One step = one decode token for every sequence of the layer (batch 256, 128
heads, P 64, N 128, 8 groups, bf16 inputs, fp32 checkpoint of 1 GiB), i.e. one
launch of the replay kernel; every 16th step folds the window into a new
checkpoint.  The timed region is whole steps on the device with the inputs
already resident (a pool of distinct seeded token inputs, cycled); the
checkpoint stream (1 GiB per step) is larger than L2, so no flush is needed.

Printed (one JSON line, rank 0): tokens/s of replay decode, the conventional
step-by-step kernel on the same layer (reads and writes the state every token)
for comparison, the roofline of the replay kernel against the measured HBM
bandwidth, an end-to-end number through the public API with host buffers, and
the CPU oracle timed on a bounded sample.

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--impl {rssm,reference}]
Multi-GPU (weak scaling, independent replicas, no collective on the data path):
  python -m torch.distributed.run --nproc-per-node N --master-addr 127.0.0.1 bench.py --gpus N
"""

from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from synth import (GDN_B256, MAMBA2_120B, SPEC_MAMBA2_B512, accepted_lengths, gdn_draft_inputs,  # noqa: E402
                   gdn_initial_state,
                   gdn_step_inputs, mamba2_draft_inputs, mamba2_initial_state, mamba2_params, mamba2_step_inputs)

WL = MAMBA2_120B
METRIC = "SSM decode tokens/s & achieved HBM GB/s at B=256, L=16 vs step-by-step kernel"
POOL = 32  # distinct token inputs cycled through the timed region


def traffic_model(wl, count_before: int) -> dict:
    """Algorithmic HBM bytes of one replay step whose sequences hold ``count_before`` records.

    checkpoint read + checkpoint write (fold steps only) + buffered records read +
    token inputs read + record appended + fp32 output written.
    """
    Bt, H, P, N, G, L = wl.batch, wl.nheads, wl.headdim, wl.dstate, wl.ngroups, wl.window
    esz = 2 if wl.in_dtype == "bf16" else 4
    state = Bt * H * P * N * 4
    rec = Bt * (H * P * esz + G * N * esz + H * 4)          # one record in the ring (x, B, dt as fp32)
    tok = Bt * (H * P * esz + 2 * G * N * esz + H * esz)     # x, B, C, dt of the token
    fold = count_before + 1 == L
    return {"state_read": state, "state_write": state if fold else 0, "ring_read": count_before * rec,
            "inputs": tok, "append": rec, "y": Bt * H * P * 4}


def verify_traffic(wl, T: int, accepted) -> float:
    """Algorithmic HBM bytes of the verify + commit rounds with the given accepted lengths, from count 0.

    Per sequence and round: checkpoint read, plus its write and the window's records when the verify
    pre-folds (count + T > L); buffered records read otherwise; T tokens' inputs read, T records appended,
    T fp32 outputs written.  Commit moves bookkeeping words only.
    """
    Bt, H, L = wl.batch, wl.nheads, wl.window
    esz = 2 if wl.in_dtype == "bf16" else 4
    if wl.kind == "mamba2":
        P, N, G = wl.headdim, wl.dstate, wl.ngroups
        state, y = H * P * N * 4, H * P * 4
        rec = H * P * esz + G * N * esz + H * 4                 # x, B, dt (fp32)
        tok = H * P * esz + 2 * G * N * esz + H * esz            # x, B, C, dt
    else:
        dk, dv = wl.dk, wl.dv
        state, y = H * dv * dk * 4, H * dv * 4
        rec = H * (dk * esz + dv * esz + 8)                      # k, v, alpha, beta (fp32)
        tok = H * (2 * dk * esz + dv * esz + 8)                  # q, k, v, alpha, beta
    count = np.zeros(Bt, np.int64)
    total = 0.0
    for acc in accepted:
        fold = count + T > L
        total += Bt * state + int(fold.sum()) * state + int(count.sum()) * rec
        total += Bt * T * (tok + rec + y)
        count = np.where(fold, 0, count) + np.asarray(acc, np.int64)
    return total


def conventional_bytes(wl) -> int:
    Bt, H, P, N, G = wl.batch, wl.nheads, wl.headdim, wl.dstate, wl.ngroups
    esz = 2 if wl.in_dtype == "bf16" else 4
    return 2 * Bt * H * P * N * 4 + Bt * (H * P * esz + 2 * G * N * esz + H * esz) + Bt * H * P * 4


def max_over_ranks(values, device=None):
    """Element-wise maximum of a list of floats over all ranks (identity when not distributed)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return [float(v) for v in values]
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(v) for v in t.cpu()]


def rank_workload(rank: int):
    """The workload rank ``rank`` decodes: the same layer with its own input seed (its own batch shard)."""
    return WL.replace(seed=WL.seed + 1000 * rank)


def weak_scaling_value(tokens_per_rank_step: int, world: int, steps: int, max_ms: float) -> float:
    """Whole-job tokens/s: every rank decodes its own batch shard; time is the slowest rank's."""
    return tokens_per_rank_step * world * steps / (max_ms * 1e-3)


def source_hash(sources) -> str:
    """sha1 of the kernel sources with comments and blank lines left out (a change of code, not of prose)."""
    import hashlib
    import re
    m = hashlib.sha1()
    for f in sources:
        for line in open(os.path.join(ROOT, "hybrid_model_ssm_gdn_b200", "csrc", f)).read().splitlines():
            code = re.sub(r"//.*$", "", line).strip()
            if code:
                m.update(code.encode() + b"\n")
    return m.hexdigest()


def profiled_traffic(summary: str, sources) -> "float | None":
    """DRAM bytes per launch from the committed ncu summary, or None if the kernel changed since it was taken."""
    import re
    path = os.path.join(ROOT, "profiles", summary)
    if not os.path.exists(path):
        return None
    text = open(path).read()
    h = re.search(r"Kernel source hash[^`]*`([0-9a-f]+)`", text)
    t = re.search(r"traffic_bytes_per_launch_window_avg:\s*([0-9.]+)", text)
    if not h or not t or h.group(1) != source_hash(sources):
        return None
    return float(t.group(1))


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return float(d["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


def gpu_selector(dev_index: int) -> str:
    """nvidia-smi ``-i`` selector of a torch device: its UUID (indices differ under CUDA_VISIBLE_DEVICES)."""
    try:
        import torch
        u = str(torch.cuda.get_device_properties(dev_index).uuid)
        return u if u.startswith("GPU-") else "GPU-" + u
    except Exception:  # noqa: BLE001 - fall back to the index
        return str(dev_index)


class ClockSampler:
    """nvidia-smi clocks and throttle reasons, sampled every 100 ms by a reader thread.

    Enter it before the warm-up: ``wait_first()`` blocks until nvidia-smi has produced a sample (its
    start-up takes longer than a short timed region), ``mark()`` brackets the timed region, and on exit
    the sampler keeps reading until one sample after the region has arrived.  The summary covers the
    samples from the one just before the region to the one just after it, so a region shorter than the
    sampling period is still described by its neighbouring samples."""

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
         "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
         "clocks_event_reasons.sw_power_cap")

    def __init__(self, selector: str):
        self.selector = selector
        self.proc = None
        self.samples = []          # (time, line)
        self.t0 = self.t1 = None

    def __enter__(self):
        import threading
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", self.selector, f"--query-gpu={self.Q}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
            return self

        def reader():
            for line in self.proc.stdout:
                if line.strip():
                    self.samples.append((time.perf_counter(), line.strip()))

        self.thread = threading.Thread(target=reader, daemon=True)
        self.thread.start()
        return self

    def wait_first(self, timeout: float = 5.0):
        t = time.perf_counter()
        while self.proc is not None and not self.samples and time.perf_counter() - t < timeout:
            time.sleep(0.01)

    def mark(self, which: str):
        if which == "start":
            self.t0 = time.perf_counter()
        else:
            self.t1 = time.perf_counter()

    def __exit__(self, *exc):
        if self.proc is None:
            return
        t = time.perf_counter()
        end = self.t1 if self.t1 is not None else t
        while not any(ts > end for ts, _ in self.samples) and time.perf_counter() - t < 1.0:
            time.sleep(0.01)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            self.proc.wait()

    def window(self):
        """Sample lines from the last one before the timed region to the first one after it."""
        if self.t0 is None:
            return [l for _, l in self.samples]
        t1 = self.t1 if self.t1 is not None else self.t0
        before = [i for i, (ts, _) in enumerate(self.samples) if ts <= self.t0]
        after = [i for i, (ts, _) in enumerate(self.samples) if ts >= t1]
        lo = before[-1] if before else 0
        hi = after[0] if after else len(self.samples) - 1
        return [l for _, l in self.samples[lo:hi + 1]]

    def summary(self):
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for l in self.window():
            f = [x.strip() for x in l.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx.append(float(f[2]))
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm)}


# ------------------------------------------------------------------------------ CPU oracle (baseline leg)

class OracleArm:
    """The float64 oracle, as it stands, decoding sequences ``first .. first + nseq - 1`` (all heads) of the
    workload."""

    def __init__(self, nseq: int, first: int = 0):
        from oracle.decoder import ReplayOracle
        self.seqs = list(range(first, first + nseq))
        S0 = mamba2_initial_state(WL, seqs=self.seqs)
        self.inputs = [{k: v[self.seqs] for k, v in mamba2_step_inputs(WL, t).items()} for t in range(4)]
        self.orc = ReplayOracle("mamba2", S0, WL.window, nheads=WL.nheads, ngroups=WL.ngroups,
                                params=mamba2_params(WL), seq_ids=self.seqs)
        self.i = 0

    def step(self):
        self.orc.step(self.inputs[self.i % len(self.inputs)])
        self.i += 1


def _limits():
    from threadpoolctl import threadpool_limits
    return threadpool_limits(1)


def host_workers(nseq: int) -> int:
    """Oracle worker processes for ``nseq`` sequences: one per usable host core, at most 32 and at most nseq."""
    try:
        cores = len(os.sched_getaffinity(0))
    except AttributeError:
        cores = os.cpu_count() or 1
    return max(1, min(cores, 32, nseq))


def _oracle_worker(first, nseq, warmup, steps, budget_s, barrier, out):
    """One host process: the oracle on its own sequences, one BLAS thread.  Times ``steps`` steps after
    ``warmup``, or (steps = 0) as many steps as fit in ``budget_s``."""
    sys.path.insert(0, ROOT)
    with _limits():
        arm = OracleArm(nseq, first)
        for _ in range(warmup):
            arm.step()
        barrier.wait()
        t0 = time.perf_counter()
        if steps:
            for _ in range(steps):
                arm.step()
        else:
            while time.perf_counter() - t0 < budget_s:
                arm.step()
        out.put((first, nseq, arm.i - warmup, time.perf_counter() - t0))


def oracle_pool(nseq_total: int, warmup: int, steps: int, budget_s: float = 0.0) -> dict:
    """The oracle on ``nseq_total`` sequences split over host worker processes (spawned: the parent may already
    hold a CUDA context), started together.  Returns tokens, the slowest worker's seconds and the cores used."""
    import multiprocessing as mp
    w = host_workers(nseq_total)
    ctx = mp.get_context("spawn")
    barrier, out = ctx.Barrier(w), ctx.Queue()
    per = [nseq_total // w + (1 if i < nseq_total % w else 0) for i in range(w)]
    firsts = [sum(per[:i]) for i in range(w)]
    procs = [ctx.Process(target=_oracle_worker, args=(firsts[i], per[i], warmup, steps, budget_s, barrier, out))
             for i in range(w)]
    for p in procs:
        p.start()
    res = [out.get(timeout=600) for _ in procs]
    for p in procs:
        p.join(timeout=60)
    tokens = sum(n * k for _, n, k, _ in res)
    secs = max(t for _, _, _, t in res)
    return {"tokens": tokens, "seconds": secs, "cores": w, "seqs": nseq_total,
            "steps": min(k for _, _, k, _ in res)}


def cpu_baseline(budget_s: float = 10.0) -> dict:
    """Oracle tokens/s on a bounded sample of the workload: one host process per core (at most 32), two
    sequences (all heads) each, whole decode steps for ~budget_s; plus the same oracle on one thread."""
    w = host_workers(64)
    r = oracle_pool(2 * w, 2, 0, budget_s)
    with _limits():
        arm = OracleArm(2)
        t0 = time.perf_counter()
        while time.perf_counter() - t0 < budget_s / 2:
            arm.step()
        dt1 = time.perf_counter() - t0
    one = len(arm.seqs) * arm.i / dt1
    return {"value": r["tokens"] / r["seconds"], "unit": "tokens/s", "cores": r["cores"], "kind": "oracle",
            "one_thread_tokens_per_s": one,
            "sample": f"{r['seqs']} of {WL.batch} sequences x all {WL.nheads} heads on {r['cores']} host processes "
                      f"(one BLAS thread each), >= {r['steps']} decode steps in {r['seconds']:.1f} s (float64 "
                      f"step-by-step + replay bookkeeping); one thread alone: {one:.1f} tokens/s"}


def arm_config(world: int) -> dict:
    """The workload of the GPU arm (the reference arm times a sample of it; see reference_config)."""
    return {"workload": "mamba2 replay decode, batch 256 per GPU, 128 heads, P 64, N 128, 8 groups, L 16, "
                        "bf16 inputs, fp32 checkpoint 1 GiB", "batch_per_gpu": WL.batch,
            "global_batch": WL.batch * world, "nheads": WL.nheads, "headdim": WL.headdim,
            "dstate": WL.dstate, "ngroups": WL.ngroups, "window": WL.window,
            "parallelism": f"replicas x{world} (batch shards, no collective)",
            "l2": "checkpoint stream (1 GiB/step) exceeds L2; no flush"}


def reference_config(nseq: int) -> dict:
    """The reference arm's config: the GPU arm's layer shape, with the sample it actually times."""
    c = {k: v for k, v in arm_config(1).items() if k not in ("batch_per_gpu", "global_batch", "parallelism", "l2")}
    c["workload"] = (f"mamba2 replay decode (oracle, host cores), {nseq} of the 256 sequences per step, 128 heads, "
                     "P 64, N 128, 8 groups, L 16, bf16 inputs, fp32 checkpoint")
    c["sampled_sequences"] = nseq
    return c


def reference_arm(args) -> dict:
    """--impl reference: the oracle timed per step on the host cores, on a sample of the sequences sized so the
    whole run takes about two minutes."""
    with _limits():
        probe = OracleArm(1)
        t0 = time.perf_counter()
        for _ in range(3):
            probe.step()
        per_seq_step = (time.perf_counter() - t0) / 3
    w = host_workers(WL.batch)
    nseq = int(max(1, min(WL.batch, 100.0 * w / ((args.steps + args.warmup) * per_seq_step))))
    r = oracle_pool(nseq, args.warmup, args.steps)
    v = r["tokens"] / r["seconds"]
    ms = r["seconds"] / args.steps * 1e3
    cb = {"value": v, "unit": "tokens/s", "cores": r["cores"], "kind": "oracle",
          "sample": f"{nseq} of {WL.batch} sequences x all {WL.nheads} heads per step on {r['cores']} host processes "
                    f"(one BLAS thread each), {args.steps} steps after {args.warmup} warm-up, {r['seconds']:.1f} s"}
    return {"impl": "reference", "metric": METRIC, "value": v, "unit": "tokens/s", "n_gpus": 0,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "ms_per_sequence_step": ms / nseq,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": reference_config(nseq),
            "cpu_baseline": cb,
            "e2e": {"value": v, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


# ------------------------------------------------------------------------------ GPU arm

def run_gpu(args, rank, world):
    import torch

    from hybrid_model_ssm_gdn_b200 import ReplaySSM, conv_mamba2_step, make_config
    torch.cuda.set_device(rank % torch.cuda.device_count())
    dev = torch.device("cuda")
    bf = torch.bfloat16
    L = WL.window
    p = mamba2_params(WL)
    A = torch.from_numpy(p["A"]).to(dev)
    D = torch.from_numpy(p["D"]).to(dev)
    layer = ReplaySSM("mamba2", WL.batch, WL.nheads, WL.headdim, WL.dstate, WL.ngroups, WL.window, 0, bf,
                      A=A, D=D)
    S0 = torch.from_numpy(mamba2_initial_state(WL)).to(dev)
    layer.load_checkpoint(S0)
    # each rank decodes its own batch shard: its own seeded inputs
    host_pool = [mamba2_step_inputs(rank_workload(rank), t) for t in range(POOL)]
    pool = [{k: torch.from_numpy(v).to(dev).to(bf) for k, v in inp.items()} for inp in host_pool]
    y = torch.empty(WL.batch, WL.nheads, WL.headdim, device=dev)
    stream = torch.cuda.current_stream()
    pos = [0]  # steps run on the layer so far (its window position is pos % L)

    def step(i):
        t = pool[i % POOL]
        layer.mamba2_step(t["x"], t["B"], t["C"], t["dt"], y)
        pos[0] += 1

    K = args.steps
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(K + 1)]
    with ClockSampler(gpu_selector(torch.cuda.current_device())) as clk:
        # warm-up: at least W steps, extended to a window boundary so that the timed region starts at window
        # position 0 (the fold falls on every L-th timed step)
        warm = -(-args.warmup // L) * L
        for i in range(warm):
            step(i)
        torch.cuda.synchronize()
        clk.wait_first()

        def timed_region(first_step):
            if world > 1:
                import torch.distributed as dist
                dist.barrier()
            torch.cuda.synchronize()
            clk.mark("start")
            ev[0].record(stream)
            for i in range(K):
                step(first_step + i)
                ev[i + 1].record(stream)
            torch.cuda.synchronize()
            clk.mark("end")
            return [ev[i].elapsed_time(ev[i + 1]) for i in range(K)], ev[0].elapsed_time(ev[K])

        count0 = pos[0] % L
        per, total_ms = timed_region(warm)
    clocks = clk.summary()
    # a region that saw a hardware or thermal slowdown is measured once more (from the next window boundary);
    # every rank takes the same decision
    bad = {"hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown"}
    retry = max_over_ranks([1.0 if bad & set(clocks["reasons"]) else 0.0], device=dev)[0] > 0
    if retry:
        with ClockSampler(gpu_selector(torch.cuda.current_device())) as clk:
            while pos[0] % L:
                step(pos[0])
            torch.cuda.synchronize()
            clk.wait_first()
            count0 = pos[0] % L
            per, total_ms = timed_region(pos[0])
        clocks = clk.summary()
        clocks["remeasured"] = True
    total_ms = max_over_ranks([total_ms], device=dev)[0]
    model = [traffic_model(WL, (count0 + i) % L) for i in range(K)]
    bytes_avg = sum(sum(m.values()) for m in model) / K
    step_ms = total_ms / K
    mean_launch_ms = sum(per) / K
    hbm_peak, peak_kind = load_peaks()
    achieved = bytes_avg / (mean_launch_ms * 1e-3) / 1e9
    fold_ms = [d for d, m in zip(per, model) if m["state_write"]]
    plain_ms = [d for d, m in zip(per, model) if not m["state_write"]]
    # the same launches weighted as in a whole window ((L - 1) plain steps, one fold), whatever K is
    window_ms = None
    if fold_ms and plain_ms:
        window_ms = ((L - 1) * statistics.mean(plain_ms) + statistics.mean(fold_ms)) / L
        window_ms = max_over_ranks([window_ms], device=dev)[0]
    err = layer.get_error()

    # conventional step-by-step kernel on the same layer (comparison)
    cfg = make_config("mamba2", WL.batch, WL.nheads, WL.headdim, WL.dstate, WL.ngroups, WL.window, 0, bf, A=A, D=D)
    S = S0.clone()
    Kc = max(16, K // 4)
    for i in range(8):
        t = pool[i % POOL]
        conv_mamba2_step(cfg, S, t["x"], t["B"], t["C"], t["dt"], y)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for i in range(Kc):
        t = pool[i % POOL]
        conv_mamba2_step(cfg, S, t["x"], t["B"], t["C"], t["dt"], y)
    e1.record(stream)
    torch.cuda.synchronize()
    conv_ms = e0.elapsed_time(e1) / Kc
    del S

    e2e = e2e_leg(layer, host_pool, pos, step, stream, dev)
    e2e_ms, conv_ms = max_over_ranks([e2e["ms_per_step"], conv_ms], device=dev)
    e2e["ms_per_step"] = e2e_ms

    tokens = WL.batch * world
    res = {
        "metric": METRIC, "value": weak_scaling_value(WL.batch, world, K, total_ms), "unit": "tokens/s",
        "n_gpus": world,
        "steps": K, "warmup": args.warmup, "ms_per_step": step_ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f32", "data": "synthetic (seeded; bf16 token inputs, fp32 checkpoint)",
        "config": dict(arm_config(world), warmup_run=warm, timed_from_window_position=count0),
        "window_weighted": None if window_ms is None else {
            "tokens_per_s": tokens / (window_ms * 1e-3), "ms_per_step": window_ms,
            "note": f"the timed launches weighted {L - 1} plain : 1 fold, as in a whole window"},
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": hbm_peak, "unit": "GB/s",
                     "frac": achieved / hbm_peak, "peak_kind": peak_kind,
                     "traffic": profiled_traffic("m2_replay_kernel__mamba2_b256_L16.md",
                                                 ("mamba2.cu", "common.cuh", "kernels.h")),
                     "kernel": "m2_replay_kernel", "bytes_per_launch": bytes_avg,
                     "mean_launch_ms": mean_launch_ms,
                     "fold_launch_ms": statistics.mean(fold_ms) if fold_ms else None,
                     "plain_launch_ms": statistics.median(plain_ms) if plain_ms else None},
        "comparison": {"conventional_tokens_per_s": tokens / (conv_ms * 1e-3), "conventional_ms_per_step": conv_ms,
                       "conventional_bytes_per_step": conventional_bytes(WL),
                       "conventional_GBps": conventional_bytes(WL) / (conv_ms * 1e-3) / 1e9,
                       "replay_speedup": conv_ms / step_ms},
        "e2e": dict(e2e, value=tokens / (e2e_ms * 1e-3), unit="tokens/s"),
        "gpu_launches": K,
        "clocks": clocks,
        "device_error": err,
    }
    return res


def e2e_leg(layer, host_pool, pos, step, stream, dev, windows: int = 4) -> dict:
    """End to end through the public API: every step's inputs are copied from pinned host memory and its output
    read back to pinned host memory inside the timed region.  The copies of neighbouring steps overlap the
    decode on separate host-to-device and device-to-host streams (double-buffered device inputs and outputs).
    Timed over whole windows from a window boundary, after one untimed window; the same copies and the step
    are also timed on their own, so the line shows which of them bounds the pipeline."""
    import torch
    bf = torch.bfloat16
    L = WL.window
    pinned = [{k: torch.from_numpy(v).to(bf).pin_memory() for k, v in inp.items()} for inp in host_pool[:8]]
    y_host = [torch.empty(WL.batch, WL.nheads, WL.headdim, dtype=torch.float32).pin_memory() for _ in range(2)]
    h2d = sum(v.numel() * v.element_size() for v in pinned[0].values())
    d2h = y_host[0].numel() * 4
    bufs = [{k: torch.empty_like(v, device=dev) for k, v in pinned[0].items()} for _ in range(2)]
    ys = [torch.empty(WL.batch, WL.nheads, WL.headdim, device=dev) for _ in range(2)]
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()

    def run(n):
        copied = [torch.cuda.Event() for _ in range(2)]
        used = [torch.cuda.Event() for _ in range(2)]
        read = [torch.cuda.Event() for _ in range(2)]

        def h2d_copy(i):
            b = i % 2
            with torch.cuda.stream(s_in):
                if i >= 2:
                    s_in.wait_event(used[b])           # step i-2 has consumed this buffer
                for k, v in pinned[i % len(pinned)].items():
                    bufs[b][k].copy_(v, non_blocking=True)
                copied[b].record(s_in)

        s_in.wait_stream(stream)
        s_out.wait_stream(stream)
        h2d_copy(0)
        for i in range(n):
            b = i % 2
            if i + 1 < n:
                h2d_copy(i + 1)
            stream.wait_event(copied[b])
            if i >= 2:
                stream.wait_event(read[b])             # y of step i-2 has been read back
            t = bufs[b]
            layer.mamba2_step(t["x"], t["B"], t["C"], t["dt"], ys[b])
            pos[0] += 1
            used[b].record(stream)
            with torch.cuda.stream(s_out):
                s_out.wait_event(used[b])
                y_host[b].copy_(ys[b], non_blocking=True)
                read[b].record(s_out)
        stream.wait_stream(s_out)

    torch.cuda.synchronize()
    run((-pos[0]) % L + L)                             # untimed: to the next window boundary, then one window
    torch.cuda.synchronize()
    Ke = windows * L
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    run(Ke)
    t1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = t0.elapsed_time(t1) / Ke

    def alone(fn, s, n=32):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        a.record(s)
        for i in range(n):
            fn(i)
        b.record(s)
        torch.cuda.synchronize()
        return a.elapsed_time(b) / n

    def copy_in(i):
        with torch.cuda.stream(s_in):
            for k, v in pinned[i % len(pinned)].items():
                bufs[0][k].copy_(v, non_blocking=True)

    def copy_out(i):
        with torch.cuda.stream(s_out):
            y_host[i % 2].copy_(ys[i % 2], non_blocking=True)

    h2d_ms = alone(copy_in, s_in)
    d2h_ms = alone(copy_out, s_out)
    while pos[0] % L:
        step(pos[0])
    step_alone = alone(lambda i: step(i), stream, 2 * L)
    return {"h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms, "steps": Ke,
            "breakdown_ms_per_step": {"h2d_copy_alone": h2d_ms, "d2h_copy_alone": d2h_ms,
                                      "decode_step_alone": step_alone},
            "h2d_GBps_alone": h2d / (h2d_ms * 1e-3) / 1e9, "d2h_GBps_alone": d2h / (d2h_ms * 1e-3) / 1e9}


# bytes per state element of each stored format: fp32, fp16, E4M3 with one fp32 scale per 64 x 128 tile,
# and NVFP4 (E2M1 codes, an E4M3 scale per 16 elements, one fp32 scale per tile)
HP_BYTES = {"f32": 4.0, "f16sr": 2.0, "f8sr": 1.0 + 4.0 / (64 * 128)}
NVFP4_BYTES = 0.5 + 1.0 / 16 + 4.0 / (64 * 128)
NVFP4D_BYTES = NVFP4_BYTES + 1.0 / 16     # plus one E4M3 column-group scale per 16 elements


def gdn_traffic(wl, count_before: int, hp: str = "f32", read: str = "same") -> float:
    """Algorithmic bytes of one GDN replay step (same terms as the Mamba-2 model) with the checkpoint stored
    as ``hp``.  Steps that do not fold read the checkpoint (``read="same"``) or the NVFP4 copy beside it
    (``"nvfp4"``); a fold reads the checkpoint and writes it and the copy.  ``"shared_nvfp4"``: the NVFP4
    copy is the checkpoint."""
    Bt, H, dk, dv, L = wl.batch, wl.nheads, wl.dk, wl.dv, wl.window
    esz = 2 if wl.in_dtype == "bf16" else 4
    elems = Bt * H * dv * dk
    ckpt = elems * (NVFP4_BYTES if read == "shared_nvfp4" else HP_BYTES[hp])
    copy = elems * {"nvfp4": NVFP4_BYTES, "nvfp4d": NVFP4D_BYTES}.get(read, 0.0)
    rec = Bt * H * (dk * esz + dv * esz + 8)
    tok = Bt * H * (2 * dk * esz + dv * esz + 8)
    fold = count_before + 1 == L
    state = ckpt + ckpt + copy if fold else (copy if read in ("nvfp4", "nvfp4d") else ckpt)
    return state + count_before * rec + tok + rec + Bt * H * dv * 4


def timed(fn, n, stream):
    import torch
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    e0.record(stream)
    for i in range(n):
        fn(i)
    e1.record(stream)
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) / n


def gdn_section(steps: int) -> dict:
    """Gated DeltaNet layer (batch 256, 32 heads, d_k = d_v = 128, L 16): replay vs conventional."""
    import torch

    from hybrid_model_ssm_gdn_b200 import ReplaySSM, conv_gdn_step, make_config
    wl, dev = GDN_B256, torch.device("cuda")
    bf = torch.bfloat16
    layer = ReplaySSM("gdn", wl.batch, wl.nheads, wl.dv, wl.dk, 1, wl.window, 0, bf)
    S0 = torch.from_numpy(gdn_initial_state(wl)).to(dev)
    layer.load_checkpoint(S0)
    pool = []
    for t in range(16):
        inp = gdn_step_inputs(wl, t)
        pool.append({k: torch.from_numpy(v).to(dev).to(torch.float32 if k in ("alpha", "beta") else bf)
                     for k, v in inp.items()})
    y = torch.empty(wl.batch, wl.nheads, wl.dv, device=dev)
    stream = torch.cuda.current_stream()

    def step(i):
        t = pool[i % 16]
        layer.gdn_step(t["q"], t["k"], t["v"], t["alpha"], t["beta"], y)

    for i in range(2 * wl.window):
        step(i)
    K = max(wl.window, steps // wl.window * wl.window)
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(K + 1)]
    torch.cuda.synchronize()
    ev[0].record(stream)
    for i in range(K):
        step(i)
        ev[i + 1].record(stream)
    torch.cuda.synchronize()
    per = [ev[i].elapsed_time(ev[i + 1]) for i in range(K)]
    ms = ev[0].elapsed_time(ev[K]) / K
    fold_ms = [d for i, d in enumerate(per) if (i + 1) % wl.window == 0]
    plain_ms = [d for i, d in enumerate(per) if (i + 1) % wl.window != 0]
    bytes_avg = sum(gdn_traffic(wl, i % wl.window) for i in range(K)) / K
    cfg = make_config("gdn", wl.batch, wl.nheads, wl.dv, wl.dk, 1, wl.window, 0, bf)
    S = S0.clone()

    def conv(i):
        t = pool[i % 16]
        conv_gdn_step(cfg, S, t["q"], t["k"], t["v"], t["alpha"], t["beta"], y)

    for i in range(4):
        conv(i)
    ms_conv = timed(conv, max(16, K // 4), stream)
    conv_bytes = 2 * S0.numel() * 4 + wl.batch * wl.nheads * (2 * wl.dk * 2 + wl.dv * 2 + 8 + wl.dv * 4)
    hbm, _ = load_peaks()
    return {"workload": "gdn replay decode, batch 256, 32 heads, d_k = d_v = 128, L 16, bf16 inputs, fp32 checkpoint",
            "tokens_per_s": wl.batch / (ms * 1e-3), "ms_per_step": ms, "GBps": bytes_avg / (ms * 1e-3) / 1e9,
            "frac_of_measured_hbm": bytes_avg / (ms * 1e-3) / 1e9 / hbm, "bytes_per_step": bytes_avg,
            "plain_launch_ms": statistics.median(plain_ms), "fold_launch_ms": statistics.mean(fold_ms),
            "conventional_tokens_per_s": wl.batch / (ms_conv * 1e-3), "conventional_ms_per_step": ms_conv,
            "conventional_GBps": conv_bytes / (ms_conv * 1e-3) / 1e9, "replay_speedup": ms_conv / ms,
            "steps": K, "device_error": layer.get_error()}


PRECISION_MODES = (("f32", "same"), ("f16sr", "same"), ("f8sr", "same"), ("f32", "nvfp4"), ("f16sr", "nvfp4"),
                   ("f8sr", "nvfp4"), ("f32", "shared_nvfp4"), ("f32", "nvfp4d"))


def precision_section(windows_timed: int = 4, modes=None) -> dict:
    """GDN layer (batch 256, 32 heads, d 128, L 16) with each checkpoint format and read mode: window-averaged
    step time, plain and fold launches, and the rate of the mode's algorithmic bytes."""
    import torch

    from hybrid_model_ssm_gdn_b200 import ReplaySSM
    wl, dev, bf = GDN_B256, torch.device("cuda"), torch.bfloat16
    S0 = torch.from_numpy(gdn_initial_state(wl)).to(dev)
    pool = []
    for t in range(16):
        inp = gdn_step_inputs(wl, t)
        pool.append({k: torch.from_numpy(v).to(dev).to(torch.float32 if k in ("alpha", "beta") else bf)
                     for k, v in inp.items()})
    y = torch.empty(wl.batch, wl.nheads, wl.dv, device=dev)
    stream = torch.cuda.current_stream()
    hbm, _ = load_peaks()
    out = {"workload": "gdn replay decode, batch 256, 32 heads, d_k = d_v = 128, L 16, bf16 inputs; checkpoint "
                       "format x read mode"}
    for hp, read in PRECISION_MODES:
        if modes and f"{hp}/{read}" not in modes:
            continue
        layer = ReplaySSM("gdn", wl.batch, wl.nheads, wl.dv, wl.dk, 1, wl.window, 0, bf, hp, read, seed=3)
        layer.load_checkpoint(S0)

        def step(i):
            t = pool[i % 16]
            layer.gdn_step(t["q"], t["k"], t["v"], t["alpha"], t["beta"], y)

        for i in range(2 * wl.window):
            step(i)
        K = wl.window * windows_timed
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(K + 1)]
        torch.cuda.synchronize()
        ev[0].record(stream)
        for i in range(K):
            step(i)
            ev[i + 1].record(stream)
        torch.cuda.synchronize()
        per = [ev[i].elapsed_time(ev[i + 1]) for i in range(K)]
        ms = ev[0].elapsed_time(ev[K]) / K
        nbytes = sum(gdn_traffic(wl, i % wl.window, hp, read) for i in range(K)) / K
        out[f"{hp}/{read}"] = {
            "ms_per_step": ms, "tokens_per_s": wl.batch / (ms * 1e-3), "bytes_per_step": nbytes,
            "GBps": nbytes / (ms * 1e-3) / 1e9, "frac_of_measured_hbm": nbytes / (ms * 1e-3) / 1e9 / hbm,
            "plain_launch_ms": statistics.median([d for i, d in enumerate(per) if (i + 1) % wl.window != 0]),
            "fold_launch_ms": statistics.mean([d for i, d in enumerate(per) if (i + 1) % wl.window == 0]),
            "device_error": layer.get_error()}
        del layer
    return out


def skip_section(windows_timed: int = 8, tau: float = 1e-2) -> dict:
    """GDN layer (batch 256, 32 heads, d 128, L 16) with fast-decaying gates (alpha = exp(-0.6 softplus(z)),
    about 0.6 on average): decay-aware read skipping off and on.  The skip pattern repeats every window (the
    inputs cycle with period L), so one untimed window of flag exports gives the skipped fraction of the
    timed steps; the byte count leaves out the skipped heads' checkpoint reads."""
    import torch

    from hybrid_model_ssm_gdn_b200 import ReplaySSM
    wl, dev, bf = GDN_B256.replace(decay_scale=0.6), torch.device("cuda"), torch.bfloat16
    L = wl.window
    S0 = torch.from_numpy(gdn_initial_state(wl)).to(dev)
    pool = []
    for t in range(L):
        inp = gdn_step_inputs(wl, t)
        pool.append({k: torch.from_numpy(v).to(dev).to(torch.float32 if k in ("alpha", "beta") else bf)
                     for k, v in inp.items()})
    y = torch.empty(wl.batch, wl.nheads, wl.dv, device=dev)
    stream = torch.cuda.current_stream()
    head_bytes = wl.dv * wl.dk * 4
    out = {"workload": "gdn replay decode, batch 256, 32 heads, d 128, L 16, bf16 inputs, fp32 checkpoint, "
                       "gates alpha = exp(-0.6 softplus(z))", "tau": tau}
    for name, t in (("off", 0.0), ("on", tau)):
        layer = ReplaySSM("gdn", wl.batch, wl.nheads, wl.dv, wl.dk, 1, L, 0, bf, skip_tau=t)
        layer.load_checkpoint(S0)

        def step(i):
            p = pool[i % L]
            layer.gdn_step(p["q"], p["k"], p["v"], p["alpha"], p["beta"], y)

        for i in range(2 * L):
            step(i)
        skipped = []  # heads skipping their read at each position of the window
        for i in range(L):
            skipped.append(int(layer.export_skip().sum().item()) if t > 0 else 0)
            step(i)
        K = L * windows_timed
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(K + 1)]
        torch.cuda.synchronize()
        ev[0].record(stream)
        for i in range(K):
            step(i)
            ev[i + 1].record(stream)
        torch.cuda.synchronize()
        ms = ev[0].elapsed_time(ev[K]) / K
        per = [sorted(ev[w * L + i].elapsed_time(ev[w * L + i + 1]) for w in range(windows_timed)) for i in range(L)]
        nbytes = sum(gdn_traffic(wl, i) - skipped[i] * head_bytes for i in range(L)) / L
        out[name] = {"ms_per_step": ms, "tokens_per_s": wl.batch / (ms * 1e-3), "bytes_per_step": nbytes,
                     "GBps": nbytes / (ms * 1e-3) / 1e9,
                     "skipped_fraction": sum(skipped) / (L * wl.batch * wl.nheads),
                     "launch_ms_by_position": [p[len(p) // 2] for p in per], "skipped_heads_by_position": skipped,
                     "device_error": layer.get_error()}
        del layer
    out["speedup"] = out["off"]["ms_per_step"] / out["on"]["ms_per_step"]
    return out


def skip_mamba2_section(windows_timed: int = 8, tau: float = 1e-2, decay_scale: float = 8.0) -> dict:
    """Mamba-2 layer (batch 256, 128 heads, P 64, N 128, 8 groups, L 16) with faster-decaying heads (A times
    ``decay_scale``): decay-aware read skipping off and on.  As in the GDN section, one untimed window of flag
    exports gives the skipped heads at each window position (the inputs cycle with period L)."""
    import torch

    from hybrid_model_ssm_gdn_b200 import ReplaySSM
    wl, dev, bf = WL.replace(decay_scale=decay_scale), torch.device("cuda"), torch.bfloat16
    L = wl.window
    p = mamba2_params(wl)
    A, D = torch.from_numpy(p["A"]).to(dev), torch.from_numpy(p["D"]).to(dev)
    S0 = torch.from_numpy(mamba2_initial_state(wl)).to(dev)
    pool = [{k: torch.from_numpy(v).to(dev).to(bf) for k, v in mamba2_step_inputs(wl, t).items()} for t in range(L)]
    y = torch.empty(wl.batch, wl.nheads, wl.headdim, device=dev)
    stream = torch.cuda.current_stream()
    head_bytes = wl.headdim * wl.dstate * 4
    out = {"workload": f"mamba2 replay decode, batch 256, 128 heads, P 64, N 128, 8 groups, L 16, bf16 inputs, "
                       f"fp32 checkpoint, A x {decay_scale}", "tau": tau}
    for name, t in (("off", 0.0), ("on", tau)):
        layer = ReplaySSM("mamba2", wl.batch, wl.nheads, wl.headdim, wl.dstate, wl.ngroups, L, 0, bf, A=A, D=D,
                          skip_tau=t)
        layer.load_checkpoint(S0)

        def step(i):
            q = pool[i % L]
            layer.mamba2_step(q["x"], q["B"], q["C"], q["dt"], y)

        for i in range(2 * L):
            step(i)
        skipped = []
        for i in range(L):
            skipped.append(int(layer.export_skip().sum().item()) if t > 0 else 0)
            step(i)
        K = L * windows_timed
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(K + 1)]
        torch.cuda.synchronize()
        ev[0].record(stream)
        for i in range(K):
            step(i)
            ev[i + 1].record(stream)
        torch.cuda.synchronize()
        ms = ev[0].elapsed_time(ev[K]) / K
        per = [sorted(ev[w * L + i].elapsed_time(ev[w * L + i + 1]) for w in range(windows_timed)) for i in range(L)]
        nbytes = sum(sum(traffic_model(wl, i).values()) - skipped[i] * head_bytes for i in range(L)) / L
        out[name] = {"ms_per_step": ms, "tokens_per_s": wl.batch / (ms * 1e-3), "bytes_per_step": nbytes,
                     "GBps": nbytes / (ms * 1e-3) / 1e9,
                     "skipped_fraction": sum(skipped) / (L * wl.batch * wl.nheads),
                     "launch_ms_by_position": [q[len(q) // 2] for q in per], "skipped_heads_by_position": skipped,
                     "device_error": layer.get_error()}
        del layer
    out["speedup"] = out["off"]["ms_per_step"] / out["on"]["ms_per_step"]
    return out


def graph_section(batches=(1, 16, 256), n_mamba2: int = 6, n_gdn: int = 2, windows: int = 4) -> dict:
    """A hybrid stack's state-space layers (6 Mamba-2 layers of the 120B-class shape and 2 GDN layers, L 16)
    decoding token by token: every layer's step launched eagerly, and the same window of steps captured
    once in a CUDA graph and replayed.  ms per token of the whole stack at several batch sizes."""
    import torch

    from hybrid_model_ssm_gdn_b200 import ReplaySSM
    dev, bf = torch.device("cuda"), torch.bfloat16
    out = {"workload": f"{n_mamba2} mamba2 layers (128 heads, P 64, N 128, 8 groups) + {n_gdn} gdn layers "
                       "(32 heads, d 128), L 16, bf16 inputs, fp32 checkpoints; eager launches vs one CUDA graph "
                       "per window"}
    L = WL.window
    for Bt in batches:
        wm, wg = WL.replace(batch=Bt), GDN_B256.replace(batch=Bt)
        p = mamba2_params(wm)
        A, D = torch.from_numpy(p["A"]).to(dev), torch.from_numpy(p["D"]).to(dev)
        Sm = torch.from_numpy(mamba2_initial_state(wm)).to(dev)
        Sg = torch.from_numpy(gdn_initial_state(wg)).to(dev)
        layers = []
        for _ in range(n_mamba2):
            c = ReplaySSM("mamba2", Bt, wm.nheads, wm.headdim, wm.dstate, wm.ngroups, L, 0, bf, A=A, D=D)
            c.load_checkpoint(Sm)
            layers.append(c)
        for _ in range(n_gdn):
            c = ReplaySSM("gdn", Bt, wg.nheads, wg.dv, wg.dk, 1, L, 0, bf)
            c.load_checkpoint(Sg)
            layers.append(c)
        del Sm, Sg
        pm = [{k: torch.from_numpy(v).to(dev).to(bf) for k, v in mamba2_step_inputs(wm, t).items()} for t in range(L)]
        pg = [{k: torch.from_numpy(v).to(dev).to(torch.float32 if k in ("alpha", "beta") else bf)
               for k, v in gdn_step_inputs(wg, t).items()} for t in range(L)]
        ym = torch.empty(Bt, wm.nheads, wm.headdim, device=dev)
        yg = torch.empty(Bt, wg.nheads, wg.dv, device=dev)

        def token(i):
            for c in layers:
                if c.kind == "mamba2":
                    t = pm[i % L]
                    c.mamba2_step(t["x"], t["B"], t["C"], t["dt"], ym)
                else:
                    t = pg[i % L]
                    c.gdn_step(t["q"], t["k"], t["v"], t["alpha"], t["beta"], yg)

        stream = torch.cuda.current_stream()
        for i in range(2 * L):
            token(i)
        ms_eager = timed(token, windows * L, stream)
        side = torch.cuda.Stream()
        side.wait_stream(stream)
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.stream(side):
            with torch.cuda.graph(graph, stream=side):
                for i in range(L):  # one window: an even number of calls per layer keeps each context's parity
                    token(i)
        stream.wait_stream(side)
        for _ in range(2):
            graph.replay()
        ms_graph = timed(lambda i: graph.replay(), windows, stream) / L
        errs = [c.get_error() for c in layers]
        out[f"B{Bt}"] = {"eager_ms_per_token": ms_eager, "graph_ms_per_token": ms_graph,
                         "graph_speedup": ms_eager / ms_graph, "launches_per_token": len(layers),
                         "device_error": max(errs)}
        del graph, layers
        torch.cuda.synchronize()
    return out


def verify_section(rounds: int, kinds=("mamba2", "gdn")) -> dict:
    """Speculative verify + commit (T = 4, 8) vs snapshot-per-draft: the Mamba-2 shape at batch 512 and the
    Gated DeltaNet layer at batch 256."""
    import torch

    from hybrid_model_ssm_gdn_b200 import ReplaySSM, make_config, snap_commit, snap_verify
    dev, bf, stream = torch.device("cuda"), torch.bfloat16, torch.cuda.current_stream()
    hbm = load_peaks()[0]
    out = {"workload": "mamba2 speculative verify + commit, batch 512, 128 heads, P 64, N 128, 8 groups, L 16",
           "gdn": {"workload": "gdn speculative verify + commit, batch 256, 32 heads, d_k = d_v = 128, L 16"}}
    for kind, wl in (("mamba2", SPEC_MAMBA2_B512), ("gdn", GDN_B256)):
        if kind not in kinds:
            continue
        if kind == "mamba2":
            p = mamba2_params(wl)
            A, D = torch.from_numpy(p["A"]).to(dev), torch.from_numpy(p["D"]).to(dev)
            S0 = torch.from_numpy(mamba2_initial_state(wl)).to(dev)
            rows, cols, G, f32_keys = wl.headdim, wl.dstate, wl.ngroups, ()
            draft_inputs = mamba2_draft_inputs
        else:
            A = D = None
            S0 = torch.from_numpy(gdn_initial_state(wl)).to(dev)
            rows, cols, G, f32_keys = wl.dv, wl.dk, 1, ("alpha", "beta")
            draft_inputs = gdn_draft_inputs
        dst = out if kind == "mamba2" else out["gdn"]
        for T in (4, 8):
            layer = ReplaySSM(kind, wl.batch, wl.nheads, rows, cols, G, wl.window, T, bf, A=A, D=D)
            layer.load_checkpoint(S0)
            drafts = [{k: torch.from_numpy(v).to(dev).to(torch.float32 if k in f32_keys else bf)
                       for k, v in draft_inputs(wl, r, T).items()} for r in range(4)]
            acc_np = [accepted_lengths(wl, r, T) for r in range(rounds)]
            accs = [torch.from_numpy(a).to(dev) for a in acc_np]
            acc_total = sum(int(a.sum()) for a in accs)
            y = torch.empty(wl.batch, T, wl.nheads, rows, device=dev)

            def rnd(i):
                layer.verify(T, y=y, **drafts[i % 4])
                layer.commit(accs[i])

            for i in range(min(8, rounds)):
                rnd(i)
            layer.load_checkpoint(S0)
            ms = timed(rnd, rounds, stream)
            err = layer.get_error()
            del layer
            # snapshot-per-draft comparison: one state read, T state writes per round
            cfg = make_config(kind, wl.batch, wl.nheads, rows, cols, G, wl.window, T, bf, A=A, D=D)
            snaps = torch.empty(wl.batch, T + 1, wl.nheads, rows, cols, device=dev)
            snaps[:, 0].copy_(S0)
            cur = torch.zeros(wl.batch, dtype=torch.int32, device=dev)

            def snap(i):
                snap_verify(cfg, snaps, cur, T, y, **drafts[i % 4])
                snap_commit(cfg, cur, accs[i])

            for i in range(min(4, rounds)):
                snap(i)
            ms_snap = timed(snap, rounds, stream)
            del snaps
            gbps = verify_traffic(wl, T, acc_np) / rounds / (ms * 1e-3) / 1e9
            dst[f"T{T}"] = {"ms_per_round": ms, "verified_tokens_per_s": wl.batch * T / (ms * 1e-3),
                            "GBps": gbps, "frac_of_measured_hbm": gbps / hbm,
                            "committed_tokens_per_s": acc_total / rounds / (ms * 1e-3),
                            "snapshot_ms_per_round": ms_snap,
                            "snapshot_committed_tokens_per_s": acc_total / rounds / (ms_snap * 1e-3),
                            "speedup_vs_snapshot": ms_snap / ms, "rounds": rounds, "device_error": err}
    return out


def window_section(windows=(4, 8, 16, 32), windows_timed: int = 8) -> dict:
    """Mamba-2 batch-256 layer at several windows L: amortised step time vs the traffic model."""
    import torch

    from hybrid_model_ssm_gdn_b200 import ReplaySSM
    dev, bf = torch.device("cuda"), torch.bfloat16
    p = mamba2_params(WL)
    A, D = torch.from_numpy(p["A"]).to(dev), torch.from_numpy(p["D"]).to(dev)
    S0 = torch.from_numpy(mamba2_initial_state(WL)).to(dev)
    pool = [{k: torch.from_numpy(v).to(dev).to(bf) for k, v in mamba2_step_inputs(WL, t).items()} for t in range(8)]
    y = torch.empty(WL.batch, WL.nheads, WL.headdim, device=dev)
    stream = torch.cuda.current_stream()
    out = {"workload": "mamba2 replay decode, batch 256, 128 heads, P 64, N 128, 8 groups, bf16 inputs, fp32 checkpoint"}
    for L in windows:
        wl = WL.replace(window=L)
        layer = ReplaySSM("mamba2", wl.batch, wl.nheads, wl.headdim, wl.dstate, wl.ngroups, L, 0, bf, A=A, D=D)
        layer.load_checkpoint(S0)

        def step(i):
            t = pool[i % 8]
            layer.mamba2_step(t["x"], t["B"], t["C"], t["dt"], y)

        for i in range(2 * L):
            step(i)
        K = L * max(windows_timed, 64 // L)
        ms = timed(step, K, stream)
        model = sum(sum(traffic_model(wl, i % L).values()) for i in range(K)) / K
        out[f"L{L}"] = {"ms_per_step": ms, "tokens_per_s": wl.batch / (ms * 1e-3), "model_bytes_per_step": model,
                        "GBps": model / (ms * 1e-3) / 1e9, "device_error": layer.get_error()}
        del layer
    return out


def batch_section(batches=(1, 2, 4, 8, 16, 32, 64, 128, 256, 512), windows_timed: int = 4) -> dict:
    """Mamba-2 layer (128 heads, P 64, N 128, 8 groups, L 16) at batch 1 .. 512: replay vs the conventional
    step-by-step kernel, window-averaged step time.  At small batches both are bound by launch and per-unit
    latency rather than by the state bytes, so the replay's gain should grow with the batch."""
    import torch

    from hybrid_model_ssm_gdn_b200 import ReplaySSM, conv_mamba2_step, make_config
    dev, bf = torch.device("cuda"), torch.bfloat16
    stream = torch.cuda.current_stream()
    out = {"workload": "mamba2 decode, 128 heads, P 64, N 128, 8 groups, L 16, bf16 inputs, fp32 state; batch sweep"}
    for Bt in batches:
        wl = WL.replace(batch=Bt)
        p = mamba2_params(wl)
        A, D = torch.from_numpy(p["A"]).to(dev), torch.from_numpy(p["D"]).to(dev)
        S0 = torch.from_numpy(mamba2_initial_state(wl)).to(dev)
        pool = [{k: torch.from_numpy(v).to(dev).to(bf) for k, v in mamba2_step_inputs(wl, t).items()} for t in range(4)]
        y = torch.empty(Bt, wl.nheads, wl.headdim, device=dev)
        layer = ReplaySSM("mamba2", Bt, wl.nheads, wl.headdim, wl.dstate, wl.ngroups, wl.window, 0, bf, A=A, D=D)
        layer.load_checkpoint(S0)

        def step(i):
            t = pool[i % 4]
            layer.mamba2_step(t["x"], t["B"], t["C"], t["dt"], y)

        for i in range(2 * wl.window):
            step(i)
        K = wl.window * windows_timed
        ms = timed(step, K, stream)
        err = layer.get_error()
        del layer
        cfg = make_config("mamba2", Bt, wl.nheads, wl.headdim, wl.dstate, wl.ngroups, wl.window, 0, bf, A=A, D=D)
        S = S0.clone()

        def conv(i):
            t = pool[i % 4]
            conv_mamba2_step(cfg, S, t["x"], t["B"], t["C"], t["dt"], y)

        for i in range(8):
            conv(i)
        ms_conv = timed(conv, K, stream)
        del S, S0
        out[f"B{Bt}"] = {"replay_ms_per_step": ms, "conventional_ms_per_step": ms_conv, "speedup": ms_conv / ms,
                         "replay_tokens_per_s": Bt / (ms * 1e-3), "device_error": err}
    return out


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=4096)
    ap.add_argument("--warmup", type=int, default=64)
    ap.add_argument("--impl", default="rssm", choices=["rssm", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--mode", action="append", default=None,
                    help="with --only precision: run only this checkpoint/read mode (e.g. f32/nvfp4); repeatable")
    ap.add_argument("--no-extra", action="store_true", help="skip the GDN, speculative-verify, precision and read-skipping sections")
    ap.add_argument("--only", choices=["gdn", "verify", "verify-mamba2", "verify-gdn", "window", "batch",
                                                  "precision", "skip", "skip-mamba2", "graph"], default=None,
                    help="run only one extra section and print its JSON (for profiling runs)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))

    if args.impl == "reference":
        # the reference arm is the CPU oracle, on rank 0 only; other ranks exit without work
        if rank == 0:
            print(json.dumps(reference_arm(args)))
        return

    if args.only is not None:
        if rank == 0:
            out = (gdn_section(args.steps) if args.only == "gdn" else
                   verify_section(args.steps) if args.only == "verify" else
                   verify_section(args.steps, (args.only.split("-")[1],)) if args.only.startswith("verify-") else
                   batch_section() if args.only == "batch" else
                   precision_section(modes=args.mode) if args.only == "precision" else
                   skip_section() if args.only == "skip" else
                   skip_mamba2_section() if args.only == "skip-mamba2" else
                   graph_section() if args.only == "graph" else window_section())
            print(json.dumps(out))
        return

    if world > 1:
        import datetime

        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    res = run_gpu(args, rank, world)
    if rank == 0 and world == 1 and not args.no_extra:
        res["gdn"] = gdn_section(min(args.steps, 1024))
        res["verify"] = verify_section(512)
        res["precision"] = precision_section()
        res["skip"] = skip_section()
        res["skip_mamba2"] = skip_mamba2_section()
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        res["cpu_baseline"] = cpu_baseline()
    if rank == 0:
        print(json.dumps(res))
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
