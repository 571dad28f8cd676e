"""Mamba-2 replay decode on the GPU vs the float64 oracle (parity tests; need a B200)."""

import numpy as np
import pytest

from gpu_harness import TOL_F32, Pair, head_rel_err
from synth import (MAMBA2_120B, MAMBA2_TINY, SPEC_MAMBA2_B512, accepted_lengths, mamba2_draft_inputs,
                   mamba2_step_inputs)

pytestmark = pytest.mark.gpu


def run_steps(p, steps, check_every=1, start=0):
    worst = 0.0
    for t in range(start, start + steps):
        y, y_ref, y_true = p.step(mamba2_step_inputs(p.wl, t))
        err = head_rel_err(y, y_true)
        worst = max(worst, err.max())
        assert err.max() <= TOL_F32, f"step {t}: rel err {err.max():.3e}"
        if check_every and (t + 1) % check_every == 0:
            p.check_bookkeeping()
    return worst


def test_tiny_every_step(cuda_ok):
    """Tiny workload (batch 4, 8 heads, P 64, N 128, L 16, fp32 inputs, zero checkpoint), 64 steps."""
    p = Pair(MAMBA2_TINY)
    run_steps(p, MAMBA2_TINY.steps)
    p.check_checkpoint()
    assert p.gpu.get_error() == (0, -1)


@pytest.mark.parametrize("L", [1, 4, 8, 32])
def test_window_sweep(cuda_ok, L):
    wl = MAMBA2_TINY.replace(window=L, init="normal", in_dtype="bf16", ngroups=2)
    p = Pair(wl)
    run_steps(p, 40)
    p.check_checkpoint()


def test_ragged_units_and_rows(cuda_ok):
    """More units than SMs and not a multiple of them; P = 40 rows (a partly filled tile)."""
    wl = MAMBA2_TINY.replace(batch=5, nheads=64, headdim=40, ngroups=4, init="normal", in_dtype="bf16")
    p = Pair(wl)
    run_steps(p, 34, check_every=17)
    p.check_checkpoint()


def test_fewer_units_than_sms(cuda_ok):
    wl = MAMBA2_TINY.replace(batch=3, nheads=2, headdim=8, ngroups=1, init="normal", in_dtype="bf16")
    p = Pair(wl)
    run_steps(p, 20)


@pytest.mark.parametrize("in_dtype", ["bf16", "f32"])
@pytest.mark.parametrize("T", [1, 4, 8])
def test_verify_commit_random(cuda_ok, T, in_dtype):
    """bf16 inputs with T > 4 take the tensor-core output path; fp32 inputs and T <= 4 the CUDA-core one."""
    wl = SPEC_MAMBA2_B512.replace(batch=6, nheads=16, ngroups=2, in_dtype=in_dtype)
    p = Pair(wl, max_draft=T)
    step = 0
    for rnd in range(12):
        y, y_ref, y_true = p.verify(T, mamba2_draft_inputs(wl, rnd, T))
        assert head_rel_err(y, y_true).max() <= TOL_F32
        p.check_bookkeeping()
        p.commit(accepted_lengths(wl, rnd, T))
        p.check_bookkeeping()
        if rnd % 3 == 2:
            for _ in range(3):
                y, y_ref, y_true = p.step(mamba2_step_inputs(wl, step))
                step += 1
                assert head_rel_err(y, y_true).max() <= TOL_F32
        p.check_bookkeeping()
    assert p.gpu.get_error() == (0, -1)


@pytest.mark.parametrize("T", [3, 8])
def test_verify_long_window_ragged_rows(cuda_ok, T):
    """L = 32 (up to 40 records per verify: three 16-record steps), P = 40 (five active row groups)."""
    wl = SPEC_MAMBA2_B512.replace(batch=5, nheads=20, headdim=40, ngroups=2, window=32)
    p = Pair(wl, max_draft=T)
    for rnd in range(14):
        y, _, y_true = p.verify(T, mamba2_draft_inputs(wl, rnd, T))
        assert head_rel_err(y, y_true).max() <= TOL_F32
        p.commit(accepted_lengths(wl, rnd, T))
        p.check_bookkeeping()
    p.check_checkpoint()
    assert p.gpu.get_error() == (0, -1)


def test_commit_full_window_then_prefold(cuda_ok):
    wl = MAMBA2_TINY.replace(batch=2, nheads=4, window=8, init="normal", in_dtype="bf16")
    p = Pair(wl, max_draft=4)
    run_steps(p, 6)
    for rnd, acc in enumerate((4, 4)):      # 6 + 4 > 8 pre-folds; then 4 + 4 == 8 fills the window
        y, _, y_true = p.verify(4, mamba2_draft_inputs(wl, rnd, 4))
        assert head_rel_err(y, y_true).max() <= TOL_F32
        p.commit(np.full(wl.batch, acc))
        p.check_bookkeeping()
    assert np.all(p.orc.count == 8)
    run_steps(p, 10, start=100)              # first step pre-folds the full window
    p.check_checkpoint()


def test_flush_mask(cuda_ok):
    wl = MAMBA2_TINY.replace(batch=4, nheads=4, init="normal", in_dtype="bf16")
    p = Pair(wl)
    run_steps(p, 5)
    p.flush(np.array([1, 0, 1, 0]))
    p.check_bookkeeping()
    p.check_checkpoint()
    run_steps(p, 20, start=5)
    p.flush()
    p.check_bookkeeping()
    p.check_checkpoint()


def test_device_errors_leave_state_untouched(cuda_ok):
    from hybrid_model_ssm_gdn_b200 import abi
    wl = MAMBA2_TINY.replace(batch=3, nheads=4, init="normal", in_dtype="bf16")
    p = Pair(wl, max_draft=2)
    run_steps(p, 3)
    p.commit(np.zeros(3, np.int32))                      # no verify pending anywhere
    assert p.gpu.get_error() == (abi.DEV_NO_VERIFY, 0)
    p.check_bookkeeping()
    p2 = Pair(wl, max_draft=2)
    p2.verify(2, mamba2_draft_inputs(wl, 0, 2))
    p2.commit(np.array([1, 3, 2]))                       # sequence 1 accepts more than T
    assert p2.gpu.get_error() == (abi.DEV_ACCEPTED, 1)
    p2.check_bookkeeping()
    y, _, y_true = p2.step(mamba2_step_inputs(wl, 0))    # sequence 1 still has its verify pending
    ok = np.array([0, 2])
    assert head_rel_err(y[ok], y_true[ok]).max() <= TOL_F32
    assert p2.gpu.get_error() == (abi.DEV_PENDING, 1)    # lowest (sequence, code), sticky
    assert p2.orc.err == (1, abi.DEV_PENDING)
    p2.check_bookkeeping()


def test_calls_before_load_are_refused(cuda_ok):
    """Until the first checkpoint load the arena is undefined: decode, commit and error reads are refused."""
    import torch

    from hybrid_model_ssm_gdn_b200 import ReplaySSM, abi
    wl = MAMBA2_TINY.replace(batch=2, nheads=4, in_dtype="bf16")
    from synth import mamba2_params
    p = mamba2_params(wl)
    layer = ReplaySSM("mamba2", wl.batch, wl.nheads, wl.headdim, 128, wl.ngroups, wl.window, 2, torch.bfloat16,
                      A=torch.from_numpy(p["A"]), D=torch.from_numpy(p["D"]))
    d = {k: torch.from_numpy(v).cuda().to(torch.bfloat16) for k, v in mamba2_step_inputs(wl, 0).items()}
    for call in (lambda: layer.mamba2_step(d["x"], d["B"], d["C"], d["dt"]),
                 lambda: layer.commit(torch.zeros(wl.batch, dtype=torch.int32, device="cuda")),
                 lambda: layer.flush(), lambda: layer.get_error()):
        with pytest.raises(abi.RSSMError) as ei:
            call()
        assert ei.value.status == 3
    layer.load_checkpoint(torch.zeros(wl.batch, wl.nheads, wl.headdim, 128, device="cuda"))
    layer.mamba2_step(d["x"], d["B"], d["C"], d["dt"])
    assert layer.get_error() == (0, -1)


@pytest.mark.slow
def test_full_size_sampled(cuda_ok):
    """The 120B-class Mamba-2 layer (batch 256, 128 heads, 1 GiB checkpoint), 1024 steps, sampled heads."""
    wl = MAMBA2_120B
    p = Pair(wl, seq_ids=[0, 77, 255], head_ids=[0, 1, 15, 16, 64, 127])
    worst = 0.0
    for t in range(wl.steps):
        y, y_ref, y_true = p.step(mamba2_step_inputs(wl, t))
        err = head_rel_err(y, y_true).max()
        worst = max(worst, err)
        assert err <= TOL_F32, f"step {t}: {err:.3e}"
        if t % 97 == 0:
            p.check_bookkeeping()
    p.check_bookkeeping()
    p.check_checkpoint()
    print(f"worst rel err {worst:.3e}")


@pytest.mark.slow
@pytest.mark.parametrize("T", [4, 8])
def test_speculative_full_size_sampled(cuda_ok, T):
    """Speculative verify + commit on the Mamba-2 shape at batch 512 (2 GiB checkpoint, 128 heads, 8 groups,
    L 16): 64 rounds with the seeded accepted lengths, so every round some of the 4096 units pre-fold.  Sampled
    sequences 0, 255, 511 and one head in each of the 8 groups: every draft output within the fp32 bound, the
    bookkeeping bit-exact after every call, the ring byte-exact and the checkpoint within 1e-5 every 16 rounds."""
    wl = SPEC_MAMBA2_B512
    heads = [0, 17, 35, 50, 64, 81, 99, 127]                  # groups 0..7
    p = Pair(wl, seq_ids=[0, 255, 511], head_ids=heads, max_draft=T)
    worst, prefolds = 0.0, 0
    for rnd in range(64):
        before = p.orc.epoch.copy()
        y, _, y_true = p.verify(T, mamba2_draft_inputs(wl, rnd, T))
        prefolds += int(np.sum(p.orc.epoch != before))
        err = head_rel_err(y, y_true).max()
        worst = max(worst, err)
        assert err <= TOL_F32, f"round {rnd}: {err:.3e}"
        p.check_bookkeeping(ring=False)
        p.commit(accepted_lengths(wl, rnd, T))
        p.check_bookkeeping(ring=(rnd % 16 == 15))
        if rnd % 16 == 15:
            p.check_checkpoint()
    assert prefolds >= 3 * (64 * T // 2 // wl.window) // 2     # about one pre-fold per 16 / (T / 2) rounds each
    assert p.gpu.get_error() == (0, -1)
    print(f"T={T}: worst rel err {worst:.3e}, pre-folds on the sampled sequences {prefolds}")


# ------------------------------------------------------------------------------------ decay-aware skipping

FAST_M2 = MAMBA2_TINY.replace(batch=5, nheads=16, ngroups=2, init="normal", in_dtype="bf16", decay_scale=8.0)


@pytest.mark.parametrize("in_dtype", ["bf16", "f32"])
def test_skip_steps_match_oracle(cuda_ok, in_dtype):
    """Steps over three windows with tau = 1e-2 on fast-decaying heads (A times 8): flags bit-exact after every
    call, outputs and checkpoints against the oracle that skips the same reads, some heads skipped and some not."""
    wl = FAST_M2.replace(in_dtype=in_dtype)
    p = Pair(wl, skip_tau=1e-2)
    skipped, calls = 0, 0
    for t in range(3 * wl.window + 5):
        skipped += int(p.orc.skip.sum())
        calls += p.orc.skip.size
        y, y_ref, _ = p.step(mamba2_step_inputs(wl, t))
        assert head_rel_err(y, y_ref).max() <= TOL_F32, f"step {t}"
        p.check_bookkeeping(ring=(t % 8 == 7))
    assert 0 < skipped < calls
    p.check_checkpoint()
    assert p.gpu.get_error() == (0, -1)


@pytest.mark.parametrize("T", [4, 8])
def test_skip_verify_commit_flush(cuda_ok, T):
    """Verify/commit rounds (T = 8 takes the tensor-core output path), steps between them and a flush, with
    skipping on: outputs against the skipping oracle, flags bit-exact after every call."""
    wl = FAST_M2
    p = Pair(wl, max_draft=T, skip_tau=2e-2)
    rng = np.random.default_rng(4)
    skipped = 0
    for rnd in range(12):
        skipped += int(p.orc.skip.sum())
        y, y_ref, _ = p.verify(T, mamba2_draft_inputs(wl, rnd, T))
        assert head_rel_err(y, y_ref).max() <= TOL_F32, f"round {rnd}"
        p.check_bookkeeping(ring=False)
        p.commit(accepted_lengths(wl, rnd, T))
        for k in range(int(rng.integers(0, 4))):
            y, y_ref, _ = p.step(mamba2_step_inputs(wl, 100 + 4 * rnd + k))
            assert head_rel_err(y, y_ref).max() <= TOL_F32
        p.check_bookkeeping(ring=True)
    assert skipped > 0
    p.flush()
    p.check_bookkeeping()
    p.check_checkpoint()
    assert p.gpu.get_error() == (0, -1)
