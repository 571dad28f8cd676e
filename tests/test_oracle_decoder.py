"""Pins for oracle.decoder: window independence, speculative-commit invariant, bookkeeping edge cases."""

import numpy as np
import pytest

from oracle.decoder import ERR_ACCEPTED, ERR_NO_VERIFY, ERR_PENDING, ReplayOracle
from synth import (GDN_B256, MAMBA2_TINY, accepted_lengths, gdn_draft_inputs, gdn_initial_state,
                   gdn_step_inputs, mamba2_draft_inputs, mamba2_params, mamba2_step_inputs)

M_WL = MAMBA2_TINY.replace(batch=3, nheads=4, headdim=8, dstate=32, init="normal")
G_WL = GDN_B256.replace(batch=3, nheads=2, dk=16, dv=8)


def _rel(a, b):
    return np.linalg.norm(a - b) / np.linalg.norm(b)


def _mamba(L, **kw):
    rng = np.random.default_rng(0)
    S0 = rng.standard_normal((M_WL.batch, M_WL.nheads, M_WL.headdim, M_WL.dstate)) * 0.05
    return ReplayOracle("mamba2", S0, L, nheads=M_WL.nheads, ngroups=M_WL.ngroups, params=mamba2_params(M_WL), **kw)


def _gdn(L, **kw):
    return ReplayOracle("gdn", gdn_initial_state(G_WL), L, nheads=G_WL.nheads, **kw)


@pytest.mark.parametrize("L", [1, 4, 8, 16, 32])
@pytest.mark.parametrize("kind", ["mamba2", "gdn"])
def test_window_independence_and_fold_schedule(kind, L):
    o = _mamba(L) if kind == "mamba2" else _gdn(L)
    gen = (lambda t: mamba2_step_inputs(M_WL, t)) if kind == "mamba2" else (lambda t: gdn_step_inputs(G_WL, t))
    for t in range(40):
        y, y_true = o.step(gen(t))
        assert _rel(y, y_true) < 2e-6                       # fp32 checkpoint at folds, f64 elsewhere
        np.testing.assert_array_equal(o.count, (t + 1) % L)
        np.testing.assert_array_equal(o.epoch, (t + 1) // L)
    assert o.err is None


@pytest.mark.parametrize("kind", ["mamba2", "gdn"])
@pytest.mark.parametrize("T", [1, 4, 8])
def test_commit_prefix_equals_decoding_prefix(kind, T):
    """verify(T) + commit(a) then decoding on == decoding only the first a drafts, for every a in 0..T."""
    L = 8
    for a in range(T + 1):
        spec = _mamba(L) if kind == "mamba2" else _gdn(L)
        plain = _mamba(L) if kind == "mamba2" else _gdn(L)
        step = (lambda t: mamba2_step_inputs(M_WL, t)) if kind == "mamba2" else (lambda t: gdn_step_inputs(G_WL, t))
        drafts = mamba2_draft_inputs(M_WL, 0, T) if kind == "mamba2" else gdn_draft_inputs(G_WL, 0, T)
        for t in range(5):                                  # leave count = 5 so that verify may pre-fold
            spec.step(step(t))
            plain.step(step(t))
        yv, yv_true = spec.verify(T, drafts)
        spec.commit(np.full(M_WL.batch, a))
        for j in range(a):
            one = {k: v[:, j] for k, v in drafts.items()}
            yp, yp_true = plain.step(one)
            np.testing.assert_allclose(yv_true[:, j], yp_true, rtol=1e-12, atol=1e-12)
            assert _rel(yv[:, j], yp) < 2e-6
        for t in range(5, 25):
            ys, ys_true = spec.step(step(t))
            yp, yp_true = plain.step(step(t))
            np.testing.assert_allclose(ys_true, yp_true, rtol=1e-11, atol=1e-12)
            assert _rel(ys, yp) < 2e-6
        np.testing.assert_allclose(spec.S_true, plain.S_true, rtol=1e-11, atol=1e-13)
        assert spec.err is None


def test_verify_prefold_and_commit_to_full_window():
    L, T = 8, 4
    o = _mamba(L)
    for t in range(6):
        o.step(mamba2_step_inputs(M_WL, t))
    np.testing.assert_array_equal(o.count, 6)
    o.verify(T, mamba2_draft_inputs(M_WL, 0, T))            # 6 + 4 > 8: fold the 6 committed records first
    np.testing.assert_array_equal(o.count, 0)
    np.testing.assert_array_equal(o.epoch, 1)
    np.testing.assert_array_equal(o.pending, T)
    o.commit(np.full(M_WL.batch, T))
    np.testing.assert_array_equal(o.count, 4)
    o.verify(T, mamba2_draft_inputs(M_WL, 1, T))            # 4 + 4 == 8: no fold
    o.commit(np.full(M_WL.batch, T))
    np.testing.assert_array_equal(o.count, 8)                # a full window after commit, not yet folded
    np.testing.assert_array_equal(o.epoch, 1)
    y, y_true = o.step(mamba2_step_inputs(M_WL, 6))          # pre-fold, then append
    np.testing.assert_array_equal(o.count, 1)
    np.testing.assert_array_equal(o.epoch, 2)
    assert _rel(y, y_true) < 2e-6


def test_bookkeeping_errors_leave_state_untouched():
    o = _mamba(8)
    o.step(mamba2_step_inputs(M_WL, 0))
    o.commit(np.zeros(M_WL.batch, np.int32))                 # commit without verify
    assert o.err == (0, ERR_NO_VERIFY)
    o2 = _gdn(8)
    o2.verify(4, gdn_draft_inputs(G_WL, 0, 4))
    y, _ = o2.step(gdn_step_inputs(G_WL, 0))                 # step while verify pending
    assert o2.err == (0, ERR_PENDING) and np.all(np.isnan(y))
    np.testing.assert_array_equal(o2.count, 0)
    o2.flush()
    np.testing.assert_array_equal(o2.count, 0)
    o2.commit(np.array([1, 7, 2]))                           # sequence 1 asks for more than T
    np.testing.assert_array_equal(o2.count, [1, 0, 2])
    np.testing.assert_array_equal(o2.pending, [0, 4, 0])
    assert o2.err == (0, ERR_PENDING)                        # lowest failing sequence is kept
    o3 = _gdn(8)
    o3.verify(2, gdn_draft_inputs(G_WL, 0, 2))
    o3.commit(np.array([0, 3, 1]))
    assert o3.err == (1, ERR_ACCEPTED)


def test_flush_masks_and_random_speculation():
    """A long random verify/commit/step/flush schedule keeps the truth-side invariant."""
    L, T = 16, 4
    o = _mamba(L)
    step_t, rnd = 0, 0
    rng = np.random.default_rng(3)
    for it in range(30):
        op = rng.integers(0, 3)
        if op == 0:
            o.step(mamba2_step_inputs(M_WL, step_t)); step_t += 1
        elif op == 1:
            y, y_true = o.verify(T, mamba2_draft_inputs(M_WL, rnd, T))
            assert _rel(y, y_true) < 2e-6
            o.commit(accepted_lengths(M_WL, rnd, T)); rnd += 1
        else:
            mask = rng.integers(0, 2, M_WL.batch).astype(bool)
            before = o.count.copy()
            o.flush(mask)
            np.testing.assert_array_equal(o.count, np.where(mask, 0, before))
        assert np.all(o.count <= L) and o.err is None


@pytest.mark.parametrize("kind", ["mamba2", "gdn"])
def test_read_copy_never_reenters_recurrence(kind):
    """Separate precision: the checkpoint and fold-step outputs are those of the fp32 run, bit for bit."""
    L = 4
    ref = _mamba(L) if kind == "mamba2" else _gdn(L)
    sep = _mamba(L, read="nvfp4") if kind == "mamba2" else _gdn(L, read="nvfp4")
    shared = _mamba(L, read="shared_nvfp4") if kind == "mamba2" else _gdn(L, read="shared_nvfp4")
    gen = (lambda t: mamba2_step_inputs(M_WL, t)) if kind == "mamba2" else (lambda t: gdn_step_inputs(G_WL, t))
    err_sep = []
    for t in range(24):
        inp = gen(t)
        y_ref, y_true = ref.step(inp)
        y_sep, _ = sep.step(inp)
        shared.step(inp)
        np.testing.assert_array_equal(sep.hp, ref.hp)
        if (t + 1) % L == 0:
            np.testing.assert_array_equal(y_sep, y_ref)     # fold step: full-precision state
        else:
            err_sep.append(_rel(y_sep, y_true))
        np.testing.assert_array_equal(shared.hp, shared.rd)
    assert 0 < max(err_sep) < 0.2


def test_fp16_checkpoint_is_on_the_fp16_grid():
    o = _gdn(4, hp="f16sr", seed=123)
    for t in range(8):
        o.step(gdn_step_inputs(G_WL, t))
    np.testing.assert_array_equal(o.hp.astype(np.float16).astype(np.float64), o.hp)
    # same seed, same words: deterministic; different seed: different roundings
    o2 = _gdn(4, hp="f16sr", seed=123)
    o3 = _gdn(4, hp="f16sr", seed=124)
    for t in range(8):
        o2.step(gdn_step_inputs(G_WL, t))
        o3.step(gdn_step_inputs(G_WL, t))
    np.testing.assert_array_equal(o.hp, o2.hp)
    assert np.any(o.hp != o3.hp)


def test_fp8_checkpoint_tiles_and_separate_read_copy():
    """FP8 checkpoint: each 64-row tile of the stored state is E4M3 grid values times one scale (its largest
    magnitude / 448), and an NVFP4 read copy beside it leaves that checkpoint unchanged."""
    import torch
    grid = torch.arange(0, 0x7F, dtype=torch.uint8).view(torch.float8_e4m3fn).float().numpy().astype(np.float64)
    o = _gdn(4, hp="f8sr", seed=5)
    sep = _gdn(4, hp="f8sr", read="nvfp4", seed=5)
    for t in range(8):
        o.step(gdn_step_inputs(G_WL, t))
        sep.step(gdn_step_inputs(G_WL, t))
        np.testing.assert_array_equal(sep.hp, o.hp)
    rows = o.hp.shape[-2]
    for r0 in range(0, rows, 64):
        tile = o.hp[..., r0:r0 + 64, :]
        s = np.abs(tile).max(axis=(-1, -2)) / 448.0
        y = np.abs(tile) / s[..., None, None]
        nearest = grid[np.clip(np.searchsorted(grid, y), 0, len(grid) - 1)]
        below = grid[np.clip(np.searchsorted(grid, y) - 1, 0, len(grid) - 1)]
        dist = np.minimum(np.abs(nearest - y), np.abs(below - y))
        assert np.all(dist <= 1e-5 * np.maximum(y, 2.0 ** -9))


# ------------------------------------------------------------------------------------ decay-aware skipping

def _halving_inputs(t, zero_alpha_at=None):
    """GDN step inputs with alpha = 1/2 for every head (products exact in fp32); optionally alpha = 0 once."""
    inp = gdn_step_inputs(G_WL, t)
    inp["alpha"] = np.full_like(inp["alpha"], 0.5 if t != zero_alpha_at else 0.0)
    return inp


def test_skip_flags_follow_the_gate_product_and_bound_the_dropped_term():
    """alpha = 1/2 makes the product over n committed records exactly 2^-n, so with tau = 1.5 * 2^-5 a head is
    flagged exactly when 5 or more records are committed, and a fold clears it.  Within the first window the
    skipping oracle differs from the non-skipping one only on calls that read a set flag, and there by at most
    tau * ||S0|| * q_scale * ||q|| per head (the whole dropped term S0 u0)."""
    L, tau = 8, 1.5 * 2.0 ** -5
    sk, ref = _gdn(L, skip_tau=tau), _gdn(L)
    S0 = gdn_initial_state(G_WL)
    for t in range(2 * L + 3):
        inp = _halving_inputs(t)
        before = sk.skip.copy()
        y, _ = sk.step(inp)
        y0, _ = ref.step(inp)
        n = (t + 1) % L
        np.testing.assert_array_equal(sk.skip, np.full((G_WL.batch, G_WL.nheads), n >= 5))
        if t < L - 1:                                   # same checkpoint on both sides until the first fold
            d = np.linalg.norm(y - y0, axis=-1)
            bound = tau * np.linalg.norm(S0, axis=(-2, -1)) * np.linalg.norm(inp["q"], axis=-1)
            assert np.all(d[~before] == 0)
            assert np.all(d[before] <= bound[before] * (1 + 1e-9))
            assert np.all(d[before] > 0)


def test_skip_with_a_zero_gate_changes_nothing():
    """With alpha = 0 at some token the checkpoint's true contribution after it is exactly zero, so skipping
    it (and writing the next checkpoint from the buffer alone) gives the non-skipping oracle's results
    exactly: the skip removes the checkpoint term and nothing else, head by head."""
    L = 8
    sk, ref = _gdn(L, skip_tau=1e-3), _gdn(L)
    for t in range(3 * L):
        inp = gdn_step_inputs(G_WL, t)
        if t % L == 2:
            inp["alpha"][:, 1] = 0.0                    # head 1 only
        y, _ = sk.step(inp)
        y0, _ = ref.step(inp)
        np.testing.assert_array_equal(y, y0)
        assert not sk.skip[:, 0].any()
        np.testing.assert_array_equal(sk.skip[:, 1], (t % L) >= 2 and (t % L) != L - 1)
    np.testing.assert_array_equal(sk.hp, ref.hp)


def test_skip_flags_under_verify_commit_and_flush():
    """Verify reads the flags but sets them from the committed records only (drafts excluded); commit leaves
    them; a pre-fold or a flush clears them."""
    L, tau = 8, 1.5 * 2.0 ** -5
    o = _gdn(L, skip_tau=tau)
    for t in range(6):
        o.step(_halving_inputs(t))
    assert o.skip.all()                                 # 6 records: 2^-6 < tau
    drafts = gdn_draft_inputs(G_WL, 0, 2)
    drafts["alpha"] = np.full_like(drafts["alpha"], 0.5)
    o.verify(2, drafts)                                 # 6 + 2 <= 8: no pre-fold
    assert o.skip.all()
    o.commit(np.full(G_WL.batch, 2))
    assert o.skip.all() and (o.count == 8).all()
    o.verify(2, drafts)                                 # 8 + 2 > 8: pre-fold, nothing committed after it
    assert not o.skip.any()
    o.commit(np.zeros(G_WL.batch, np.int64))
    for t in range(5):
        o.step(_halving_inputs(10 + t))
    assert o.skip.all()
    o.flush()
    assert not o.skip.any() and (o.count == 0).all()


# ------------------------------------------------------------------------------------ Mamba-2 decay-aware skipping

M2_TAU = float(np.exp(-2.25))          # ln(tau) lies between -2.5 and -2.0


def _mamba_A(L, A, **kw):
    """The Mamba-2 oracle of _mamba with per-head A replaced (fp32 values)."""
    p = dict(mamba2_params(M_WL))
    p["A"] = np.broadcast_to(np.asarray(A, np.float32), (M_WL.nheads,)).copy()
    rng = np.random.default_rng(0)
    S0 = rng.standard_normal((M_WL.batch, M_WL.nheads, M_WL.headdim, M_WL.dstate)) * 0.05
    return ReplayOracle("mamba2", S0, L, nheads=M_WL.nheads, ngroups=M_WL.ngroups, params=p, **kw), S0


def _const_dt(t, dt=0.0625, draft=None):
    inp = mamba2_step_inputs(M_WL, t) if draft is None else mamba2_draft_inputs(M_WL, t, draft)
    inp["dt"] = np.full_like(inp["dt"], dt)
    return inp


def test_mamba2_skip_flags_follow_the_decay_and_bound_the_dropped_term():
    """A = -8 and dt = 1/16 make A * (sum of dt) over n committed records exactly -n/2 in fp32, so with
    ln(tau) = -2.25 a head is flagged exactly when 5 or more records are committed, and a fold clears it.
    Within the first window the skipping oracle differs from the non-skipping one only on calls that read a
    set flag, and there by at most tau * ||S0|| * ||C|| per head (the whole dropped term exp(A s) S0 C)."""
    L = 8
    sk, S0 = _mamba_A(L, -8.0, skip_tau=M2_TAU)
    ref, _ = _mamba_A(L, -8.0)
    for t in range(2 * L + 3):
        inp = _const_dt(t)
        before = sk.skip.copy()
        y, _ = sk.step(inp)
        y0, _ = ref.step(inp)
        n = (t + 1) % L
        np.testing.assert_array_equal(sk.skip, np.full((M_WL.batch, M_WL.nheads), n >= 5))
        if t < L - 1:                                   # same checkpoint on both sides until the first fold
            d = np.linalg.norm(y - y0, axis=-1)
            c = np.linalg.norm(inp["C"][:, 0], axis=-1)[:, None]          # one group
            bound = M2_TAU * np.linalg.norm(S0, axis=(-2, -1)) * c
            assert np.all(d[~before] == 0)
            assert np.all(d[before] <= bound[before] * (1 + 1e-9))
            assert np.all(d[before] > 0)


def test_mamba2_skip_with_a_vanishing_decay_changes_nothing():
    """With A dt = -1000 on one head, exp(A dt) is exactly zero in float64, so that head's checkpoint contributes
    nothing once a record is buffered: skipping its read (and folding from the buffer alone) gives the
    non-skipping oracle's outputs and checkpoints exactly, and the other heads are never flagged."""
    L = 8
    A = np.array([-1.0, -1e4, -1.0, -1.0], np.float32)
    sk, _ = _mamba_A(L, A, skip_tau=1e-3)
    ref, _ = _mamba_A(L, A)
    for t in range(3 * L):
        inp = mamba2_step_inputs(M_WL, t)
        inp["dt"][:, 1] = 0.1
        y, _ = sk.step(inp)
        y0, _ = ref.step(inp)
        np.testing.assert_array_equal(y, y0)
        assert not sk.skip[:, [0, 2, 3]].any()
        np.testing.assert_array_equal(sk.skip[:, 1], (t % L) != L - 1)
    np.testing.assert_array_equal(sk.hp, ref.hp)


def test_mamba2_skip_flags_under_verify_commit_and_flush():
    """Verify sets the flags from the committed records only (drafts excluded); commit leaves them; a pre-fold
    or a flush clears them."""
    L = 8
    o, _ = _mamba_A(L, -8.0, skip_tau=M2_TAU)
    for t in range(6):
        o.step(_const_dt(t))
    assert o.skip.all()                                 # 6 records: -3 < -2.25
    o.verify(2, _const_dt(0, draft=2))                  # 6 + 2 <= 8: no pre-fold
    assert o.skip.all()
    o.commit(np.full(M_WL.batch, 2))
    assert o.skip.all() and (o.count == 8).all()
    o.verify(2, _const_dt(1, draft=2))                  # 8 + 2 > 8: pre-fold, nothing committed after it
    assert not o.skip.any()
    o.commit(np.zeros(M_WL.batch, np.int64))
    for t in range(4):
        o.step(_const_dt(10 + t))
    assert not o.skip.any()                             # 4 records: -2 > -2.25
    o.step(_const_dt(20))
    assert o.skip.all()
    o.flush()
    assert not o.skip.any() and (o.count == 0).all()


def test_skip_threshold_is_the_fp32_log():
    """ln(tau) is the double-precision log of the fp32 threshold, rounded once to fp32."""
    import math
    o, _ = _mamba_A(8, -1.0, skip_tau=1e-2)
    assert o.ln_tau == np.float32(math.log(float(np.float32(1e-2))))
    assert o.ln_tau.dtype == np.float32 and abs(float(o.ln_tau) - math.log(1e-2)) < 1e-6
