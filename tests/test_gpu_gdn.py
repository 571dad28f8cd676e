"""Gated DeltaNet replay decode on the GPU vs the float64 oracle (parity tests; need a B200)."""

import numpy as np
import pytest
import torch

from gpu_harness import TOL_F32, Pair, head_rel_err
from oracle import lowprec as lp
from oracle.philox import sr_words
from synth import GDN_B256, GDN_LOWPREC, accepted_lengths, gdn_draft_inputs, gdn_step_inputs

pytestmark = pytest.mark.gpu

SMALL = GDN_B256.replace(batch=4, nheads=4)


def run_steps(p, steps, start=0, check_every=1, tol=TOL_F32, ref="true"):
    worst = 0.0
    for t in range(start, start + steps):
        y, y_ref, y_true = p.step(gdn_step_inputs(p.wl, t))
        err = head_rel_err(y, y_true if ref == "true" else y_ref)
        worst = max(worst, err.max())
        assert err.max() <= tol, f"step {t}: rel err {err.max():.3e}"
        if check_every and (t + 1) % check_every == 0:
            p.check_bookkeeping()
    return worst


def test_small_every_step(cuda_ok):
    p = Pair(SMALL)
    run_steps(p, 48)
    p.check_checkpoint()
    assert p.gpu.get_error() == (0, -1)


@pytest.mark.parametrize("L", [1, 4, 8, 32])
def test_window_sweep(cuda_ok, L):
    p = Pair(SMALL.replace(window=L, batch=3))
    run_steps(p, 40)
    p.check_checkpoint()


def test_ragged_rows_and_heads(cuda_ok):
    """d_v = 40 (one partial 64-row tile), 6 heads (a partial unit), fp32 inputs, 5 sequences."""
    wl = SMALL.replace(batch=5, nheads=6, dv=40, in_dtype="f32")
    p = Pair(wl)
    run_steps(p, 34, check_every=17)
    p.check_checkpoint()


@pytest.mark.parametrize("dv,nheads,L,T", [(40, 3, 16, 4), (96, 5, 16, 8), (128, 3, 5, 4), (72, 2, 1, 1),
                                            (128, 2, 16, 2), (96, 3, 12, 8)])
def test_chunked_fold_shapes(cuda_ok, dv, nheads, L, T):
    """The fold of an fp32 checkpoint with bf16 inputs runs in the chunked form (Z = S K^T, U = RT T^T,
    S' = a S + W K on the tensor cores, one group of four warps per tile): partial 16-row blocks (d_v = 40, 72),
    a 32-row tile (96), windows that fold 16, 12, 5 and 1 records, and verify rounds of 1 to 8 drafts whose
    pre-folds take every committed count from 1 to L (their outputs then come from the chunked fold result)."""
    wl = SMALL.replace(batch=3, nheads=nheads, dv=dv, window=L)
    p = Pair(wl, max_draft=T)
    run_steps(p, 2 * L + 3, check_every=L)
    p.check_checkpoint()
    for rnd in range(8):
        y, _, y_true = p.verify(T, gdn_draft_inputs(wl, rnd, T))
        assert head_rel_err(y, y_true).max() <= TOL_F32
        p.commit(accepted_lengths(wl, rnd, T))
        p.check_bookkeeping()
    p.check_checkpoint()
    assert p.gpu.get_error() == (0, -1)


def test_many_units(cuda_ok):
    """More units than SMs, not a multiple of them (151 sequences x 2 units)."""
    wl = SMALL.replace(batch=151, nheads=8)
    p = Pair(wl, seq_ids=[0, 75, 150])
    run_steps(p, 20, check_every=10)
    p.check_checkpoint()


@pytest.mark.parametrize("T", [1, 2, 4, 8])
def test_verify_commit_random(cuda_ok, T):
    wl = SMALL.replace(batch=5, nheads=3)
    p = Pair(wl, max_draft=T)
    step = 0
    for rnd in range(10):
        y, _, y_true = p.verify(T, gdn_draft_inputs(wl, rnd, T))
        assert head_rel_err(y, y_true).max() <= TOL_F32
        p.check_bookkeeping()
        p.commit(accepted_lengths(wl, rnd, T))
        p.check_bookkeeping()
        if rnd % 3 == 1:
            for _ in range(3):
                y, _, y_true = p.step(gdn_step_inputs(wl, step))
                step += 1
                assert head_rel_err(y, y_true).max() <= TOL_F32
    p.check_checkpoint()
    assert p.gpu.get_error() == (0, -1)


@pytest.mark.parametrize("T,in_dtype,L,dv", [(8, "f32", 16, 128), (8, "bf16", 32, 96), (3, "bf16", 32, 96),
                                              (5, "bf16", 8, 128)])
def test_verify_paths(cuda_ok, T, in_dtype, L, dv):
    """bf16 and fp32 inputs, 3 to 8 outputs per row; L = 32 gives up to 40 records per verify, d_v = 96 leaves a
    32-row tile."""
    wl = SMALL.replace(batch=3, nheads=3, window=L, dv=dv, in_dtype=in_dtype)
    p = Pair(wl, max_draft=T)
    for rnd in range(12):
        y, _, y_true = p.verify(T, gdn_draft_inputs(wl, rnd, T))
        assert head_rel_err(y, y_true).max() <= TOL_F32
        p.commit(accepted_lengths(wl, rnd, T))
        p.check_bookkeeping()
    p.check_checkpoint()
    assert p.gpu.get_error() == (0, -1)


def test_flush_mask(cuda_ok):
    p = Pair(SMALL)
    run_steps(p, 5)
    p.flush(np.array([1, 0, 0, 1]))
    p.check_bookkeeping()
    p.check_checkpoint()
    run_steps(p, 12, start=5)
    p.flush()
    p.check_bookkeeping()
    p.check_checkpoint()


# ------------------------------------------------------------------------------------ precision converters

def _edge_state(shape, seed):
    rng = np.random.default_rng(seed)
    S = (rng.standard_normal(shape) * 10.0 ** rng.uniform(-7, 2, shape[:-1] + (1,))).astype(np.float32)
    S[0, 0, 3] = 0.0                                             # a zero row
    S[0, 0, 5, :16] = 0.0                                        # a zero block
    S[0, 1, 7, :4] = [65504.0, -70000.0, 3e-6, -1e-8]            # saturation, fp16 subnormals
    S[0, 1, 9] = np.float16(0.125).astype(np.float32)            # on the fp16 grid
    S[1, 2, 64:] = 0.0                                           # an all-zero 64-row tile (scale 1)
    return S


@pytest.mark.parametrize("hp,read", [("f16sr", "nvfp4"), ("f32", "shared_nvfp4"), ("f16sr", "same"),
                                     ("f8sr", "same"), ("f8sr", "nvfp4"), ("f32", "nvfp4d"), ("f8sr", "nvfp4d")])
def test_load_converters_bit_exact(cuda_ok, hp, read):
    wl = SMALL.replace(batch=2, nheads=3, dv=128)
    S = _edge_state((2, 3, 128, 128), 1)
    p = Pair(wl, hp=hp, read=read, seed=0xABCDEF0123456789, S0=S)
    ex = p.gpu.export(state=True, ring=False)["S"].cpu().numpy()
    if read == "shared_nvfp4":
        np.testing.assert_array_equal(ex, lp.nvfp4_roundtrip_state(S))
    elif hp in ("f16sr", "f8sr"):
        units = (np.arange(2)[:, None] * 3 + np.arange(3)[None, :])
        words = sr_words(0xABCDEF0123456789, units, 0, 128 * 128).reshape(2, 3, 128, 128)
        want = (lp.fp16_stochastic_round(S, words).astype(np.float32) if hp == "f16sr"
                else lp.fp8_quantize_state(S, words)["values"])
        np.testing.assert_array_equal(ex, want)
    if read != "same":
        rc = p.gpu.export_read_copy()
        q = (lp.nvfp4d_quantize_state if read == "nvfp4d" else lp.nvfp4_quantize_state)(S)
        if read == "nvfp4d":
            np.testing.assert_array_equal(p.gpu.export_column_scales().cpu().numpy(), q["colscales"])
        np.testing.assert_array_equal(rc["packed"].cpu().numpy(), q["packed"])
        np.testing.assert_array_equal(rc["scales"].cpu().numpy(), q["scales"])
        np.testing.assert_array_equal(rc["g"].cpu().numpy(), q["g"])


# ------------------------------------------------------------------------------------ separate precision

# Bounds for the low-precision modes, GPU against the oracle in the same mode.
#
# Without stochastic rounding the two differ only in the fold's arithmetic (fp32 on the GPU, float64 in the
# oracle): now and then an element of the new state lands on the other side of an NVFP4 decision, which moves
# it by one E2M1 step (at most a third of its block's maximum).  The converters themselves are pinned bit for
# bit (tests/test_gpu_fold_converters.py).
# * fp32 checkpoint with a separate copy: the copy is re-made from the checkpoint at every fold, so a flip
#   lasts until the next fold and does not feed back.  After each fold the GPU's copy (the quantisation of its
#   exported checkpoint) is compared with the oracle's element by element: every difference is at most one
#   E2M1 step of its block (0.4 of the block maximum allows for a block scale decided the other way too), the
#   differing codes are at most FLIP_CODE_RATE of all, and the outputs of every head whose copy matches
#   are held to the fp32 bound; a head with a flip to TOL_FLIP.
# * shared NVFP4 checkpoint: a flip feeds the next fold, so only the per-head cap and the fraction of
#   outputs above 1e-4 apply.
TOL_FLIP = 1e-2
FLIP_FRACTION = 0.02
FLIP_CODE_RATE = 2e-5   # measured: at most 3 of 1.6 M codes (1.8e-6), small, full-batch and verify cases
TOL_CKPT_G = 1e-5   # tile scales, relative: the bound of the checkpoint after folds
# With stochastic rounding the oracle's trajectory is one sample among many: one rounding decision taken
# differently changes the checkpoint by one fp16 (or E4M3) step, and the trajectories then differ within the
# seed-to-seed spread.  The criterion is the mean error against that spread (at most twice it, plus the fp32
# bound); the per-head cap only catches a gross error.  Measured: at most 1.8e-2 per head, mean at most
# 1.6e-4 against spreads of 3e-3 to 7e-2.
TOL_SR_HEAD = 3e-2


class CopyFlips:
    """Per sampled (sequence, head): does the GPU's read copy differ from the oracle's (fp32 checkpoint with a
    separate NVFP4 copy)?  Re-evaluated after every call that folds; counts the elements whose code or scale
    differs.  The GPU's copy is the quantisation of its exported checkpoint (pinned bit for bit elsewhere), the
    oracle's that of its fp32 checkpoint, so both are formed here by the oracle's quantiser and compared code by
    code (a tile scale differs only by the fold's error: checked, not counted)."""

    def __init__(self, p, read):
        self.p, self.read = p, read
        self.flipped = np.zeros((len(p.seq_ids), len(p.head_ids)), bool)
        self.n_diff = self.n_codes = 0

    def after(self, folded):
        """folded: per sampled sequence, did this call fold (epoch changed)."""
        if not folded.any():
            return
        S_gpu = self.p.selected_state()
        S_orc = np.asarray(self.p.orc.hp, np.float64)[..., :S_gpu.shape[2], :].astype(np.float32)
        quant = lp.nvfp4d_quantize_state if self.read == "nvfp4d" else lp.nvfp4_quantize_state
        qg, qo = quant(S_gpu), quant(S_orc)
        diff = qg["codes"] != qo["codes"]
        diff |= np.repeat(qg["scales"] != qo["scales"], 16, axis=-1)
        if self.read == "nvfp4d":
            diff |= np.repeat(qg["colscales"] != qo["colscales"], 16, axis=-2)[..., :diff.shape[-2], :]
        # the tile scales follow the tile maxima, within the fold's error; with equal codes and block scales such
        # a difference moves every value of the tile by the same small factor and no output by more than it
        assert np.all(np.abs(qg["g"].astype(np.float64) / qo["g"] - 1.0) <= TOL_CKPT_G), "tile scale"
        if self.read == "nvfp4":
            vg, vo = lp.nvfp4_roundtrip_state(S_gpu), lp.nvfp4_roundtrip_state(S_orc)
            bm = np.maximum(np.abs(vg), np.abs(vo)).reshape(*vg.shape[:-1], -1, 16).max(-1)
            step = np.repeat(bm, 16, axis=-1)
            assert np.all(np.abs(vg - vo)[diff] <= 0.4 * step[diff]), "a copy difference larger than one E2M1 step"
        d = diff[folded]
        self.n_diff += int(d.sum())
        self.n_codes += d.size
        self.flipped[folded] = d.any(axis=(-2, -1))

    def rate(self):
        return self.n_diff / max(self.n_codes, 1)


def track_lowprec(wl, hp, read, steps, seq_ids=None, head_ids=None):
    """Steps a low-precision context beside the oracle in the same mode (on the sampled sequences and heads).
    With stochastic rounding the oracle's trajectory is one sample among many, so the GPU is held to the
    spread between two oracle seeds (mean error at most twice the seed-to-seed mean, plus the fp32 bound);
    without it, to rare single-code NVFP4 flips, counted element by element where the checkpoint is fp32.
    Returns the per-output errors."""
    from oracle.decoder import ReplayOracle
    from synth import gdn_initial_state
    p = Pair(wl, seq_ids=seq_ids, head_ids=head_ids, hp=hp, read=read, seed=7)
    other = None
    if hp in ("f16sr", "f8sr"):
        S_sel = gdn_initial_state(wl, seqs=p.seq_ids)[:, p.head_ids]
        other = ReplayOracle("gdn", S_sel, wl.window, nheads=wl.nheads, seq_ids=p.seq_ids, head_ids=p.head_ids,
                             hp=hp, read=read, seed=8)
    errs, spread = [], []
    cap = TOL_SR_HEAD if other is not None else TOL_FLIP
    flips = CopyFlips(p, read) if hp == "f32" and read in ("nvfp4", "nvfp4d") else None
    for t in range(steps):
        inp = gdn_step_inputs(wl, t)
        e0 = p.orc.epoch.copy()
        y, y_ref, y_true = p.step(inp)
        err = head_rel_err(y, y_ref)
        errs.append(err.ravel())
        assert err.max() <= cap, f"step {t}: {err.max():.3e}"
        if flips is not None:
            folded = p.orc.epoch != e0
            exact = ~flips.flipped | folded[:, None]   # a fold step's outputs come from the fp32 fold result
            assert err[exact].max(initial=0.0) <= TOL_F32, f"step {t}: {err[exact].max():.3e} on a matching copy"
            flips.after(folded)
        if other is not None:
            y_other, _ = other.step({k: v[p.seq_ids] for k, v in inp.items()})
            spread.append(head_rel_err(y_other, y_ref).ravel())
        p.check_bookkeeping(ring=(t % 8 == 7))
    errs = np.concatenate(errs)
    frac = float(np.mean(errs > TOL_F32))
    print(f"{hp}/{read}: max {errs.max():.3e}, median {np.median(errs):.3e}, fraction above 1e-4 {frac:.4f}")
    if other is not None:
        spread = np.concatenate(spread)
        print(f"  seed-to-seed spread: mean {spread.mean():.3e}, GPU mean {errs.mean():.3e}")
        assert errs.mean() <= 2 * spread.mean() + TOL_F32
    elif flips is not None:
        print(f"  copy codes differing from the oracle's: {flips.n_diff} of {flips.n_codes} ({flips.rate():.2e})")
        assert flips.rate() <= FLIP_CODE_RATE
    else:
        assert frac <= FLIP_FRACTION
    return p, errs


@pytest.mark.parametrize("hp,read", [("f32", "nvfp4"), ("f16sr", "nvfp4"), ("f16sr", "same"), ("f32", "shared_nvfp4"),
                                     ("f8sr", "same"), ("f8sr", "nvfp4"), ("f32", "nvfp4d"), ("f16sr", "nvfp4d")])
def test_lowprec_modes_track_oracle(cuda_ok, hp, read):
    track_lowprec(GDN_LOWPREC.replace(batch=4, nheads=4, window=8), hp, read, 48)


@pytest.mark.slow
@pytest.mark.parametrize("hp,read", [("f32", "nvfp4"), ("f16sr", "nvfp4"), ("f8sr", "nvfp4")])
def test_lowprec_full_batch_sampled(cuda_ok, hp, read):
    """The separate-precision GDN layer at full size (batch 256, 32 heads, d 128, L 16), four windows, on
    sampled sequences and heads; after the last fold the sampled read copies are the NVFP4 quantisation of
    the fp32 fold result (in fp32-checkpoint mode, of the exported checkpoint), bit for bit."""
    wl = GDN_LOWPREC
    p, _ = track_lowprec(wl, hp, read, 4 * wl.window, seq_ids=[0, 128, 255], head_ids=[0, 13, 31])
    if hp == "f32":
        S = p.selected_state()
        rc = p.gpu.export_read_copy()
        sel_s, sel_h = torch.from_numpy(p.seq_ids).cuda(), torch.from_numpy(p.head_ids).cuda()
        q = lp.nvfp4_quantize_state(S)
        for key in ("packed", "scales", "g"):
            got = rc[key].index_select(0, sel_s).index_select(1, sel_h).cpu().numpy()
            np.testing.assert_array_equal(got, q[key], err_msg=key)
    assert p.gpu.get_error() == (0, -1)


@pytest.mark.parametrize("hp,read", [("f32", "nvfp4"), ("f16sr", "same"), ("f8sr", "nvfp4")])
def test_verify_lowprec_modes(cuda_ok, hp, read):
    """8-draft verify reading an NVFP4 copy, an fp16 or an E4M3 checkpoint against the method-mirroring oracle, with the
    flip-aware bound of the step test."""
    wl = GDN_LOWPREC.replace(batch=3, nheads=4, window=8)
    p = Pair(wl, hp=hp, read=read, seed=7, max_draft=8)
    errs = []
    cap = TOL_FLIP if hp == "f32" else TOL_SR_HEAD
    flips = CopyFlips(p, read) if hp == "f32" else None
    for rnd in range(10):
        e0 = p.orc.epoch.copy()
        y, y_ref, _ = p.verify(8, gdn_draft_inputs(wl, rnd, 8))
        err = head_rel_err(y, y_ref)                        # (sequence, draft, head)
        assert err.max() <= cap, f"round {rnd}: {err.max():.3e}"
        errs.append(err.ravel())
        if flips is not None:
            folded = p.orc.epoch != e0                      # pre-folded: outputs from the fp32 fold result
            exact = (~flips.flipped | folded[:, None])[:, None, :]
            assert np.broadcast_to(err <= TOL_F32, err.shape)[np.broadcast_to(exact, err.shape)].all(), \
                f"round {rnd}: error above the fp32 bound on a matching copy"
            flips.after(folded)
        p.commit(accepted_lengths(wl, rnd, 8))
        p.check_bookkeeping(ring=False)
    errs = np.concatenate(errs)
    print(f"verify {hp}/{read}: max {errs.max():.3e}, fraction above 1e-4 {float(np.mean(errs > TOL_F32)):.4f}")
    if flips is not None:
        print(f"  copy codes differing from the oracle's: {flips.n_diff} of {flips.n_codes} ({flips.rate():.2e})")
        assert flips.rate() <= FLIP_CODE_RATE
    assert p.gpu.get_error() == (0, -1)


# ------------------------------------------------------------------------------------ decay-aware skipping

FAST_DECAY = SMALL.replace(batch=5, nheads=8, decay_scale=0.6)   # alpha spread over (0.2, 1)


@pytest.mark.parametrize("hp,read", [("f32", "same"), ("f32", "nvfp4"), ("f8sr", "same")])
def test_skip_steps_match_oracle(cuda_ok, hp, read):
    """Steps over three windows with tau = 1e-2 on fast-decaying gates: flags bit-exact after every call, outputs
    and checkpoints against the oracle that skips the same reads, and some heads really skipped."""
    wl = FAST_DECAY
    p = Pair(wl, hp=hp, read=read, seed=5, skip_tau=1e-2)
    tol = TOL_F32 if hp == "f32" and read == "same" else TOL_FLIP if hp == "f32" else TOL_SR_HEAD
    skipped, worst = 0, 0.0
    for t in range(3 * wl.window + 5):
        skipped += int(p.orc.skip.sum())
        y, y_ref, _ = p.step(gdn_step_inputs(wl, t))
        worst = max(worst, head_rel_err(y, y_ref).max())
        assert head_rel_err(y, y_ref).max() <= tol, f"step {t}"
        p.check_bookkeeping(ring=(t % 8 == 7))
    print(f"skip {hp}/{read}: max {worst:.3e}")
    assert skipped > 0
    if hp == "f32":
        p.check_checkpoint()
    assert p.gpu.get_error() == (0, -1)


def test_skip_verify_commit_flush(cuda_ok):
    """Random verify/commit rounds with T in {1, 2, 4, 8}, steps between them and a flush, with skipping on."""
    wl = FAST_DECAY
    p = Pair(wl, max_draft=8, seed=5, skip_tau=2e-2)
    rng = np.random.default_rng(3)
    skipped = 0
    for rnd in range(12):
        T = int(rng.choice([1, 2, 4, 8]))
        skipped += int(p.orc.skip.sum())
        y, y_ref, _ = p.verify(T, gdn_draft_inputs(wl, rnd, T))
        assert head_rel_err(y, y_ref).max() <= TOL_F32, f"round {rnd}"
        p.check_bookkeeping(ring=False)
        p.commit(accepted_lengths(wl, rnd, T))
        for k in range(int(rng.integers(0, 4))):
            y, y_ref, _ = p.step(gdn_step_inputs(wl, 100 + 4 * rnd + k))
            assert head_rel_err(y, y_ref).max() <= TOL_F32
        p.check_bookkeeping(ring=True)
    assert skipped > 0
    p.flush()
    p.check_bookkeeping()
    p.check_checkpoint()
    assert p.gpu.get_error() == (0, -1)


@pytest.mark.slow
def test_full_size_sampled(cuda_ok):
    """The GDN layer (batch 256, 32 heads, d 128, L 16), 1024 steps, sampled sequences and heads."""
    wl = GDN_B256
    p = Pair(wl, seq_ids=[0, 128, 255], head_ids=[0, 5, 31])
    worst = run_steps(p, wl.steps, check_every=101)
    p.check_bookkeeping()
    p.check_checkpoint()
    print(f"worst rel err {worst:.3e}")
