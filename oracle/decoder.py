"""Checkpoint + input-buffer bookkeeping of ReplaySSM decoding (oracle; test infrastructure only).

What the pages fix:

* The state is a checkpoint plus a buffer of recent inputs; most steps append
  their inputs and compute the output from checkpoint and buffer without
  writing state back ("Hybrid-model decoding has a new bottleneck", Synopsis
  and Interpretation, second paragraph).
* Only a full buffer folds the buffered inputs into the checkpoint ("SSM
  decoding stops writing state every step", Synopsis and Interpretation, second
  paragraph; "NVIDIA and Dao AI Lab speed up hybrid-model decoding", third
  paragraph: a new checkpoint after 16 tokens in the tested setup).
* Speculative verification needs only outputs, with no intermediate states,
  and the accepted prefix is committed by advancing the buffer pointer
  ("Hybrid-model decoding has a new bottleneck", Interpretation, third
  paragraph; "SSM decoding stops writing state every step", Interpretation,
  third paragraph).
* The recurrence checkpoint and the copy read for outputs may differ in
  precision; non-flush outputs depend on the approximate copy ("Hybrid-model
  decoding has a new bottleneck", Interpretation, fourth paragraph; "SSM
  decoding stops writing state every step", Perspective, second paragraph).

Readings taken where the pages are silent (per sequence; L = window):

* step: if count == L (only after a commit) fold first; write the record to
  slot count; count += 1; if count == L fold now (eager fold) and take y from
  the new state, else take y by replay from the checkpoint and slots
  0..count-1.
* verify(T): if count + T > L fold the committed records first; write the T
  drafts to slots count..count+T-1 without moving count; output y for every
  draft; pending = T.
* commit(a): requires a pending verify and 0 <= a <= pending; count += a;
  pending = 0.  Nothing else moves.
* flush: fold the committed records (if any) into the checkpoint.
* A fold resets count to 0 and adds 1 to epoch.  A call on a sequence in a
  state that forbids it (step, verify or flush with a verify pending; commit
  without one; accepted length out of range) leaves that sequence untouched,
  writes none of its outputs, and records an error: the error word keeps the
  lowest sequence index that ever failed, with its code (the lowest code if
  that sequence failed in several ways).
* Outputs of a call that folds come from the freshly folded state at full
  precision; the stored checkpoint is read for folding, the read copy for
  outputs of calls that do not fold.

Precision modes: hp = "f32" (fp32 checkpoint), "f16sr" (fp16 with stochastic
rounding, random words from Philox4x32-10 with counter (sequence*H + head,
new epoch, element/4, 0) and the 64-bit seed as key) or "f8sr" (E4M3 with a
per-64-row-tile scale and the same stochastic rounding); read = "same" (outputs
read the checkpoint), "nvfp4" (separate NVFP4 read copy, re-quantised from the
fp32 fold result at every fold), "nvfp4d" (the same with two-axis scales:
column-group scales along the channel axis and block scales along the state
axis, see lowprec) or "shared_nvfp4" (the NVFP4 copy is also the checkpoint
the recurrence continues from; contrast mode).  The copies are quantised tile
by tile, a tile being 64 consecutive rows of one head's state.

Decay-aware read skipping (``skip_tau`` > 0): a head whose decay over the
buffered inputs has fallen below a threshold may skip reading the checkpoint,
which then counts as zero; a fold of such a head writes the new checkpoint
from the buffer alone ("SSM decoding stops writing state every step",
Perspective, first paragraph, names this as a next step for heads whose decay
is negligible, and fixes no rule).  Reading taken: after
each step, verify or flush, a head's flag is set from the committed records of
the current window, and the next call reads it:

* GDN: iff the product of alpha over those records, taken in fp32 in record
  order, is below ``skip_tau``.  The product only falls as records are added,
  so the skipped term S0 u0 of any later output has norm at most
  skip_tau * ||S0|| * q_scale * ||q|| (each (I - beta k k^T) has norm <= 1 for
  ||k|| = 1, 0 <= beta <= 2).
* Mamba-2: iff A_h * s < ln(skip_tau), with s the fp32 sum of dt over those
  records in record order, the product A_h * s taken in fp32, and ln(skip_tau)
  the double-precision natural log of the fp32 threshold rounded once to fp32.
  Then the product of dA = exp(dt A_h) over the records is exp(A_h s) <
  skip_tau up to that rounding, and it only falls as records are added (A_h <
  0 < dt), so the skipped term exp(A_h s(m, e)) S0 C of any later output has
  norm at most about skip_tau * ||S0|| * ||C||.

Commit leaves the flags alone; a fold that empties the window clears them.

Two outputs are produced per call: ``y`` mirrors the method (folds at the
points above, state rounded to its stored formats, replay in float64) and
``y_true`` is conventional step-by-step decoding in float64 with no rounding
of the state.  In fp32 mode the pages' invariant says the two agree up to
floating-point differences; the tests check it.
"""

from __future__ import annotations

import math

import numpy as np

from . import lowprec
from . import recurrence as rc
from .philox import sr_words

ERR_PENDING = 1        # step / verify / flush while a verify is pending
ERR_NO_VERIFY = 2      # commit without a pending verify
ERR_ACCEPTED = 3       # accepted length outside 0..pending


class ReplayOracle:
    """Per-layer oracle over a subset of sequences (``seq_ids``) and heads (``head_ids``).

    kind: "mamba2" or "gdn".  S0: initial checkpoint, [nb][nh][rows][cols] for
    the selected sequences and heads.  params: Mamba-2 {"A", "D"} over all
    heads (selected by head_ids here); GDN uses ``q_scale``.
    Inputs to ``step`` / ``verify`` carry every head of the selected sequences
    (leading [nb] or [nb][T]); Mamba-2 B and C carry every group.
    """

    def __init__(self, kind, S0, window, *, nheads, ngroups=1, params=None, seq_ids=None, head_ids=None,
                 hp="f32", read="same", seed=0, q_scale=1.0, skip_tau=0.0):
        assert kind in ("mamba2", "gdn")
        assert skip_tau >= 0
        assert hp in ("f32", "f16sr", "f8sr") and read in ("same", "nvfp4", "nvfp4d", "shared_nvfp4")
        self.kind, self.L, self.H, self.G = kind, int(window), int(nheads), int(ngroups)
        S0 = np.asarray(S0, np.float64)
        self.nb = S0.shape[0]
        self.seq_ids = np.arange(self.nb) if seq_ids is None else np.asarray(seq_ids)
        self.head_ids = np.arange(self.H) if head_ids is None else np.asarray(head_ids)
        self.nh = len(self.head_ids)
        assert S0.shape[1] == self.nh
        self.head_group = [int(h) // (self.H // self.G) for h in self.head_ids]
        self.params = params or {}
        if kind == "mamba2":
            self.A = np.asarray(self.params["A"], np.float64)[self.head_ids]
            self.D = np.asarray(self.params["D"], np.float64)[self.head_ids]
        self.q_scale = float(q_scale)
        self.hp_mode, self.read_mode, self.seed = hp, read, int(seed)
        self.skip_tau = np.float32(skip_tau)
        self.ln_tau = np.float32(math.log(float(self.skip_tau))) if skip_tau > 0 else np.float32(0)

        self.S_true = S0.copy()
        self.count = np.zeros(self.nb, np.int64)
        self.epoch = np.zeros(self.nb, np.int64)
        # loading a checkpoint writes it in the stored formats like a fold that produces epoch 0
        self.hp = np.empty_like(S0)
        self.rd = np.empty_like(S0)
        for b in range(self.nb):
            self._store(b, S0[b])
        self.pending = np.zeros(self.nb, np.int64)
        self.skip = np.zeros((self.nb, self.nh), bool)       # decay-aware skip flags, read by the next call
        self.err = None                      # (seq, code) of the lowest failing sequence
        self.ring = [[None] * self.L for _ in range(self.nb)]   # per sequence, per slot: record dict
        self._drafts_true = [None] * self.nb                    # truth-side draft records awaiting commit

    # ------------------------------------------------------------------ helpers
    def _select(self, inp, b, lead=()):
        """Record of sequence index b (position in the subset) restricted to the selected heads."""
        idx = (b,) + lead
        if self.kind == "mamba2":
            return {"x": np.asarray(inp["x"][idx])[self.head_ids], "B": np.asarray(inp["B"][idx]),
                    "C": np.asarray(inp["C"][idx]), "dt": np.asarray(inp["dt"][idx])[self.head_ids]}
        return {"q": np.asarray(inp["q"][idx])[self.head_ids], "k": np.asarray(inp["k"][idx])[self.head_ids],
                "v": np.asarray(inp["v"][idx])[self.head_ids], "alpha": np.asarray(inp["alpha"][idx])[self.head_ids],
                "beta": np.asarray(inp["beta"][idx])[self.head_ids]}

    def _fold(self, S, recs):
        if not recs:
            return np.asarray(S, np.float64)
        if self.kind == "mamba2":
            return rc.mamba2_fold(S, recs, self.A, self.head_group)
        return rc.gdn_fold(S, recs)

    def _replay(self, S, recs, cur):
        if self.kind == "mamba2":
            return rc.mamba2_replay_output(S, recs, cur["C"], self.A, self.D, self.head_group)
        return rc.gdn_replay_output(S, recs, cur["q"], self.q_scale)

    def _output(self, S, cur):
        if self.kind == "mamba2":
            return rc.mamba2_output(S, cur["C"], cur["x"], self.D, self.head_group)
        return rc.gdn_output(S, cur["q"], self.q_scale)

    def _true_step(self, S, rec):
        if self.kind == "mamba2":
            return rc.mamba2_step(S, rec["x"], rec["B"], rec["C"], rec["dt"], self.A, self.D, self.head_group)
        return rc.gdn_step(S, rec["q"], rec["k"], rec["v"], rec["alpha"], rec["beta"], self.q_scale)

    def _ckpt(self, S, b):
        """The checkpoint as a call reads it: heads flagged for skipping contribute zero."""
        if not self.skip[b].any():
            return S
        return np.where(self.skip[b][:, None, None], 0.0, S)

    def _update_skip(self, b):
        """Flags for the next call from the committed records, in order: GDN, fp32 product of alpha < skip_tau;
        Mamba-2, A_h times the fp32 sum of dt < ln(skip_tau), in fp32."""
        if self.skip_tau <= 0:
            return
        recs = self.ring[b][: self.count[b]]
        if self.kind == "gdn":
            prod = np.ones(self.nh, np.float32)
            for rec in recs:
                prod = (prod * np.asarray(rec["alpha"], np.float32)).astype(np.float32)
            self.skip[b] = prod < self.skip_tau
            return
        s = np.zeros(self.nh, np.float32)
        for rec in recs:
            s = (s + np.asarray(rec["dt"], np.float32)).astype(np.float32)
        self.skip[b] = (self.A.astype(np.float32) * s).astype(np.float32) < self.ln_tau

    def _read_copy(self, S32):
        if self.read_mode == "nvfp4d":
            return lowprec.nvfp4d_roundtrip_state(S32).astype(np.float64)
        return lowprec.nvfp4_roundtrip_state(S32).astype(np.float64)

    def _store(self, b, S_new):
        """Write a fold result for sequence b into the stored formats."""
        S32 = np.asarray(S_new, np.float64).astype(np.float32)
        if self.read_mode == "shared_nvfp4":
            self.hp[b] = self.rd[b] = self._read_copy(S32)
            return
        if self.hp_mode == "f32":
            self.hp[b] = S32.astype(np.float64)
        else:
            units = int(self.seq_ids[b]) * self.H + self.head_ids.astype(np.int64)
            n = S32.shape[-1] * S32.shape[-2]
            words = sr_words(self.seed, units, int(self.epoch[b]), n).reshape(S32.shape)
            if self.hp_mode == "f16sr":
                self.hp[b] = lowprec.fp16_stochastic_round(S32, words).astype(np.float64)
            else:
                self.hp[b] = lowprec.fp8_quantize_state(S32, words)["values"].astype(np.float64)
        self.rd[b] = self.hp[b] if self.read_mode == "same" else self._read_copy(S32)

    def _error(self, b, code):
        s = int(self.seq_ids[b])
        if self.err is None or (s, code) < self.err:
            self.err = (s, code)

    # ------------------------------------------------------------------ calls
    def step(self, inp):
        """One decode token per selected sequence.  Returns (y, y_true), each [nb][nh][rows]."""
        rows = self.S_true.shape[2]
        y = np.full((self.nb, self.nh, rows), np.nan)
        y_true = np.full_like(y, np.nan)
        for b in range(self.nb):
            if self.pending[b]:
                self._error(b, ERR_PENDING)
                continue
            rec = self._select(inp, b)
            self.S_true[b], y_true[b] = self._true_step(self.S_true[b], rec)
            folded = False
            S = self._ckpt(self.rd[b], b)
            if self.count[b] == self.L:                               # pre-fold (after a commit)
                S = self._fold(self._ckpt(self.hp[b], b), self.ring[b][: self.L])
                self.count[b] = 0
                self.epoch[b] += 1
                folded = True
            elif self.count[b] + 1 == self.L:
                S = self._ckpt(self.hp[b], b)
            self.ring[b][self.count[b]] = rec
            self.count[b] += 1
            if self.count[b] == self.L:                               # eager fold
                S = self._fold(S, self.ring[b][: self.L])
                self.count[b] = 0
                self.epoch[b] += 1
                y[b] = self._output(S, rec)
                folded = True
            else:
                y[b] = self._replay(S, self.ring[b][: self.count[b]], rec)
            if folded:
                self._store(b, S)
            self._update_skip(b)
        return y, y_true

    def verify(self, T, inp):
        """T draft tokens per selected sequence (inputs [nb][T]...).  Returns (y, y_true), [nb][T][nh][rows]."""
        assert 1 <= T <= self.L
        rows = self.S_true.shape[2]
        y = np.full((self.nb, T, self.nh, rows), np.nan)
        y_true = np.full_like(y, np.nan)
        for b in range(self.nb):
            if self.pending[b]:
                self._error(b, ERR_PENDING)
                continue
            S = self._ckpt(self.rd[b], b)
            if self.count[b] + T > self.L:                            # make room: fold committed records
                S = self._fold(self._ckpt(self.hp[b], b), self.ring[b][: self.count[b]])
                self.count[b] = 0
                self.epoch[b] += 1
                self._store(b, S)
            c = int(self.count[b])
            recs = [self._select(inp, b, (j,)) for j in range(T)]
            for j in range(T):
                self.ring[b][c + j] = recs[j]
            St = self.S_true[b]
            for j in range(T):
                y[b, j] = self._replay(S, self.ring[b][: c + j + 1], recs[j])
                St, y_true[b, j] = self._true_step(St, recs[j])
            self._drafts_true[b] = recs
            self.pending[b] = T
            self._update_skip(b)
        return y, y_true

    def commit(self, accepted):
        accepted = np.asarray(accepted)
        for b in range(self.nb):
            a = int(accepted[b])
            if not self.pending[b]:
                self._error(b, ERR_NO_VERIFY)
                continue
            if a < 0 or a > self.pending[b]:
                self._error(b, ERR_ACCEPTED)
                continue
            for rec in self._drafts_true[b][:a]:
                self.S_true[b], _ = self._true_step(self.S_true[b], rec)
            self.count[b] += a
            self.pending[b] = 0
            self._drafts_true[b] = None

    def flush(self, mask=None):
        for b in range(self.nb):
            if mask is not None and not mask[b]:
                continue
            if self.pending[b]:
                self._error(b, ERR_PENDING)
                continue
            if self.count[b]:
                S = self._fold(self._ckpt(self.hp[b], b), self.ring[b][: self.count[b]])
                self.count[b] = 0
                self.epoch[b] += 1
                self._store(b, S)
                self._update_skip(b)

    # ------------------------------------------------------------------ inspection
    def live_slots(self, b):
        """Number of ring slots holding committed or pending records of sequence b."""
        return int(self.count[b] + self.pending[b])
