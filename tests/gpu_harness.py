"""Drive the CUDA library and the CPU oracle side by side on the same seeded inputs (GPU tests only).

The oracle runs on a chosen subset of sequences and heads (every head of a
sequence is independent), so full-size workloads are checked on sampled
outputs the oracle can compute one by one.
"""

from __future__ import annotations

import numpy as np
import torch

from hybrid_model_ssm_gdn_b200 import ReplaySSM
from oracle.decoder import ReplayOracle
from synth import gdn_initial_state, mamba2_initial_state, mamba2_params

# Tolerance for fp32 state: per (step, sequence, head), ||y_gpu - y_ref|| / ||y_ref|| over the head's rows.
TOL_F32 = 1e-4
# Stored checkpoint vs the oracle's fp32-rounded fold, per (sequence, head).
TOL_CKPT = 1e-5


def torch_dtype(wl):
    return torch.bfloat16 if wl.in_dtype == "bf16" else torch.float32


def dev(a, dtype):
    """numpy float32 array (values exact in dtype) -> contiguous CUDA tensor of dtype."""
    return torch.from_numpy(np.ascontiguousarray(a)).to("cuda").to(dtype).contiguous()


def head_rel_err(y, ref):
    y = np.asarray(y, np.float64)
    ref = np.asarray(ref, np.float64)
    num = np.linalg.norm(y - ref, axis=-1)
    den = np.linalg.norm(ref, axis=-1)
    return num / np.maximum(den, 1e-300)


class Pair:
    """A GPU ReplaySSM context and a ReplayOracle over (seq_ids x head_ids)."""

    def __init__(self, wl, seq_ids=None, head_ids=None, max_draft=0, hp="f32", read="same", seed=0,
                 S0=None, skip_tau=0.0):
        self.wl = wl
        self.kind = wl.kind
        self.seq_ids = np.arange(wl.batch) if seq_ids is None else np.asarray(seq_ids)
        self.head_ids = np.arange(wl.nheads) if head_ids is None else np.asarray(head_ids)
        self.dt = torch_dtype(wl)
        if self.kind == "mamba2":
            self.params = mamba2_params(wl)
            S_full = mamba2_initial_state(wl) if S0 is None else S0
            self.gpu = ReplaySSM("mamba2", wl.batch, wl.nheads, wl.headdim, 128, wl.ngroups, wl.window, max_draft,
                                 self.dt, hp, read, seed, 1.0, torch.from_numpy(self.params["A"]),
                                 torch.from_numpy(self.params["D"]), skip_tau=skip_tau)
            S_sel = S_full[self.seq_ids][:, self.head_ids]
            self.orc = ReplayOracle("mamba2", S_sel, wl.window, nheads=wl.nheads, ngroups=wl.ngroups,
                                    params=self.params, seq_ids=self.seq_ids, head_ids=self.head_ids, hp=hp,
                                    read=read, seed=seed, skip_tau=skip_tau)
        else:
            S_full = gdn_initial_state(wl) if S0 is None else S0
            self.gpu = ReplaySSM("gdn", wl.batch, wl.nheads, wl.dv, 128, 1, wl.window, max_draft, self.dt, hp, read,
                                 seed, wl.q_scale, skip_tau=skip_tau)
            S_sel = S_full[self.seq_ids][:, self.head_ids]
            self.orc = ReplayOracle("gdn", S_sel, wl.window, nheads=wl.nheads, seq_ids=self.seq_ids,
                                    head_ids=self.head_ids, hp=hp, read=read, seed=seed, q_scale=wl.q_scale,
                                    skip_tau=skip_tau)
        self.gpu.load_checkpoint(torch.from_numpy(np.ascontiguousarray(S_full, np.float32)).cuda())

    # ------------------------------------------------------------------ inputs
    def _dev_inputs(self, inp):
        f32 = {"alpha", "beta"}
        return {k: dev(v, torch.float32 if k in f32 else self.dt) for k, v in inp.items()}

    def _sel(self, inp):
        return {k: v[self.seq_ids] for k, v in inp.items()}

    def _pick(self, y, lead_axes=1):
        y = y.cpu().numpy()
        y = y[self.seq_ids]
        return y[:, :, self.head_ids] if lead_axes == 2 else y[:, self.head_ids]

    # ------------------------------------------------------------------ calls
    def step(self, inp):
        d = self._dev_inputs(inp)
        if self.kind == "mamba2":
            y = self.gpu.mamba2_step(d["x"], d["B"], d["C"], d["dt"])
        else:
            y = self.gpu.gdn_step(d["q"], d["k"], d["v"], d["alpha"], d["beta"])
        y_ref, y_true = self.orc.step(self._sel(inp))
        return self._pick(y), y_ref, y_true

    def verify(self, T, inp):
        d = self._dev_inputs(inp)
        if self.kind == "mamba2":
            y = self.gpu.verify(T, x=d["x"], B=d["B"], C=d["C"], dt=d["dt"])
        else:
            y = self.gpu.verify(T, q=d["q"], k=d["k"], v=d["v"], alpha=d["alpha"], beta=d["beta"])
        y_ref, y_true = self.orc.verify(T, self._sel(inp))
        return self._pick(y, 2), y_ref, y_true

    def commit(self, accepted):
        self.gpu.commit(torch.from_numpy(np.asarray(accepted, np.int32)).cuda())
        self.orc.commit(np.asarray(accepted)[self.seq_ids])

    def flush(self, mask=None):
        self.gpu.flush(None if mask is None else torch.from_numpy(np.asarray(mask, np.uint8)).cuda())
        self.orc.flush(None if mask is None else np.asarray(mask)[self.seq_ids])

    # ------------------------------------------------------------------ state checks
    def check_bookkeeping(self, ring=True):
        """count / epoch / pending bit-exact; live ring slots byte-equal to the oracle's records."""
        ex = self.gpu.export(state=False, ring=ring)
        meta = ex["meta"].cpu().numpy()[self.seq_ids]
        np.testing.assert_array_equal(meta[:, 0], self.orc.count)
        np.testing.assert_array_equal(meta[:, 1], self.orc.epoch)
        np.testing.assert_array_equal(meta[:, 2], self.orc.pending)
        if self.orc.skip_tau > 0:
            flags = self.gpu.export_skip().cpu().numpy()[self.seq_ids][:, self.head_ids]
            np.testing.assert_array_equal(flags.astype(bool), self.orc.skip, err_msg="skip flags")
        if not ring:
            return
        fields = (("x", "x", True), ("dt", "dt", True), ("B", "B", False)) if self.kind == "mamba2" else \
            (("k", "k", True), ("v", "v", True), ("alpha", "alpha", True), ("beta", "beta", True))
        sel = torch.from_numpy(self.seq_ids).cuda()
        views = {name: ex["ring_" + name].index_select(0, sel).float().cpu().numpy() for name, _, _ in fields}
        for i in range(len(self.seq_ids)):
            for slot in range(self.orc.live_slots(i)):
                rec = self.orc.ring[i][slot]
                for name, key, per_head in fields:
                    got = views[name][i][:, slot]
                    want = np.asarray(rec[key], np.float32)
                    if per_head:
                        got = got[self.head_ids]
                    np.testing.assert_array_equal(got, want, err_msg=f"ring {name} seq {i} slot {slot}")

    def selected_state(self):
        """The exported fp32 checkpoint of the sampled sequences and heads (sliced on the device)."""
        S = self.gpu.export(state=True, ring=False)["S"]
        S = S.index_select(0, torch.from_numpy(self.seq_ids).cuda())
        return S.index_select(1, torch.from_numpy(self.head_ids).cuda()).cpu().numpy()

    def check_checkpoint(self, tol=TOL_CKPT):
        S = self.selected_state()
        rows = S.shape[2]
        err = head_rel_err(S.reshape(S.shape[0], S.shape[1], -1),
                           self.orc.hp[..., :rows, :].reshape(S.shape[0], S.shape[1], -1))
        assert err.max() <= tol, f"checkpoint rel err {err.max():.3e}"
        return err.max()
