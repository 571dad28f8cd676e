"""In-house comparison kernels (conventional step-by-step, snapshot-per-draft) vs the float64 truth (need a B200)."""

import numpy as np
import pytest
import torch

from gpu_harness import TOL_F32, dev, head_rel_err
from hybrid_model_ssm_gdn_b200 import conv_gdn_step, conv_mamba2_step, make_config, snap_commit, snap_verify
from oracle import recurrence as rc
from synth import (GDN_B256, MAMBA2_TINY, accepted_lengths, gdn_draft_inputs, gdn_initial_state, gdn_step_inputs,
                   mamba2_draft_inputs, mamba2_initial_state, mamba2_params, mamba2_step_inputs)

pytestmark = pytest.mark.gpu


def test_conventional_mamba2(cuda_ok):
    wl = MAMBA2_TINY.replace(batch=3, nheads=8, ngroups=2, init="normal", in_dtype="bf16")
    p = mamba2_params(wl)
    A, D = torch.from_numpy(p["A"]).cuda(), torch.from_numpy(p["D"]).cuda()
    cfg = make_config("mamba2", wl.batch, wl.nheads, wl.headdim, 128, wl.ngroups, wl.window, 0, torch.bfloat16, A=A, D=D)
    S0 = mamba2_initial_state(wl)
    S = torch.from_numpy(S0).cuda()
    S_ref = S0.astype(np.float64)
    hg = [h // (wl.nheads // wl.ngroups) for h in range(wl.nheads)]
    y = torch.empty(wl.batch, wl.nheads, wl.headdim, device="cuda")
    for t in range(20):
        inp = mamba2_step_inputs(wl, t)
        d = {k: dev(v, torch.bfloat16) for k, v in inp.items()}
        conv_mamba2_step(cfg, S, d["x"], d["B"], d["C"], d["dt"], y)
        S_ref, y_ref = rc.mamba2_step(S_ref, inp["x"], inp["B"], inp["C"], inp["dt"], p["A"], p["D"], hg)
        assert head_rel_err(y.cpu().numpy(), y_ref).max() <= TOL_F32
    err = head_rel_err(S.cpu().numpy().reshape(wl.batch, wl.nheads, -1), S_ref.reshape(wl.batch, wl.nheads, -1))
    assert err.max() <= 1e-5


def test_conventional_gdn(cuda_ok):
    wl = GDN_B256.replace(batch=3, nheads=4, dv=96)
    cfg = make_config("gdn", wl.batch, wl.nheads, wl.dv, 128, 1, wl.window, 0, torch.bfloat16)
    S0 = gdn_initial_state(wl)
    S = torch.from_numpy(S0).cuda()
    S_ref = S0.astype(np.float64)
    y = torch.empty(wl.batch, wl.nheads, wl.dv, device="cuda")
    for t in range(20):
        inp = gdn_step_inputs(wl, t)
        d = {k: dev(v, torch.float32 if k in ("alpha", "beta") else torch.bfloat16) for k, v in inp.items()}
        conv_gdn_step(cfg, S, d["q"], d["k"], d["v"], d["alpha"], d["beta"], y)
        S_ref, y_ref = rc.gdn_step(S_ref, inp["q"], inp["k"], inp["v"], inp["alpha"], inp["beta"])
        assert head_rel_err(y.cpu().numpy(), y_ref).max() <= TOL_F32


@pytest.mark.parametrize("T", [4, 8])
def test_snapshot_per_draft_mamba2(cuda_ok, T):
    """One state read and T snapshot writes per verify; commit moves the live slot to the accepted draft."""
    wl = MAMBA2_TINY.replace(batch=4, nheads=8, ngroups=2, init="normal", in_dtype="bf16")
    p = mamba2_params(wl)
    A, D = torch.from_numpy(p["A"]).cuda(), torch.from_numpy(p["D"]).cuda()
    cfg = make_config("mamba2", wl.batch, wl.nheads, wl.headdim, 128, wl.ngroups, wl.window, T, torch.bfloat16, A=A, D=D)
    S0 = mamba2_initial_state(wl)
    snaps = torch.zeros(wl.batch, T + 1, wl.nheads, wl.headdim, 128, device="cuda")
    snaps[:, 0].copy_(torch.from_numpy(S0))
    cur = torch.zeros(wl.batch, dtype=torch.int32, device="cuda")
    S_ref = S0.astype(np.float64)
    hg = [h // (wl.nheads // wl.ngroups) for h in range(wl.nheads)]
    y = torch.empty(wl.batch, T, wl.nheads, wl.headdim, device="cuda")
    for rnd in range(6):
        dr = mamba2_draft_inputs(wl, rnd, T)
        d = {k: dev(v, torch.bfloat16) for k, v in dr.items()}
        snap_verify(cfg, snaps, cur, T, y, x=d["x"], B=d["B"], C=d["C"], dt=d["dt"])
        acc = accepted_lengths(wl, rnd, T)
        states = [S_ref]
        for j in range(T):
            Sj, yj = rc.mamba2_step(states[-1], dr["x"][:, j], dr["B"][:, j], dr["C"][:, j], dr["dt"][:, j],
                                    p["A"], p["D"], hg)
            states.append(Sj)
            assert head_rel_err(y[:, j].cpu().numpy(), yj).max() <= TOL_F32
        snap_commit(cfg, cur, torch.from_numpy(acc).cuda())
        S_ref = np.stack([states[a][b] for b, a in enumerate(acc)])
        live = snaps[torch.arange(wl.batch), cur.long()].cpu().numpy()
        err = head_rel_err(live.reshape(wl.batch, wl.nheads, -1), S_ref.reshape(wl.batch, wl.nheads, -1))
        assert err.max() <= 1e-5


@pytest.mark.parametrize("T", [4, 8])
def test_snapshot_per_draft_gdn(cuda_ok, T):
    """GDN snapshot-per-draft verify and its commit against the float64 recurrence."""
    wl = GDN_B256.replace(batch=3, nheads=4, dv=96)
    cfg = make_config("gdn", wl.batch, wl.nheads, wl.dv, 128, 1, wl.window, T, torch.bfloat16)
    S0 = gdn_initial_state(wl)
    snaps = torch.zeros(wl.batch, T + 1, wl.nheads, wl.dv, 128, device="cuda")
    snaps[:, 0].copy_(torch.from_numpy(S0))
    cur = torch.zeros(wl.batch, dtype=torch.int32, device="cuda")
    S_ref = S0.astype(np.float64)
    y = torch.empty(wl.batch, T, wl.nheads, wl.dv, device="cuda")
    for rnd in range(5):
        dr = gdn_draft_inputs(wl, rnd, T)
        d = {k: dev(v, torch.float32 if k in ("alpha", "beta") else torch.bfloat16) for k, v in dr.items()}
        snap_verify(cfg, snaps, cur, T, y, **d)
        acc = accepted_lengths(wl, rnd, T)
        states = [S_ref]
        for j in range(T):
            Sj, yj = rc.gdn_step(states[-1], dr["q"][:, j], dr["k"][:, j], dr["v"][:, j], dr["alpha"][:, j],
                                 dr["beta"][:, j])
            states.append(Sj)
            assert head_rel_err(y[:, j].cpu().numpy(), yj).max() <= TOL_F32
        snap_commit(cfg, cur, torch.from_numpy(acc).cuda())
        S_ref = np.stack([states[a][b] for b, a in enumerate(acc)])
        live = snaps[torch.arange(wl.batch), cur.long()].cpu().numpy()
        err = head_rel_err(live.reshape(wl.batch, wl.nheads, -1), S_ref.reshape(wl.batch, wl.nheads, -1))
        assert err.max() <= 1e-5
