"""The library under CUDA-graph replay and with several contexts on several streams (need a B200)."""

import numpy as np
import pytest
import torch

from gpu_harness import TOL_F32, Pair, head_rel_err
from synth import (GDN_B256, MAMBA2_TINY, SPEC_MAMBA2_B512, accepted_lengths, gdn_step_inputs, mamba2_draft_inputs,
                   mamba2_step_inputs)

pytestmark = pytest.mark.gpu


def test_graph_replay_of_a_window(cuda_ok):
    """A whole window (15 plain steps and the fold) captured once and replayed three times matches the
    oracle run over the same 48 steps: the unit counter re-arms itself and the bookkeeping ping-pong
    returns to its parity after an even number of calls."""
    wl = MAMBA2_TINY.replace(batch=5, nheads=16, ngroups=2, init="normal", in_dtype="bf16")
    p = Pair(wl)
    n = wl.window
    inputs = [mamba2_step_inputs(wl, t) for t in range(n)]
    dev_in = [p._dev_inputs(inp) for inp in inputs]
    ys = [torch.empty(wl.batch, wl.nheads, wl.headdim, device="cuda") for _ in range(n)]
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.stream(side):
        with torch.cuda.graph(graph, stream=side):
            for t in range(n):
                d = dev_in[t]
                p.gpu.mamba2_step(d["x"], d["B"], d["C"], d["dt"], ys[t])
    torch.cuda.current_stream().wait_stream(side)
    for rep in range(3):
        graph.replay()
        torch.cuda.synchronize()
        for t in range(n):
            y_ref, y_true = p.orc.step(p._sel(inputs[t]))
            assert head_rel_err(p._pick(ys[t]), y_true).max() <= TOL_F32, f"replay {rep} step {t}"
        p.check_bookkeeping()
    p.check_checkpoint()
    assert p.gpu.get_error() == (0, -1)
    del graph


def test_two_contexts_two_streams(cuda_ok):
    """A Mamba-2 context verifying on one stream and a GDN context stepping on another, interleaved."""
    wl_m = SPEC_MAMBA2_B512.replace(batch=4, nheads=16, ngroups=2)
    wl_g = GDN_B256.replace(batch=4, nheads=4)
    pm, pg = Pair(wl_m, max_draft=4), Pair(wl_g)
    sm, sg = torch.cuda.Stream(), torch.cuda.Stream()
    sm.wait_stream(torch.cuda.current_stream())
    sg.wait_stream(torch.cuda.current_stream())
    for rnd in range(8):
        with torch.cuda.stream(sm):
            dm = mamba2_draft_inputs(wl_m, rnd, 4)
            ym, _, ym_true = pm.verify(4, dm)
            pm.commit(accepted_lengths(wl_m, rnd, 4))
        with torch.cuda.stream(sg):
            for k in range(3):
                yg, _, yg_true = pg.step(gdn_step_inputs(wl_g, 3 * rnd + k))
                assert head_rel_err(yg, yg_true).max() <= TOL_F32
        assert head_rel_err(ym, ym_true).max() <= TOL_F32
    torch.cuda.synchronize()
    pm.check_bookkeeping()
    pg.check_bookkeeping()
    pm.check_checkpoint()
    pg.check_checkpoint()
    assert pm.gpu.get_error() == (0, -1)
    assert pg.gpu.get_error() == (0, -1)
    np.testing.assert_array_equal(pm.orc.pending, 0)
