"""Bounded waits end a launch cleanly (need a B200).

Every wait of the replay kernels on an asynchronous copy or on another warp gives up after a bounded number
of clock cycles, records RSSM_DEV_TIMEOUT in the context's error word, drains the block's copies in flight
and returns.  A test hook makes one launch's tile stage never fill (the producer arms the stage's barrier and
issues no copy into it): the consumer warps waiting on it run out of time.  Nothing faults or hangs; the
wait bound is shortened to about a millisecond for the test.  After the timeout the launch has returned,
the unit scheduler's counter is re-armed for the next launch, and reloading the checkpoint gives a context
that decodes in parity with a fresh oracle.
"""

import numpy as np
import pytest
import torch

from gpu_harness import TOL_F32, Pair, head_rel_err
from hybrid_model_ssm_gdn_b200 import abi
from synth import GDN_B256, MAMBA2_TINY, gdn_step_inputs, mamba2_step_inputs

pytestmark = pytest.mark.gpu

CASES = {
    "mamba2": (MAMBA2_TINY.replace(batch=6, nheads=16, ngroups=2, init="normal", in_dtype="bf16"), mamba2_step_inputs),
    "gdn": (GDN_B256.replace(batch=6, nheads=8), gdn_step_inputs),
}


def _sched_words(layer):
    """The unit counter and the finished-block count, read from the arena (they follow the bookkeeping words)."""
    off = (2 * layer.batch * 16 + 255) // 256 * 256
    return layer.arena[off:off + 16].view(torch.int32).cpu().numpy()


@pytest.mark.parametrize("kind", ["mamba2", "gdn"])
def test_a_stage_that_never_fills_times_out_and_the_context_recovers(cuda_ok, kind, monkeypatch):
    wl, inputs = CASES[kind]
    monkeypatch.setenv("RSSM_WAIT_CYCLES", "2000000")
    monkeypatch.setenv("RSSM_WITHHOLD_TILE", "2")
    p = Pair(wl)                                   # the context reads both at creation
    monkeypatch.delenv("RSSM_WITHHOLD_TILE")
    monkeypatch.delenv("RSSM_WAIT_CYCLES")
    for t in range(3):                             # the first launch withholds a stage in every block
        p.step(inputs(wl, t))
    code, seq = p.gpu.get_error()                  # synchronises: the launches have returned
    assert code == abi.DEV_TIMEOUT and 0 <= seq < wl.batch
    words = _sched_words(p.gpu)
    assert words[0] == seq * 16 + abi.DEV_TIMEOUT
    assert words[1] == 0 and words[2] == 0         # the unit counter is re-armed
    # reload: the context decodes in parity with a fresh oracle and the error word is clean
    q = Pair(wl)
    p.gpu.load_checkpoint(torch.from_numpy(np.ascontiguousarray(
        q.orc.S_true.astype(np.float32))).cuda())
    for t in range(2 * wl.window + 3):
        inp = inputs(wl, 50 + t)
        y, _, y_true = q.step(inp)                 # q's own context and oracle advance too
        d = q._dev_inputs(inp)
        if kind == "mamba2":
            y2 = p.gpu.mamba2_step(d["x"], d["B"], d["C"], d["dt"])
        else:
            y2 = p.gpu.gdn_step(d["q"], d["k"], d["v"], d["alpha"], d["beta"])
        assert head_rel_err(q._pick(y2), y_true).max() <= TOL_F32, f"step {t}"
    assert p.gpu.get_error() == (0, -1)
    assert q.gpu.get_error() == (0, -1)
