"""The precision converters inside the GDN fold, pinned bit for bit (need a B200).

The separate-precision mode writes, at every fold, the recurrence checkpoint in its stored format and the NVFP4
read copy re-quantised from the fp32 fold result ("Hybrid-model decoding has a new bottleneck", Interpretation,
fourth paragraph; Perspective, second paragraph).  The converters at checkpoint load are pinned elsewhere; these
tests pin the ones inside the fold kernel, which quantise in registers with a tile maximum shared by eight warps.

* fp32 checkpoint + NVFP4 read copy: after every call that folds, the exported read copy (codes, E4M3 block
  scales, tile scales) must equal the oracle's NVFP4 quantisation of the exported fp32 checkpoint, bit for bit.
* fp16-SR and E4M3-SR checkpoints: a companion context with an fp32 checkpoint runs the same fold from the same
  stored values (the low-precision checkpoint, exported and loaded into it at each window boundary), so its
  exported checkpoint is the fp32 fold result the low-precision context rounded.  The companion keeps the
  two-axis read copy: that instance folds with the same sequential row update as the low-precision checkpoints
  (an fp32 checkpoint read as it is or through the one-axis copy folds in the chunked form, whose rounding
  differs).  The low-precision checkpoint
  must equal the oracle's stochastic rounding of that result with the Philox words of (sequence x head, epoch
  written, element / 4), bit for bit, and its read copy the oracle's NVFP4 quantisation of it.
* shared NVFP4: the same, with the shared copy as the state.

The fold arithmetic itself is checked against the float64 oracle by the parity tests (checkpoint within 1e-5).
"""

import numpy as np
import pytest
import torch

from gpu_harness import Pair
from hybrid_model_ssm_gdn_b200 import ReplaySSM
from oracle import lowprec as lp
from oracle.philox import sr_words
from synth import GDN_LOWPREC, accepted_lengths, gdn_draft_inputs, gdn_initial_state, gdn_step_inputs

pytestmark = pytest.mark.gpu

SEED = 0x5EED0123456789AB


def _gpu_inputs(inp, dtype):
    return {k: torch.from_numpy(np.ascontiguousarray(v)).cuda().to(torch.float32 if k in ("alpha", "beta") else dtype)
            for k, v in inp.items()}


def _step(layer, inp, dtype):
    d = _gpu_inputs(inp, dtype)
    return layer.gdn_step(d["q"], d["k"], d["v"], d["alpha"], d["beta"])


def _read_copy_matches(layer, S, read="nvfp4"):
    rc = layer.export_read_copy()
    q = (lp.nvfp4d_quantize_state if read == "nvfp4d" else lp.nvfp4_quantize_state)(S)
    np.testing.assert_array_equal(rc["packed"].cpu().numpy(), q["packed"], err_msg="NVFP4 codes")
    np.testing.assert_array_equal(rc["scales"].cpu().numpy(), q["scales"], err_msg="E4M3 block scales")
    np.testing.assert_array_equal(rc["g"].cpu().numpy(), q["g"], err_msg="tile scales")
    if read == "nvfp4d":
        np.testing.assert_array_equal(layer.export_column_scales().cpu().numpy(), q["colscales"],
                                      err_msg="column-group scales")


@pytest.mark.parametrize("read", ["nvfp4", "nvfp4d"])
@pytest.mark.parametrize("dv,nheads", [(128, 5), (96, 3), (40, 2)])
def test_fold_read_copy_is_the_quantised_checkpoint(cuda_ok, dv, nheads, read):
    """fp32 checkpoint + NVFP4 copy (one-axis or two-axis scales): steps over three windows, a verify that
    pre-folds and a masked flush; after every call that folds, copy == quantisation of the checkpoint exactly
    (d_v = 96 leaves a 32-row tile, d_v = 40 a tile with a partial 16-row group)."""
    wl = GDN_LOWPREC.replace(batch=3, nheads=nheads, dv=dv, window=8)
    p = Pair(wl, hp="f32", read=read, max_draft=4)
    folds = 0
    for t in range(3 * wl.window):
        e0 = p.orc.epoch.copy()
        p.step(gdn_step_inputs(wl, t))
        if np.any(p.orc.epoch != e0):
            folds += 1
            _read_copy_matches(p.gpu, p.gpu.export(state=True, ring=False)["S"].cpu().numpy(), read)
    p.step(gdn_step_inputs(wl, 100))
    p.verify(4, gdn_draft_inputs(wl, 0, 4))
    p.commit(np.full(wl.batch, 4))
    p.verify(4, gdn_draft_inputs(wl, 1, 4))                  # 5 + 4 > 8: pre-folds the committed records
    _read_copy_matches(p.gpu, p.gpu.export(state=True, ring=False)["S"].cpu().numpy(), read)
    p.commit(accepted_lengths(wl, 1, 4))
    p.flush(np.array([1, 0, 1]))
    _read_copy_matches(p.gpu, p.gpu.export(state=True, ring=False)["S"].cpu().numpy(), read)
    p.check_bookkeeping(ring=False)
    assert folds == 3
    assert p.gpu.get_error() == (0, -1)


@pytest.mark.parametrize("hp,read", [("f16sr", "same"), ("f16sr", "nvfp4"), ("f8sr", "same"), ("f8sr", "nvfp4"),
                                     ("f32", "shared_nvfp4"), ("f16sr", "nvfp4d")])
@pytest.mark.parametrize("dv", [128, 96])
def test_fold_rounding_is_the_oracle_rounding_of_the_fp32_fold(cuda_ok, hp, read, dv):
    wl = GDN_LOWPREC.replace(batch=3, nheads=5, dv=dv, window=8)
    bf = torch.bfloat16
    S0 = torch.from_numpy(gdn_initial_state(wl)).cuda()
    low = ReplaySSM("gdn", wl.batch, wl.nheads, wl.dv, 128, 1, wl.window, 0, bf, hp, read, SEED)
    ref = ReplaySSM("gdn", wl.batch, wl.nheads, wl.dv, 128, 1, wl.window, 0, bf, "f32", "nvfp4d", SEED)
    low.load_checkpoint(S0)
    units = np.arange(wl.batch)[:, None] * wl.nheads + np.arange(wl.nheads)[None, :]
    n = wl.dv * 128
    for w in range(3):
        ref.load_checkpoint(low.export(state=True, ring=False)["S"])   # same stored values, window empty
        for t in range(wl.window):
            inp = gdn_step_inputs(wl, w * wl.window + t)
            y_low = _step(low, inp, bf)
            y_ref = _step(ref, inp, bf)
        # the fold step's output comes from the fp32 fold result in both contexts
        torch.testing.assert_close(y_low, y_ref, rtol=0, atol=0)
        S32 = ref.export(state=True, ring=False)["S"].cpu().numpy()
        got = low.export(state=True, ring=False)
        assert np.all(got["meta"].cpu().numpy()[:, 1] == w + 1)
        S_low = got["S"].cpu().numpy()
        if hp == "f16sr":
            words = sr_words(SEED, units, w + 1, n).reshape(S32.shape)
            want = lp.fp16_stochastic_round(S32, words).astype(np.float32)
        elif hp == "f8sr":
            words = sr_words(SEED, units, w + 1, n).reshape(S32.shape)
            want = lp.fp8_quantize_state(S32, words)["values"]
        else:
            want = lp.nvfp4_roundtrip_state(S32)
        np.testing.assert_array_equal(S_low, want, err_msg=f"window {w}: stored checkpoint")
        if read != "same":
            _read_copy_matches(low, S32, read)
    assert low.get_error() == (0, -1) and ref.get_error() == (0, -1)
