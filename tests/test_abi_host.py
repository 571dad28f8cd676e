"""The C-ABI library loads, exports every declared entry point, and validates on the host (no GPU needed)."""

import ctypes as C
import os
import re

import pytest

from hybrid_model_ssm_gdn_b200 import abi
from hybrid_model_ssm_gdn_b200.build import build

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "rssm.h")


@pytest.fixture(scope="module")
def lib():
    build()
    return abi.load()


def declared_functions():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"^\s*(?:rssm_status|const char \*)\s*(rssm_\w+)\s*\(", text, re.M)))


def test_every_declared_symbol_is_exported(lib):
    names = declared_functions()
    assert len(names) >= 18
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) <= set(abi._SIGS) | {"rssm_last_cuda_error"}


def _cfg(**kw):
    base = dict(kind=abi.MAMBA2, batch=2, nheads=4, headdim=64, dstate=128, ngroups=2, window=16, max_draft=4,
                in_dtype=abi.BF16, hp=abi.HP_F32, read=abi.READ_SAME, seed=0, q_scale=1.0, A=16, D=16)
    base.update(kw)
    return abi.Config(**base)


def _arena(lib, **kw):
    n = C.c_size_t(0)
    st = lib.rssm_arena_bytes(C.byref(_cfg(**kw)), C.byref(n))
    return st, n.value


def test_arena_size_and_validation(lib):
    st, n = _arena(lib)
    assert st == 0
    # checkpoint 2*4*64*128*4 bytes dominates; the ring holds 2L slots per head / group
    assert n >= 2 * 4 * 64 * 128 * 4 + 2 * 4 * 32 * 64 * 2 + 2 * 2 * 32 * 128 * 2
    assert _arena(lib, dstate=64)[0] == 2               # only N = 128 is built
    assert _arena(lib, headdim=12)[0] == 2              # rows must be a multiple of 8
    assert _arena(lib, headdim=72)[0] == 2              # Mamba-2 tiles hold at most 64 rows
    assert _arena(lib, ngroups=3)[0] == 2               # H % G
    assert _arena(lib, window=33)[0] == 2
    assert _arena(lib, window=4, max_draft=5)[0] == 2   # T_max <= L
    assert _arena(lib, A=None)[0] == 1
    assert _arena(lib, kind=7)[0] == 1
    assert _arena(lib, kind=abi.GDN, headdim=128, ngroups=1, A=None, D=None)[0] == 0
    assert _arena(lib, kind=abi.GDN, headdim=128, ngroups=2)[0] == 2


def test_precision_and_skip_modes_validation(lib):
    """The FP8 checkpoint is a GDN mode: Mamba-2 contexts refuse it.  Decay-aware skipping serves both kinds; a
    negative, NaN or infinite threshold is an argument error.  The FP8 arena holds a quarter of the fp32
    checkpoint plus one fp32 scale per 64-row tile; skipping adds one flag byte per head."""
    gdn = dict(kind=abi.GDN, headdim=128, ngroups=1, A=None, D=None)
    assert _arena(lib, hp=abi.HP_F8_SR)[0] == 3
    st, m_plain = _arena(lib)
    st2, m_skip = _arena(lib, skip_tau=1e-3)
    assert st == st2 == 0 and 2 * 4 <= m_skip - m_plain <= 256
    assert _arena(lib, skip_tau=-1.0)[0] == 1
    assert _arena(lib, skip_tau=-1.0, **gdn)[0] == 1
    assert _arena(lib, skip_tau=float("nan"), **gdn)[0] == 1
    assert _arena(lib, skip_tau=float("inf"), **gdn)[0] == 1
    _, n32 = _arena(lib, **gdn)
    st, n8 = _arena(lib, hp=abi.HP_F8_SR, **gdn)
    assert st == 0
    state = 2 * 4 * 128 * 128
    assert n32 - n8 >= state * 3 - 256 and n32 - n8 <= state * 3 + 256
    st, nsk = _arena(lib, skip_tau=1e-2, **gdn)
    assert st == 0 and 2 * 4 <= nsk - n32 <= 256
    assert _arena(lib, hp=5, **gdn)[0] == 1


def test_null_arguments_are_rejected_without_launch(lib):
    assert lib.rssm_create(None, None, 0, None) == 1
    assert lib.rssm_create(C.byref(_cfg()), None, 0, C.byref(C.c_void_p())) == 1
    assert lib.rssm_destroy(None) == 1
    assert lib.rssm_mamba2_step(None, None, None, None, None, None, None) == 1
    assert lib.rssm_commit(None, None, None) == 1
    assert lib.rssm_export_skip(None, None, None) == 1
    code, seq = C.c_int(), C.c_int()
    assert lib.rssm_get_error(None, C.byref(code), C.byref(seq), None) == 1
    assert lib.rssm_conv_mamba2_step(C.byref(_cfg()), None, None, None, None, None, None, None) == 1


def test_binding_input_sizes_match_the_workloads():
    """The binding's per-input element counts (checked before any device call, so that a short buffer cannot
    be overrun) agree with the seeded workloads that the tests and the bench pass, for steps and drafts."""
    import types

    import numpy as np
    import torch

    from hybrid_model_ssm_gdn_b200 import ReplaySSM, _dev
    from synth import GDN_B256, MAMBA2_120B, gdn_draft_inputs, gdn_step_inputs, mamba2_draft_inputs, mamba2_step_inputs

    for wl, step, drafts in ((MAMBA2_120B.replace(batch=3), mamba2_step_inputs, mamba2_draft_inputs),
                             (GDN_B256.replace(batch=3, nheads=4), gdn_step_inputs, gdn_draft_inputs)):
        m2 = wl.kind == "mamba2"
        fake = types.SimpleNamespace(batch=wl.batch, nheads=wl.nheads, rows=wl.headdim if m2 else wl.dv,
                                     dstate=128, ngroups=wl.ngroups if m2 else 1)
        for name, v in step(wl, 0).items():
            assert ReplaySSM._need(fake, name, (wl.batch,)) == np.asarray(v).size, name
        for name, v in drafts(wl, 0, 4).items():
            assert ReplaySSM._need(fake, name, (wl.batch, 4)) == np.asarray(v).size, name
    with pytest.raises(ValueError, match="needs at least 8 elements"):
        _dev(torch.zeros(7), torch.float32, "x", 8)


def test_short_per_head_parameters_are_rejected_before_any_device_call():
    """Mamba-2 contexts read nheads floats from A and D through raw pointers: shorter tensors are refused on the
    host, before the binding touches the device."""
    import torch

    from hybrid_model_ssm_gdn_b200 import ReplaySSM
    ok, short = torch.full((4,), -1.0), torch.zeros(3)
    for A, D, name in ((short, ok, "A"), (ok, short, "D"), (None, ok, "A")):
        with pytest.raises(ValueError, match=f"{name}: needs at least 4 elements"):
            ReplaySSM("mamba2", 2, 4, 64, 128, 1, 16, 0, torch.bfloat16, A=A, D=D)
