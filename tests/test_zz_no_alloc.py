"""The scheduler self-test entry point, which needs no caller device memory."""

import ctypes as C

import pytest

from hybrid_model_ssm_gdn_b200 import abi, sched_probe
from hybrid_model_ssm_gdn_b200.build import build


def test_probe_rejects_bad_counts():
    """Argument checks happen on the host, before any device work (no GPU needed)."""
    build()
    lib = abi.load()
    per_block = (C.c_int * 4)()
    bad = C.c_int(0)
    pb, pbad = C.cast(per_block, C.c_void_p), C.cast(C.pointer(bad), C.c_void_p)
    for units, blocks in ((0, 4), (1 << 16 + 1, 4), (10, 0), (10, 1025)):
        assert lib.rssm_sched_probe(units, blocks, pb, pbad, None) == 1
    assert lib.rssm_sched_probe(10, 4, None, pbad, None) == 1
    assert lib.rssm_sched_probe(10, 4, pb, None, None) == 1


@pytest.mark.gpu
@pytest.mark.parametrize("units,blocks", [(5000, 148), (10, 64), (1 << 16, 1024), (1, 1)])
def test_every_unit_drawn_once_and_counter_rearmed(cuda_ok, units, blocks):
    for _ in range(3):  # the last block of each launch re-arms the counter for the next one
        per_block, bad = sched_probe(units, blocks)
        assert bad == 0
        assert sum(per_block) == units
        assert min(per_block) >= 0
