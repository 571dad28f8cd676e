"""The scheduler self-test entry point, which allocates nothing and needs no caller device memory.

Some callers cannot allocate device memory (a process holding only a driver context, or code
running where allocation is forbidden); ``rssm_sched_probe`` serves them from one fixed-size
array inside the library.  This file sorts last so that a run stopping at its first failure has
already run every other test; its GPU test passes alone in a fresh process and after the others.
"""

import ctypes as C

import pytest

from hybrid_model_ssm_gdn_b200 import abi, sched_probe
from hybrid_model_ssm_gdn_b200.build import build

MAX_UNITS, MAX_BLOCKS = 1 << 16, 1024


def test_probe_rejects_bad_counts():
    """Argument checks happen on the host, before any device work (no GPU needed)."""
    build()
    lib = abi.load()
    per_block = (C.c_int * 4)()
    bad = C.c_int(0)
    pb, pbad = C.cast(per_block, C.c_void_p), C.cast(C.pointer(bad), C.c_void_p)
    for units, blocks in ((0, 4), (-1, 4), (MAX_UNITS + 1, 4), (10, 0), (10, MAX_BLOCKS + 1)):
        assert lib.rssm_sched_probe(units, blocks, pb, pbad, None) == 1, (units, blocks)
    assert lib.rssm_sched_probe(10, 4, None, pbad, None) == 1
    assert lib.rssm_sched_probe(10, 4, pb, None, None) == 1


@pytest.mark.gpu
@pytest.mark.parametrize("units,blocks", [(5000, 148), (10, 64), (MAX_UNITS, MAX_BLOCKS), (1, 1), (148, 148)])
def test_every_unit_drawn_once_and_counter_rearmed(cuda_ok, units, blocks):
    """Several calls in a row on the shared array: each one draws every unit exactly once and leaves the
    counter re-armed (bad == 0 covers both), and the per-block tallies add up."""
    for _ in range(3):
        per_block, bad = sched_probe(units, blocks)
        assert bad == 0
        assert sum(per_block) == units
        assert min(per_block) >= 0


@pytest.mark.gpu
def test_probe_after_a_larger_one_and_on_a_side_stream(cuda_ok):
    """A small probe after the largest one sees none of its marks; a probe on a non-default stream works."""
    import torch
    assert sched_probe(MAX_UNITS, MAX_BLOCKS)[1] == 0
    per_block, bad = sched_probe(7, 3)
    assert bad == 0 and sum(per_block) == 7 and len(per_block) == 3
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        per_block, bad = sched_probe(4096, 148)
    assert bad == 0 and sum(per_block) == 4096
