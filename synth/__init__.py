"""Seeded synthetic inputs for the ReplaySSM decode path (see ``synth.workloads``)."""

from .workloads import *  # noqa: F401,F403
