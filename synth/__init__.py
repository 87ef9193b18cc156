"""Seeded synthetic inputs for the draft/verify hot path.

This package only draws random numbers and lays them out; it computes no step of
the method (no attention, no quantisation, no acceptance).  Both the fp64 oracle
tests and the CUDA path take their inputs from here, so the two sides see the
same bytes.
"""
from .configs import CONFIGS, AttnConfig, LoopConfig, get_config  # noqa: F401
from . import gen  # noqa: F401
