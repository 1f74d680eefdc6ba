"""Seeded synthetic workloads for the sparse MoE FFN forward.

A module of its own: it serves both the CUDA path's tests and bench and the
oracle's tests, and holds the input recipe only (shapes and random draws), none
of the layer's arithmetic.
"""

from .configs import CONFIGS, DEFAULT_WORKLOAD, PERF_WORKLOADS, MoEConfig  # noqa: F401
from .inputs import MoEInputs, make_inputs, make_tokens, router_inputs, skew_offsets  # noqa: F401
