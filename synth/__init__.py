"""Seeded synthetic inputs for the VDN hybrid attention forward.

This package holds only the workload shapes and the random draws that both the
CUDA path and the CPU oracle consume.  It contains none of the method's
arithmetic.
"""
from .inputs import CONFIGS, Config, make_inputs, sample_rows  # noqa: F401
