"""Seeded synthetic inputs for the VDN hybrid attention forward.

This package holds only the workload shapes and the random draws that both the
CUDA path and the CPU oracle consume.  It contains none of the method's
arithmetic.
"""
from .inputs import (CONFIGS, Config, grid_shape, make_inputs, make_prep_inputs,  # noqa: F401
                     make_text_queries, sample_rows)
