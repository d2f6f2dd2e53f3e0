"""Seeded synthetic workloads for the LSRM native-sparse-attention layer.

This package only builds inputs: token layouts (block offsets, integer 3D
lattice coordinates) and seeded bf16 tensors.  It holds none of the layer's
arithmetic and is shared by the CUDA path's tests/bench and by the oracle's
tests, which is the only code the two sides have in common.
"""
from .nsa_workloads import (  # noqa: F401
    Workload,
    make_workload,
    lsrm_layout,
    camera_inputs,
    speed3r_layout,
    WORKLOAD_NAMES,
    gen_lib,
    bf16_bits_to_f32,
)
