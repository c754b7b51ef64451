"""Routed Mixture-of-Experts FFN forward pass for NVIDIA B200 (sm_100a).

The compute path is the CUDA library ``libmoe_b200.so`` (C ABI in
include/moe_b200.h); ``native`` is its ctypes binding.  ``workloads`` and
``synth`` describe and draw the seeded synthetic inputs.
"""
from . import workloads  # noqa: F401
