"""Seeded synthetic inputs for the VDN hybrid attention layer.

This package is shared by the CUDA path's tests/bench and by the oracle's
tests. It only draws random numbers and shapes them (including the per-token
key normalisation that the workloads specify as a property of the inputs); it
holds none of the layer's arithmetic.
"""
from .configs import WORKLOADS, Workload, get_workload  # noqa: F401
from .generate import make_inputs, to_f64  # noqa: F401
