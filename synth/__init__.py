"""Seeded synthetic inputs for the sparse MoE layer forward.

This package only draws numbers (``synth.c`` defines the generator) and
describes the workloads' shapes and value distributions; it contains no step
of the layer itself.  The CUDA path's tests and benchmark and the CPU oracle
consume the exact bit patterns produced here, so a (seed, tag, index) triple
always names the same value.
"""
from .gen import build, default_threads, normal, uniform_int, word  # noqa: F401
from .workloads import TAGS, WORKLOADS, Workload, layer_inputs, sparseclip_inputs  # noqa: F401
