"""Seeded synthetic workloads for the routed block-sparse attention path.

This package only draws random inputs with the shapes, value distributions and
structure of the workloads the Velox pages describe (chunked video-diffusion KV
caches, sparse geometric overlap scores, coverage flags).  It holds none of the
method's arithmetic: no pooling, no softmax, no routing, no attention.  Both the
CPU oracle (through the tests) and the CUDA path (through the tests, the bench
and the smoke run) receive their inputs from here.
"""

from .configs import CONFIGS, Workload, RouteParams, sweep_workload, config
from .generate import make_inputs, make_current, Inputs

__all__ = ["CONFIGS", "Workload", "RouteParams", "sweep_workload", "config",
           "make_inputs", "make_current", "Inputs"]
