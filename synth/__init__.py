"""Seeded synthetic workloads for the hybrid CSA/HCA decode path.

This package only draws numbers: it holds the named workload shapes and the
seeded generators that fill their input tensors.  It contains none of the
method's arithmetic (no compression, scoring, selection or attention), so
both the CUDA library's tests and the CPU oracle can be fed from it without
sharing any computation.
"""

from .workloads import SPECS, Spec, Workload, mxfp4_random, spec_by_name  # noqa: F401
