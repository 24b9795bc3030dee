"""Seeded synthetic inputs for the hybrid sparse + linear decode path.

This module holds no arithmetic of the attention method.  It only draws the
queries, keys and values of the synthetic workloads from a counter-based
generator, so that any slice of any tensor can be regenerated on its own.

Two implementations of the same generator exist and produce identical bits:

* ``syngen.host``   -- numpy, used by the tests and by the CPU oracle's inputs;
* ``syngen.device`` -- a small CUDA library (``libsyngen.so``) that fills the
  device-resident KV caches of the large workloads directly in HBM.

Both evaluate the same fixed sequence of correctly rounded fp64 operations
(add, multiply, divide, square root, exponent extraction), so their outputs
agree bit for bit; a GPU test checks that on sampled slices.
"""

from .configs import WORKLOADS, Workload, get_workload  # noqa: F401
