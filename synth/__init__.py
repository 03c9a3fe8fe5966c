"""Seeded synthetic inputs for the residual-binarization layers.

This module is shared by the fp64 oracle's tests and by the CUDA path's tests
and bench. It holds shapes, value distributions and seeds only: none of the
method's arithmetic (no signs, scales, residuals or products) lives here.

Every tensor is addressed by (workload, layer, matrix, tensor) and drawn from
its own child seed of one root seed, so any tensor can be regenerated alone.
Two back ends exist:

* ``host``: numpy PCG64 streams (used by the parity tests, whose CPU copies
  feed both the oracle and, after an upload, the kernels);
* ``device``: torch's Philox generator on a CUDA device (used by the bench to
  build multi-gigabyte layer stacks quickly; sampled rows are copied back to
  the host when the oracle has to see them).

The two back ends draw different numbers from the same seed; a test picks one
and uses it for both sides.
"""
from .configs import (  # noqa: F401
    ROOT_SEED,
    WORKLOADS,
    Workload,
    MatrixSpec,
    child_seed,
    host_weight,
    host_activations,
    device_weight,
    device_activations,
    host_rows,
)
