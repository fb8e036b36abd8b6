"""B200-native selective scan (S6) forward: a C-ABI CUDA library for sm_100a and its binding.

``selective_scan_fwd`` (in ``selective_state_space_13_b200.scan``) runs the whole scan --
Delta = softplus(delta_raw + bias), Abar = exp(Delta*A), Bbar*u = Delta*B*u, the recurrence,
the C readout with the D skip, the direction merge and the silu(z) gate -- in hand-written CUDA
kernels behind ``include/selective_scan.h``.  Importing this package does not load the CUDA
library; the first call does, and it raises if the library is missing.
"""

from .workloads import (DIR_COLUMN, DIR_COLUMN_REVERSE, DIR_FORWARD, DIR_REVERSE,  # noqa: F401
                        WORKLOADS)

__all__ = ["DIR_FORWARD", "DIR_REVERSE", "DIR_COLUMN", "DIR_COLUMN_REVERSE", "WORKLOADS"]
