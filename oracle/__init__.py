"""Float64 CPU oracle for the gain-weighted residual memory scan.

TEST INFRASTRUCTURE ONLY: imported by tests/, __graft_entry__.smoke() and
bench.py's CPU baseline, never by the product package.  See ``oracle.scan``
for what it computes, the readings it takes and the pins that hold it.
"""

from .backward import (scan_delta_backward, scan_kalman_diag_backward, scan_kalman_full_backward,
                       scan_kalman_iso_backward)
from .hola import hola_cache_read, rms_norm, top_w_indices
from .scan import (decode_step, diag_update, iso_update, kalman_update, scan_delta, scan_kalman_diag,
                   scan_kalman_full, scan_kalman_iso)

__all__ = ["scan_delta", "scan_kalman_full", "scan_kalman_diag", "scan_kalman_iso", "decode_step", "kalman_update",
           "diag_update", "iso_update", "hola_cache_read", "rms_norm", "top_w_indices", "scan_delta_backward",
           "scan_kalman_diag_backward", "scan_kalman_iso_backward", "scan_kalman_full_backward"]
