"""Failure detection on the GPU without faulting it.

Every wait of the tensor-core kernels on an mbarrier is bounded; on expiry the
kernel records KDN_ERR_TIMEOUT in the status word, frees its tensor memory and
returns.  kdn_selftest_wait_timeout takes that path on purpose (a wait on an
mbarrier nothing arrives at, nothing in flight, a limit of a few microseconds),
so these tests read the timeout back and then check that the context is still
usable.  No test here traps, faults or hangs a GPU.
"""

import pytest
import torch

from delta_rule_recurrent_scan_b200 import kdn
from delta_rule_recurrent_scan_b200.workloads import WORKLOADS, make_scan_inputs
from parity import TOL, compare, run_gpu, run_oracle

pytestmark = pytest.mark.gpu
DEV = "cuda"


def test_bounded_wait_expires_sets_timeout_and_the_context_stays_usable():
    ws = torch.empty(kdn.workspace_bytes("delta", 1, 2, 130, 64, 64), dtype=torch.uint8, device=DEV)
    kdn.selftest_wait_timeout(ws, wait_cycles=20_000)
    assert kdn.read_device_status(ws) == kdn.KDN_ERR_TIMEOUT
    # the next scan clears the word and runs normally on the same context
    w = WORKLOADS["gdn_d64"]
    x = make_scan_inputs(w, seed=21, device=DEV, B=1, H=2, L=130)
    o, m, S = kdn.scan_delta(x["q"], x["k"], x["v"], x["beta"], a=x["a"], workspace=ws)
    assert kdn.read_device_status(ws) == kdn.KDN_OK
    compare({"o": o, "m": m, "S": S}, run_oracle("delta", x), TOL["bf16"])


def test_timeout_in_the_no_alloc_status_word():
    """A NULL workspace addresses the static status word of the no-alloc entry point."""
    kdn.selftest_wait_timeout(None, wait_cycles=20_000)
    assert kdn.read_device_status(None) == kdn.KDN_ERR_TIMEOUT


def test_wait_limit_is_validated_on_the_host():
    ws = torch.empty(256, dtype=torch.uint8, device=DEV)
    for bad in (0, -5, 3_000_000_000):
        with pytest.raises(kdn.KdnError) as e:
            kdn.selftest_wait_timeout(ws, wait_cycles=bad)
        assert e.value.status == kdn.KDN_ERR_INVALID_ARG


@pytest.mark.parametrize("variant", ["delta", "kalman_diag", "kalman_full", "kalman_iso"])
def test_entry_points_leave_the_current_device_unchanged(variant):
    """The library launches on the state's device and restores the caller's current device; on a
    one-GPU machine that is the same-device case (the switching logic itself is checked on the host)."""
    before = torch.cuda.current_device()
    w = WORKLOADS["gdn_d128"].with_(variant=variant, qn=1e-3)
    x = make_scan_inputs(w, seed=22, device=DEV, B=1, H=1, L=70)
    run_gpu(variant, x)
    ws = torch.empty(256, dtype=torch.uint8, device=DEV)
    kdn.read_device_status(ws)
    assert torch.cuda.current_device() == before
