"""Device-side failure detection without a fault: a bounded wait that nothing
completes runs out, the kernel records it and returns, the host reads
GDN_ERR_TIMEOUT, and the context keeps working."""

import pytest
import torch

from frame_wise_gated_b200 import api
from tests import gdn_testutil as U

pytestmark = pytest.mark.gpu


def test_bounded_wait_reports_timeout_and_context_survives():
    api.check_device_status()                      # clean start
    api.selftest_wait(arrive=True, limit_ns=1_000_000)
    api.check_device_status()                      # completed wait: no status
    api.selftest_wait(arrive=False, limit_ns=1_000_000)
    with pytest.raises(api.GdnError) as ei:
        api.check_device_status()
    assert ei.value.status == api.GDN_ERR_TIMEOUT
    api.check_device_status()                      # the word was cleared
    # the context is still usable: a normal scan runs and matches the oracle
    arr = U.random_case(91, 1, 1, 4, 64, 128, bf16=True, state=True)
    d = U.dev_inputs(arr, True)
    out, st = api.frame_scan_fwd_ex(d["q"], d["k"], d["v"], d["beta"], d["gamma"], d["state"])
    torch.cuda.synchronize()
    api.check_device_status()
    o_ref, _ = U.oracle_slab(arr, 0, 0, True)
    assert U.rel_frob_per_frame(U.host(out[0, 0]), o_ref) < U.TOL_BF16


def test_selftest_rejects_long_limits():
    with pytest.raises(api.GdnError):
        api.selftest_wait(arrive=False, limit_ns=10**10)
