"""Failure detection without a GPU fault.

Every device wait in the library is bounded: after its cycle budget it ORs
STRATA_DEV_TIMEOUT into the caller's status word, raises the CTA's abort
flag (so later waits of that CTA return at once) and lets the CTA finish.
strata_selftest_wait runs those same waits in one CTA on an mbarrier that
nothing arrives at (or, as a control, one whose phase completes), with a
short budget, so the timeout path runs for real: no trap, no assert, no
hang, and the context stays usable for the next call.
"""
import time

import pytest

import expert_ffn_execution_b200 as sm
from expert_ffn_execution_b200._binding import EINVAL, ETIMEOUT, OK


def test_selftest_argument_checks():
    # rejected on the host before any launch: budget above the kernels' own,
    # or missing buffers
    assert sm.strata_selftest_wait(5_000_000_000, 0, 1 << 20, 1 << 20, stream=0,
                                   check=False) == EINVAL
    assert sm.strata_selftest_wait(1000, 0, None, 1 << 20, stream=0, check=False) == EINVAL
    assert sm.strata_selftest_wait(1000, 0, 1 << 20, None, stream=0, check=False) == EINVAL


@pytest.mark.gpu
def test_bounded_wait_times_out_and_context_stays_usable():
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = torch.full((2,), -1, dtype=torch.int32, device="cuda")
    # control: the phase completes, both waits succeed, the status is clean
    sm.strata_selftest_wait(2_000_000, 1, status, out)
    torch.cuda.synchronize()
    assert out.tolist() == [1, 1]
    assert sm.strata_read_status(status) == OK
    # nothing arrives: the first wait runs out (about 1 ms at 2e6 cycles),
    # the second returns at once on the abort flag
    t0 = time.perf_counter()
    sm.strata_selftest_wait(2_000_000, 0, status, out)
    torch.cuda.synchronize()
    elapsed = time.perf_counter() - t0
    assert out.tolist() == [0, 0]
    assert sm.strata_read_status(status) == ETIMEOUT
    assert elapsed < 1.0, elapsed
    # the context is usable: a fresh status word and an ordinary layer call
    import moe_inputs as mi
    c = mi.CONFIGS[0]
    inp = mi.make_layer(0, 1, layer=0, device="cuda", E=16)
    hid = torch.empty(1, c.H, dtype=torch.bfloat16, device="cuda")
    status2 = torch.zeros(1, dtype=torch.int32, device="cuda")
    sm.moe_rmsnorm(inp.x, 1, c.H, c.eps, hid)
    torch.cuda.synchronize()
    assert torch.isfinite(hid.float()).all()
    assert sm.strata_read_status(status2) == OK
