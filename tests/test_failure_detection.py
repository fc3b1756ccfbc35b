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
    # an unknown mode, or missing buffers
    assert sm.strata_selftest_wait(5_000_000_000, 0, 1 << 20, 1 << 20, stream=0,
                                   check=False) == EINVAL
    assert sm.strata_selftest_wait(1000, 3, 1 << 20, 1 << 20, stream=0, check=False) == EINVAL
    assert sm.strata_selftest_wait(1000, -1, 1 << 20, 1 << 20, stream=0, check=False) == EINVAL
    assert sm.strata_selftest_wait(1000, 0, None, 1 << 20, stream=0, check=False) == EINVAL
    assert sm.strata_selftest_wait(1000, 0, 1 << 20, None, stream=0, check=False) == EINVAL


def _usable_after_timeout(torch):
    """An ordinary call with a fresh status word runs cleanly: the routing of
    one token through moe_route, whose kernels take dev_status."""
    import moe_inputs as mi
    c = mi.CONFIGS[0]
    T, E, k, H = 1, 16, 4, c.H
    inp = mi.make_layer(0, T, layer=0, device="cuda", E=E)
    dev = "cuda"
    status2 = torch.zeros(1, dtype=torch.int32, device=dev)
    hid = torch.empty(T, H, dtype=torch.bfloat16, device=dev)
    ids = torch.full((T, k), -1, dtype=torch.int32, device=dev)
    w = torch.empty(T, k, dtype=torch.float32, device=dev)
    counts = torch.empty(E, dtype=torch.int32, device=dev)
    offsets = torch.empty(E + 1, dtype=torch.int32, device=dev)
    perm = torch.empty(T * k, dtype=torch.int32, device=dev)
    inv = torch.empty(T * k, dtype=torch.int32, device=dev)
    active = torch.empty(E + 1, dtype=torch.int32, device=dev)
    n = max(sm.moe_route_workspace_size(T, H, E, k), 256)
    wsb = torch.empty(n, dtype=torch.uint8, device=dev)
    sm.moe_route(inp.x, T, H, c.eps, inp.w_router, inp.bias, E, k, hid, ids, w, counts, offsets,
                 perm, inv, active, wsb, n, status2)
    torch.cuda.synchronize()
    assert sm.strata_read_status(status2) == OK
    assert torch.isfinite(hid.float()).all()
    got = ids[0].tolist()
    assert len(set(got)) == k and all(0 <= e < E for e in got)
    assert int(offsets[E]) == T * k


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
    _usable_after_timeout(torch)


@pytest.mark.gpu
def test_counter_wait_times_out_and_context_stays_usable():
    """The cross-CTA counter wait (the fused decode kernel's wait for another
    CTA's h rows) on a counter nobody raises: it gives up within its budget,
    reports STRATA_DEV_TIMEOUT, and the next call runs cleanly."""
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = torch.full((2,), -1, dtype=torch.int32, device="cuda")
    t0 = time.perf_counter()
    sm.strata_selftest_wait(2_000_000, 2, status, out)
    torch.cuda.synchronize()
    elapsed = time.perf_counter() - t0
    assert out.tolist() == [0, 0]
    assert sm.strata_read_status(status) == ETIMEOUT
    assert elapsed < 1.0, elapsed
    _usable_after_timeout(torch)
