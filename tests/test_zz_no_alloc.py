"""moe_experts_static_scratch: the decode expert path with its scratch in the
library's fixed array instead of a caller's workspace.

On the GPU its output is compared with moe_experts (the workspace entry point)
on the same routing, for two calls in a row with different shapes, so the
second call runs over the first call's leftovers in the shared array.  Both
entry points run the same deterministic kernels with the scratch at another
address, so the outputs must agree bit for bit (which is within the
per-token relative L2 bar of the parity tests, and stricter).  The size limit
is a host check and is tested without a GPU.
"""
import numpy as np
import pytest

import expert_ffn_execution_b200 as sm
from expert_ffn_execution_b200._binding import EINVAL, EUNSUPPORTED
from tests.harness import OUT_REL_L2, rel_l2_rows

MAX_SCRATCH_HALFS = 1 << 20  # T*k*I limit of the static array (2 MiB of fp16)


def _fake_weights(E, H, I, fmt=sm.FMT_Q2_32):
    # a 256-byte-aligned address that is never dereferenced: the calls below
    # return before any device work
    stride = (sm.strata_expert_bytes(fmt, H, I) + 255) // 256 * 256
    return sm.qweights(fmt, E, H, I, 1 << 20, stride)


def test_rejects_sizes_beyond_the_array():
    w = _fake_weights(64, 256, 4096)
    p = 1 << 20
    # 16 * 32 * 4096 fp16 = 4 MiB > 2 MiB
    rc = sm.moe_experts_static_scratch(p, w, p, p, p, 16, 32, p, p, stream=0, check=False)
    assert rc == EUNSUPPORTED
    # T beyond the decode path
    w = _fake_weights(64, 256, 256)
    rc = sm.moe_experts_static_scratch(p, w, p, p, p, sm.DECODE_MAX_T + 1, 1, p, p, stream=0,
                                       check=False)
    assert rc == EUNSUPPORTED
    # exactly at the limit passes the size check (and then fails on a null y)
    w = _fake_weights(64, 256, 2048)
    assert 16 * 32 * 2048 == MAX_SCRATCH_HALFS
    rc = sm.moe_experts_static_scratch(p, w, p, p, p, 16, 32, None, p, stream=0, check=False)
    assert rc == EINVAL


def _routed(config, T, seed_layer):
    """Inputs and routing of one layer through the existing entry points."""
    import moe_inputs as mi
    import torch
    dev = "cuda"
    c = mi.CONFIGS[config]
    inp = mi.make_layer(config, T, layer=seed_layer, device=dev)
    H, I, k = c.H, c.I, c.k
    E = inp.w_router.shape[1]
    qw = sm.qweights(c.fmt, E, H, I, inp.experts, inp.experts.stride(0))
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    P = T * k
    r = {
        "T": T, "k": k, "H": H, "qw": qw, "status": status,
        "hidden": torch.empty(T, H, dtype=torch.bfloat16, device=dev),
        "ids": torch.empty(T, k, dtype=torch.int32, device=dev),
        "w": torch.empty(T, k, dtype=torch.float32, device=dev),
        "counts": torch.empty(E, dtype=torch.int32, device=dev),
        "offsets": torch.empty(E + 1, dtype=torch.int32, device=dev),
        "perm": torch.empty(P, dtype=torch.int32, device=dev),
        "inv": torch.empty(P, dtype=torch.int32, device=dev),
        "active": torch.empty(E + 1, dtype=torch.int32, device=dev),
        "inp": inp,
    }
    nb = max(sm.moe_route_workspace_size(T, H, E, k), 256)
    rws = torch.empty(nb, dtype=torch.uint8, device=dev)
    sm.moe_route(inp.x, T, H, c.eps, inp.w_router, inp.bias, E, k, r["hidden"], r["ids"], r["w"],
                 r["counts"], r["offsets"], r["perm"], r["inv"], r["active"], rws, nb, status)
    r["y_ref"] = torch.empty(P, H, dtype=torch.float32, device=dev)
    nb = sm.moe_experts_workspace_size(qw, T, k)
    ews = torch.empty(nb, dtype=torch.uint8, device=dev)
    sm.moe_experts(r["hidden"], qw, r["offsets"], r["perm"], r["active"], T, k, r["y_ref"], ews,
                   nb, status)
    r["y"] = torch.full((P, H), float("nan"), dtype=torch.float32, device=dev)
    return r


@pytest.mark.gpu
def test_matches_workspace_entry_point_on_two_calls_in_a_row():
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    # first call: the larger scratch footprint (4-bit codebook, T=8, k=6, I=2048);
    # second call: a smaller one (2-bit, T=4, k=10, I=640) over its leftovers
    runs = [_routed(4, 8, 3), _routed(1, 4, 5)]
    torch.cuda.synchronize()
    alloc0 = torch.cuda.memory_allocated()
    reserved0 = torch.cuda.memory_reserved()
    for r in runs:
        sm.moe_experts_static_scratch(r["hidden"], r["qw"], r["offsets"], r["perm"], r["active"],
                                      r["T"], r["k"], r["y"], r["status"])
    torch.cuda.synchronize()
    assert torch.cuda.memory_allocated() == alloc0
    assert torch.cuda.memory_reserved() == reserved0
    for r in runs:
        assert sm.strata_read_status(r["status"]) == 0
        y = r["y"].cpu().numpy()
        y_ref = r["y_ref"].cpu().numpy()
        assert np.isfinite(y).all()
        err = rel_l2_rows(y, y_ref)
        assert err.max() <= OUT_REL_L2, err.max()
        assert torch.equal(r["y"], r["y_ref"]), "not bit-identical to moe_experts"
