"""CPU checks of the C-ABI library: it loads, exports every symbol the header
declares, agrees on blob sizes, and rejects bad arguments on the host before
anything is enqueued (no kernel launches; no GPU needed)."""
import os
import re

import numpy as np
import pytest

import expert_ffn_execution_b200 as sm
import moe_inputs
import oracle
from expert_ffn_execution_b200 import _binding as B
from tests.harness import check_routing

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def header_symbols():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            txt = open(os.path.join(ROOT, "include", fn)).read()
            names |= set(re.findall(r"STRATA_API\s+[\w\s\*]+?\b((?:moe|strata)_\w+)\s*\(", txt))
    return names


def test_library_exports_every_declared_symbol():
    lib = sm.load()
    declared = header_symbols()
    assert len(declared) >= 16
    for name in declared:
        assert hasattr(lib, name), name
    assert declared == set(B.exported_symbols())


def test_abi_version_and_status_strings():
    assert sm.abi_version() == 1
    assert sm.status_string(0) == "ok"
    assert sm.status_string(1) == "invalid argument"
    assert sm.status_string(6) == "fp16 intermediate overflowed"
    assert sm.status_string(99) == "unknown status"


@pytest.mark.parametrize("fmt,H,I", [(1, 2560, 640), (2, 2560, 640), (2, 4096, 2048), (1, 128, 128),
                                     (3, 2560, 640), (3, 4096, 2048), (3, 128, 128)])
def test_expert_bytes_agree(fmt, H, I):
    assert sm.strata_expert_bytes(fmt, H, I) == moe_inputs.expert_bytes(fmt, H, I)
    assert sm.strata_expert_bytes(fmt, H, I) == oracle.expert_bytes(fmt, H, I)
    assert sm.strata_expert_bytes(4, H, I) == 0
    assert sm.strata_expert_bytes(0, H, I) == 0
    assert sm.strata_expert_bytes(fmt, H + 16, I) == 0


def test_host_validation_rejects_bad_arguments():
    """Every one of these returns STRATA_EINVAL from the host checks."""
    E = B.EINVAL
    assert sm.moe_rmsnorm(None, -1, 2560, 1e-6, None, stream=0, check=False) == E
    assert sm.moe_rmsnorm(None, 1, 2561, 1e-6, None, stream=0, check=False) == E
    assert sm.moe_rmsnorm(None, 1, 2560, 1e-6, None, stream=0, check=False) == E
    assert sm.moe_router_topk(None, None, None, 1, 2560, 512, 0, None, None, None, None, 0, None,
                              stream=0, check=False) == E
    assert sm.moe_router_topk(None, None, None, 1, 2560, 511, 10, None, None, None, None, 0,
                              None, stream=0, check=False) == E
    assert sm.moe_router_topk(None, None, None, 1, 2560, 512, 33, None, None, None, None, 0,
                              None, stream=0, check=False) == E
    assert sm.moe_bucket(None, 1, 11, 10, None, None, None, None, None, None, 0, None, stream=0,
                         check=False) == E
    w = sm.qweights(1, 512, 2560, 640, 0, 1536000)  # NULL base
    assert sm.moe_experts(None, w, None, None, None, 1, 10, None, None, 0, None, stream=0,
                          check=False) == E
    w = sm.qweights(1, 512, 2560, 640, 256, 1536000 - 256)  # stride too small
    assert sm.moe_experts(None, w, None, None, None, 1, 10, None, None, 0, None, stream=0,
                          check=False) == E
    w = sm.qweights(3, 512, 2560, 640, 256, 1536000)  # unknown format
    assert sm.moe_experts(None, w, None, None, None, 1, 10, None, None, 0, None, stream=0,
                          check=False) == E
    assert sm.moe_combine(None, 7, None, None, None, 0, None, 1, 10, 2560, None, None, None,
                          stream=0, check=False) == E
    assert sm.moe_combine(None, 0, None, None, None, 0, None, 1, 10, 2560, None, 0x1000, None,
                          stream=0, check=False) == E  # residual_out without residual


def test_empty_batch_is_a_noop():
    """T == 0 returns STRATA_OK without touching any pointer."""
    assert sm.moe_rmsnorm(None, 0, 2560, 1e-6, None, stream=0) == 0
    assert sm.moe_router_topk(None, None, None, 0, 2560, 512, 10, None, None, None, None, 0,
                              None, stream=0) == 0
    w = sm.qweights(1, 512, 2560, 640, 256, 1536000)
    assert sm.moe_experts(None, w, None, None, None, 0, 10, None, None, 0, None, stream=0) == 0
    assert sm.moe_combine(None, 0, None, None, None, 0, None, 0, 10, 2560, None, None, None,
                          stream=0) == 0


def test_workspace_queries():
    assert sm.moe_router_topk_workspace_size(4, 2560, 512, 10) >= 40 * 4 * 512 * 4
    assert sm.moe_bucket_workspace_size(4, 10, 512) == 0
    assert sm.moe_bucket_workspace_size(8192, 10, 512) >= 320 * 512 * 4
    w = sm.qweights(1, 512, 2560, 640, 256, 1536000)
    assert sm.moe_experts_workspace_size(w, 4, 10) >= 40 * 640 * 2
    assert sm.moe_layer_workspace_size(4, 512, 10, w, None) > 0


def test_near_tie_rule():
    """The routing comparison accepts swaps only inside the tie band (twice
    the router-logit tolerance, absolute plus relative), and a token whose
    ids are not the top-k of the GPU's own logits is a mismatch."""
    L = np.array([[3.0, 2.0, 1.0, 0.5], [1.0, 1.0 + 1e-7, 0.2, 0.1],
                  [0.01, 0.01 + 5e-5, -0.3, -0.4], [0.5, 0.5 + 1e-3, 0.1, 0.0]])
    ok, near, bad = check_routing(L, np.array([[0, 1], [1, 0], [1, 0], [1, 0]]), 2)
    assert ok and near == [] and bad == []
    # swaps of logits 1e-7 apart, and of small logits 5e-5 apart (inside the
    # absolute part of the band), are near ties
    ok, near, bad = check_routing(L, np.array([[0, 1], [0, 1], [0, 1], [1, 0]]), 2)
    assert ok and near == [1, 2]
    # a gap of 1e-3 at 0.5 and a gap of 1 are outside the band
    ok, near, bad = check_routing(L, np.array([[1, 0], [1, 0], [1, 0], [0, 1]]), 2)
    assert not ok and bad == [0, 3]
    # ids that are not the top-k of the GPU's own logits
    G = L.astype(np.float32)
    ok, near, bad = check_routing(L, np.array([[0, 1], [0, 1], [1, 0], [1, 0]]), 2, gpu_logits=G)
    assert not ok and bad == [1]
    ok, near, bad = check_routing(L, np.array([[0, 1], [1, 0], [1, 0], [1, 0]]), 2, gpu_logits=G)
    assert ok and bad == []
