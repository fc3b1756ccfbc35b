"""Shared helpers for the GPU parity tests: run the C-ABI calls one by one on
seeded inputs and compare with the oracle.  Imports torch lazily so the CPU
suite can import the pure helpers."""
from __future__ import annotations

import numpy as np

NEAR_TIE_REL = 1e-5       # near-tie band on oracle logits (relative)
TOPK_W_ATOL = 1e-5        # |GPU w - oracle w|
OUT_REL_L2 = 5e-3         # per-token relative L2 of the layer output


def rel_l2_rows(a, b):
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    num = np.sqrt(((a - b) ** 2).sum(-1))
    den = np.sqrt((b ** 2).sum(-1))
    return num / np.maximum(den, 1e-30)


def check_routing(oracle_logits, gpu_ids, k):
    """Compare GPU top-k ids with the oracle's logits.

    A token is exact if the GPU ids equal the oracle's sorted top-k (logit
    descending, index ascending).  It is a near-tie if two adjacent logits
    among the oracle's top k+1 differ by less than NEAR_TIE_REL relative; a
    near-tie token is accepted when, position by position, the GPU's expert
    has an oracle logit within the tie band of the oracle's logit at that
    rank.  Returns (ok, near_tie_tokens, mismatched_tokens)."""
    L = np.asarray(oracle_logits, np.float64)
    T, E = L.shape
    ids = np.asarray(gpu_ids)
    near, bad = [], []
    for t in range(T):
        order = sorted(range(E), key=lambda e: (-L[t, e], e))
        ref = order[:k]
        if list(ids[t]) == ref:
            continue
        top = [L[t, e] for e in order[:min(E, k + 1)]]
        tie = any(abs(top[i] - top[i + 1]) < NEAR_TIE_REL * max(abs(top[i]), abs(top[i + 1]))
                  for i in range(len(top) - 1))
        ok = tie and len(set(ids[t])) == k and all(
            0 <= ids[t, j] < E and abs(L[t, ids[t, j]] - top[j]) <=
            NEAR_TIE_REL * max(abs(top[j]), 1e-30) for j in range(k))
        (near if ok else bad).append(t)
    return len(bad) == 0, near, bad
