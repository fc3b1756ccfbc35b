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


def oracle_topk_order(logits, k):
    """The oracle's ranking of the first k+1 experts per token (logit
    descending, expert index ascending on equal logits): int [T, k+1]."""
    L = np.asarray(logits, np.float64)
    T, E = L.shape
    idx = np.broadcast_to(np.arange(E), (T, E))
    order = np.lexsort((idx, -L), axis=-1)
    return order[:, :min(E, k + 1)]


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
    order = oracle_topk_order(L, k)
    exact = (order[:, :k] == ids).all(axis=1)
    near, bad = [], []
    for t in np.nonzero(~exact)[0]:
        top = [L[t, e] for e in order[t]]
        tie = any(abs(top[i] - top[i + 1]) < NEAR_TIE_REL * max(abs(top[i]), abs(top[i + 1]))
                  for i in range(len(top) - 1))
        ok = tie and len(set(ids[t])) == k and all(
            0 <= ids[t, j] < E and abs(L[t, ids[t, j]] - top[j]) <=
            NEAR_TIE_REL * max(abs(top[j]), 1e-30) for j in range(k))
        (near if ok else bad).append(int(t))
    return len(bad) == 0, near, bad


def near_tie_report(oracle_logits, gpu_ids, k, max_list=32):
    """Tokens whose oracle logits of ranks k and k+1 (or any two adjacent
    ranks among the first k+1) lie within the near-tie band, whether or not
    the GPU's ids differ there: [(token, rank, relative gap)]."""
    L = np.asarray(oracle_logits, np.float64)
    order = oracle_topk_order(L, k)
    top = np.take_along_axis(L, order, axis=1)
    gap = np.abs(top[:, :-1] - top[:, 1:])
    scale = np.maximum(np.abs(top[:, :-1]), np.abs(top[:, 1:]))
    rel = gap / np.maximum(scale, 1e-30)
    hits = np.argwhere(rel < NEAR_TIE_REL)
    return [(int(t), int(r), float(rel[t, r])) for t, r in hits[:max_list]]


def parallel_rows(fn, n_rows, chunk, workers=None):
    """Run fn(lo, hi) over row ranges [lo, hi) in a thread pool (the oracle's
    C calls release the GIL) and return the results in order."""
    import concurrent.futures as cf
    import os
    ranges = [(lo, min(n_rows, lo + chunk)) for lo in range(0, n_rows, chunk)]
    with cf.ThreadPoolExecutor(max_workers=workers or os.cpu_count() or 4) as ex:
        return list(ex.map(lambda r: fn(*r), ranges))


def stratified_tokens(counts, offsets, perm, k, T, n=256, tile=128, seed=0):
    """A token sample for the full-size prefill checks: every token of the
    least-loaded non-empty expert and of the tail (last partial 128-token
    tile) of the most-loaded expert, tokens of the most-loaded expert's full
    tiles, tail tokens of other experts, then uniform random tokens up to n
    (sorted, unique)."""
    counts = np.asarray(counts)
    offsets = np.asarray(offsets)
    perm = np.asarray(perm)
    rng = np.random.default_rng(seed)
    pick = set()

    def toks_of(e, lo=None, hi=None):
        s0, s1 = int(offsets[e]), int(offsets[e + 1])
        lo = s0 if lo is None else lo
        hi = s1 if hi is None else hi
        return [int(perm[s]) // k for s in range(lo, hi)]

    nz = np.nonzero(counts)[0]
    emax = int(nz[np.argmax(counts[nz])])
    emin = int(nz[np.argmin(counts[nz])])
    pick.update(toks_of(emin)[:32])
    c = int(counts[emax])
    tail0 = int(offsets[emax]) + (c // tile) * tile
    pick.update(toks_of(emax, tail0)[:32])
    full = toks_of(emax, int(offsets[emax]), tail0)
    if full:
        pick.update(rng.choice(full, min(32, len(full)), replace=False).tolist())
    others = rng.choice(nz, min(32, len(nz)), replace=False)
    for e in others:
        c = int(counts[e])
        t0 = int(offsets[e]) + (c // tile) * tile
        tt = toks_of(int(e), t0) or toks_of(int(e))
        pick.add(int(tt[-1]))
    rest = [t for t in rng.permutation(T).tolist() if t not in pick]
    pick.update(rest[:max(0, n - len(pick))])
    return np.array(sorted(pick), dtype=np.int64)
