"""Shared helpers for the GPU parity tests: run the C-ABI calls one by one on
seeded inputs and compare with the oracle.  Imports torch lazily so the CPU
suite can import the pure helpers."""
from __future__ import annotations

import numpy as np

# Router logits: the kernels sum H bf16 x bf16 products in fp32 (about H/16
# sequential fp32 additions of K16 partial sums); the oracle sums in fp64 and
# rounds once.  With |x w| summing to about 40 at the workloads' magnitudes
# (H <= 4096, W_r ~ N(0, 0.02), RMS-normalised x), four standard deviations of
# that rounding walk, sqrt(H/16) * 2^-24 * 40 * 4, come to about 1e-4.
ROUTER_LOGIT_ATOL = 1e-4
ROUTER_LOGIT_RTOL = 1e-4
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


def logit_tol(ref):
    """Tolerance on a GPU router logit against the oracle's value `ref`."""
    return ROUTER_LOGIT_ATOL + ROUTER_LOGIT_RTOL * np.abs(ref)


def tie_band(a, b):
    """Two oracle logits closer than this may be ranked either way by a kernel
    whose logits each lie within logit_tol of the oracle's."""
    return 2.0 * (ROUTER_LOGIT_ATOL + ROUTER_LOGIT_RTOL * max(abs(a), abs(b)))


def check_routing(oracle_logits, gpu_ids, k, gpu_logits=None):
    """Compare GPU top-k ids with the oracle's logits.

    The top-k is a decision taken on floating-point logits, so it is checked
    in the precision the kernel takes it in: when the GPU's own logits are
    given, its ids must be their top-k (logit descending, index ascending)
    exactly, for every token.  Against the oracle, a token is exact if the
    GPU ids equal the oracle's sorted top-k; otherwise it is accepted as a
    near tie when the GPU's ids are k distinct experts and, rank by rank, the
    GPU's expert has an oracle logit within tie_band of the oracle's logit at
    that rank.  Returns (ok, near_tie_tokens, mismatched_tokens); a token
    whose ids are not the top-k of the GPU's logits counts as mismatched."""
    L = np.asarray(oracle_logits, np.float64)
    T, E = L.shape
    ids = np.asarray(gpu_ids)
    bad = set()
    if gpu_logits is not None:
        own = oracle_topk_order(np.asarray(gpu_logits, np.float64), k)[:, :k]
        bad.update(int(t) for t in np.nonzero(~(own == ids).all(axis=1))[0])
    order = oracle_topk_order(L, k)
    exact = (order[:, :k] == ids).all(axis=1)
    near = []
    for t in np.nonzero(~exact)[0]:
        top = [L[t, e] for e in order[t]]
        ok = len(set(ids[t].tolist())) == k and all(
            0 <= ids[t, j] < E and abs(L[t, ids[t, j]] - top[j]) <= tie_band(L[t, ids[t, j]], top[j])
            for j in range(k))
        if ok and int(t) not in bad:
            near.append(int(t))
        else:
            bad.add(int(t))
    bad = sorted(bad)
    return len(bad) == 0, near, bad


def near_tie_report(oracle_logits, gpu_ids, k, max_list=32):
    """Tokens with two adjacent logits among the oracle's first k+1 inside
    the tie band, whether or not the GPU's ids differ there:
    [(token, rank, gap)], gap the absolute difference of the two logits."""
    L = np.asarray(oracle_logits, np.float64)
    order = oracle_topk_order(L, k)
    top = np.take_along_axis(L, order, axis=1)
    gap = np.abs(top[:, :-1] - top[:, 1:])
    scale = np.maximum(np.abs(top[:, :-1]), np.abs(top[:, 1:]))
    band = 2.0 * (ROUTER_LOGIT_ATOL + ROUTER_LOGIT_RTOL * scale)
    hits = np.argwhere(gap < band)
    return [(int(t), int(r), float(gap[t, r])) for t, r in hits[:max_list]]


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
