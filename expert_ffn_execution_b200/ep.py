"""Expert parallelism for the routed-expert FFN layer.

The pages run experts on several devices ("path D", multi-GPU peer experts,
lcz.me/topic/2153; the walk-through's layer split over 2-3 GPUs); they give
no data path for it.  This module is one: the E experts of a layer are split
into G contiguous ranges, one per rank, and every rank

  1. routes its own tokens (RMSNorm, router, top-k, bucket: moe_route);
  2. lays out the hidden row of each of its (token, slot) pairs in sorted
     (expert-major) order (moe_gather_rows).  With contiguous expert ranges
     the sorted order is also ordered by destination rank, so the rows for
     rank d are one contiguous run whose length follows from the bucket's
     offsets;
  3. exchanges row counts, then rows and the rows' local expert ids, with an
     all-to-all into buffers on the receiving rank (NCCL over NVLink on
     GPUs; no kernel reads another GPU's memory);
  4. runs its local experts on the rows it received, each row one token
     routed to one expert (moe_bucket with k = 1, moe_experts), and puts the
     outputs back in the order received (moe_gather_rows with the inverse
     of that local sort);
  5. sends the outputs back with the reverse all-to-all, which delivers them
     in the sorted order the rows left in, and combines its own tokens in
     the fixed slot order, with the shared expert and the residual
     (moe_combine).

The arithmetic of every step is the single-rank layer's: only the row
traffic is added.  Compute is delegated to a backend (CudaEPBackend: the
library's kernels; tests substitute a host implementation) and the
exchange to an exchange object (DistExchange: torch.distributed
all_to_all_single; tests also use an in-process one).
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np
import torch


def expert_ranges(E: int, G: int):
    """Contiguous expert range [lo, hi) of each of G ranks (sizes differ by at
    most one)."""
    if G < 1 or E < G:
        raise ValueError(f"cannot split {E} experts over {G} ranks")
    return [(r * E // G, (r + 1) * E // G) for r in range(G)]


def send_counts(offsets, ranges):
    """Rows this rank sends to each rank: the pairs routed to that rank's
    experts, read off the bucket offsets (int [E+1])."""
    off = np.asarray(offsets)
    return [int(off[hi] - off[lo]) for lo, hi in ranges]


def sorted_local_ids(offsets, ranges):
    """For every sorted position s: the local index (on its owner rank) of
    the expert the position belongs to."""
    off = np.asarray(offsets, np.int64)
    P = int(off[-1])
    out = np.empty(P, np.int32)
    for lo, hi in ranges:
        for e in range(lo, hi):
            out[off[e]:off[e + 1]] = e - lo
    return out


@dataclass
class Dispatch:
    """What one rank keeps between sending its rows and combining."""
    x: object            # the layer input (residual stream)
    route: dict          # hidden, ids, w, counts, offsets, perm, inv (backend tensors)
    rows: object         # [P, H] hidden rows of the pairs, sorted order
    ids: object          # [P] local expert id of each row on its owner rank
    counts: list         # rows sent to each rank
    shared_y: object     # the shared expert's output for this rank's tokens, or None


class EPLayer:
    """One layer's experts range on this rank; `backend` does the compute."""

    def __init__(self, backend, E: int, k: int, rank: int, world: int):
        self.be = backend
        self.E, self.k, self.rank, self.G = E, k, rank, world
        self.ranges = expert_ranges(E, world)
        self.lo, self.hi = self.ranges[rank]

    def prepare(self, x) -> Dispatch:
        r = self.be.route(x)
        off = self.be.to_host(r["offsets"]).astype(np.int64)
        P = int(off[-1])
        rows = self.be.gather_pairs(r["hidden"], r["perm"], self.k, P)
        ids = self.be.from_host(sorted_local_ids(off, self.ranges))
        shared = self.be.shared(r["hidden"])
        return Dispatch(x, r, rows, ids, send_counts(off, self.ranges), shared)

    def compute(self, recv_rows, recv_ids):
        return self.be.local_experts(recv_rows, recv_ids)

    def finish(self, d: Dispatch, y_sorted):
        return self.be.combine(y_sorted, d.route, d.shared_y, d.x)

    def forward(self, x, exchange):
        d = self.prepare(x)
        recv_counts = exchange.counts(d.counts)
        recv_rows = exchange.rows(d.rows, d.counts, recv_counts)
        recv_ids = exchange.rows(d.ids, d.counts, recv_counts)
        y_recv = self.compute(recv_rows, recv_ids)
        y_sorted = exchange.rows(y_recv, recv_counts, d.counts)
        return self.finish(d, y_sorted)


class DistExchange:
    """All-to-all of row blocks over a torch.distributed process group: rows
    for rank d are the d-th contiguous run of the send buffer; received rows
    land in a new local buffer, source rank by source rank.  Every rank
    takes the same collective steps in the same order."""

    def __init__(self, group=None):
        import torch.distributed as dist
        self.dist = dist
        self.group = group

    def counts(self, send):
        dev = self._device()
        t = torch.tensor(send, dtype=torch.int64, device=dev)
        out = torch.empty_like(t)
        self.dist.all_to_all_single(out, t, group=self.group)
        return [int(v) for v in out.tolist()]

    def rows(self, send, send_counts, recv_counts):
        send = send.contiguous()
        shape = (int(sum(recv_counts)),) + tuple(send.shape[1:])
        out = torch.empty(shape, dtype=send.dtype, device=send.device)
        # 16-bit rows travel as bytes (not every backend moves 16-bit types)
        s, o = send, out
        if send.element_size() == 2:
            s, o = send.view(torch.uint8), out.view(torch.uint8)
        self.dist.all_to_all_single(o, s, list(recv_counts), list(send_counts), group=self.group)
        return out

    def _device(self):
        if self.dist.get_backend(self.group) == "nccl":
            return torch.device("cuda", torch.cuda.current_device())
        return torch.device("cpu")


def forward_in_process(layers, xs):
    """All G ranks of one layer in one process, the exchange done by copies:
    the same data path as DistExchange, for a single device or the host."""
    G = len(layers)
    ds = [layers[r].prepare(xs[r]) for r in range(G)]
    starts = [np.concatenate([[0], np.cumsum(d.counts)]) for d in ds]

    def block(t, r, d):  # rows rank r sends to rank d
        return t[int(starts[r][d]):int(starts[r][d + 1])]

    cat = torch.cat
    recv_rows = [cat([block(ds[s].rows, s, d) for s in range(G)]) for d in range(G)]
    recv_ids = [cat([block(ds[s].ids, s, d) for s in range(G)]) for d in range(G)]
    y_recv = [layers[d].compute(recv_rows[d], recv_ids[d]) for d in range(G)]
    # rank d's received rows are source-major: split them back per source
    outs = []
    for r in range(G):
        parts = []
        for d in range(G):
            rc = [ds[s].counts[d] for s in range(G)]
            o = int(sum(rc[:r]))
            parts.append(y_recv[d][o:o + rc[r]])
        outs.append(layers[r].finish(ds[r], cat(parts)))
    return outs


class CudaEPBackend:
    """The library's kernels for one rank: full router weights, the rank's
    expert range [lo, hi) of the layer's blob array, an optional shared
    expert.  Tensors live on the current CUDA device."""

    def __init__(self, w_router, bias, experts, fmt, H, I, k, lo, hi, shared=None,
                 shared_fmt=None, eps=1e-6):
        from . import _binding as sm
        self.sm = sm
        self.dev = experts.device
        self.wr, self.bias, self.k, self.eps = w_router, bias, k, eps
        self.H, self.I, self.fmt = H, I, fmt
        self.E = w_router.shape[1]
        self.loc = experts[lo:hi]  # a view: the rank's experts, back to back
        self.El = hi - lo
        self.qw = sm.qweights(fmt, self.El, H, I, self.loc, self.loc.stride(0))
        self.sqw = (sm.qweights(shared_fmt, 1, H, I, shared, shared.stride(0))
                    if shared is not None else None)
        self.status = torch.zeros(1, dtype=torch.int32, device=self.dev)

    def to_host(self, t):
        return t.cpu().numpy()

    def from_host(self, a):
        return torch.as_tensor(a).to(self.dev)

    def _ws(self, n):
        return torch.empty(max(int(n), 256), dtype=torch.uint8, device=self.dev)

    def route(self, x):
        sm, T, H, E, k, dev = self.sm, x.shape[0], self.H, self.E, self.k, self.dev
        P = T * k
        r = {"hidden": torch.empty(T, H, dtype=torch.bfloat16, device=dev),
             "ids": torch.empty(T, k, dtype=torch.int32, device=dev),
             "w": torch.empty(T, k, dtype=torch.float32, device=dev),
             "counts": torch.empty(E, dtype=torch.int32, device=dev),
             "offsets": torch.empty(E + 1, dtype=torch.int32, device=dev),
             "perm": torch.empty(max(P, 1), dtype=torch.int32, device=dev),
             "inv": torch.empty(max(P, 1), dtype=torch.int32, device=dev),
             "active": torch.empty(E + 1, dtype=torch.int32, device=dev)}
        ws = self._ws(sm.moe_route_workspace_size(T, H, E, k))
        sm.moe_route(x, T, H, self.eps, self.wr, self.bias, E, k, r["hidden"], r["ids"], r["w"],
                     r["counts"], r["offsets"], r["perm"], r["inv"], r["active"], ws, ws.numel(),
                     self.status)
        return r

    def gather_pairs(self, hidden, perm, k, P):
        sm = self.sm
        rows = torch.empty(P, self.H, dtype=torch.bfloat16, device=self.dev)
        sm.moe_gather_rows(hidden, sm.DTYPE_BF16, hidden.shape[0], self.H, perm, k, P, rows,
                           sm.DTYPE_BF16, self.status)
        return rows

    def shared(self, hidden):
        if self.sqw is None:
            return None
        sm, T = self.sm, hidden.shape[0]
        ydt = torch.float32 if T <= sm.DECODE_MAX_T else torch.float16
        y = torch.empty(T, self.H, dtype=ydt, device=self.dev)
        ws = self._ws(sm.moe_shared_expert_workspace_size(self.sqw, T))
        sm.moe_shared_expert(hidden, self.sqw, T, y, ws, ws.numel(), self.status)
        if ydt == torch.float16:  # the combine takes one dtype for y and shared_y: fp32
            y32 = torch.empty(T, self.H, dtype=torch.float32, device=self.dev)
            idx = torch.arange(T, dtype=torch.int32, device=self.dev)
            sm.moe_gather_rows(y, sm.DTYPE_F16, T, self.H, idx, 1, T, y32, sm.DTYPE_F32,
                               self.status)
            y = y32
        return y

    def local_experts(self, rows, lid):
        """Rows received from every rank, one expert each (local id): the
        routed experts as T = R tokens with k = 1, outputs fp32 in the order
        received."""
        sm, R, H, dev = self.sm, rows.shape[0], self.H, self.dev
        y_recv = torch.empty(R, H, dtype=torch.float32, device=dev)
        if R == 0:
            return y_recv
        El = self.El
        counts = torch.empty(El, dtype=torch.int32, device=dev)
        offsets = torch.empty(El + 1, dtype=torch.int32, device=dev)
        perm = torch.empty(R, dtype=torch.int32, device=dev)
        inv = torch.empty(R, dtype=torch.int32, device=dev)
        active = torch.empty(El + 1, dtype=torch.int32, device=dev)
        ids = lid.to(torch.int32).reshape(R, 1).contiguous()
        bw = self._ws(sm.moe_bucket_workspace_size(R, 1, El))
        sm.moe_bucket(ids, R, 1, El, counts, offsets, perm, inv, active, bw, bw.numel(),
                      self.status)
        decode = R <= sm.DECODE_MAX_T
        y = torch.empty(R, H, dtype=torch.float32 if decode else torch.float16, device=dev)
        ew = self._ws(sm.moe_experts_workspace_size(self.qw, R, 1))
        sm.moe_experts(rows, self.qw, offsets, perm, active, R, 1, y, ew, ew.numel(),
                       self.status)
        sm.moe_gather_rows(y, sm.DTYPE_F32 if decode else sm.DTYPE_F16, R, H, inv, 1, R, y_recv,
                           sm.DTYPE_F32, self.status)
        return y_recv

    def combine(self, y_sorted, r, shared_y, x):
        sm, T, H, k = self.sm, x.shape[0], self.H, self.k
        out = torch.empty(T, H, dtype=torch.bfloat16, device=self.dev)
        res = torch.empty(T, H, dtype=torch.float32, device=self.dev)
        sm.moe_combine(y_sorted, sm.DTYPE_F32, r["inv"], r["w"], shared_y, sm.DTYPE_F32, x, T, k,
                       H, out, res, self.status)
        return out, res
