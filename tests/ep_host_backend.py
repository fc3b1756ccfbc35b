"""Host stand-in for the compute of expert parallelism: the oracle's routing,
expert FFN and combine behind the backend interface of
expert_ffn_execution_b200.ep, so the exchange logic can run on CPU ranks
(gloo) and in process.  Test infrastructure only."""
from __future__ import annotations

import numpy as np
import torch

import oracle


class OracleEPBackend:
    def __init__(self, wr_u16, bias, blobs, fmt, H, I, k, lo, hi, shared_blob=None,
                 shared_fmt=0, eps=1e-6):
        self.wr, self.bias, self.fmt, self.H, self.I, self.k = wr_u16, bias, fmt, H, I, k
        self.E = wr_u16.shape[1]
        self.blobs = {e: blobs[e] for e in range(lo, hi)}  # this rank's experts only
        self.lo, self.hi = lo, hi
        self.shared_blob, self.shared_fmt, self.eps = shared_blob, shared_fmt, eps

    def to_host(self, t):
        return t.numpy()

    def from_host(self, a):
        return torch.as_tensor(np.ascontiguousarray(a))

    def route(self, x):
        hid = oracle.rmsnorm(x.numpy(), self.eps)
        lg = oracle.router_logits(hid, self.wr, self.bias)
        ids, w = oracle.topk(lg, self.k)
        counts, offsets, perm, inv = oracle.bucket(ids, self.E)
        t = torch.as_tensor
        return {"hidden": t(hid.view(np.int16)), "ids": t(ids), "w": t(w), "counts": t(counts),
                "offsets": t(offsets), "perm": t(perm), "inv": t(inv)}

    def gather_pairs(self, hidden, perm, k, P):
        return hidden[perm[:P].long() // k].contiguous()

    def shared(self, hidden):
        if self.shared_blob is None:
            return None
        hid = hidden.numpy().view(np.uint16)
        return torch.as_tensor(np.stack([oracle.expert_ffn(self.shared_fmt, self.shared_blob,
                                                           self.H, self.I, hid[t])
                                         for t in range(hid.shape[0])]))

    def local_experts(self, rows, lid):
        R = rows.shape[0]
        out = np.zeros((R, self.H), np.float32)
        r16 = rows.numpy().view(np.uint16)
        for i in range(R):
            e = self.lo + int(lid[i])
            assert self.lo <= e < self.hi, (e, self.lo, self.hi)
            out[i] = oracle.expert_ffn(self.fmt, self.blobs[e], self.H, self.I, r16[i])
        return torch.as_tensor(out)

    def combine(self, y_sorted, r, shared_y, x):
        inv = r["inv"].numpy()
        y_pairs = y_sorted.numpy()[inv]
        sh = None if shared_y is None else shared_y.numpy()
        of, ob, res = oracle.combine(y_pairs, r["w"].numpy(), sh, x.numpy())
        return torch.as_tensor(ob.view(np.int16)), torch.as_tensor(res)
