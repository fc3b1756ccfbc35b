"""Device-memory plumbing around the C ABI: torch owns the buffers, the
library's kernels do the work.  No arithmetic of the layer happens here."""
from __future__ import annotations

from dataclasses import dataclass

import torch

from . import _binding as B


@dataclass
class ExpertWeights:
    """E expert blobs stored back to back: uint8 [E, stride] on the device."""
    blobs: torch.Tensor
    fmt: int
    hidden: int
    inter: int

    def __post_init__(self):
        need = B.strata_expert_bytes(self.fmt, self.hidden, self.inter)
        if self.blobs.dtype != torch.uint8 or self.blobs.dim() != 2 or self.blobs.shape[1] < need:
            raise ValueError("blobs must be uint8 [E, >= expert_bytes]")
        self.qw = B.qweights(self.fmt, self.blobs.shape[0], self.hidden, self.inter,
                             self.blobs.data_ptr(), self.blobs.stride(0))

    @property
    def num_experts(self) -> int:
        return self.blobs.shape[0]


class MoELayer:
    """One routed-expert FFN layer: router W_r bf16 [H, E], optional bias fp32
    [E], routed experts and an optional shared expert."""

    def __init__(self, w_router: torch.Tensor, bias: torch.Tensor | None, experts: ExpertWeights,
                 k: int, shared: ExpertWeights | None = None, eps: float = 1e-6):
        self.w_router = w_router.contiguous()
        self.bias = None if bias is None else bias.contiguous()
        self.experts = experts
        self.shared = shared
        self.k = k
        self.eps = eps
        self.E = experts.num_experts
        self.H = experts.hidden
        self._ws = {}

    def workspace(self, T: int) -> torch.Tensor:
        if T not in self._ws:
            n = B.moe_layer_workspace_size(T, self.E, self.k, self.experts.qw,
                                           None if self.shared is None else self.shared.qw)
            self._ws[T] = torch.empty(max(n, 256), dtype=torch.uint8, device=self.w_router.device)
        return self._ws[T]

    def forward(self, x: torch.Tensor, out: torch.Tensor | None = None,
                residual_out: torch.Tensor | None = None, topk_ids: torch.Tensor | None = None,
                topk_w: torch.Tensor | None = None, dev_status: torch.Tensor | None = None,
                stream=None) -> torch.Tensor:
        T = x.shape[0]
        if out is None:
            out = torch.empty(T, self.H, dtype=torch.bfloat16, device=x.device)
        ws = self.workspace(T)
        B.moe_layer_forward(x, T, self.w_router, self.bias, self.E, self.k, self.experts.qw,
                            None if self.shared is None else self.shared.qw, self.eps, out,
                            residual_out, topk_ids, topk_w, ws, ws.numel(), dev_status, stream)
        return out
