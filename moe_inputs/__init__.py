"""Seeded synthetic inputs for the routed-expert FFN layer.

This module is shared by the CUDA path's tests/bench and by the oracle's
tests.  It holds none of the layer's arithmetic: it draws random tensors with
the workloads' sizes and value distributions and writes them in the expert
blob byte layout (a storage format, restated here from its definition in
include/strata_moe.h):

  one expert = gate codes | gate scales | up codes | up scales |
               down codes | down scales, each plane on a 256-byte boundary;
  gate/up are [I rows x H], down is [H rows x I]; codes are uint8 planes
  ([N][K/4] for the 2-bit format, [N][K/2] for the 4-bit codebook format),
  scales are fp16 [N][K/32], or for the MXFP4 format (4-bit E2M1 codes laid
  out like the 4-bit codebook format) one E8M0 byte per block, [N][K/32].

Random codes are uniform bytes, which makes every 2-bit code uniform in 0..3
and every 4-bit code uniform in 0..15.  Scales are U[lo, hi] rounded to fp16;
MXFP4 scales are E8M0 exponents e uniform over the integers with 2^(e-127) in
[lo, hi] (lo and hi powers of two).

Workloads (the five layer configurations this library is measured on):
  C0  H=2560 E=512 I=640 k=10, T=1, 2-bit experts d~U[0.005,0.02], no bias
  C1  48 stacked C0-shape layers, T=4, Zipf(s=1.1) router bias per layer
  C2  one C0-shape layer, T=8192, Zipf(s=1.1) bias
  C3  C2 plus a shared expert (same shape) in the 4-bit codebook format,
      d~U[0.0005,0.002]; also T=1 and T=4
  C4  H=4096 E=256 I=2048 k=6, 4-bit codebook routed + shared experts,
      d~U[0.0005,0.002], Zipf(s=1.0) bias, x rounded to bf16; T=1, 4, 8192
  C6  the C1/C2 layer with MXFP4 routed experts, scales 2^-9..2^-6, Zipf(s=1.1)
      bias; T=1, 4, 8192 (the native-MXFP4 model tier's expert format)
x ~ N(0,1) fp32 (then RMSNorm inside the layer); W_r ~ N(0, 0.02) bf16 [H, E].
Zipf bias: a seeded permutation gives each expert a popularity rank r in
1..E and bias[e] = -0.5 * s * ln(r_e) (half the log of a Zipf(s) probability,
without its normalising constant, which shifts every logit equally).
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import torch

FMT_Q2 = 1
FMT_Q4CB = 2
FMT_MXFP4 = 3


def _round256(x: int) -> int:
    return (x + 255) & ~255


def plane_layout(fmt: int, H: int, I: int):
    """[(name, offset, nbytes, rows, K, kind)] for the six planes, and the
    blob size.  kind is 'codes' or 'scales'."""
    if fmt not in (FMT_Q2, FMT_Q4CB, FMT_MXFP4):
        raise ValueError(f"unknown format {fmt}")
    if H % 32 or I % 32:
        raise ValueError("H and I must be multiples of 32")
    planes = []
    off = 0
    for name, rows, K in (("gate", I, H), ("up", I, H), ("down", H, I)):
        nc = rows * (K // 4 if fmt == FMT_Q2 else K // 2)
        planes.append((name, off, nc, rows, K, "codes"))
        off = _round256(off + nc)
        ns = rows * (K // 32) * (1 if fmt == FMT_MXFP4 else 2)
        planes.append((name, off, ns, rows, K, "scales"))
        off = _round256(off + ns)
    return planes, off


def expert_bytes(fmt: int, H: int, I: int) -> int:
    return plane_layout(fmt, H, I)[1]


@dataclass
class LayerConfig:
    name: str
    H: int
    E: int
    I: int
    k: int
    fmt: int
    d_range: tuple
    Ts: tuple
    layers: int = 1
    zipf_s: float | None = None
    shared_fmt: int | None = None
    shared_d_range: tuple | None = None
    x_bf16: bool = False
    eps: float = 1e-6
    notes: str = ""
    extra: dict = field(default_factory=dict)


CONFIGS = {
    0: LayerConfig("C0", 2560, 512, 640, 10, FMT_Q2, (0.005, 0.02), (1,),
                   notes="single layer, decode T=1"),
    1: LayerConfig("C1", 2560, 512, 640, 10, FMT_Q2, (0.005, 0.02), (4,), layers=48,
                   zipf_s=1.1, notes="48 stacked layers, T=4 verify window"),
    2: LayerConfig("C2", 2560, 512, 640, 10, FMT_Q2, (0.005, 0.02), (8192,),
                   zipf_s=1.1, notes="prefill chunk T=8192"),
    3: LayerConfig("C3", 2560, 512, 640, 10, FMT_Q2, (0.005, 0.02), (8192, 1, 4),
                   zipf_s=1.1, shared_fmt=FMT_Q4CB, shared_d_range=(0.0005, 0.002),
                   notes="C2 plus a 4-bit-codebook shared expert"),
    4: LayerConfig("C4", 4096, 256, 2048, 6, FMT_Q4CB, (0.0005, 0.002), (1, 4, 8192),
                   zipf_s=1.0, shared_fmt=FMT_Q4CB, shared_d_range=(0.0005, 0.002),
                   x_bf16=True, notes="large experts, 4-bit codebook"),
    # the other reading of config 3: every expert, routed and shared, in the
    # 4-bit codebook format at E = 512 (reported beside C3, not a parity gate)
    5: LayerConfig("C3b", 2560, 512, 640, 10, FMT_Q4CB, (0.0005, 0.002), (1, 4),
                   zipf_s=1.1, shared_fmt=FMT_Q4CB, shared_d_range=(0.0005, 0.002),
                   notes="C3 with 4-bit-codebook routed experts"),
    6: LayerConfig("C6", 2560, 512, 640, 10, FMT_MXFP4, (2.0**-9, 2.0**-6), (1, 4, 8192),
                   zipf_s=1.1, notes="C1/C2 layer with MXFP4 routed experts"),
}


def seed_for(config: int, layer: int, part: str) -> int:
    parts = {"x": 1, "router": 2, "bias": 3, "experts": 4, "shared": 5, "xstep": 6}
    return ((1000 + config) * 100003 + layer * 7919 + parts[part] * 104729) % (2**62)


def _gen(device, seed: int) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def gen_x(T: int, H: int, seed: int, device="cpu", bf16_first: bool = False) -> torch.Tensor:
    """x ~ N(0,1) fp32 [T, H] (optionally rounded through bf16)."""
    x = torch.randn(T, H, generator=_gen(device, seed), device=device, dtype=torch.float32)
    if bf16_first:
        x = x.to(torch.bfloat16).to(torch.float32)
    return x


def gen_router(H: int, E: int, seed: int, device="cpu") -> torch.Tensor:
    """W_r ~ N(0, 0.02) as bf16 [H, E]."""
    w = torch.randn(H, E, generator=_gen(device, seed), device=device, dtype=torch.float32)
    return (w * 0.02).to(torch.bfloat16)


def gen_zipf_bias(E: int, s: float, seed: int, device="cpu") -> torch.Tensor:
    """bias[e] = -0.5 * s * ln(rank_e), ranks a seeded permutation of 1..E."""
    ranks = torch.randperm(E, generator=_gen("cpu", seed)).to(torch.float64) + 1.0
    bias = -0.5 * s * torch.log(ranks)
    return bias.to(torch.float32).to(device)


def gen_experts(fmt: int, E: int, H: int, I: int, d_range, seed: int, device="cpu",
                out: torch.Tensor | None = None) -> torch.Tensor:
    """E expert blobs as uint8 [E, expert_bytes]: uniform random code bytes,
    fp16 scales U[lo, hi] (MXFP4: E8M0 bytes for the powers of two in
    [lo, hi]).  Writes into `out` if given."""
    planes, nbytes = plane_layout(fmt, H, I)
    if out is None:
        out = torch.empty(E, nbytes, dtype=torch.uint8, device=device)
    assert out.shape == (E, nbytes) and out.dtype == torch.uint8
    g = _gen(out.device, seed)
    lo, hi = d_range
    out.zero_()
    for name, off, n, rows, K, kind in planes:
        if kind == "codes":
            out[:, off:off + n] = torch.randint(0, 256, (E, n), generator=g, device=out.device,
                                                dtype=torch.uint8)
        elif fmt == FMT_MXFP4:
            e_lo = 127 + int(round(math.log2(lo)))
            e_hi = 127 + int(round(math.log2(hi)))
            out[:, off:off + n] = torch.randint(e_lo, e_hi + 1, (E, n), generator=g,
                                                device=out.device, dtype=torch.uint8)
        else:
            cnt = n // 2
            d = torch.rand(E, cnt, generator=g, device=out.device, dtype=torch.float32)
            d = (d * (hi - lo) + lo).to(torch.float16)
            out[:, off:off + n] = d.view(torch.uint8).view(E, n)
    return out


@dataclass
class LayerInputs:
    x: torch.Tensor            # fp32 [T, H]
    w_router: torch.Tensor     # bf16 [H, E]
    bias: torch.Tensor | None  # fp32 [E]
    experts: torch.Tensor      # uint8 [E, expert_bytes]
    shared: torch.Tensor | None  # uint8 [1, expert_bytes]


def make_layer(config: int, T: int, layer: int = 0, device="cpu", E: int | None = None,
               with_experts: bool = True) -> LayerInputs:
    c = CONFIGS[config]
    E = c.E if E is None else E
    x = gen_x(T, c.H, seed_for(config, layer, "x"), device, c.x_bf16)
    wr = gen_router(c.H, E, seed_for(config, layer, "router"), device)
    bias = (gen_zipf_bias(E, c.zipf_s, seed_for(config, layer, "bias"), device)
            if c.zipf_s is not None else None)
    ex = (gen_experts(c.fmt, E, c.H, c.I, c.d_range, seed_for(config, layer, "experts"), device)
          if with_experts else None)
    sh = None
    if c.shared_fmt is not None and with_experts:
        sh = gen_experts(c.shared_fmt, 1, c.H, c.I, c.shared_d_range,
                         seed_for(config, layer, "shared"), device)
    return LayerInputs(x, wr, bias, ex, sh)

