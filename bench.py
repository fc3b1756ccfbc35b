#!/usr/bin/env python3
"""Benchmark of the routed-expert FFN layer on B200.

Default workload (the headline configuration): 48 stacked MoE layers of the
hidden-2560 / 512-expert / width-640 / top-10 shape with 2-bit (Q2_32) expert
weights, 37.75 GB resident in HBM, T = 4 tokens per step (one token plus
three speculative drafts verified together).  One step = for each layer
RMSNorm -> router/top-k -> bucket -> experts -> combine + residual add, each
layer a call sequence of the library's C ABI, captured into a CUDA graph.

Prints one JSON line (rank 0).  `value` is whole-job tokens/s with the inputs
resident in HBM, device-timed with CUDA events over exactly --steps steps
between a barrier + synchronize on both sides (max over ranks).  `e2e` is the
same metric with each step's input copied host->device from pinned memory
and its result copied back inside the timed region.  `roofline` is the
moe_experts stage (decode: the counter reset and the fused gate/up + down
kernel, or the gate/up and down kernels) measured live with
external CUDA events captured in the step graphs, against algorithmic bytes.

--impl reference times the CPU oracle (the only reference implementation this
layer has) on the host cores, on a bounded sample of the same workload.
Multi-GPU (torchrun): every rank holds its own copy of the model and runs its
own token batches (replicas, weak scaling); there is no collective on the
data path.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import moe_inputs as mi  # noqa: E402

PEAKS_FILE = os.path.join(ROOT, "MEASURED_PEAKS.json")
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0
METRIC = "MoE-layer tokens/s; decode HBM GB/s and prefill TFLOPS as % of B200 peak"
NCU_TRAFFIC_FILE = os.path.join(ROOT, "profiles", "traffic.json")


def peaks():
    try:
        with open(PEAKS_FILE) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), float(p["bf16_tflops"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, FALLBACK_BF16_TFLOPS, "fallback"


def sustained_tflops():
    try:
        with open(PEAKS_FILE) as f:
            return float(json.load(f)["bf16_tflops_sustained"])
    except Exception:
        return 1400.0


def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def replica_input_seed(config, rank, g):
    """Seed of input batch g on a rank: every replica runs its own tokens."""
    return mi.seed_for(config, 1000 * rank + g, "xstep")


def max_over_ranks(values, device):
    """Element-wise max of `values` over all ranks (the slowest rank sets the
    job's time); the values themselves with one rank."""
    dist = torch.distributed
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return [float(v) for v in values]
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(v) for v in t.tolist()]


def job_tokens_per_s(tokens_per_step_per_rank, steps, world, ms):
    """Whole-job throughput: the tokens all ranks processed / the job time."""
    return tokens_per_step_per_rank * steps * world / (ms * 1e-3)


class Clocks:
    """Samples nvidia-smi clocks and throttle reasons during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.dev = device_index
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.dev), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.2)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        rows = []
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) >= 9:
                rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}

        def num(s):
            try:
                return float(s)
            except ValueError:
                return None
        sm = [num(r[1]) for r in rows if num(r[1])]
        mx = max((num(r[2]) for r in rows if num(r[2])), default=None)
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx,
                "reasons": reasons, "samples": len(rows)}


# ---------------------------------------------------------------- model
class DecodeStack:
    """L layers of one configuration, weights generated on the device."""

    def __init__(self, config: int, T: int, layers: int, device):
        import expert_ffn_execution_b200 as sm
        self.sm = sm
        self.c = mi.CONFIGS[config]
        self.config, self.T, self.L, self.dev = config, T, layers, device
        c = self.c
        self.H, self.E, self.I, self.k = c.H, c.E, c.I, c.k
        self.ebytes = mi.expert_bytes(c.fmt, c.H, c.I)
        self.wr, self.bias, self.experts, self.qw, self.shared, self.sqw = [], [], [], [], [], []
        for l in range(layers):
            inp = mi.make_layer(config, T, layer=l, device=device, with_experts=False)
            self.wr.append(inp.w_router)
            self.bias.append(inp.bias)
            ex = mi.gen_experts(c.fmt, c.E, c.H, c.I, c.d_range, mi.seed_for(config, l, "experts"),
                                device)
            self.experts.append(ex)
            self.qw.append(sm.qweights(c.fmt, c.E, c.H, c.I, ex, ex.stride(0)))
            if c.shared_fmt is not None:
                sh = mi.gen_experts(c.shared_fmt, 1, c.H, c.I, c.shared_d_range,
                                    mi.seed_for(config, l, "shared"), device)
                self.shared.append(sh)
                self.sqw.append(sm.qweights(c.shared_fmt, 1, c.H, c.I, sh, sh.stride(0)))
            else:
                self.shared.append(None)
                self.sqw.append(None)
        torch.cuda.synchronize()
        T, H, E, k = self.T, self.H, self.E, self.k
        P = T * k
        dev = device
        self.decode = T <= sm.DECODE_MAX_T
        ydt = torch.float32 if self.decode else torch.float16
        self.ydtype = sm.DTYPE_F32 if self.decode else sm.DTYPE_F16
        self.hidden = torch.empty(T, H, dtype=torch.bfloat16, device=dev)
        self.ids = torch.empty(T, k, dtype=torch.int32, device=dev)
        self.w = torch.empty(T, k, dtype=torch.float32, device=dev)
        self.counts = torch.empty(E, dtype=torch.int32, device=dev)
        self.offsets = torch.empty(E + 1, dtype=torch.int32, device=dev)
        self.perm = torch.empty(P, dtype=torch.int32, device=dev)
        self.inv = torch.empty(P, dtype=torch.int32, device=dev)
        self.y = torch.empty(P, H, dtype=ydt, device=dev)
        self.shy = torch.empty(T, H, dtype=ydt, device=dev) if c.shared_fmt else None
        self.out = torch.empty(T, H, dtype=torch.bfloat16, device=dev)
        self.xa = torch.empty(T, H, dtype=torch.float32, device=dev)
        self.xb = torch.empty(T, H, dtype=torch.float32, device=dev)
        n = max(sm.moe_route_workspace_size(T, H, E, k),
                sm.moe_experts_workspace_size(self.qw[0], T, k),
                sm.moe_shared_expert_workspace_size(self.sqw[0], T) if self.sqw[0] else 0)
        self.ws = torch.empty(int(n) + 256, dtype=torch.uint8, device=dev)
        self.status = torch.zeros(1, dtype=torch.int32, device=dev)
        self.launches_per_step = None

    def step(self, x_in, x_out, active_bufs=None, events=None):
        """Enqueue one step (all layers): x_out = x_in after L layers."""
        sm, T, H, E, k = self.sm, self.T, self.H, self.E, self.k
        st = self.status
        ws, wn = self.ws, self.ws.numel()
        cur = x_in
        for l in range(self.L):
            nxt = x_out if l == self.L - 1 else (self.xa if (l % 2 == 0) else self.xb)
            act = active_bufs[l]
            sm.moe_route(cur, T, H, self.c.eps, self.wr[l], self.bias[l], E, k, self.hidden,
                         self.ids, self.w, self.counts, self.offsets, self.perm, self.inv, act,
                         ws, wn, st)
            if events is not None:
                events[l][0].record()
            sm.moe_experts(self.hidden, self.qw[l], self.offsets, self.perm, act, T, k, self.y, ws,
                           wn, st)
            if events is not None:
                events[l][1].record()
            if self.sqw[l] is not None:
                sm.moe_shared_expert(self.hidden, self.sqw[l], T, self.shy, ws, wn, st)
            sm.moe_combine(self.y, self.ydtype, self.inv, self.w, self.shy, self.ydtype, cur, T, k,
                           H, self.out, nxt, st)
            cur = nxt


def kernels_per_layer(T, k, shared):
    """Kernel launches the library enqueues per layer.  Decode (T <= 16):
    moe_route 2 (logits with RMSNorm; top-k and bucket), experts 2 (counter
    reset and the fused gate/up + down kernel, or gate/up and down), shared
    expert 2, combine 1.  Prefill: moe_route 7 (RMSNorm,
    router GEMM, top-k, bucket histogram, column scan, offsets, scatter),
    experts 4 (plan, gather, gate/up GEMM, down GEMM), shared expert 4,
    combine 1."""
    if T <= 16:
        return 2 + 2 + 1 + (2 if shared else 0)
    return 7 + 4 + 1 + (4 if shared else 0)


def run_ours(args):
    ws_, rank, local = dist_env()
    if ws_ > 1:
        import datetime
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    cfg = mi.CONFIGS[args.config]
    T = args.tokens or cfg.Ts[0]
    L = args.layers or cfg.layers
    stack = DecodeStack(args.config, T, L, dev)
    prefill = T > stack.sm.DECODE_MAX_T
    H, E, k = stack.H, stack.E, stack.k
    G = min(args.steps, args.graphs)
    # distinct seeded inputs per graph, per rank
    xs = [mi.gen_x(T, H, replica_input_seed(args.config, rank, g), dev, cfg.x_bf16)
          for g in range(G)]
    x_out = [torch.empty(T, H, dtype=torch.float32, device=dev) for _ in range(G)]
    actives = [[torch.empty(E + 1, dtype=torch.int32, device=dev) for _ in range(L)]
               for _ in range(G)]
    events = [[(torch.cuda.Event(enable_timing=True, external=True),
                torch.cuda.Event(enable_timing=True, external=True)) for _ in range(L)]
              for _ in range(G)]
    # eager warm-up (also loads the library), then capture one graph per input
    s = torch.cuda.Stream(device=dev)
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        for g in range(G):
            stack.step(xs[g], x_out[g], actives[g])
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    # Only graph 0 records the experts-stage events: an event node between two
    # kernels breaks their programmatic overlap, so the other graphs run the
    # step uninstrumented and the stage is timed on every G-th step.
    graphs = []
    for g in range(G):
        gr = torch.cuda.CUDAGraph()
        with torch.cuda.graph(gr, stream=s):
            stack.step(xs[g], x_out[g], actives[g], events[g] if g == 0 else None)
        graphs.append(gr)
    torch.cuda.synchronize()
    st = torch.cuda.current_stream()
    for i in range(args.warmup):
        graphs[i % G].replay()
    torch.cuda.synchronize()
    if int(stack.status.item()) != 0:
        raise SystemExit(f"device status {int(stack.status.item())} after warm-up")
    # the bucket of the last layer accounts for every (token, slot) pair
    if int(stack.offsets[E].item()) != T * k:
        raise SystemExit(f"bucket total {int(stack.offsets[E].item())} != T*k = {T * k}")

    def barrier():
        if ws_ > 1:
            torch.distributed.barrier()

    # device-timed region
    clocks = Clocks(local)
    clocks.start()
    barrier()
    torch.cuda.synchronize()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(st)
    for i in range(args.steps):
        graphs[i % G].replay()
    t1.record(st)
    torch.cuda.synchronize()
    barrier()
    clk = clocks.stop()
    ms = t0.elapsed_time(t1)
    # moe_experts stage durations from the last replay of graph 0
    durs, bytes_ = [], []
    for l in range(L):
        durs.append(events[0][l][0].elapsed_time(events[0][l][1]) * 1e-3)
        U = int(actives[0][l][0].item())
        bytes_.append(U * stack.ebytes + T * H * 2 + T * k * H * 4)
    # prefill: algorithmic flops of the expert GEMMs (routed + shared)
    flops = 6.0 * H * stack.I * T * k + (6.0 * H * stack.I * T if cfg.shared_fmt else 0.0)
    # end-to-end: pinned host input -> device, step, result -> pinned host
    hx = [xs[g].cpu().pin_memory() for g in range(G)]
    hout = [torch.empty(T, H, dtype=torch.float32).pin_memory() for _ in range(G)]
    barrier()
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(st)
    for i in range(args.steps):
        g = i % G
        xs[g].copy_(hx[g], non_blocking=True)
        graphs[g].replay()
        hout[g].copy_(x_out[g], non_blocking=True)
    e1.record(st)
    torch.cuda.synchronize()
    barrier()
    e2e_ms = e0.elapsed_time(e1)
    if int(stack.status.item()) != 0:
        raise SystemExit(f"device status {int(stack.status.item())}")
    ms, e2e_ms = max_over_ranks([ms, e2e_ms], dev)
    value = job_tokens_per_s(T, args.steps, ws_, ms)
    e2e = job_tokens_per_s(T, args.steps, ws_, e2e_ms)
    hbm, bf16, src = peaks()
    bf16_sus = sustained_tflops()
    avg_dur = sum(durs) / len(durs)
    avg_bytes = sum(bytes_) / len(bytes_)
    achieved = avg_bytes / avg_dur / 1e9
    if prefill:
        achieved_tf = flops / avg_dur / 1e12
    traffic = None
    try:
        with open(NCU_TRAFFIC_FILE) as f:
            tr = json.load(f)
        traffic = tr.get(f"C{args.config}_T{T}")
    except Exception:
        pass
    result = None
    if rank == 0:
        cpu = None
        if ws_ == 1 and not args.no_cpu_baseline:
            cpu = cpu_baseline(stack, xs[0], args)
        result = {
            "metric": METRIC, "value": round(value, 2), "unit": "tokens/s", "n_gpus": ws_,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms / args.steps, 4),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f16",
            "data": "synthetic (seeded; random-init weights of the stated shape)",
            "config": {"workload": f"C{args.config}: {L} stacked MoE layers, H={H}, E={E}, "
                                   f"I={stack.I}, top-{k}, "
                                   f"{'Q2_32' if cfg.fmt == 1 else 'Q4CB_32'} experts "
                                   f"({L * E * stack.ebytes / 1e9:.2f} GB), T={T} tokens per step",
                       "layers": L, "T": T, "tokens_per_step_per_gpu": T,
                       "parallelism": f"replicas x{ws_}",
                       "accumulate": "f32", "weights": "2.5 bits/weight" if cfg.fmt == 1 else "4.5 bits/weight",
                       "l2": "no flush: per-step weight stream (~%.1f GB) >> 126 MB L2"
                             % (sum(bytes_[:L]) / 1e9) if not prefill else
                             "no flush: per-step working set (weights + activations) > 1 GB",
                       "graphs": G},
            "e2e": {"value": round(e2e, 2), "unit": "tokens/s",
                    "h2d_bytes_per_step": T * H * 4, "d2h_bytes_per_step": T * H * 4},
            "gpu_launches": kernels_per_layer(T, k, cfg.shared_fmt is not None) * L * args.steps,
            "roofline": ({"kernel": "moe_experts decode stage (fused gate/up + down kernel)",
                          "bound": "hbm", "achieved": round(achieved, 1), "peak": hbm,
                          "unit": "GB/s", "frac": round(achieved / hbm, 4),
                          "peak_source": f"{src} (MEASURED_PEAKS.json hbm_gbs, burst)"
                          if src == "measured" else "fallback 6.65 TB/s",
                          "avg_launch_us": round(avg_dur * 1e6, 3),
                          "timed": "external CUDA events around moe_experts of every layer in "
                                   "one of the G replayed step graphs",
                          "algorithmic_bytes_per_launch": int(avg_bytes),
                          "traffic": traffic} if not prefill else
                         {"kernel": "moe_experts prefill stage (plan, gather, tcgen05 gate/up "
                                    "and down grouped GEMMs)",
                          "bound": "tensor", "achieved": round(achieved_tf, 1),
                          "peak": bf16_sus, "unit": "TFLOP/s",
                          "frac": round(achieved_tf / bf16_sus, 4),
                          "frac_of_burst": round(achieved_tf / bf16, 4),
                          "peak_source": "MEASURED_PEAKS.json bf16_tflops_sustained (fp16 "
                                         "kind::f16 runs at the bf16 rate)",
                          "avg_launch_us": round(avg_dur * 1e6, 3),
                          "timed": "external CUDA events around moe_experts of every layer in "
                                   "one of the G replayed step graphs",
                          "algorithmic_flops_per_launch": flops,
                          "traffic": traffic}),
            "clocks": clk,
        }
        if cpu is not None:
            result["cpu_baseline"] = cpu
        print(json.dumps(result), flush=True)
    for gr in graphs:
        del gr
    graphs.clear()
    if ws_ > 1:
        torch.distributed.destroy_process_group()
    return result


# ---------------------------------------------------------------- CPU side
def oracle_sample(config, T, layers, device_stack=None, target_s=15.0, x0=None):
    """Time the oracle on the workload until about target_s seconds of CPU
    work: decode (T <= 16) runs whole layers of the stack in order; prefill
    runs 16-token slices of the first layer.  Returns (tokens/s of the whole
    workload, description, threads)."""
    import numpy as np

    import oracle
    c = mi.CONFIGS[config]
    x = (x0.cpu() if x0 is not None else mi.gen_x(T, c.H, mi.seed_for(config, 0, "xstep"))).numpy()
    spent, n = 0.0, 0

    def layer_inputs(l):
        if device_stack is not None:
            wr = device_stack.wr[l].cpu().view(torch.int16).numpy().view(np.uint16)
            bias = None if device_stack.bias[l] is None else device_stack.bias[l].cpu().numpy()
            blobs = device_stack.experts[l].cpu().numpy()
            sh = None if device_stack.shared[l] is None else device_stack.shared[l][0].cpu().numpy()
        else:
            inp = mi.make_layer(config, 1, layer=l, device="cpu")
            wr = inp.w_router.view(torch.int16).numpy().view(np.uint16)
            bias = None if inp.bias is None else inp.bias.numpy()
            blobs = inp.experts.numpy()
            sh = None if inp.shared is None else inp.shared[0].numpy()
        return wr, bias, blobs, sh

    if T <= 16:
        for l in range(layers):
            wr, bias, blobs, sh = layer_inputs(l)
            t0 = time.perf_counter()
            hid = oracle.rmsnorm(x, c.eps)
            r = oracle.moe_layer(hid, wr, bias, c.E, c.k, c.fmt, c.I, blobs,
                                 shared_fmt=c.shared_fmt or 0, shared_blob=sh, residual=x)
            spent += time.perf_counter() - t0
            n += 1
            x = r["residual_out"]
            if spent >= target_s:
                break
        per_layer = spent / n
        return (T / (per_layer * layers),
                f"{n} of {layers} layers, T={T}, scaled to a {layers}-layer step "
                f"({per_layer:.3f} s per layer)", min(oracle.num_threads(), T))
    wr, bias, blobs, sh = layer_inputs(0)
    tok = 0
    while spent < target_s and tok < T:
        sl = x[tok:tok + 16]
        t0 = time.perf_counter()
        hid = oracle.rmsnorm(sl, c.eps)
        oracle.moe_layer(hid, wr, bias, c.E, c.k, c.fmt, c.I, blobs,
                         shared_fmt=c.shared_fmt or 0, shared_blob=sh, residual=sl)
        spent += time.perf_counter() - t0
        tok += sl.shape[0]
    return (tok / (spent * layers), f"{tok} of {T} tokens of layer 0 in 16-token slices, "
            f"scaled to {layers} layer(s)", min(oracle.num_threads(), 16))


def cpu_baseline(stack, x0, args):
    tok_s, desc, cores = oracle_sample(args.config, stack.T, stack.L, stack, args.cpu_seconds, x0)
    return {"value": round(tok_s, 4), "unit": "tokens/s", "cores": cores, "kind": "oracle",
            "sample": desc}


def run_reference(args):
    """The oracle as the reference arm.  One step times a bounded unit of the
    workload: one token's router logits + softmax/top-k and ONE of its k
    expert FFNs (cycling over tokens, experts and two cached layers), plus
    that token's combine; the step time of the full workload is then
    L x (router + k x expert + combine) per token."""
    import numpy as np

    import oracle
    ws_, rank, _ = dist_env()
    if rank != 0:
        return None
    cfg = mi.CONFIGS[args.config]
    T = args.tokens or cfg.Ts[0]
    L = args.layers or cfg.layers
    cached = []
    for l in range(min(L, 2)):
        inp = mi.make_layer(args.config, T, layer=l, device="cpu")
        hid = oracle.rmsnorm(inp.x.numpy(), cfg.eps)
        wr = inp.w_router.view(torch.int16).numpy().view(np.uint16)
        bias = None if inp.bias is None else inp.bias.numpy()
        cached.append((hid, wr, bias, inp.experts.numpy(),
                       None if inp.shared is None else inp.shared[0].numpy()))
    t_router, t_expert, t_comb = [], [], []

    def unit(i, record):
        hid, wr, bias, blobs, sh = cached[i % len(cached)]
        t = (i // len(cached)) % T
        j = (i // (len(cached) * T)) % cfg.k
        a = time.perf_counter()
        lg = oracle.router_logits(hid[t:t + 1], wr, bias)
        ids, w = oracle.topk(lg, cfg.k)
        b = time.perf_counter()
        y = oracle.expert_ffn(cfg.fmt, blobs[ids[0, j]], cfg.H, cfg.I, hid[t])
        if sh is not None and j == 0:
            y = y + oracle.expert_ffn(cfg.shared_fmt, sh, cfg.H, cfg.I, hid[t])
        c = time.perf_counter()
        oracle.combine(np.repeat(y[None, :], cfg.k, 0), w)
        d = time.perf_counter()
        if record:
            t_router.append(b - a)
            t_expert.append(c - b)
            t_comb.append(d - c)

    for i in range(args.warmup):
        unit(i, False)
    wall0 = time.perf_counter()
    for i in range(args.steps):
        unit(i, True)
    wall = time.perf_counter() - wall0
    per_tok_layer = (statistics.mean(t_router) + cfg.k * statistics.mean(t_expert)
                     + statistics.mean(t_comb))
    step_s = per_tok_layer * L * T
    value = T / step_s
    res = {"metric": METRIC, "value": round(value, 4), "unit": "tokens/s", "n_gpus": ws_,
           "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(step_s * 1e3, 3),
           "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
           "data": "synthetic (seeded; random-init weights of the stated shape)",
           "config": {"workload": f"C{args.config}: {L} stacked MoE layers, H={cfg.H}, E={cfg.E}, "
                                  f"I={cfg.I}, top-{cfg.k}, T={T} tokens per step",
                      "layers": L, "T": T},
           "impl": "reference",
           "cpu_baseline": {"value": round(value, 4), "unit": "tokens/s", "cores": 1,
                            "kind": "oracle",
                            "sample": f"{args.steps} units of one token's router+top-k and one "
                                      f"of its {cfg.k} expert FFNs (+combine), cycling over "
                                      f"{len(cached)} cached layers; scaled to {L} layers x "
                                      f"{cfg.k} experts x {T} tokens ({wall:.1f} s wall)"},
           "e2e": {"value": round(value, 4), "unit": "tokens/s", "h2d_bytes_per_step": 0,
                   "d2h_bytes_per_step": 0}}
    print(json.dumps(res), flush=True)
    return res


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--config", type=int, default=1)
    ap.add_argument("--tokens", type=int, default=0)
    ap.add_argument("--layers", type=int, default=0)
    ap.add_argument("--graphs", type=int, default=8)
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    if args.warmup < 3:
        raise SystemExit("--warmup must be >= 3")
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
