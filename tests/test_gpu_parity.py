"""GPU parity: the CUDA path through the C ABI against the CPU oracle.

Inputs are the seeded synthetic workloads of moe_inputs, generated on the
device; the oracle receives the same bytes (hidden rows, router weights, the
blobs of the experts the routing touched).  Bars:
  - RMSNorm: within one bf16 ulp of the oracle.
  - Router: top-k ids exact except listed near-ties (oracle logits of two
    adjacent ranks within 1e-5 relative); weights within 1e-5.
  - Bucket: counts, offsets, perm, inv bit-exact vs the oracle on the GPU's ids.
  - Combine: bit-exact vs the oracle given the GPU's expert outputs.
  - Expert outputs and the layer output: per-token relative L2 <= 5e-3 vs the
    oracle run with the GPU's ids (teacher forcing).
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("needs a CUDA GPU", allow_module_level=True)

import expert_ffn_execution_b200 as sm  # noqa: E402
import moe_inputs as mi  # noqa: E402
import oracle  # noqa: E402
from expert_ffn_execution_b200._binding import EOVERFLOW, EUNSUPPORTED  # noqa: E402
from tests.harness import (OUT_REL_L2, TOPK_W_ATOL, check_routing, logit_tol, parallel_rows,  # noqa: E402
                           rel_l2_rows, stratified_tokens)

pytestmark = pytest.mark.gpu
DEV = "cuda"


def u16(t):
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def ws(nbytes):
    return torch.empty(max(int(nbytes), 256), dtype=torch.uint8, device=DEV)


class Run:
    """One layer through the individual C-ABI calls, all intermediates kept."""

    def __init__(self, config, T, layer=0, E=None, x=None):
        self.c = mi.CONFIGS[config]
        self.inp = mi.make_layer(config, T, layer=layer, device=DEV, E=E)
        if x is not None:
            self.inp.x = x
        self.T, self.H, self.I, self.k = T, self.c.H, self.c.I, self.c.k
        self.E = self.inp.w_router.shape[1]
        self.status = torch.zeros(1, dtype=torch.int32, device=DEV)
        self.qw = sm.qweights(self.c.fmt, self.E, self.H, self.I, self.inp.experts,
                              self.inp.experts.stride(0))
        self.sqw = None
        if self.inp.shared is not None:
            self.sqw = sm.qweights(self.c.shared_fmt, 1, self.H, self.I, self.inp.shared,
                                   self.inp.shared.stride(0))

    def run(self):
        T, H, E, k, I = self.T, self.H, self.E, self.k, self.I
        st = self.status
        self.hidden = torch.empty(T, H, dtype=torch.bfloat16, device=DEV)
        sm.moe_rmsnorm(self.inp.x, T, H, self.c.eps, self.hidden)
        self.ids = torch.empty(T, k, dtype=torch.int32, device=DEV)
        self.w = torch.empty(T, k, dtype=torch.float32, device=DEV)
        self.logits = torch.empty(T, E, dtype=torch.float32, device=DEV)
        rw = ws(sm.moe_router_topk_workspace_size(T, H, E, k))
        sm.moe_router_topk(self.hidden, self.inp.w_router, self.inp.bias, T, H, E, k, self.ids,
                           self.w, self.logits, rw, rw.numel(), st)
        P = T * k
        self.counts = torch.empty(E, dtype=torch.int32, device=DEV)
        self.offsets = torch.empty(E + 1, dtype=torch.int32, device=DEV)
        self.perm = torch.empty(max(P, 1), dtype=torch.int32, device=DEV)
        self.inv = torch.empty(max(P, 1), dtype=torch.int32, device=DEV)
        self.active = torch.empty(E + 1, dtype=torch.int32, device=DEV)
        bw = ws(sm.moe_bucket_workspace_size(T, k, E))
        sm.moe_bucket(self.ids, T, k, E, self.counts, self.offsets, self.perm, self.inv,
                      self.active, bw, bw.numel(), st)
        decode = T <= sm.DECODE_MAX_T
        ydt = torch.float32 if decode else torch.float16
        self.ydtype = sm.DTYPE_F32 if decode else sm.DTYPE_F16
        self.y = torch.empty(max(P, 1), H, dtype=ydt, device=DEV)
        ew = ws(sm.moe_experts_workspace_size(self.qw, T, k))
        sm.moe_experts(self.hidden, self.qw, self.offsets, self.perm, self.active, T, k, self.y,
                       ew, ew.numel(), st)
        self.shy = None
        if self.sqw is not None:
            self.shy = torch.empty(T, H, dtype=ydt, device=DEV)
            sw = ws(sm.moe_shared_expert_workspace_size(self.sqw, T))
            sm.moe_shared_expert(self.hidden, self.sqw, T, self.shy, sw, sw.numel(), st)
        self.out = torch.empty(T, H, dtype=torch.bfloat16, device=DEV)
        self.zero = torch.zeros(T, H, dtype=torch.float32, device=DEV)
        self.acc = torch.empty(T, H, dtype=torch.float32, device=DEV)
        sm.moe_combine(self.y, self.ydtype, self.inv, self.w, self.shy, self.ydtype, self.zero, T,
                       k, H, self.out, self.acc, st)
        torch.cuda.synchronize()
        assert sm.strata_read_status(self.status) == 0
        return self

    def blobs_for(self, ids):
        return {int(e): self.inp.experts[int(e)].cpu().numpy() for e in np.unique(ids)}


def check_layer(r: Run, sample=None):
    """Full check of one run.  RMSNorm, router logits, top-k ids and weights
    and the bucket are checked on every token; `sample` = token indices for
    the combine, expert-output and layer-output checks (all tokens if None).
    Returns the per-token relative L2 of the layer output on the sample."""
    T, H, E, k = r.T, r.H, r.E, r.k
    hid = u16(r.hidden)
    # RMSNorm within one bf16 ulp
    ref_h = oracle.rmsnorm(r.inp.x.cpu().numpy(), r.c.eps)
    a = oracle.bf16_bits_to_f32(hid).astype(np.float64)
    b = oracle.bf16_bits_to_f32(ref_h).astype(np.float64)
    ulp = 2.0 ** (np.floor(np.log2(np.maximum(np.abs(b), 1e-30))) - 7)
    assert np.all(np.abs(a - b) <= ulp), "rmsnorm beyond one bf16 ulp"
    # router on the GPU's hidden, every token (the oracle in token chunks on
    # the host's cores)
    wr = u16(r.inp.w_router)
    bias = None if r.inp.bias is None else r.inp.bias.cpu().numpy()
    ref_lg = np.concatenate(parallel_rows(
        lambda lo, hi: oracle.router_logits(hid[lo:hi], wr, bias), T, 256))
    gl = r.logits.cpu().numpy()
    assert np.all(np.abs(gl - ref_lg) <= logit_tol(ref_lg)), "router logits"
    gids = r.ids.cpu().numpy()
    ok, near, bad = check_routing(ref_lg, gids, k, gpu_logits=gl)
    assert ok, f"routing mismatch on tokens {bad[:10]}"
    if near:
        print(f"near-tie tokens: {near}")
    ref_ids_gpu_logits, ref_w = oracle.topk(gl, k)
    np.testing.assert_array_equal(ref_ids_gpu_logits, gids)
    assert np.abs(r.w.cpu().numpy() - ref_w).max() <= TOPK_W_ATOL
    # bucket bit-exact on the GPU's ids (all tokens)
    counts, offsets, perm, inv = oracle.bucket(gids, E)
    np.testing.assert_array_equal(r.counts.cpu().numpy(), counts)
    np.testing.assert_array_equal(r.offsets.cpu().numpy(), offsets)
    np.testing.assert_array_equal(r.perm.cpu().numpy()[:T * k], perm)
    np.testing.assert_array_equal(r.inv.cpu().numpy()[:T * k], inv)
    act = r.active.cpu().numpy()
    nz = np.nonzero(counts)[0]
    assert act[0] == len(nz)
    np.testing.assert_array_equal(act[1:1 + len(nz)], nz)
    toks = np.arange(T) if sample is None else np.asarray(sample)
    # combine bit-exact given the GPU's y (sampled tokens)
    rows = inv.reshape(T, k)[toks]
    yg = r.y[torch.as_tensor(rows.reshape(-1), device=DEV).long()].float().cpu().numpy()
    sh = None if r.shy is None else r.shy[torch.as_tensor(toks, device=DEV).long()].float().cpu().numpy()
    of, ob, _ = oracle.combine(yg, r.w.cpu().numpy()[toks], sh)
    np.testing.assert_array_equal(u16(r.out)[toks], ob)
    np.testing.assert_array_equal(r.acc.cpu().numpy()[toks], of)
    # expert outputs and the layer output vs the oracle (teacher-forced ids)
    blobs = r.blobs_for(gids[toks])
    pairs = [(i, int(t), j) for i, t in enumerate(toks) for j in range(k)]

    def expert_errs(lo, hi):
        out = []
        for i, t, j in pairs[lo:hi]:
            e = int(gids[t, j])
            ref_y = oracle.expert_ffn(r.c.fmt, blobs[e], H, r.I, hid[t])
            out.append((rel_l2_rows(yg[i * k + j], ref_y), t, j, e))
        return out
    for errs in parallel_rows(expert_errs, len(pairs), 16):
        for err, t, j, e in errs:
            assert err <= OUT_REL_L2, (t, j, e, float(err))
    sb = None if r.inp.shared is None else r.inp.shared[0].cpu().numpy()
    if sb is not None:
        def shared_errs(lo, hi):
            return [(rel_l2_rows(sh[i], oracle.expert_ffn(r.c.shared_fmt, sb, H, r.I,
                                                          hid[toks[i]])), int(toks[i]))
                    for i in range(lo, hi)]
        for errs in parallel_rows(shared_errs, len(toks), 8):
            for err, t in errs:
                assert err <= OUT_REL_L2, ("shared", t, float(err))
    ref = oracle.moe_layer(hid[toks], wr, bias, E, k, r.c.fmt, r.I, blobs,
                           shared_fmt=r.c.shared_fmt or 0, shared_blob=sb,
                           forced_ids=gids[toks])
    got = oracle.bf16_bits_to_f32(u16(r.out)[toks])
    err = rel_l2_rows(got, ref["out_f32"])
    assert err.max() <= OUT_REL_L2, f"max per-token rel L2 {err.max():.3e}"
    return err


@pytest.mark.parametrize("config,T", [(0, 1), (1, 4), (3, 1), (3, 4), (4, 1), (4, 4), (4, 8),
                                      (4, 16), (5, 1), (5, 4), (6, 1), (6, 4)])
def test_decode_layer_parity(config, T):
    """Configs 0, 1, 3 and 4 at their decode token counts, config 5
    ("C3b": the all-4-bit-codebook reading of config 3 at E = 512) and config
    6 (MXFP4 routed experts), each checked on every token with the parity
    bars."""
    r = Run(config, T).run()
    err = check_layer(r)
    print(f"C{config} T={T}: max rel L2 {err.max():.2e}")


@pytest.mark.parametrize("T", [2, 7, 8, 9, 15, 16])
def test_decode_ragged_token_counts(T):
    """Token counts on both sides of the 8-column MMA tile, up to the decode
    maximum (two column tiles)."""
    check_layer(Run(1, T).run())


@pytest.mark.parametrize("T", [7, 9, 16])
def test_mxfp4_decode_ragged_token_counts(T):
    """MXFP4 experts at token counts on both sides of the 8-column tile."""
    check_layer(Run(6, T).run())


def test_mxfp4_decode_top_of_exact_scale_range():
    """MXFP4 down-projection scales raised by 2^19 to E8M0 bytes 137..140,
    the top of the range where the kernels' fp16 weight e2m1 * 2^(e-127) is
    exact (6 * 2^13 = 49152 < 65504); y is fp32 on the decode path, so
    parity holds as for ordinary scales."""
    r = Run(6, 4)
    planes, _ = mi.plane_layout(r.c.fmt, r.H, r.I)
    _, off, n, _, _, _ = [pl for pl in planes if pl[0] == "down" and pl[5] == "scales"][0]
    r.inp.experts[:, off:off + n] += 19
    assert int(r.inp.experts[:, off:off + n].max()) == 140
    r.run()
    check_layer(r)


def test_mxfp4_decode_needs_h_multiple_of_512():
    """MXFP4 at H = 2304 (a multiple of 256, not of 512): the decode path
    reports STRATA_EUNSUPPORTED before launching anything."""
    H, I, E, T, k = 2304, 640, 4, 2, 2
    nb = sm.strata_expert_bytes(sm.FMT_MXFP4_32, H, I)
    blobs = torch.zeros(E, nb, dtype=torch.uint8, device=DEV)
    qw = sm.qweights(sm.FMT_MXFP4_32, E, H, I, blobs, blobs.stride(0))
    hid = torch.zeros(T, H, dtype=torch.bfloat16, device=DEV)
    offs = torch.tensor([0, 2, 4, 4, 4], dtype=torch.int32, device=DEV)
    perm = torch.arange(T * k, dtype=torch.int32, device=DEV)
    act = torch.tensor([2, 0, 1, 0, 0], dtype=torch.int32, device=DEV)
    y = torch.empty(T * k, H, dtype=torch.float32, device=DEV)
    ew = ws(sm.moe_experts_workspace_size(qw, T, k))
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    rc = sm.moe_experts(hid, qw, offs, perm, act, T, k, y, ew, ew.numel(), st, check=False)
    assert rc == EUNSUPPORTED


def test_decode_small_expert_count_and_k1():
    """E = 8 experts, every token on several: many tokens per expert."""
    r = Run(0, 16, E=8)
    r.k = 1
    r.run()
    check_layer(r)


def test_decode_large_down_scales():
    """Down-projection block scales of 82..328 (2^14 times the C1 range, on
    both sides of 128): the 2-bit decode's fp16 products d*(c-1.5) stay in
    range and parity holds as for ordinary scales.  Gate/up scales stay as
    generated so that h stays well inside fp16."""
    r = Run(1, 4)
    planes, _ = mi.plane_layout(r.c.fmt, r.H, r.I)
    _, off, n, _, _, _ = [pl for pl in planes if pl[0] == "down" and pl[5] == "scales"][0]
    d = r.inp.experts[:, off:off + n].view(torch.float16)
    d.mul_(2.0 ** 14)
    big = (d.abs() >= 128).float().mean().item()
    assert 0.2 < big < 0.9, big  # both forms are exercised
    r.run()
    check_layer(r)


@pytest.mark.parametrize("T", [4, 64])
def test_fp16_overflow_flagged(T):
    """Gate/up block scales times 2^12 push the SwiGLU output h past the fp16
    range: h is stored as inf and the call reports STRATA_EOVERFLOW (decode at
    T = 4, prefill at T = 64)."""
    c = mi.CONFIGS[1]
    inp = mi.make_layer(1, T, layer=0, device=DEV)
    planes, _ = mi.plane_layout(c.fmt, c.H, c.I)
    for name in ("gate", "up"):
        _, off, n, _, _, _ = [pl for pl in planes if pl[0] == name and pl[5] == "scales"][0]
        inp.experts[:, off:off + n].view(torch.float16).mul_(2.0 ** 12)
    H, E, k, I = c.H, inp.w_router.shape[1], c.k, c.I
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    hid = torch.empty(T, H, dtype=torch.bfloat16, device=DEV)
    ids = torch.empty(T, k, dtype=torch.int32, device=DEV)
    w = torch.empty(T, k, device=DEV)
    counts = torch.empty(E, dtype=torch.int32, device=DEV)
    offs = torch.empty(E + 1, dtype=torch.int32, device=DEV)
    perm = torch.empty(T * k, dtype=torch.int32, device=DEV)
    inv = torch.empty(T * k, dtype=torch.int32, device=DEV)
    act = torch.empty(E + 1, dtype=torch.int32, device=DEV)
    rw = ws(sm.moe_route_workspace_size(T, H, E, k))
    sm.moe_route(inp.x, T, H, c.eps, inp.w_router, inp.bias, E, k, hid, ids, w, counts, offs,
                 perm, inv, act, rw, rw.numel(), st)
    assert sm.strata_read_status(st) == 0
    qw = sm.qweights(c.fmt, E, H, I, inp.experts, inp.experts.stride(0))
    decode = T <= sm.DECODE_MAX_T
    y = torch.empty(T * k, H, dtype=torch.float32 if decode else torch.float16, device=DEV)
    ew = ws(sm.moe_experts_workspace_size(qw, T, k))
    sm.moe_experts(hid, qw, offs, perm, act, T, k, y, ew, ew.numel(), st)
    torch.cuda.synchronize()
    assert sm.strata_read_status(st) == EOVERFLOW


@pytest.mark.parametrize("config,T", [(1, 4), (4, 8)])
def test_decode_deterministic(config, T):
    a = Run(config, T).run()
    b = Run(config, T).run()
    for x, y in ((a.ids, b.ids), (a.perm, b.perm), (a.y, b.y), (a.out, b.out)):
        assert torch.equal(x, y)


def test_layer_forward_matches_steps():
    """moe_layer_forward gives bit-identical results to the individual calls,
    and residual_out = x + acc."""
    for config, T in ((1, 4), (3, 4)):
        r = Run(config, T).run()
        E, k, H = r.E, r.k, r.H
        layer = sm.MoELayer(r.inp.w_router, r.inp.bias,
                            sm.ExpertWeights(r.inp.experts, r.c.fmt, H, r.I), k,
                            None if r.inp.shared is None else
                            sm.ExpertWeights(r.inp.shared, r.c.shared_fmt, H, r.I), r.c.eps)
        res = torch.empty(T, H, dtype=torch.float32, device=DEV)
        ids = torch.empty(T, k, dtype=torch.int32, device=DEV)
        out = layer.forward(r.inp.x, residual_out=res, topk_ids=ids, dev_status=r.status)
        torch.cuda.synchronize()
        assert torch.equal(out, r.out) and torch.equal(ids, r.ids)
        assert torch.equal(res, r.inp.x + r.acc)


def test_stacked_layers_teacher_forced():
    """Config 1's 48-layer stack (first 6 layers here): each layer's input is
    the previous GPU layer's residual output; every layer is checked."""
    c = mi.CONFIGS[1]
    x = mi.gen_x(4, c.H, mi.seed_for(1, 0, "xstep"), DEV)
    for layer in range(6):
        r = Run(1, 4, layer=layer, x=x).run()
        check_layer(r)
        x = (x + r.acc).contiguous()


def test_dev_status_clean_and_invalid_ids_flagged():
    """Out-of-range ids are skipped and flagged in dev_status, never trapped."""
    T, k, E = 4, 2, 16
    ids = torch.tensor([[0, 1], [2, 99], [3, 4], [5, -1]], dtype=torch.int32, device=DEV)
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    counts = torch.empty(E, dtype=torch.int32, device=DEV)
    offsets = torch.empty(E + 1, dtype=torch.int32, device=DEV)
    perm = torch.full((T * k,), -7, dtype=torch.int32, device=DEV)
    inv = torch.empty(T * k, dtype=torch.int32, device=DEV)
    active = torch.empty(E + 1, dtype=torch.int32, device=DEV)
    sm.moe_bucket(ids, T, k, E, counts, offsets, perm, inv, active, None, 0, st)
    torch.cuda.synchronize()
    assert sm.strata_read_status(st) == 5
    assert int(offsets[-1]) == 6 and int(counts.sum()) == 6
    assert inv[3].item() == -1 and inv[7].item() == -1


@pytest.mark.parametrize("config,T", [(1, 1), (1, 4), (1, 16), (4, 4), (4, 16)])
def test_route_matches_separate_calls(config, T):
    """moe_route (the fused decode routing kernel for T <= 16) gives the same
    bits as moe_rmsnorm -> moe_router_topk -> moe_bucket."""
    r = Run(config, T).run()
    E, k, H = r.E, r.k, r.H
    hid = torch.empty(T, H, dtype=torch.bfloat16, device=DEV)
    ids = torch.empty(T, k, dtype=torch.int32, device=DEV)
    w = torch.empty(T, k, dtype=torch.float32, device=DEV)
    counts = torch.empty(E, dtype=torch.int32, device=DEV)
    offsets = torch.empty(E + 1, dtype=torch.int32, device=DEV)
    perm = torch.empty(T * k, dtype=torch.int32, device=DEV)
    inv = torch.empty(T * k, dtype=torch.int32, device=DEV)
    active = torch.empty(E + 1, dtype=torch.int32, device=DEV)
    wsb = ws(sm.moe_route_workspace_size(T, H, E, k))
    sm.moe_route(r.inp.x, T, H, r.c.eps, r.inp.w_router, r.inp.bias, E, k, hid, ids, w, counts,
                 offsets, perm, inv, active, wsb, wsb.numel(), r.status)
    torch.cuda.synchronize()
    assert sm.strata_read_status(r.status) == 0
    assert torch.equal(hid, r.hidden) and torch.equal(ids, r.ids) and torch.equal(w, r.w)
    assert torch.equal(counts, r.counts) and torch.equal(offsets, r.offsets)
    assert torch.equal(perm, r.perm[:T * k]) and torch.equal(inv, r.inv[:T * k])
    nact = int(active[0])
    assert torch.equal(active[:1 + nact], r.active[:1 + nact])


# ---------------------------------------------------------------- prefill (T > 16)
@pytest.mark.parametrize("T,E", [(17, 16), (100, 16), (300, 16), (300, 512)])
def test_prefill_ragged(T, E):
    """Tensor-core path at sizes that span several 128-token tiles per expert
    (E = 16: ~T*10/16 tokens each) and ragged tails, checked on every token."""
    r = Run(1, T, E=E).run()
    err = check_layer(r)
    print(f"prefill T={T} E={E}: max rel L2 {err.max():.2e}")


@pytest.mark.parametrize("T,E", [(17, 16), (300, 16)])
def test_mxfp4_prefill_ragged(T, E):
    """MXFP4 experts on the tensor-core path, every token checked."""
    check_layer(Run(6, T, E=E).run())


def test_prefill_one_expert_takes_everything():
    """All tokens routed to one expert (k = 1, E = 8, a bias of +50 on expert 1):
    a single expert with T tokens = many full tiles plus a tail."""
    T = 1000
    r = Run(1, T, E=8)
    r.k = 1
    r.inp.bias = torch.tensor([0.0, 50.0, 0, 0, 0, 0, 0, 0], device=DEV)
    r.run()
    assert int(r.counts[1]) == T
    check_layer(r, sample=np.arange(0, T, 37))


@pytest.mark.parametrize("config", [2, 3, 4, 6])
def test_prefill_full_size(config):
    """The T = 8192 prefill chunks (2-bit routed; + 4-bit shared expert; 4-bit
    large experts; MXFP4 routed) at full size: RMSNorm, router logits, top-k ids and weights
    and the bucket on all 8192 tokens; combine, expert outputs and layer
    output on a stratified sample of 256 tokens (the least-loaded expert's
    tokens, the most-loaded expert's full tiles and last partial tile, the
    tail token of other experts, then uniform random tokens)."""
    r = Run(config, 8192).run()
    sample = stratified_tokens(r.counts.cpu().numpy(), r.offsets.cpu().numpy(),
                               r.perm.cpu().numpy(), r.k, r.T, n=256, seed=config)
    err = check_layer(r, sample=sample)
    print(f"C{config} T=8192: max rel L2 {err.max():.2e} over {len(sample)} tokens")


def test_prefill_32k_chunk():
    """A 32768-token prefill chunk of config 2's layer (the walk-through's
    opt-in chunk size, section 7; 327,680 token-expert pairs): RMSNorm,
    routing and bucket on every token, the rest on a stratified sample."""
    r = Run(2, 32768).run()
    sample = stratified_tokens(r.counts.cpu().numpy(), r.offsets.cpu().numpy(),
                               r.perm.cpu().numpy(), r.k, r.T, n=256, seed=32)
    err = check_layer(r, sample=sample)
    print(f"C2 T=32768: max rel L2 {err.max():.2e} over {len(sample)} tokens")


def test_prefill_deterministic():
    a = Run(2, 2048).run()
    b = Run(2, 2048).run()
    for x, y in ((a.ids, b.ids), (a.perm, b.perm), (a.y, b.y), (a.out, b.out)):
        assert torch.equal(x, y)
