"""Pins of the CPU oracle to things other than itself (no GPU).

Each test checks the oracle against a fact fixed outside the oracle: values
worked out by hand from the format definition (tests/golden), brute force on
tiny inputs, a float64 textbook MLP built by an independent numpy decoder,
exact identities (k = E identical experts, exact scaling, permutations),
library routines (numpy's stable argsort) and the closed-form sizes the pages
print.  The mistakes each one catches are named in its docstring.
"""
import itertools
import math
import os

import numpy as np
import pytest

import oracle
from oracle import FMT_MXFP4, FMT_Q2, FMT_Q4CB, bf16_bits_to_f32, f32_to_bf16_bits

KV = np.array([-127, -104, -83, -65, -49, -35, -22, -10, 1, 13, 25, 38, 53, 69, 89, 113],
              np.float64)
# FP4 E2M1 values of codes 0..15, read off the OCP MX v1.0 element table
E2M1 = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6, -0.0, -0.5, -1, -1.5, -2, -3, -4, -6], np.float64)


def scale_bytes(fmt):
    return 1 if fmt == FMT_MXFP4 else 2


# ------------------------------------------------------------ independent decoder
def np_layout(fmt, H, I):
    """Plane offsets written out from the blob definition (not the oracle's)."""
    def r256(x):
        return -(-x // 256) * 256
    out, off = {}, 0
    for name, rows, K in (("gate", I, H), ("up", I, H), ("down", H, I)):
        nc = rows * K * (2 if fmt == FMT_Q2 else 4) // 8
        out[name] = (off, None, rows, K)
        off = r256(off + nc)
        out[name] = (out[name][0], off, rows, K)
        off = r256(off + rows * K // 32 * scale_bytes(fmt))
    return out, off


def np_dequant(fmt, blob, H, I, name):
    """Vectorised float64 decode of one matrix [rows, K]."""
    lay, _ = np_layout(fmt, H, I)
    co, so, rows, K = lay[name]
    if fmt == FMT_MXFP4:
        e = blob[so:so + rows * K // 32].astype(np.int64).reshape(rows, K // 32)
        d = np.where(e == 255, np.nan, np.ldexp(1.0, e - 127))
    else:
        d = blob[so:so + rows * K // 32 * 2].view(np.float16).astype(np.float64).reshape(
            rows, K // 32)
    if fmt == FMT_Q2:
        b = blob[co:co + rows * K // 4].reshape(rows, K // 4)
        c = np.stack([(b >> (2 * i)) & 3 for i in range(4)], axis=-1).reshape(rows, K)
        v = c.astype(np.float64) - 1.5
    else:
        b = blob[co:co + rows * K // 2].reshape(rows, K // 2)
        c = np.stack([b & 15, b >> 4], axis=-1).reshape(rows, K)
        v = (E2M1 if fmt == FMT_MXFP4 else KV)[c]
    return v * np.repeat(d, 32, axis=1)


def rand_blob(rng, fmt, H, I, d_lo=0.005, d_hi=0.02):
    lay, n = np_layout(fmt, H, I)
    blob = rng.integers(0, 256, n, dtype=np.uint8)
    for name, (co, so, rows, K) in lay.items():
        if fmt == FMT_MXFP4:  # E8M0 exponents, d_lo..d_hi read as powers of two
            e = rng.integers(127 + int(math.log2(d_lo)), 128 + int(math.log2(d_hi)),
                             rows * K // 32)
            blob[so:so + rows * K // 32] = e.astype(np.uint8)
            continue
        d = rng.uniform(d_lo, d_hi, rows * K // 32).astype(np.float16)
        blob[so:so + d.nbytes] = d.view(np.uint8)
    return blob


def rand_hidden(rng, T, H):
    return f32_to_bf16_bits(rng.standard_normal((T, H)).astype(np.float32))


def read_golden(path):
    recs = []
    with open(path) as f:
        for line in f:
            if not line.strip() or line.startswith("#"):
                continue
            name, codes, scale, vals = [s.strip() for s in line.split("|")]
            recs.append((name, bytes.fromhex(codes.replace(" ", "")), int(scale, 16),
                         np.array([float(v) for v in vals.split()], np.float64)))
    return recs


def blob_with_first_row(fmt, H, I, which, codes, scale_bits):
    """A zero blob whose matrix `which` row 0, block 0, holds the given bytes."""
    lay, n = np_layout(fmt, H, I)
    blob = np.zeros(n, np.uint8)
    co, so, rows, K = lay[("gate", "up", "down")[which]]
    blob[co:co + len(codes)] = np.frombuffer(codes, np.uint8)
    if fmt == FMT_MXFP4:
        blob[so] = scale_bits
    else:
        blob[so:so + 2] = np.array([scale_bits], np.uint16).view(np.uint8)
    return blob


# ------------------------------------------------------------ dequantisation
@pytest.mark.parametrize("fmt,fname", [(FMT_Q2, "q2_blocks.txt"), (FMT_Q4CB, "q4cb_blocks.txt"),
                                      (FMT_MXFP4, "mxfp4_blocks.txt")])
@pytest.mark.parametrize("which", [0, 1, 2])
def test_dequant_hand_built_blocks(golden_dir, fmt, fname, which):
    """Known codes and scales decode to the hand-worked values in every matrix.
    Catches: wrong bit/nibble order, wrong offset (-1.5), wrong codebook entry,
    wrong fp16 decode, wrong plane offsets for gate/up/down; for MXFP4 a wrong
    E2M1 field split, exponent bias, subnormal value, sign, or E8M0 bias/NaN."""
    H, I = 64, 32
    for name, codes, sbits, expect in read_golden(os.path.join(golden_dir, fname)):
        blob = blob_with_first_row(fmt, H, I, which, codes, sbits)
        row = oracle.dequant_row(fmt, blob, H, I, which, 0)
        np.testing.assert_array_equal(row[:32].astype(np.float64), expect, err_msg=name)


def test_dequant_matches_independent_decoder():
    """The oracle's row decode equals the numpy decoder on random blobs, all
    rows of all three matrices, every format (exact)."""
    rng = np.random.default_rng(1)
    for fmt in (FMT_Q2, FMT_Q4CB, FMT_MXFP4):
        H, I = 96, 64
        blob = rand_blob(rng, fmt, H, I, *((2.0**-9, 2.0**-6) if fmt == FMT_MXFP4
                                           else (0.005, 0.02)))
        for which, name in enumerate(("gate", "up", "down")):
            ref = np_dequant(fmt, blob, H, I, name)
            got = np.stack([oracle.dequant_row(fmt, blob, H, I, which, r)
                            for r in range(ref.shape[0])])
            np.testing.assert_array_equal(got.astype(np.float64), ref)


def test_dequant_planes_are_distinct():
    """gate, up and down are read from their own planes: give each plane its
    own scale and check which one comes back."""
    H, I = 64, 32
    lay, n = np_layout(FMT_Q2, H, I)
    blob = np.zeros(n, np.uint8)
    for scale, name in zip((1.0, 2.0, 4.0), ("gate", "up", "down")):
        co, so, rows, K = lay[name]
        blob[co:co + rows * K // 4] = 0xFF  # every code 3 -> +1.5 d
        blob[so:so + rows * K // 32 * 2] = np.full(rows * K // 32, scale,
                                                   np.float16).view(np.uint8)
    for which, scale in enumerate((1.0, 2.0, 4.0)):
        row = oracle.dequant_row(FMT_Q2, blob, H, I, which, 1)
        assert np.all(row == np.float32(1.5 * scale))


def test_mxfp4_sign_and_scale_steps():
    """MXFP4 properties fixed by the format: setting a code's bit 3 negates
    the element; adding 1 to a block's E8M0 byte doubles its 32 elements
    exactly and leaves the other blocks alone; codes 0..7 increase strictly.
    Catches: sign taken from the wrong bit, a scale indexed by the wrong
    block, a scale that is not a power of two."""
    rng = np.random.default_rng(11)
    H, I = 96, 64
    blob = rand_blob(rng, FMT_MXFP4, H, I, 2.0**-9, 2.0**-6)
    lay, _ = np_layout(FMT_MXFP4, H, I)
    for which, name in enumerate(("gate", "up", "down")):
        co, so, rows, K = lay[name]
        r = 3
        base = oracle.dequant_row(FMT_MXFP4, blob, H, I, which, r).astype(np.float64)
        neg = blob.copy()
        neg[co + r * K // 2:co + (r + 1) * K // 2] ^= 0x88
        np.testing.assert_array_equal(
            oracle.dequant_row(FMT_MXFP4, neg, H, I, which, r), -base)
        dbl = blob.copy()
        dbl[so + r * K // 32 + 1] += 1
        got = oracle.dequant_row(FMT_MXFP4, dbl, H, I, which, r).astype(np.float64)
        np.testing.assert_array_equal(got[32:64], 2 * base[32:64])
        np.testing.assert_array_equal(np.delete(got, np.s_[32:64]), np.delete(base, np.s_[32:64]))
    mono = blob.copy()
    co, so, rows, K = lay["gate"]
    mono[co:co + 4] = [0x10, 0x32, 0x54, 0x76]
    v = oracle.dequant_row(FMT_MXFP4, mono, H, I, 0, 0)[:8]
    assert np.all(np.diff(v) > 0) and v[0] == 0


# ------------------------------------------------------------ sizes
def read_sizes(golden_dir):
    d = {}
    with open(os.path.join(golden_dir, "page_sizes.txt")) as f:
        for line in f:
            if line.strip() and not line.startswith("#"):
                name, val, _ = [s.strip() for s in line.split("|")]
                d[name] = float(val)
    return d


def test_page_closed_forms(golden_dir):
    """The pages' own totals follow from their geometry: 1,382,400 B per expert
    is 2.25 bits/weight; 48 x 10 x blob = 0.66 GB per token; 24,576 x blob =
    34.0 GB; 1 GB / blob ~ 700 experts."""
    s = read_sizes(golden_dir)
    weights = 3 * s["hidden"] * s["expert_width"]
    assert s["pages_q2_0_blob_bytes"] * 8 / weights == pytest.approx(2.25)
    assert s["layers"] * s["experts_per_layer"] == s["total_experts"]
    per_tok = s["layers"] * s["experts_per_token"] * s["pages_q2_0_blob_bytes"] / 1e9
    assert round(per_tok, 2) == s["routed_read_per_token_gb"]
    assert round(s["total_experts"] * s["pages_q2_0_blob_bytes"] / 1e9, 1) == s["routed_store_gb"]
    assert abs(1e9 / s["pages_q2_0_blob_bytes"] - s["experts_per_gb"]) < 0.05 * s["experts_per_gb"]


def test_blob_sizes_closed_form():
    """Blob bytes = 3 H I bits/8 (2.5 bits for Q2_32, 4.5 for Q4CB_32) when the
    planes are already 256-byte multiples; 48 x 512 Q2 experts ~ 38 GB."""
    assert oracle.expert_bytes(FMT_Q2, 2560, 640) == 3 * 2560 * 640 * 5 // 16 == 1536000
    assert oracle.expert_bytes(FMT_Q4CB, 2560, 640) == 3 * 2560 * 640 * 9 // 16 == 2764800
    # MXFP4: 4 bits per element and an 8-bit scale per 32 -> 4.25 bits/weight
    assert oracle.expert_bytes(FMT_MXFP4, 2560, 640) == 3 * 2560 * 640 * 17 // 32 == 2611200
    assert oracle.expert_bytes(FMT_MXFP4, 4096, 2048) == 3 * 4096 * 2048 * 17 // 32
    assert oracle.expert_bytes(FMT_Q4CB, 4096, 2048) == 14155776
    assert round(48 * 512 * 1536000 / 2**30, 2) == 35.16  # 37.75 GB
    assert oracle.expert_bytes(FMT_Q2, 64, 32) == np_layout(FMT_Q2, 64, 32)[1]


# ------------------------------------------------------------ rmsnorm
def test_rmsnorm_closed_form():
    """x = (3, 4, 0, 0): mean square 6.25, rms 2.5, so xhat = (1.2, 1.6, 0, 0)
    up to eps; the bf16 result is within half an ulp of the exact value."""
    x = np.array([[3.0, 4.0, 0.0, 0.0], [-2.0, -2.0, -2.0, -2.0]], np.float32)
    eps = 1e-6
    out = bf16_bits_to_f32(oracle.rmsnorm(x, eps)).astype(np.float64)
    exact = x / np.sqrt((x.astype(np.float64) ** 2).mean(1, keepdims=True) + eps)
    ulp = 2.0 ** (np.floor(np.log2(np.maximum(np.abs(exact), 1e-30))) - 7)
    assert np.all(np.abs(out - exact) <= 0.5 * ulp + 1e-30)
    assert out[0, 0] == 1.203125 and out[0, 1] == 1.6015625 and out[1, 0] == -1.0


# ------------------------------------------------------------ router / top-k
def test_router_logits_exact_small_integers():
    """Integer-valued bf16 operands: the logits are exact sums; bias adds."""
    rng = np.random.default_rng(2)
    T, H, E = 3, 64, 6
    hid = rng.integers(-8, 9, (T, H)).astype(np.float32)
    wr = rng.integers(-8, 9, (H, E)).astype(np.float32)
    bias = np.array([0.5, -1.0, 0.0, 2.0, 0.25, -0.75], np.float32)
    got = oracle.router_logits(f32_to_bf16_bits(hid), f32_to_bf16_bits(wr), bias)
    ref = hid.astype(np.float64) @ wr.astype(np.float64) + bias
    np.testing.assert_array_equal(got.astype(np.float64), ref)


def brute_topk(logits, k):
    """Definition: e is chosen iff fewer than k experts beat it, where e' beats
    e when l[e'] > l[e], or l[e'] == l[e] and e' < e.  Listed by rank."""
    E = len(logits)
    rank = [sum(1 for f in range(E) if logits[f] > logits[e] or (logits[f] == logits[e] and f < e))
            for e in range(E)]
    chosen = sorted([e for e in range(E) if rank[e] < k], key=lambda e: rank[e])
    num = np.array([math.exp(float(logits[e])) for e in chosen])
    return np.array(chosen, np.int32), num / num.sum()


def test_topk_brute_force_all_k():
    """Oracle top-k and renormalised weights equal the rank definition and the
    softmax over the chosen logits, for every k, with planted exact ties.
    Catches: wrong tie-break, wrong order, missing renormalisation, softmax
    over the wrong set."""
    rng = np.random.default_rng(3)
    for trial in range(40):
        E = int(rng.integers(2, 13))
        lg = rng.standard_normal(E).astype(np.float32)
        if trial % 2 == 0 and E >= 4:  # planted exact ties
            lg[1] = lg[3]
            lg[E - 1] = lg[0]
        for k in range(1, E + 1):
            ids, w = oracle.topk(lg[None, :], k)
            bid, bw = brute_topk(lg, k)
            np.testing.assert_array_equal(ids[0], bid)
            np.testing.assert_allclose(w[0].astype(np.float64), bw, rtol=2e-7, atol=0)


def test_topk_special_cases():
    """k = 1 gives weight exactly 1; k = E gives the full softmax; two chosen
    experts get 1/(1+exp(l2-l1)); equal W_r columns tie to the lower index."""
    lg = np.array([[0.3, 1.2, -0.5, 1.2, 0.9]], np.float32)
    ids, w = oracle.topk(lg, 1)
    assert ids[0, 0] == 1 and w[0, 0] == 1.0
    ids, w = oracle.topk(lg, 2)
    assert list(ids[0]) == [1, 3] and np.allclose(w[0], [0.5, 0.5], rtol=0, atol=1e-7)
    ids, w = oracle.topk(lg, 5)
    p = np.exp(lg[0].astype(np.float64))
    np.testing.assert_allclose(w[0], (p / p.sum())[ids[0]], rtol=1e-6)
    ids, w = oracle.topk(np.array([[2.0, 1.0, 0.0]], np.float32), 2)
    assert np.isclose(w[0, 0], 1 / (1 + math.exp(-1.0)), rtol=1e-7)
    # ties through the router: identical columns 2 and 4
    rng = np.random.default_rng(4)
    wr = rng.standard_normal((32, 6)).astype(np.float32) * 0.1
    wr[:, 4] = wr[:, 2]
    hid = rand_hidden(rng, 4, 32)
    lgt = oracle.router_logits(hid, f32_to_bf16_bits(wr))
    for t in range(4):
        ids, _ = oracle.topk(lgt[t:t + 1], 6)
        pos = list(ids[0])
        assert pos.index(2) == pos.index(4) - 1


def test_bias_changes_selection_and_weights():
    """The bias is part of the logits: it can move a lower raw score into the
    top-k and it enters the weights."""
    hid = f32_to_bf16_bits(np.ones((1, 32), np.float32))
    wr = np.zeros((32, 3), np.float32)
    wr[:, 0] = 1 / 32  # raw logits (1, 0, 0)
    bias = np.array([0.0, 1.5, 0.0], np.float32)
    lg = oracle.router_logits(hid, f32_to_bf16_bits(wr), bias)
    np.testing.assert_array_equal(lg[0], np.array([1.0, 1.5, 0.0], np.float32))
    ids, w = oracle.topk(lg, 1)
    assert ids[0, 0] == 1
    ids, w = oracle.topk(lg, 2)
    assert list(ids[0]) == [1, 0]
    assert np.isclose(w[0, 0], 1 / (1 + math.exp(-0.5)), rtol=1e-7)


# ------------------------------------------------------------ bucket
def test_bucket_invariants_and_stable_sort():
    """counts sum to T*k, offsets are their exclusive scan ending at T*k, perm
    equals numpy's stable argsort of the ids, inv inverts perm."""
    rng = np.random.default_rng(5)
    for T, k, E in ((1, 1, 1), (3, 2, 4), (64, 10, 512), (37, 6, 256), (5, 4, 4)):
        ids = np.stack([rng.permutation(E)[:k] for _ in range(T)]).astype(np.int32)
        counts, offsets, perm, inv = oracle.bucket(ids, E)
        assert counts.sum() == T * k and offsets[0] == 0 and offsets[-1] == T * k
        assert np.all(np.diff(offsets) == counts)
        np.testing.assert_array_equal(counts, np.bincount(ids.ravel(), minlength=E))
        np.testing.assert_array_equal(perm, np.argsort(ids.ravel(), kind="stable"))
        np.testing.assert_array_equal(inv[perm], np.arange(T * k))


# ------------------------------------------------------------ expert FFN and layer
def textbook_mlp(fmt, blob, H, I, x_bits):
    x = bf16_bits_to_f32(x_bits).astype(np.float64)
    wg, wu, wd = (np_dequant(fmt, blob, H, I, n) for n in ("gate", "up", "down"))
    g, u = wg @ x, wu @ x
    return wd @ (g / (1 + np.exp(-g)) * u)


D_RANGE = {FMT_Q2: (0.005, 0.02), FMT_Q4CB: (0.0005, 0.002), FMT_MXFP4: (2.0**-9, 2.0**-6)}


@pytest.mark.parametrize("fmt", [FMT_Q2, FMT_Q4CB, FMT_MXFP4])
def test_expert_ffn_matches_textbook_mlp(fmt):
    """E = 1: one expert equals the float64 SwiGLU MLP y = Wd (silu(Wg x) * Wu x)
    built from the independent decoder, with H != I so a transposed operand
    cannot pass.  Catches: gate/up swapped, wrong activation, transposes."""
    rng = np.random.default_rng(6)
    H, I = 96, 64
    for _ in range(3):
        blob = rand_blob(rng, fmt, H, I, *D_RANGE[fmt])
        x = rand_hidden(rng, 1, H)[0]
        ref = textbook_mlp(fmt, blob, H, I, x)
        y32 = oracle.expert_ffn(fmt, blob, H, I, x, acc64=False).astype(np.float64)
        y64 = oracle.expert_ffn(fmt, blob, H, I, x, acc64=True).astype(np.float64)
        scale = np.abs(ref).max()
        assert np.abs(y64 - ref).max() <= 1e-6 * scale
        assert np.abs(y32 - ref).max() <= 1e-4 * scale


def layer_case(rng, T=6, H=64, I=32, E=8, k=3, fmt=FMT_Q2):
    hid = rand_hidden(rng, T, H)
    wr = f32_to_bf16_bits((rng.standard_normal((H, E)) * 0.2).astype(np.float32))
    blobs = np.stack([rand_blob(rng, fmt, H, I) for _ in range(E)])
    return hid, wr, blobs


def test_k_equals_E_identical_experts_is_dense_mlp():
    """k = E with every expert identical: the routing weights sum to 1, so the
    layer equals one dense SwiGLU MLP (float64 textbook)."""
    rng = np.random.default_rng(7)
    H, I, E = 64, 32, 5
    hid = rand_hidden(rng, 4, H)
    wr = f32_to_bf16_bits((rng.standard_normal((H, E)) * 0.3).astype(np.float32))
    one = rand_blob(rng, FMT_Q2, H, I)
    r = oracle.moe_layer(hid, wr, None, E, E, FMT_Q2, I, np.stack([one] * E), acc64=True)
    for t in range(4):
        ref = textbook_mlp(FMT_Q2, one, H, I, hid[t])
        np.testing.assert_allclose(r["out_f32"][t], ref, rtol=0, atol=1e-6 * np.abs(ref).max())


def test_layer_equals_weighted_sum_of_textbook_experts():
    """out[t] = sum_j w_j y_j with the router's ids and weights, each y_j the
    textbook MLP of expert ids[t, j]."""
    rng = np.random.default_rng(8)
    hid, wr, blobs = layer_case(rng)
    H, I, E, k = 64, 32, 8, 3
    r = oracle.moe_layer(hid, wr, None, E, k, FMT_Q2, I, blobs, acc64=True)
    lg = oracle.router_logits(hid, wr)
    for t in range(hid.shape[0]):
        bid, bw = brute_topk(lg[t], k)
        np.testing.assert_array_equal(r["ids"][t], bid)
        ref = sum(bw[j] * textbook_mlp(FMT_Q2, blobs[bid[j]], H, I, hid[t]) for j in range(k))
        np.testing.assert_allclose(r["out_f32"][t], ref, rtol=0, atol=2e-6 * np.abs(ref).max())


def test_down_scale_doubling_doubles_output_exactly():
    """Doubling every W_down scale (exact in fp16) doubles y, out_f32 and the
    bf16 output bit for bit.  Catches: a down scale that is not applied."""
    rng = np.random.default_rng(9)
    hid, wr, blobs = layer_case(rng)
    H, I, E, k = 64, 32, 8, 3
    lay, _ = np_layout(FMT_Q2, H, I)
    co, so, rows, K = lay["down"]
    b2 = blobs.copy()
    d = b2[:, so:so + rows * K // 32 * 2].copy().view(np.float16)
    b2[:, so:so + rows * K // 32 * 2] = (d * np.float16(2)).view(np.uint8)
    r1 = oracle.moe_layer(hid, wr, None, E, k, FMT_Q2, I, blobs)
    r2 = oracle.moe_layer(hid, wr, None, E, k, FMT_Q2, I, b2)
    np.testing.assert_array_equal(r2["out_f32"], 2 * r1["out_f32"])
    np.testing.assert_array_equal(bf16_bits_to_f32(r2["out_bf16"]),
                                  2 * bf16_bits_to_f32(r1["out_bf16"]))


def test_expert_relabelling_and_token_permutation_invariance():
    """Relabelling experts (W_r columns and blobs together) leaves out
    unchanged; permuting tokens permutes out; both bit for bit."""
    rng = np.random.default_rng(10)
    hid, wr, blobs = layer_case(rng)
    E, k, I = 8, 3, 32
    r = oracle.moe_layer(hid, wr, None, E, k, FMT_Q2, I, blobs)
    pe = rng.permutation(E)
    r2 = oracle.moe_layer(hid, wr[:, pe], None, E, k, FMT_Q2, I, blobs[pe])
    np.testing.assert_array_equal(r2["out_bf16"], r["out_bf16"])
    np.testing.assert_array_equal(pe[r2["ids"]], r["ids"])
    pt = rng.permutation(hid.shape[0])
    r3 = oracle.moe_layer(hid[pt], wr, None, E, k, FMT_Q2, I, blobs)
    np.testing.assert_array_equal(r3["out_bf16"], r["out_bf16"][pt])


def test_shared_expert_adds_with_weight_one():
    """The shared expert's output is added once, unweighted."""
    rng = np.random.default_rng(11)
    hid, wr, blobs = layer_case(rng)
    E, k, H, I = 8, 3, 64, 32
    sh = rand_blob(rng, FMT_Q4CB, H, I, 0.0005, 0.002)
    r0 = oracle.moe_layer(hid, wr, None, E, k, FMT_Q2, I, blobs, acc64=True)
    r1 = oracle.moe_layer(hid, wr, None, E, k, FMT_Q2, I, blobs, shared_fmt=FMT_Q4CB,
                          shared_blob=sh, acc64=True)
    for t in range(hid.shape[0]):
        ref = textbook_mlp(FMT_Q4CB, sh, H, I, hid[t])
        np.testing.assert_allclose(r1["out_f32"][t] - r0["out_f32"][t], ref, rtol=0,
                                   atol=1e-5 * np.abs(ref).max())


def test_combine_order_and_residual():
    """The combine sums j = 0..k-1 in order in fp32: (1e8 + 1) - 1e8 is 0 in
    that order (1 is lost) but 1 in any order that adds the 1 last.  The
    residual output is residual + acc."""
    y = np.zeros((3, 8), np.float32)
    y[0], y[1], y[2] = 1e8, 1.0, -1e8
    w = np.ones((1, 3), np.float32)
    res = np.full((1, 8), 0.5, np.float32)
    of, ob, ro = oracle.combine(y, w, residual=res)
    assert np.all(of == 0.0) and np.all(ro == 0.5)
    of, _, _ = oracle.combine(y[[0, 2, 1]], w)
    assert np.all(of == 1.0)


def test_forced_ids_reuse_router_weights():
    """With forced ids equal to the router's own choice the layer is unchanged;
    with the two best swapped the output is unchanged up to fp32 order."""
    rng = np.random.default_rng(12)
    hid, wr, blobs = layer_case(rng)
    E, k, I = 8, 3, 32
    r = oracle.moe_layer(hid, wr, None, E, k, FMT_Q2, I, blobs)
    r2 = oracle.moe_layer(hid, wr, None, E, k, FMT_Q2, I, blobs, forced_ids=r["ids"])
    np.testing.assert_array_equal(r2["out_f32"], r["out_f32"])
    sw = r["ids"][:, [1, 0, 2]]
    r3 = oracle.moe_layer(hid, wr, None, E, k, FMT_Q2, I, blobs, forced_ids=sw)
    np.testing.assert_allclose(r3["out_f32"], r["out_f32"], rtol=1e-6, atol=1e-7)


def test_missing_blob_is_an_error():
    rng = np.random.default_rng(13)
    hid, wr, blobs = layer_case(rng, T=2)
    with pytest.raises(ValueError):
        oracle.moe_layer(hid, wr, None, 8, 3, FMT_Q2, 32, {0: blobs[0]})
