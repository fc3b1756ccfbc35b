"""Expert parallelism on CPU: the exchange logic of expert_ffn_execution_b200.ep
with the oracle as the compute backend, in process and as two gloo ranks.
The layer split over G ranks must give the single-rank layer's output bit
for bit (the same expert and combine arithmetic; only rows move), with
every rank's routing identical to the single-rank routing."""
import os
import socket

import numpy as np
import pytest
import torch

import moe_inputs as mi
import oracle
from expert_ffn_execution_b200 import ep
from tests.ep_host_backend import OracleEPBackend

H, I, E, K = 256, 128, 16, 4


def _u16(t):
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


def _layer(seed, fmt=mi.FMT_Q2, shared=False, E_=E):
    wr = _u16(mi.gen_router(H, E_, seed))
    bias = mi.gen_zipf_bias(E_, 1.1, seed + 1).numpy()
    d = {mi.FMT_Q2: (0.005, 0.02), mi.FMT_Q4CB: (0.0005, 0.002),
         mi.FMT_MXFP4: (2.0**-9, 2.0**-6)}[fmt]
    blobs = mi.gen_experts(fmt, E_, H, I, d, seed + 2).numpy()
    sb = mi.gen_experts(mi.FMT_Q4CB, 1, H, I, (0.0005, 0.002), seed + 3).numpy()[0] if shared else None
    return wr, bias, blobs, sb


def _reference(x, wr, bias, blobs, fmt, sb, E_=E):
    hid = oracle.rmsnorm(x.numpy())
    return oracle.moe_layer(hid, wr, bias, E_, K, fmt, I, blobs,
                            shared_fmt=mi.FMT_Q4CB if sb is not None else 0, shared_blob=sb,
                            residual=x.numpy())


def _backends(G, wr, bias, blobs, fmt, sb, E_=E):
    return [OracleEPBackend(wr, bias, blobs, fmt, H, I, K, lo, hi, sb,
                            mi.FMT_Q4CB if sb is not None else 0)
            for lo, hi in ep.expert_ranges(E_, G)]


def test_ranges_counts_and_local_ids():
    assert ep.expert_ranges(16, 2) == [(0, 8), (8, 16)]
    assert ep.expert_ranges(10, 3) == [(0, 3), (3, 6), (6, 10)]
    with pytest.raises(ValueError):
        ep.expert_ranges(2, 3)
    offsets = np.array([0, 2, 2, 5, 6, 9, 9, 9, 12, 12, 13])  # E = 10, P = 13
    rng = ep.expert_ranges(10, 3)
    assert ep.send_counts(offsets, rng) == [5, 4, 4]
    lid = ep.sorted_local_ids(offsets, rng)
    # positions 0-1 expert 0, 2-4 expert 2, 5 expert 3 (rank 1 local 0), 6-8 expert 4,
    # 9-11 expert 7 (rank 2 local 1), 12 expert 9 (rank 2 local 3)
    np.testing.assert_array_equal(lid, [0, 0, 2, 2, 2, 0, 1, 1, 1, 1, 1, 1, 3])


@pytest.mark.parametrize("G,T,fmt,shared", [(2, 5, mi.FMT_Q2, False), (3, 4, mi.FMT_Q2, True),
                                            (4, 1, mi.FMT_Q4CB, False), (1, 3, mi.FMT_Q2, True),
                                            (2, 4, mi.FMT_MXFP4, True)])
def test_in_process_split_equals_single_rank(G, T, fmt, shared):
    wr, bias, blobs, sb = _layer(100 + G, fmt, shared)
    xs = [mi.gen_x(T, H, 200 + r) for r in range(G)]
    layers = [ep.EPLayer(b, E, K, r, G)
              for r, b in enumerate(_backends(G, wr, bias, blobs, fmt, sb))]
    outs = ep.forward_in_process(layers, xs)
    for r in range(G):
        ref = _reference(xs[r], wr, bias, blobs, fmt, sb)
        out, res = outs[r]
        np.testing.assert_array_equal(out.numpy().view(np.uint16), ref["out_bf16"])
        np.testing.assert_array_equal(res.numpy(), ref["residual_out"])


def test_in_process_rank_with_no_rows():
    """A bias that routes every token to rank 0's experts: rank 1 receives
    nothing and sends nothing back; the split still equals the single rank."""
    G, T = 2, 6
    wr, bias, blobs, _ = _layer(7)
    bias = np.where(np.arange(E) < E // 2, 40.0, 0.0).astype(np.float32)
    xs = [mi.gen_x(T, H, 300 + r) for r in range(G)]
    layers = [ep.EPLayer(b, E, K, r, G)
              for r, b in enumerate(_backends(G, wr, bias, blobs, mi.FMT_Q2, None))]
    d0 = layers[0].prepare(xs[0])
    assert d0.counts[1] == 0
    outs = ep.forward_in_process(layers, xs)
    for r in range(G):
        ref = _reference(xs[r], wr, bias, blobs, mi.FMT_Q2, None)
        np.testing.assert_array_equal(outs[r][0].numpy().view(np.uint16), ref["out_bf16"])


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _gloo_rank(rank, world, port, q):
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        wr, bias, blobs, sb = _layer(55, mi.FMT_Q2, True)
        lo, hi = ep.expert_ranges(E, world)[rank]
        be = OracleEPBackend(wr, bias, blobs, mi.FMT_Q2, H, I, K, lo, hi, sb, mi.FMT_Q4CB)
        layer = ep.EPLayer(be, E, K, rank, world)
        x = mi.gen_x(3 + 2 * rank, H, 400 + rank)
        out, res = layer.forward(x, ep.DistExchange())
        ref = _reference(x, wr, bias, blobs, mi.FMT_Q2, sb)
        ok = (np.array_equal(out.numpy().view(np.uint16), ref["out_bf16"]) and
              np.array_equal(res.numpy(), ref["residual_out"]))
        q.put((rank, ok, None))
    except Exception as e:  # reported to the parent
        q.put((rank, False, repr(e)))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_equal_single_rank():
    """Two CPU ranks, each with its own tokens (3 and 5) and half the experts,
    exchanging rows with all_to_all_single over gloo."""
    ctx = torch.multiprocessing.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_gloo_rank, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    got = [q.get(timeout=240) for _ in procs]
    for p in procs:
        p.join(timeout=60)
    for rank, ok, err in sorted(got):
        assert ok, f"rank {rank}: {err}"
