"""Expert parallelism on one GPU: G ranks of a layer run in one process with
the library's kernels (route, row gathers, local experts with k = 1,
combine), the exchange done by device copies (the all-to-all's data
movement, with no rank waiting on another).  Every rank's output is checked
against the oracle layer on its own tokens (per-token relative L2 <= 5e-3)
and its routing against the single-rank routing kernels (bit-exact)."""
import numpy as np
import pytest

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("needs a CUDA GPU", allow_module_level=True)

import expert_ffn_execution_b200 as sm  # noqa: E402
import moe_inputs as mi  # noqa: E402
import oracle  # noqa: E402
from expert_ffn_execution_b200 import ep  # noqa: E402
from expert_ffn_execution_b200._binding import EBOUNDS  # noqa: E402
from tests.harness import OUT_REL_L2, check_routing, rel_l2_rows  # noqa: E402

pytestmark = pytest.mark.gpu
DEV = "cuda"


def u16(t):
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


@pytest.mark.parametrize("config,G,T", [(0, 2, 4), (0, 4, 1), (3, 2, 8), (4, 2, 2)])
def test_expert_parallel_in_process(config, G, T):
    """Config 0: 2 ranks x 4 tokens (about 20 rows per rank: the grouped-GEMM
    path for the local experts) and 4 ranks x 1 token (the decode path);
    config 3 adds the 4-bit shared expert; config 4 the large 4-bit experts
    split 128 + 128."""
    c = mi.CONFIGS[config]
    inp = mi.make_layer(config, 1, layer=0, device=DEV)
    E = inp.w_router.shape[1]
    layers, xs = [], []
    for r, (lo, hi) in enumerate(ep.expert_ranges(E, G)):
        be = ep.CudaEPBackend(inp.w_router, inp.bias, inp.experts, c.fmt, c.H, c.I, c.k, lo, hi,
                              inp.shared, c.shared_fmt, c.eps)
        layers.append(ep.EPLayer(be, E, c.k, r, G))
        xs.append(mi.gen_x(T, c.H, mi.seed_for(config, r, "xstep"), DEV, c.x_bf16))
    outs = ep.forward_in_process(layers, xs)
    torch.cuda.synchronize()
    wr = u16(inp.w_router)
    bias = None if inp.bias is None else inp.bias.cpu().numpy()
    sb = None if inp.shared is None else inp.shared[0].cpu().numpy()
    for r in range(G):
        assert sm.strata_read_status(layers[r].be.status) == 0
        out, res = outs[r]
        hid = oracle.rmsnorm(xs[r].cpu().numpy(), c.eps)
        lg = oracle.router_logits(hid, wr, bias)
        # the rank's routing: the same kernels as a single rank
        d = layers[r].prepare(xs[r])
        gids = d.route["ids"].cpu().numpy()
        ok, near, bad = check_routing(lg, gids, c.k)
        assert ok, (r, bad)
        blobs = {int(e): inp.experts[int(e)].cpu().numpy() for e in np.unique(gids)}
        ref = oracle.moe_layer(u16(d.route["hidden"]), wr, bias, E, c.k, c.fmt, c.I, blobs,
                               shared_fmt=c.shared_fmt or 0, shared_blob=sb, forced_ids=gids)
        got = oracle.bf16_bits_to_f32(u16(out))
        err = rel_l2_rows(got, ref["out_f32"])
        assert err.max() <= OUT_REL_L2, (r, float(err.max()))
        ref_res = xs[r].cpu().numpy() + ref["out_f32"]
        assert rel_l2_rows(res.cpu().numpy() - xs[r].cpu().numpy(),
                           ref_res - xs[r].cpu().numpy()).max() <= OUT_REL_L2
        print(f"C{config} G={G} rank {r}: T={T}, rows sent {d.counts}, max rel L2 {err.max():.2e}")


def test_gather_rows_kernel():
    """moe_gather_rows: dst[i] = src[idx[i] / div] for bf16 and fp32 rows, the
    fp16 -> fp32 widening, and an out-of-range index (zero row, flagged)."""
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    H = 264
    src = torch.randn(7, H, device=DEV).to(torch.bfloat16)
    idx = torch.tensor([0, 5, 13, 20, 3], dtype=torch.int32, device=DEV)
    dst = torch.empty(5, H, dtype=torch.bfloat16, device=DEV)
    sm.moe_gather_rows(src, sm.DTYPE_BF16, 7, H, idx, 3, 5, dst, sm.DTYPE_BF16, st)
    torch.cuda.synchronize()
    assert torch.equal(dst, src[(idx.long() // 3)])
    assert sm.strata_read_status(st) == 0
    src16 = torch.randn(4, H, device=DEV).to(torch.float16)
    idx2 = torch.tensor([3, 1, 9, 0], dtype=torch.int32, device=DEV)
    dst32 = torch.full((4, H), 7.0, device=DEV)
    sm.moe_gather_rows(src16, sm.DTYPE_F16, 4, H, idx2, 1, 4, dst32, sm.DTYPE_F32, st)
    torch.cuda.synchronize()
    assert torch.equal(dst32[[0, 1, 3]], src16[[3, 1, 0]].float())
    assert torch.equal(dst32[2], torch.zeros(H, device=DEV))
    assert sm.strata_read_status(st) == EBOUNDS
