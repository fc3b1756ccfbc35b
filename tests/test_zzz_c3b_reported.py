"""C3b: the other reading of config 3, with every expert (routed and shared)
in the 4-bit codebook format at E = 512.  The reading taken for C3 keeps the
routed experts 2-bit; this one is run and its parity reported beside it, not
used as a gate: the test fails only on a device error or a non-finite
output, and prints the per-token relative L2 of the expert outputs and the
layer output against the oracle (teacher-forced ids)."""
import numpy as np
import pytest

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("needs a CUDA GPU", allow_module_level=True)

import oracle  # noqa: E402
from tests.harness import rel_l2_rows  # noqa: E402
from tests.test_gpu_parity import DEV, Run, u16  # noqa: E402

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("T", [1, 4])
def test_c3b_all_codebook_reported(T):
    r = Run(5, T).run()  # asserts a clean device status
    out = oracle.bf16_bits_to_f32(u16(r.out))
    assert np.isfinite(out).all()
    H, k = r.H, r.k
    hid = u16(r.hidden)
    gids = r.ids.cpu().numpy()
    inv = r.inv.cpu().numpy()[:T * k]
    yg = r.y[torch.as_tensor(inv, device=DEV).long()].float().cpu().numpy()
    blobs = r.blobs_for(gids)
    ey = max(float(rel_l2_rows(yg[t * k + j],
                               oracle.expert_ffn(r.c.fmt, blobs[int(gids[t, j])], H, r.I,
                                                 hid[t])))
             for t in range(T) for j in range(k))
    sb = r.inp.shared[0].cpu().numpy()
    wr = u16(r.inp.w_router)
    ref = oracle.moe_layer(hid, wr, r.inp.bias.cpu().numpy(), r.E, k, r.c.fmt, r.I, blobs,
                           shared_fmt=r.c.shared_fmt, shared_blob=sb, forced_ids=gids)
    eo = float(rel_l2_rows(out, ref["out_f32"]).max())
    print(f"C3b T={T}: expert outputs max rel L2 {ey:.2e}, layer output max rel L2 {eo:.2e}")
