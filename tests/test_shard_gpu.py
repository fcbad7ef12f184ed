"""Context-sharded decode on one GPU: the context of every sequence is cut
into slices (as if held by different GPUs), each slice's partial (M, Z, O) is
computed by lca_decode_partial from its own copy of those cache rows, and
lca_merge_partials merges them; the result must match the oracle's whole
decode, and the slices' anchors its anchors.  The slices are computed one
after another on one device (no kernel waits on another), so this needs one
GPU; the exchange between ranks is covered on CPU (test_context_shard.py)."""
import numpy as np
import pytest

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

import kv_compression_b200 as kvc  # noqa: E402
import workloads  # noqa: E402
from gpu_helpers import (BF16_TOL, F32_TOL, DeviceInputs, compare, make_plan, oracle_lca,  # noqa: E402
                         to_device)
from kv_compression_b200.shard import slice_bounds  # noqa: E402

pytestmark = pytest.mark.gpu

CASES = [  # (B, H, L, g, w, dtype, parts)
    (2, 128, 3000, 16, 200, "bf16", 3),
    (2, 16, 2000, 8, 100, "bf16", 4),
    (1, 128, 1000, 64, 0, "bf16", 2),
    (2, 4, 900, 8, 64, "f32", 3),
    (2, 128, 700, 16, 800, "bf16", 2),    # nothing condensed
    (1, 16, 500, 4, 60, "bf16", 1),       # one part: the whole decode
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "B{}_H{}_L{}_g{}_w{}_{}_x{}".format(*c))
def test_sliced_partials_merge_to_the_oracle(case):
    B, H, L, g, w, dt, parts = case
    kw = dict(d_c=64, d_r=16) if dt == "f32" else {}
    wl = workloads.small("shard", B=B, H=H, L=L, g=g, w=w, dtype=dt, seed=L + parts, **kw)
    x = workloads.generate(wl)
    d = DeviceInputs(x)
    plan = make_plan(wl)
    slices = slice_bounds(L, g, w, parts)
    mzs, os_, ancs = [], [], []
    for (pos0, n) in slices:
        c_sl = to_device(np.ascontiguousarray(x.c_kv[:, pos0:pos0 + n]))
        k_sl = to_device(np.ascontiguousarray(x.k_r[:, pos0:pos0 + n]))
        ng = kvc.slice_groups(L, g, w, pos0, n)
        mz = torch.empty(B, H, 2, device="cuda")
        po = torch.empty(B, H, wl.d_c, device="cuda")
        anc = torch.full((B, H, max(ng, 1)), -1, dtype=torch.int32, device="cuda")
        plan.decode_partial(d.q_c, d.q_r, c_sl, k_sl, n, pos0, L, g, w, mz, po, anc if ng else None)
        mzs.append(mz); os_.append(po); ancs.append(anc[:, :, :ng])
    all_mz = torch.stack(mzs).contiguous()
    all_o = torch.stack(os_).contiguous()
    out = torch.empty(B, H, wl.d_c, device="cuda")
    plan.merge_partials(parts, all_mz, all_o, out)
    torch.cuda.synchronize()
    assert plan.device_error() == kvc.LCA_OK
    ref = oracle_lca(x, g, w)
    got_anc = torch.cat(ancs, dim=2).cpu().numpy()
    compare(out.cpu().numpy().astype(np.float64), got_anc, ref, F32_TOL if dt == "f32" else BF16_TOL,
            exact_anchors=dt == "f32", x=x, g=g)


def test_partial_refuses_a_cut_group():
    wl = workloads.small("shard", B=1, H=16, L=500, g=16, w=20, seed=3)
    x = workloads.generate(wl)
    d = DeviceInputs(x)
    plan = make_plan(wl)
    mz = torch.empty(1, 16, 2, device="cuda")
    po = torch.empty(1, 16, 512, device="cuda")
    assert kvc.slice_groups(500, 16, 20, 8, 100) == -1
    with pytest.raises(kvc.LcaError):
        plan.decode_partial(d.q_c, d.q_r, d.c_kv, d.k_r, 100, 8, 500, 16, 20, mz, po, None)
