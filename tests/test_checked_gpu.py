"""The range-checked debug build (liblca_checked.so, -DLCA_CHECKS) on the
small parity cases of every kernel: each guarded shared-memory, tensor-memory,
ring-slot, anchor and workspace index must pass its check (a failed check is
reported as LCA_ERR_DEVICE_CHECK and the access skipped, never a trap), and
the results must still match the oracle."""
import numpy as np
import pytest

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

import kv_compression_b200 as kvc  # noqa: E402
import workloads  # noqa: E402
from gpu_helpers import (BF16_TOL, F32_TOL, DeviceInputs, compare, oracle_dense, oracle_lca,  # noqa: E402
                         rel_err, run_dense, run_lca, to_device)
from kv_compression_b200 import build as kbuild  # noqa: E402
from kv_compression_b200.shard import slice_bounds  # noqa: E402
from oracle import oracle as orc  # noqa: E402

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def checked_lib():
    return kbuild.build_checked()


def _plan(wl, lib_path, opts=None):
    plan = kvc.Plan(wl.B, wl.H, wl.d_c, wl.d_r, wl.dtype, wl.L, lib_path=lib_path)
    for k, v in (opts or {}).items():
        plan.set(k, v)
    return plan


CASES = [  # (B, H, L, g, w, kernel code, NUM_CTAS)
    (2, 128, 1000, 16, 100, 3, 0),
    (5, 128, 130, 2, 3, 3, 0),
    (3, 128, 777, 64, 0, 3, 0),
    (4, 128, 1000, 16, 50, 3, 6),     # ranges across sequences
    (2, 16, 1000, 16, 100, 2, 0),
    (3, 16, 777, 64, 0, 2, 0),
    (4, 32, 1000, 16, 50, 2, 6),
    (2, 16, 300, 8, 40, 1, 0),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "B{}_H{}_L{}_g{}_w{}_k{}_n{}".format(*c))
def test_checked_build_parity(case, checked_lib):
    B, H, L, g, w, kern, n = case
    wl = workloads.small("chk", B=B, H=H, L=L, g=g, w=w, seed=L + B)
    x = workloads.generate(wl)
    opts = {kvc.OPT_KERNEL: kern}
    if n:
        opts[kvc.OPT_NUM_CTAS] = n
    plan = _plan(wl, checked_lib, opts)
    d = DeviceInputs(x)
    out, anc = run_lca(plan, d, g, w)            # asserts device_error() == LCA_OK
    compare(out, anc, oracle_lca(x, g, w), BF16_TOL, exact_anchors=False, x=x, g=g)
    dense = run_dense(plan, d)
    assert plan.device_error() == kvc.LCA_OK
    assert rel_err(dense, oracle_dense(x)) <= BF16_TOL


def test_checked_build_fp32_and_stored_and_slices(checked_lib):
    wt = workloads.WORKLOADS["tiny_f32"]
    xt = workloads.generate(wt)
    pt = _plan(wt, checked_lib)
    out, anc = run_lca(pt, DeviceInputs(xt), wt.g, wt.w)
    compare(out, anc, oracle_lca(xt, wt.g, wt.w), F32_TOL, exact_anchors=True)
    # stored cache: build + decode
    wl = workloads.small("chk", B=2, H=128, L=1500, g=16, w=100, seed=1)
    x = workloads.generate(wl)
    d = DeviceInputs(x)
    plan = _plan(wl, checked_lib)
    R = kvc.stored_rows(wl.L, wl.g, wl.w)
    c_st = torch.empty(wl.B, R, wl.d_c, dtype=torch.bfloat16, device="cuda")
    k_st = torch.empty(wl.B, R, wl.d_r, dtype=torch.bfloat16, device="cuda")
    anc_st = torch.empty(wl.B, wl.n_groups, dtype=torch.int32, device="cuda")
    plan.build_stored(d.q_c, d.q_r, d.c_kv, d.k_r, wl.L, wl.g, wl.w, c_st, k_st, anc_st)
    o = torch.empty(wl.B, wl.H, wl.d_c, device="cuda")
    plan.decode_stored(d.q_c, d.q_r, c_st, k_st, R, wl.n_groups, 0.0, o)
    torch.cuda.synchronize()
    assert plan.device_error() == kvc.LCA_OK
    # slices and the merge
    mzs, os_ = [], []
    for (pos0, n) in slice_bounds(wl.L, wl.g, wl.w, 3):
        c_sl = to_device(np.ascontiguousarray(x.c_kv[:, pos0:pos0 + n]))
        k_sl = to_device(np.ascontiguousarray(x.k_r[:, pos0:pos0 + n]))
        ng = kvc.slice_groups(wl.L, wl.g, wl.w, pos0, n)
        mz = torch.empty(wl.B, wl.H, 2, device="cuda")
        po = torch.empty(wl.B, wl.H, wl.d_c, device="cuda")
        an = torch.empty(wl.B, wl.H, max(ng, 1), dtype=torch.int32, device="cuda")
        plan.decode_partial(d.q_c, d.q_r, c_sl, k_sl, n, pos0, wl.L, wl.g, wl.w, mz, po, an if ng else None)
        mzs.append(mz); os_.append(po)
    out = torch.empty(wl.B, wl.H, wl.d_c, device="cuda")
    plan.merge_partials(3, torch.stack(mzs).contiguous(), torch.stack(os_).contiguous(), out)
    torch.cuda.synchronize()
    assert plan.device_error() == kvc.LCA_OK
    ref = oracle_lca(x, wl.g, wl.w)
    assert rel_err(out.cpu().numpy().astype(np.float64), ref.out) <= BF16_TOL


@pytest.mark.parametrize("H", [128, 16, 4])
def test_checked_build_paged_and_prefill(H, checked_lib):
    """The paged decode (ragged lengths, NaN rows outside the sequences) and a
    prefill chunk on the range-checked build: no check fires, oracle parity."""
    dt = "f32" if H == 4 else "bf16"
    kw = dict(d_c=64, d_r=16) if dt == "f32" else {}
    lengths = [700, 65, 1, 300]
    wl = workloads.small("chk_paged", B=4, H=H, L=700, g=8, w=40, dtype=dt, seed=9, **kw)
    x = workloads.generate(wl)
    cache = workloads.paged_layout(x, lengths, 64, seed=9)
    plan = _plan(wl, checked_lib)
    stride = kvc.num_groups(wl.L, 8, 40)
    out = torch.empty(wl.B, H, wl.d_c, device="cuda")
    anc = torch.empty(wl.B, H, stride, dtype=torch.int32, device="cuda")
    c_pool, k_pool = to_device(cache.c_pool), to_device(cache.k_pool)
    table = torch.from_numpy(cache.block_table).cuda()
    plan.decode_paged(to_device(x.q_c), to_device(x.q_r), c_pool, k_pool, 64, table,
                      torch.from_numpy(cache.seq_lens).cuda(), 8, 40, out, anc)
    torch.cuda.synchronize()
    assert plan.device_error() == kvc.LCA_OK
    ref = orc.lca_paged(x.q_c, x.q_r, cache.c_pool, cache.k_pool, cache.block_table, cache.seq_lens, 64, 8, 40)
    tol = F32_TOL if dt == "f32" else BF16_TOL
    assert rel_err(out.cpu().numpy().astype(np.float64), ref.out) <= tol
    # a prefill chunk: the 4 queries at positions 200 .. 203 of sequence 0
    plan.prefill_paged(to_device(x.q_c), to_device(x.q_r), c_pool, k_pool, 64, table[0].contiguous(), 200, 8, 40,
                       out, anc)
    torch.cuda.synchronize()
    assert plan.device_error() == kvc.LCA_OK
    pre = orc.lca_prefill(x.q_c, x.q_r, cache.c_pool, cache.k_pool, cache.block_table[0], 200, 64, 8, 40)
    assert rel_err(out.cpu().numpy().astype(np.float64), pre.out) <= tol


def test_checked_build_gqa(checked_lib):
    x = workloads.generate_gqa(2, 28, 4, 128, 128, 900, "bf16", 3)
    plan = kvc.Plan(2, 28, 128, 128, "bf16", 900, lib_path=checked_lib)
    nG = kvc.num_groups(900, 16, 100)
    out = torch.empty(2, 28, 128, device="cuda")
    anc = torch.empty(2, 28, nG, dtype=torch.int32, device="cuda")
    plan.decode_gqa(to_device(x.q), to_device(x.k), to_device(x.v), 900, 4, 16, 100, out, anc)
    torch.cuda.synchronize()
    assert plan.device_error() == kvc.LCA_OK
    ref = orc.lca_gqa(x.q, x.k, x.v, 16, 100)
    assert rel_err(out.cpu().numpy().astype(np.float64), ref.out) <= BF16_TOL
