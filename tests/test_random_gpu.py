"""Seeded random cases of the paged decode, the prefill and the GQA decode on
the GPU against the oracle: shapes, lengths, page sizes, groups and windows
drawn from a fixed generator (numpy default_rng(2026)), so every run checks the
same cases.  Bars as for the fixed cases: <= 2e-2 (bf16) / 1e-5 (fp32) max
relative error, bf16 anchors gated by the oracle's top-2 gap."""
import numpy as np
import pytest

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

import kv_compression_b200 as kvc  # noqa: E402
import workloads  # noqa: E402
from gpu_helpers import BF16_TOL, F32_TOL, rel_err, to_device  # noqa: E402
from oracle import oracle as orc  # noqa: E402
from test_paged_gpu import PagedDevice, _check_sequences, _run  # noqa: E402

pytestmark = pytest.mark.gpu

_RNG = np.random.default_rng(2026)
PAGED = []
for _ in range(10):
    H = int(_RNG.choice([128, 16, 32, 4]))
    dt = "f32" if H == 4 else "bf16"
    B = int(_RNG.integers(1, 5))
    lengths = [int(x) for x in _RNG.integers(1, 2500, size=B)]
    ps = int(_RNG.choice([64, 128, 192, 256]))
    g = int(_RNG.choice([1, 2, 4, 8, 16, 32, 64]))
    w = int(_RNG.choice([0, 1, 17, 64, 300]))
    PAGED.append((H, dt, lengths, ps, g, w, int(_RNG.integers(1 << 20))))
GQA = []
for _ in range(8):
    H_kv = int(_RNG.choice([1, 2, 4, 8]))
    r = int(_RNG.choice([1, 2, 3, 5, 7, 8, 12, 16]))
    dt = str(_RNG.choice(["bf16", "f32"]))
    d_k = int(_RNG.choice([64, 96, 128]))
    d_v = int(_RNG.choice([32, 64, 128]))
    L = int(_RNG.integers(1, 3000))
    g = int(_RNG.choice([1, 2, 4, 8, 16, 32, 64]))
    w = int(_RNG.choice([0, 5, 100, 1000]))
    GQA.append((int(_RNG.integers(1, 4)), H_kv * r, H_kv, d_k, d_v, L, g, w, dt, int(_RNG.integers(1 << 20))))


@pytest.mark.parametrize("case", PAGED, ids=lambda c: "H{}_{}_L{}_ps{}_g{}_w{}".format(
    c[0], c[1], "-".join(map(str, c[2])), c[3], c[4], c[5]))
def test_random_paged(case):
    H, dt, lengths, ps, g, w, seed = case
    kw = dict(d_c=64, d_r=16) if dt == "f32" else {}
    wl = workloads.small("rnd_paged", B=len(lengths), H=H, L=max(lengths), g=g, w=w, dtype=dt, seed=seed, **kw)
    x = workloads.generate(wl)
    cache = workloads.paged_layout(x, lengths, ps, seed=seed)
    d = PagedDevice(x, cache)
    plan = kvc.Plan(wl.B, wl.H, wl.d_c, wl.d_r, wl.dtype, wl.L)
    stride = kvc.num_groups(wl.L, g, w)
    st, got, anc = _run(plan, wl, d, ps, g, w, stride)
    assert st == kvc.LCA_OK, f"device error {st} at site {plan.device_error_site():#x}"
    ref = orc.lca_paged(x.q_c, x.q_r, cache.c_pool, cache.k_pool, cache.block_table, cache.seq_lens, ps, g, w)
    _check_sequences(x, ref, got, anc, lengths, g, w, F32_TOL if dt == "f32" else BF16_TOL)
    # the last sequence's final tokens as a prefill chunk over its own pages
    n = min(4, lengths[-1])
    pos0 = lengths[-1] - n
    q_c, q_r = x.q_c[:n] if n <= wl.B else None, x.q_r[:n] if n <= wl.B else None
    if q_c is None or n < 1:
        return
    pplan = kvc.Plan(n, wl.H, wl.d_c, wl.d_r, wl.dtype, wl.L)
    out = torch.empty(n, wl.H, wl.d_c, device="cuda")
    panc = torch.full((n, wl.H, max(stride, 1)), -7, dtype=torch.int32, device="cuda")
    row = torch.from_numpy(cache.block_table[-1].copy()).cuda()
    pplan.prefill_paged(to_device(q_c), to_device(q_r), d.c_pool, d.k_pool, ps, row, pos0, g, w, out,
                        panc if stride > 0 else None)
    torch.cuda.synchronize()
    assert pplan.device_error() == kvc.LCA_OK
    pre = orc.lca_prefill(q_c, q_r, cache.c_pool, cache.k_pool, cache.block_table[-1], pos0, ps, g, w)
    assert rel_err(out.cpu().numpy().astype(np.float64), pre.out) <= (F32_TOL if dt == "f32" else BF16_TOL)


@pytest.mark.parametrize("case", GQA, ids=lambda c: "B{}_H{}_kv{}_dk{}_dv{}_L{}_g{}_w{}_{}".format(*c[:9]))
def test_random_gqa(case):
    B, H, H_kv, d_k, d_v, L, g, w, dt, seed = case
    x = workloads.generate_gqa(B, H, H_kv, d_k, d_v, L, dt, seed)
    plan = kvc.Plan(B, H, d_v, d_k, dt, L)
    nG = kvc.num_groups(L, g, w)
    out = torch.empty(B, H, d_v, device="cuda")
    anc = torch.empty(B, H, max(nG, 1), dtype=torch.int32, device="cuda")
    plan.decode_gqa(to_device(x.q), to_device(x.k), to_device(x.v), L, H_kv, g, w, out, anc if nG else None)
    torch.cuda.synchronize()
    assert plan.device_error() == kvc.LCA_OK
    ref = orc.lca_gqa(x.q, x.k, x.v, g, w)
    assert rel_err(out.cpu().numpy().astype(np.float64), ref.out) <= (F32_TOL if dt == "f32" else BF16_TOL)
    if nG:
        a = anc.cpu().numpy()[:, :, :nG]
        lo = (np.arange(nG) * g)[None, None, :]
        assert np.all((a >= lo) & (a < lo + g))
        if dt == "f32":
            assert np.array_equal(a, ref.anchor)
        else:
            gate = ref.tie_gap > 1e-3 * ref.max_abs_s[..., None]
            assert np.array_equal(a[gate], ref.anchor[gate])
