"""The stored, head-shared condensed cache on the GPU against the oracle.

lca_build_stored / lca_condense condense groups once with the head-mean score
of a query and store (c_bar_j, k_{a_j}); lca_decode_stored attends over
[stored || window] with an optional bias on the condensed logits.  The
oracle runs the same pipeline in double precision from the same inputs
(oracle.lca_stored); nothing the GPU produced is fed to it.  Bars: stored
latents within bf16 storage rounding plus fp32 accumulation (1e-2 of the
row's largest value), stored RoPE keys and window rows bit-exact copies,
anchors exact where the head-mean top-2 gap exceeds 1e-3 of max |s_bar| and
otherwise in-group and within that gate of the maximum, decode outputs
<= 2e-2 (bf16) / 1e-5 (fp32) max relative error.  The seeds are chosen so
that no group's head-mean top-2 gap is below 5e-4 of max |s_bar| (asserted),
so that every stored key is the oracle's and the end-to-end outputs are
comparable."""
import math

import numpy as np
import pytest

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

import kv_compression_b200 as kvc  # noqa: E402
import workloads  # noqa: E402
from gpu_helpers import (ANCHOR_GAP, BF16_TOL, F32_TOL, DeviceInputs, Guarded, OUT_SENTINEL,  # noqa: E402
                         make_plan, rel_err)
from oracle import oracle as orc  # noqa: E402
from workloads import bf16_bits_to_f32  # noqa: E402

pytestmark = pytest.mark.gpu

STORE_TOL = 1e-2

# (B, H, L, g, w, dtype, seed, kernel the decode runs)
CASES = [
    (2, 128, 1500, 16, 100, "bf16", 1, "tcgen05_pair"),
    (1, 128, 4000, 32, 256, "bf16", 1, "tcgen05_pair"),
    (3, 16, 2000, 4, 300, "bf16", 12, "tcgen05"),
    (2, 128, 900, 64, 64, "bf16", 1, "tcgen05_pair"),
    (2, 4, 700, 8, 50, "f32", 0, "simt"),
]


def _wl(B, H, L, g, w, dt, seed):
    kw = dict(d_c=64, d_r=16) if dt == "f32" else {}
    return workloads.small("stored", B=B, H=H, L=L, g=g, w=w, dtype=dt, seed=seed, **kw)


def _wide(a):
    return bf16_bits_to_f32(a).astype(np.float64) if a.dtype == np.uint16 else a.astype(np.float64)


def _torch_dtype(wl):
    return torch.bfloat16 if wl.dtype == "bf16" else torch.float32


def _host(t: torch.Tensor) -> np.ndarray:
    t = t.cpu()
    return t.float().numpy().astype(np.float64) if t.dtype == torch.bfloat16 else t.numpy().astype(np.float64)


def _build(plan, wl, d):
    R = kvc.stored_rows(wl.L, wl.g, wl.w)
    nG = wl.n_groups
    c_st = torch.empty(wl.B, R, wl.d_c, dtype=_torch_dtype(wl), device="cuda")
    k_st = torch.empty(wl.B, R, wl.d_r, dtype=_torch_dtype(wl), device="cuda")
    anc = torch.full((wl.B, max(nG, 1)), -1, dtype=torch.int32, device="cuda")
    plan.build_stored(d.q_c, d.q_r, d.c_kv, d.k_r, wl.L, wl.g, wl.w, c_st, k_st, anc if nG else None)
    torch.cuda.synchronize()
    return R, c_st, k_st, anc[:, :nG]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "B{}_H{}_L{}_g{}_w{}_{}".format(*c[:6]))
def test_build_and_decode_stored(case):
    B, H, L, g, w, dt, seed, kernel = case
    wl = _wl(B, H, L, g, w, dt, seed)
    x = workloads.generate(wl)
    d = DeviceInputs(x)
    plan = make_plan(wl)
    nG = wl.n_groups
    R, c_st, k_st, anc = _build(plan, wl, d)
    cb, ka, an, gap, mx = orc.condense_shared(x.q_c, x.q_r, x.c_kv, x.k_r, g, 0, nG)
    assert np.all(gap > 5e-4 * mx[:, None]), "seed has a head-mean near-tie; pick another"
    # anchors, stored keys (copies of the anchors' rows), stored latents
    got_anc = anc.cpu().numpy()
    assert np.array_equal(got_anc, an)
    kst, cst = _host(k_st), _host(c_st)
    assert np.array_equal(kst[:, :nG], _wide(x.k_r)[np.arange(B)[:, None], an])
    assert rel_err(cst[:, :nG], cb) <= STORE_TOL
    # window rows: copies of tokens [n_G g, L)
    assert np.array_equal(cst[:, nG:], _wide(x.c_kv)[:, nG * g:])
    assert np.array_equal(kst[:, nG:], _wide(x.k_r)[:, nG * g:])
    # decode a second query over the stored cache, with and without the log g bias
    wq = wl.with_(seed=seed + 1000)
    xq = workloads.generate(wq)
    dq = DeviceInputs(xq)
    tol = F32_TOL if dt == "f32" else BF16_TOL
    for bias in (0.0, math.log(g)):
        ref = orc.lca_stored(x.q_c, x.q_r, x.c_kv, x.k_r, g, w, q_c=xq.q_c, q_r=xq.q_r, bias=bias)
        out = Guarded((B, H, wl.d_c), torch.float32, float("nan"), OUT_SENTINEL)
        assert plan.kernel(R, 1, 0) == kernel
        plan.decode_stored(dq.q_c, dq.q_r, c_st, k_st, R, nG, bias, out.t)
        torch.cuda.synchronize()
        assert plan.device_error() == kvc.LCA_OK
        out.check()
        err = rel_err(out.t.cpu().numpy().astype(np.float64), ref.out)
        # fp32 latents are stored in fp32: the oracle keeps doubles, so the
        # stored rounding is 2^-24; bf16 storage rounds c_bar to 8 bits
        assert err <= (tol if dt == "f32" else BF16_TOL), (bias, err)


def test_condense_on_eviction_into_a_ring():
    """lca_condense on a middle range of groups, written at a row offset of a
    larger stored buffer (as when a group leaves the window), equals the
    oracle's condensation of those groups; rows outside stay untouched."""
    wl = _wl(2, 128, 1500, 16, 100, "bf16", 1)
    x = workloads.generate(wl)
    d = DeviceInputs(x)
    plan = make_plan(wl)
    j0, n, rows, row0 = 20, 37, 100, 41
    sentinel = -7.0
    c_dst = torch.full((wl.B, rows, wl.d_c), sentinel, dtype=torch.bfloat16, device="cuda")
    k_dst = torch.full((wl.B, rows, wl.d_r), sentinel, dtype=torch.bfloat16, device="cuda")
    anc = torch.full((wl.B, n), -1, dtype=torch.int32, device="cuda")
    plan.condense(d.q_c, d.q_r, d.c_kv, d.k_r, wl.L, wl.g, j0, n, c_dst, k_dst, rows, row0, anc)
    torch.cuda.synchronize()
    cb, ka, an, gap, mx = orc.condense_shared(x.q_c, x.q_r, x.c_kv, x.k_r, wl.g, j0, n)
    gate = gap > ANCHOR_GAP * mx[:, None]
    got = anc.cpu().numpy()
    assert np.array_equal(got[gate], an[gate])
    c, k = _host(c_dst), _host(k_dst)
    assert rel_err(c[:, row0:row0 + n], cb) <= STORE_TOL
    assert np.array_equal(k[:, row0:row0 + n][gate], ka[gate])
    assert np.all(c[:, :row0] == sentinel) and np.all(c[:, row0 + n:] == sentinel)
    assert np.all(k[:, :row0] == sentinel) and np.all(k[:, row0 + n:] == sentinel)


def test_stored_decode_with_log_g_bias_is_dense_for_identical_groups():
    """Groups of identical tokens: with bias log g the stored decode is exactly
    dense attention over all L tokens (here against mla_decode's oracle)."""
    wl = _wl(2, 128, 640, 8, 64, "bf16", 3)
    x = workloads.generate(wl)
    nG = wl.n_groups
    for j in range(nG):
        x.c_kv[:, j * 8:(j + 1) * 8] = x.c_kv[:, j * 8:j * 8 + 1]
        x.k_r[:, j * 8:(j + 1) * 8] = x.k_r[:, j * 8:j * 8 + 1]
    d = DeviceInputs(x)
    plan = make_plan(wl)
    R, c_st, k_st, anc = _build(plan, wl, d)
    assert np.array_equal(anc.cpu().numpy(), np.tile(np.arange(nG) * 8, (wl.B, 1)))
    out = torch.empty(wl.B, wl.H, wl.d_c, device="cuda")
    plan.decode_stored(d.q_c, d.q_r, c_st, k_st, R, nG, math.log(8), out)
    torch.cuda.synchronize()
    ref = orc.mla(x.q_c, x.q_r, x.c_kv, x.k_r)
    assert rel_err(out.cpu().numpy().astype(np.float64), ref) <= BF16_TOL


def test_stored_argument_errors():
    wl = _wl(1, 16, 256, 16, 16, "bf16", 5)
    x = workloads.generate(wl)
    d = DeviceInputs(x)
    plan = make_plan(wl)
    lib = kvc.load_library()
    buf = torch.empty(1, 512, 512, dtype=torch.bfloat16, device="cuda")
    P = lambda t: t.data_ptr()  # noqa: E731
    s = torch.cuda.current_stream().cuda_stream
    # (j0 + n) g > L
    assert lib.lca_condense(plan.handle, P(d.q_c), P(d.q_r), P(d.c_kv), P(d.k_r), 256, 16, 10, 7,
                            P(buf), P(buf), 512, 0, P(buf), s) == 1
    # dst_row0 + n > dst_rows
    assert lib.lca_condense(plan.handle, P(d.q_c), P(d.q_r), P(d.c_kv), P(d.k_r), 256, 16, 0, 4,
                            P(buf), P(buf), 3, 0, P(buf), s) == 1
    # n_cond > n_rows
    out = torch.empty(1, 16, 512, device="cuda")
    assert lib.lca_decode_stored(plan.handle, P(d.q_c), P(d.q_r), P(buf), P(buf), 10, 11, 0.0, P(out),
                                 s) == 1
    assert kvc.stored_rows(32768, 16, 1024) == 1984 + 1024
    assert kvc.stored_rows(10, 4, 20) == 10
