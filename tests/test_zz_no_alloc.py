"""lca_decode_noalloc, the allocation-free entry point, against lca_decode.

lca_decode_noalloc runs the kernels of lca_decode with a fixed file-scope
device scratch in place of a plan's workspace.  Two calls in a row (the
second finds the scratch as the first left it) must each agree with
lca_decode on the same inputs.  The file name sorts last, so pytest collects
it after every other test; it passes run alone as well.
"""
import ctypes

import numpy as np
import pytest

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

import kv_compression_b200 as kvc  # noqa: E402
import workloads  # noqa: E402
from gpu_helpers import (ANC_SENTINEL, BF16_TOL, F32_TOL, OUT_SENTINEL, DeviceInputs,  # noqa: E402
                         Guarded, make_plan, rel_err, run_lca)

pytestmark = pytest.mark.gpu


def _vp(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def run_noalloc(wl, d, g, w):
    lib = kvc.load_library()
    nG = kvc.num_groups(wl.L, g, w)
    out = Guarded((wl.B, wl.H, wl.d_c), torch.float32, float("nan"), OUT_SENTINEL)
    anc = Guarded((wl.B, wl.H, max(nG, 1)), torch.int32, -7, ANC_SENTINEL)
    dt = kvc.LCA_BF16 if wl.dtype == "bf16" else kvc.LCA_F32
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    st = lib.lca_decode_noalloc(wl.B, wl.H, wl.d_c, wl.d_r, dt, _vp(d.q_c), _vp(d.q_r),
                                _vp(d.c_kv), _vp(d.k_r), wl.L, g, w, _vp(out.t),
                                _vp(anc.t) if nG > 0 else None, stream)
    assert st == kvc.LCA_OK, kvc.STATUS.get(st, st)
    torch.cuda.synchronize()
    out.check()
    anc.check()
    return out.t.cpu().numpy().astype(np.float64), anc.t.cpu().numpy()[:, :, :nG]


@pytest.mark.parametrize("wl,tol", [
    (workloads.small("na_bf16", B=3, H=32, L=5000, g=16, w=300, seed=41), BF16_TOL),
    (workloads.small("na_pair", B=2, H=128, L=3000, g=16, w=300, seed=44), BF16_TOL),
    (workloads.small("na_f32", B=2, H=4, L=1500, g=8, w=100, d_c=64, d_r=16, dtype="f32",
                     seed=42), F32_TOL),
])
def test_noalloc_matches_lca_decode_twice(wl, tol):
    x = workloads.generate(wl)
    d = DeviceInputs(x)
    ref_out, ref_anc = run_lca(make_plan(wl), d, wl.g, wl.w)
    for _ in range(2):
        got_out, got_anc = run_noalloc(wl, d, wl.g, wl.w)
        assert np.all(np.isfinite(got_out))
        err = rel_err(got_out, ref_out)
        assert err <= tol, f"relative difference {err:.3e} > {tol:.1e}"
        assert np.array_equal(got_anc, ref_anc)


def test_noalloc_rejects_shapes_beyond_its_scratch():
    lib = kvc.load_library()
    buf = torch.zeros(16, dtype=torch.uint8, device="cuda")
    p = _vp(buf)
    # B * H * d_c = 64 * 128 * 1024 floats > the 4 Mi floats of partial outputs
    st = lib.lca_decode_noalloc(64, 128, 1024, 64, kvc.LCA_BF16, p, p, p, p, 16, 1, 0, p, p, None)
    assert st == kvc.LCA_ERR_UNSUPPORTED
    # small d_c: the partial outputs would fit, the (max, sum) pairs would not
    # (B * H = 64 * 256 > 8192 slot-heads); refused before any launch
    st = lib.lca_decode_noalloc(64, 256, 64, 16, kvc.LCA_BF16, p, p, p, p, 16, 1, 0, p, p, None)
    assert st == kvc.LCA_ERR_UNSUPPORTED


def test_noalloc_small_latent_at_the_pair_limit():
    """d_c = 64 with B * H = 8192 slot-heads: exactly what the (max, sum) region
    holds for one slot per sequence.  It must run inside the scratch (guard
    regions intact) and match lca_decode."""
    wl = workloads.small("na_edge", B=64, H=128, L=40, g=4, w=8, d_c=64, d_r=16, dtype="f32",
                         seed=43)
    x = workloads.generate(wl)
    d = DeviceInputs(x)
    ref_out, ref_anc = run_lca(make_plan(wl), d, wl.g, wl.w)
    got_out, got_anc = run_noalloc(wl, d, wl.g, wl.w)
    assert rel_err(got_out, ref_out) <= F32_TOL
    assert np.array_equal(got_anc, ref_anc)
