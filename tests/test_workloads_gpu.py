"""The five full-size workloads, in the launch configuration the benchmark
times, against the oracle on sampled sequences and heads (the oracle computes
those outputs one by one), plus properties checked over every output."""
import numpy as np
import pytest

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

import kv_compression_b200 as kvc  # noqa: E402
import workloads  # noqa: E402
from gpu_helpers import (BF16_TOL, DeviceInputs, compare, make_plan, oracle_lca,  # noqa: E402
                         run_lca)

pytestmark = pytest.mark.gpu


def _anchors_in_their_groups(anc: np.ndarray, g: int) -> None:
    nG = anc.shape[-1]
    lo = (np.arange(nG) * g)[None, None, :]
    assert np.all((anc >= lo) & (anc < lo + g))


def _check(name, rows, heads, points=None):
    wl = workloads.WORKLOADS[name]
    x = workloads.generate(wl, threads=16)
    d = DeviceInputs(x)
    plan = make_plan(wl)
    results = []
    for (g, w) in (points or [(wl.g, wl.w)]):
        assert plan.kernel(wl.L, g, w) == "tcgen05"
        out, anc = run_lca(plan, d, g, w)
        assert np.all(np.isfinite(out))
        _anchors_in_their_groups(anc, g)
        ref = oracle_lca(x, g, w, rows=rows, heads=heads)
        sub_out = out[rows][:, heads] if heads is not None else out[rows]
        sub_anc = anc[rows][:, heads] if heads is not None else anc[rows]
        results.append((g, w, compare(sub_out, sub_anc, ref, BF16_TOL, exact_anchors=False)))
        del out, anc
    return x, results


def test_v2lite_full():
    wl = workloads.WORKLOADS["v2lite"]
    _check("v2lite", rows=list(range(wl.B)), heads=None)


def test_v2_sampled():
    _check("v2", rows=[0, 31], heads=[0, 1, 63, 100, 127])


def test_needle_sampled_and_tie_break():
    wl = workloads.WORKLOADS["needle"]
    x, _ = _check("needle", rows=[0, 3], heads=[0, 17, 64, 127])
    d = DeviceInputs(x)
    plan = make_plan(wl)
    _, anc = run_lca(plan, d, wl.g, wl.w)
    win0 = wl.n_groups * wl.g
    pairs = 0
    for b in range(wl.B):
        pos = x.needle_pos[b]
        for j in np.unique(pos[pos < win0] // wl.g):
            planted = pos[(pos // wl.g) == j]
            a = anc[b, :, j]
            # identical planted rows score identically: an anchor on a planted
            # token must be the lowest planted index of its group
            on_planted = np.isin(a, planted)
            assert np.all(a[on_planted] == planted.min())
            pairs += len(planted) > 1
    assert pairs > 0, "no group holds two needles; the tie-break is untested"


def test_sweep_sampled():
    wl = workloads.WORKLOADS["sweep"]
    _check("sweep", rows=[0, 15], heads=[0, 7, 15], points=list(wl.sweep))
