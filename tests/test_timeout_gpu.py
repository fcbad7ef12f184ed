"""Failure detection without a GPU fault: the tcgen05 kernel's bounded waits.

The plan's debug switch makes the TMA producer skip its first load, so the
MMA issuer's wait for it can never complete.  With a 50 ms bound the kernel
must record a timeout in the device error word, stop, free its TMEM and
exit; the host reads LCA_ERR_DEVICE_TIMEOUT, and the context stays usable:
the next normal call on the same plan is correct.
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

import kv_compression_b200 as kvc  # noqa: E402
import workloads  # noqa: E402
from gpu_helpers import BF16_TOL, DeviceInputs, compare, make_plan, oracle_lca, run_lca  # noqa: E402

pytestmark = pytest.mark.gpu


def test_wait_timeout_is_reported_and_recovers():
    wl = workloads.small("t", B=2, H=16, L=1000, g=16, w=100, seed=21)
    x = workloads.generate(wl)
    d = DeviceInputs(x)
    plan = make_plan(wl, {kvc.OPT_WAIT_TIMEOUT_NS: 50_000_000, kvc.OPT_DEBUG_SKIP_LOAD: 1})
    out = torch.zeros(wl.B, wl.H, wl.d_c, device="cuda")
    anc = torch.zeros(wl.B, wl.H, wl.n_groups, dtype=torch.int32, device="cuda")
    plan.decode(d.q_c, d.q_r, d.c_kv, d.k_r, wl.L, wl.g, wl.w, out, anc)
    assert plan.device_error() == kvc.LCA_ERR_DEVICE_TIMEOUT
    assert plan.device_error() == kvc.LCA_OK          # the error word was cleared
    plan.set(kvc.OPT_DEBUG_SKIP_LOAD, 0)
    got, got_anc = run_lca(plan, d, wl.g, wl.w)
    compare(got, got_anc, oracle_lca(x, wl.g, wl.w), BF16_TOL, exact_anchors=False)


def test_pair_kernel_wait_timeout_is_reported_and_recovers():
    """The same on the two-CTA kernel (H = 128): the producer of each CTA skips
    its first K_R load, so the score MMA issuer's wait runs out; the peer CTA's
    waits for the partial scores run out in turn.  Both CTAs record the
    timeout, leave their loops, meet at the cluster barrier and free TMEM."""
    wl = workloads.small("t", B=2, H=128, L=1000, g=16, w=100, seed=22)
    x = workloads.generate(wl)
    d = DeviceInputs(x)
    plan = make_plan(wl, {kvc.OPT_WAIT_TIMEOUT_NS: 50_000_000, kvc.OPT_DEBUG_SKIP_LOAD: 1})
    assert plan.kernel(wl.L, wl.g, wl.w) == "tcgen05_pair"
    out = torch.zeros(wl.B, wl.H, wl.d_c, device="cuda")
    anc = torch.zeros(wl.B, wl.H, wl.n_groups, dtype=torch.int32, device="cuda")
    plan.decode(d.q_c, d.q_r, d.c_kv, d.k_r, wl.L, wl.g, wl.w, out, anc)
    assert plan.device_error() == kvc.LCA_ERR_DEVICE_TIMEOUT
    assert plan.device_error() == kvc.LCA_OK
    plan.set(kvc.OPT_DEBUG_SKIP_LOAD, 0)
    got, got_anc = run_lca(plan, d, wl.g, wl.w)
    compare(got, got_anc, oracle_lca(x, wl.g, wl.w), BF16_TOL, exact_anchors=False)
