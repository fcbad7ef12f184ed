"""The roofline arithmetic of bench.py, checked by hand from the workload shapes.

Algorithmic bytes per launch: the cache read once (C_KV and K_R, bf16), the
queries, the fp32 output and the int32 anchors.  Algorithmic flops per context
token: 2 H (d_c + d_r) for the scores plus 2 H d_c for the folded P.C.
"""
import os
import sys
from types import SimpleNamespace

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
import workloads  # noqa: E402


@pytest.mark.parametrize("name,expected", [
    # 8*32768*576*2 + 8*16*576*2 + 8*16*512*4 + 8*16*1984*4
    ("v2lite", 301989888 + 147456 + 262144 + 1015808),
    # 32*65536*576*2 + 32*128*576*2 + 32*128*512*4 + 32*128*3968*4
    ("v2", 2415919104 + 4718592 + 8388608 + 65011712),
    # 4*131072*576*2 + 4*128*576*2 + 4*128*512*4 + 4*128*3968*4
    ("needle", 603979776 + 589824 + 1048576 + 8126464),
])
def test_algorithmic_bytes(name, expected):
    assert bench.algorithmic_bytes(workloads.WORKLOADS[name]) == expected


def test_v2lite_bytes_match_the_documented_figure():
    assert bench.algorithmic_bytes(workloads.WORKLOADS["v2lite"]) == 303_415_296


@pytest.mark.parametrize("name,gflop", [("v2lite", 9.127), ("v2", 584.1), ("needle", 146.0)])
def test_algorithmic_flops(name, gflop):
    assert bench.algorithmic_flops(workloads.WORKLOADS[name]) / 1e9 == pytest.approx(gflop, rel=1e-3)


def test_sweep_points_change_only_g_and_w():
    wl = workloads.WORKLOADS["sweep"]
    pt = bench.with_point(wl, SimpleNamespace(g=64, w=4096))
    assert (pt.g, pt.w) == (64, 4096)
    assert (pt.B, pt.H, pt.L, pt.d_c, pt.d_r, pt.seed) == (wl.B, wl.H, wl.L, wl.d_c, wl.d_r, wl.seed)
    assert pt.n_groups == (wl.L - 4096) // 64
    same = bench.with_point(wl, SimpleNamespace(g=None, w=None))
    assert (same.g, same.w) == (wl.g, wl.w)
    # the anchors shrink with n_G; the cache bytes do not
    assert bench.algorithmic_bytes(pt) < bench.algorithmic_bytes(wl)
    assert bench.algorithmic_flops(pt) == bench.algorithmic_flops(wl)


def test_profiled_traffic_only_for_its_workload():
    assert bench.profiled_traffic(workloads.WORKLOADS["needle"]) is None
    t = bench.profiled_traffic(workloads.WORKLOADS["v2lite"])
    if t is not None:   # None once the kernel sources change after the capture
        alg = bench.algorithmic_bytes(workloads.WORKLOADS["v2lite"])
        assert alg <= t < 1.1 * alg
