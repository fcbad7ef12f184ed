"""GPU parity: the CUDA kernels (through the C ABI) against the CPU oracle on
the same seeded inputs.  Bars: fp32 latents -- anchors bit-exact, max relative
error <= 1e-5; bf16 latents with fp32 accumulation -- max relative error
<= 2e-2, anchors exact wherever the oracle's top-2 score gap exceeds
1e-3 * max|s| (elsewhere fp32 rounding may legitimately pick the other token).
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

import kv_compression_b200 as kvc  # noqa: E402
import workloads  # noqa: E402
from gpu_helpers import (BF16_TOL, F32_TOL, DeviceInputs, compare, make_plan, oracle_dense,  # noqa: E402
                         oracle_lca, rel_err, run_dense, run_lca)

pytestmark = pytest.mark.gpu

# (B, H, L, g, w): several 128-token tiles, ragged tails, every group-size path
SMALL = [
    (2, 16, 1000, 16, 100),     # ragged tail (1000 = 7*128 + 104)
    (1, 32, 4096, 4, 512),      # two head blocks
    (3, 16, 777, 64, 0),        # groups spanning two warps, no window
    (2, 16, 2048, 128, 7),      # one group per tile, leftovers join the window
    (1, 16, 300, 1, 0),         # g = 1: every token its own group
    (2, 16, 500, 8, 600),       # w >= L: nothing condensed
    (5, 16, 130, 2, 3),         # many short sequences
    (4, 48, 1500, 32, 64),      # three head blocks
    (1, 16, 1, 1, 0),           # a single token
    (2, 16, 129, 32, 1),        # one full tile plus one token
]


def _ids(c):
    return "B{}_H{}_L{}_g{}_w{}".format(*c)


@pytest.mark.parametrize("case", SMALL, ids=_ids)
@pytest.mark.parametrize("kernel", ["tcgen05", "simt"])
def test_small_bf16(case, kernel):
    B, H, L, g, w = case
    wl = workloads.small("t", B=B, H=H, L=L, g=g, w=w, seed=B * 1000 + L)
    x = workloads.generate(wl)
    plan = make_plan(wl, {kvc.OPT_FORCE_SIMT: 1} if kernel == "simt" else None)
    assert plan.kernel(L, g, w) == kernel
    out, anc = run_lca(plan, DeviceInputs(x), g, w)
    ref = oracle_lca(x, g, w)
    compare(out, anc, ref, BF16_TOL, exact_anchors=False, x=x, g=g)


# (B, H, L, g, w) for the two-CTA kernel (128 heads per cluster, 64-token tiles)
PAIR = [
    (2, 128, 1000, 16, 100),    # ragged tail (1000 = 15*64 + 40)
    (1, 128, 4096, 4, 512),
    (3, 128, 777, 64, 0),       # a group spans both token halves, no window
    (2, 128, 2048, 32, 7),      # leftovers join the window
    (1, 128, 300, 1, 0),        # g = 1: every token its own group
    (2, 128, 500, 8, 600),      # w >= L: nothing condensed
    (5, 128, 130, 2, 3),        # many short sequences
    (1, 256, 1500, 16, 64),     # two head blocks
    (1, 128, 1, 1, 0),          # a single token
    (2, 128, 65, 32, 1),        # one full tile plus one token
    (2, 128, 96, 32, 0),        # a tile whose second half is past L
]


@pytest.mark.parametrize("case", PAIR, ids=_ids)
def test_pair_kernel_small(case):
    """The two-CTA kernel (d_c split across a cluster, partial scores and P
    exchanged through distributed shared memory) against the oracle."""
    B, H, L, g, w = case
    wl = workloads.small("t", B=B, H=H, L=L, g=g, w=w, seed=B * 1000 + L + 7)
    x = workloads.generate(wl)
    plan = make_plan(wl)
    assert plan.kernel(L, g, w) == "tcgen05_pair"
    out, anc = run_lca(plan, DeviceInputs(x), g, w)
    ref = oracle_lca(x, g, w)
    compare(out, anc, ref, BF16_TOL, exact_anchors=False, x=x, g=g)


def test_pair_kernel_matches_the_16_head_kernel():
    """At H = 128 both tensor-core kernels take the shape; they must agree with
    each other as closely as each agrees with the oracle."""
    wl = workloads.small("t", B=2, H=128, L=3000, g=16, w=200, seed=21)
    x = workloads.generate(wl)
    d = DeviceInputs(x)
    a_pair, anc_pair = run_lca(make_plan(wl, {kvc.OPT_KERNEL: 3}), d, wl.g, wl.w)
    a_tc, anc_tc = run_lca(make_plan(wl, {kvc.OPT_KERNEL: 2}), d, wl.g, wl.w)
    ref = oracle_lca(x, wl.g, wl.w)
    compare(a_pair, anc_pair, ref, BF16_TOL, exact_anchors=False, x=x, g=wl.g)
    compare(a_tc, anc_tc, ref, BF16_TOL, exact_anchors=False, x=x, g=wl.g)
    assert rel_err(a_pair, a_tc) <= BF16_TOL


def test_pair_kernel_rescale():
    """Scores that rise by far more than the rescale threshold inside a range:
    token rows late in the sequence are scaled so that their scores exceed the
    first tile's maximum by ~30 (natural log units), which forces the reference
    max to rise and both CTAs to rescale the affected heads' O rows."""
    wl = workloads.small("t", B=1, H=128, L=2048, g=16, w=128, seed=23)
    x = workloads.generate(wl)
    from workloads import bf16_bits_to_f32, f32_to_bf16_bits
    c = bf16_bits_to_f32(x.c_kv).copy()
    k = bf16_bits_to_f32(x.k_r).copy()
    qdir = np.concatenate([bf16_bits_to_f32(x.q_c[0, :64]), bf16_bits_to_f32(x.q_r[0, :64])], axis=1)
    u = qdir.mean(axis=0)
    u /= np.linalg.norm(u)
    for t in (700, 1300, 1333, 1990):       # several rises, one in the window
        row = (40.0 * np.sqrt(576.0) * u).astype(np.float32)
        c[0, t] = row[:512]
        k[0, t] = row[512:]
    x.c_kv = f32_to_bf16_bits(c)
    x.k_r = f32_to_bf16_bits(k)
    d = DeviceInputs(x)
    plan = make_plan(wl)
    assert plan.kernel(wl.L, wl.g, wl.w) == "tcgen05_pair"
    out, anc = run_lca(plan, d, wl.g, wl.w)
    ref = oracle_lca(x, wl.g, wl.w)
    compare(out, anc, ref, BF16_TOL, exact_anchors=False, x=x, g=wl.g)
    for n in (2, 4):                          # fewer, longer ranges: rises mid-range
        out, anc = run_lca(make_plan(wl, {kvc.OPT_NUM_CTAS: n}), d, wl.g, wl.w)
        compare(out, anc, ref, BF16_TOL, exact_anchors=False, x=x, g=wl.g)


def test_pair_rescales_and_part_ends_back_to_back():
    """Short sequences (five tiles, the last partial) whose scores rise past the
    rescale threshold in every tile: the O issuer's rescale decisions come tile
    after tile, and with few clusters a sequence part ends every few tiles of
    a range, so the shippers' write-outs, the decisions and the rescales follow
    each other closely.  Repeated at several cluster counts, for g = 16 and 64."""
    from workloads import bf16_bits_to_f32, f32_to_bf16_bits
    for g, w, seed in ((16, 40, 31), (64, 44, 32)):
        wl = workloads.small("t", B=6, H=128, L=300, g=g, w=w, seed=seed)
        x = workloads.generate(wl)
        c = bf16_bits_to_f32(x.c_kv).copy()
        k = bf16_bits_to_f32(x.k_r).copy()
        for b in range(wl.B):
            qdir = np.concatenate([bf16_bits_to_f32(x.q_c[b]), bf16_bits_to_f32(x.q_r[b])], axis=1)
            u = qdir.mean(axis=0)
            u /= np.linalg.norm(u)
            for n, t in enumerate((20, 84, 148, 212, 276)):     # one rise in each tile
                row = (12.0 * (n + 1) * np.sqrt(576.0) * u).astype(np.float32)
                c[b, t] = row[:512]
                k[b, t] = row[512:]
        x.c_kv = f32_to_bf16_bits(c)
        x.k_r = f32_to_bf16_bits(k)
        d = DeviceInputs(x)
        ref = oracle_lca(x, wl.g, wl.w)
        for n in (2, 4, 10, 148):
            plan = make_plan(wl, {kvc.OPT_NUM_CTAS: n})
            assert plan.kernel(wl.L, wl.g, wl.w) == "tcgen05_pair"
            for _ in range(3):
                out, anc = run_lca(plan, d, wl.g, wl.w)
                compare(out, anc, ref, BF16_TOL, exact_anchors=False, x=x, g=wl.g)


def test_pair_ranges_spanning_sequences():
    """Few clusters: every tile range of the two-CTA kernel crosses sequence
    boundaries (query reloads, partials in several slots)."""
    wl = workloads.small("t", B=4, H=128, L=1000, g=16, w=50, seed=27)
    x = workloads.generate(wl)
    d = DeviceInputs(x)
    ref = oracle_lca(x, wl.g, wl.w)
    for n in (2, 4, 6, 12, 32, 148):
        plan = make_plan(wl, {kvc.OPT_NUM_CTAS: n})
        assert plan.kernel(wl.L, wl.g, wl.w) == "tcgen05_pair"
        out, anc = run_lca(plan, d, wl.g, wl.w)
        compare(out, anc, ref, BF16_TOL, exact_anchors=False, x=x, g=wl.g)


def test_pair_short_ranges_repeatable():
    """Ranges of one and two tiles with a partial last tile (L = 3000): each
    range's partial is written out only after the O of both its tiles is
    complete.  Repeated runs at several cluster counts must all match the
    oracle (a missed wait shows up as rows that differ from run to run)."""
    for L, w, seed in ((3000, 300, 44), (3000, 200, 21)):
        wl = workloads.small("t", B=2, H=128, L=L, g=16, w=w, seed=seed)
        x = workloads.generate(wl)
        d = DeviceInputs(x)
        ref = oracle_lca(x, wl.g, wl.w)
        for n in (124, 126, 148, 40):
            plan = make_plan(wl, {kvc.OPT_NUM_CTAS: n})
            assert plan.kernel(wl.L, wl.g, wl.w) == "tcgen05_pair"
            for _ in range(3):
                out, anc = run_lca(plan, d, wl.g, wl.w)
                compare(out, anc, ref, BF16_TOL, exact_anchors=False, x=x, g=wl.g)


def test_ranges_spanning_sequences():
    """Few CTAs: every tile range crosses sequence boundaries (query reloads)."""
    wl = workloads.small("t", B=4, H=32, L=1000, g=16, w=50, seed=7)
    x = workloads.generate(wl)
    d = DeviceInputs(x)
    ref = oracle_lca(x, wl.g, wl.w)
    for n in (2, 3, 6, 16):
        plan = make_plan(wl, {kvc.OPT_NUM_CTAS: n})
        out, anc = run_lca(plan, d, wl.g, wl.w)
        compare(out, anc, ref, BF16_TOL, exact_anchors=False, x=x, g=wl.g)


def test_tiny_f32_config():
    """The tiny fp32 workload in full: anchors bit-exact, relative error <= 1e-5."""
    wl = workloads.WORKLOADS["tiny_f32"]
    x = workloads.generate(wl)
    plan = make_plan(wl)
    assert plan.kernel(wl.L, wl.g, wl.w) == "simt"
    d = DeviceInputs(x)
    out, anc = run_lca(plan, d, wl.g, wl.w)
    ref = oracle_lca(x, wl.g, wl.w)
    compare(out, anc, ref, F32_TOL, exact_anchors=True)
    dense = run_dense(plan, d)
    assert rel_err(dense, oracle_dense(x)) <= F32_TOL


@pytest.mark.parametrize("kernel", ["tcgen05", "simt", "tcgen05_pair"])
def test_dense_bf16(kernel):
    H = 128 if kernel == "tcgen05_pair" else 16
    wl = workloads.small("t", B=2, H=H, L=1500, g=1, w=0, seed=11)
    x = workloads.generate(wl)
    plan = make_plan(wl, {kvc.OPT_KERNEL: kvc.KERNEL_CODES[kernel]})
    out = run_dense(plan, DeviceInputs(x))
    assert rel_err(out, oracle_dense(x)) <= BF16_TOL


def test_lca_equals_dense_when_nothing_condensed():
    wl = workloads.small("t", B=2, H=16, L=900, g=16, w=900, seed=12)
    x = workloads.generate(wl)
    plan = make_plan(wl)
    d = DeviceInputs(x)
    a, _ = run_lca(plan, d, 16, 900)
    b = run_dense(plan, d)
    assert rel_err(a, b) <= 1e-6


def test_host_buffer_entry_point():
    wl = workloads.small("t", B=2, H=16, L=1000, g=16, w=100, seed=13)
    x = workloads.generate(wl)
    plan = make_plan(wl)
    nG = kvc.num_groups(wl.L, wl.g, wl.w)

    def host(a):
        t = torch.from_numpy(a.view(np.int16) if a.dtype == np.uint16 else a)
        return t.pin_memory()
    out = torch.empty(wl.B, wl.H, wl.d_c, dtype=torch.float32).pin_memory()
    anc = torch.empty(wl.B, wl.H, nG, dtype=torch.int32).pin_memory()
    plan.decode_host(host(x.q_c), host(x.q_r), host(x.c_kv), host(x.k_r), wl.L, wl.g, wl.w, out, anc)
    ref = oracle_lca(x, wl.g, wl.w)
    compare(out.numpy().astype(np.float64), anc.numpy(), ref, BF16_TOL, exact_anchors=False, x=x,
            g=wl.g)


def test_argument_errors():
    wl = workloads.small("t", B=1, H=16, L=256, g=16, w=16, seed=14)
    x = workloads.generate(wl)
    d = DeviceInputs(x)
    plan = make_plan(wl)
    out = torch.empty(1, 16, 512, device="cuda")
    anc = torch.empty(1, 16, 256, dtype=torch.int32, device="cuda")   # room for any g here
    lib = kvc.load_library()
    h = plan.handle
    s = torch.cuda.current_stream().cuda_stream
    P = lambda t: t.data_ptr()  # noqa: E731
    args = [P(d.q_c), P(d.q_r), P(d.c_kv), P(d.k_r)]
    assert lib.lca_decode(h, *args, 256, 16, 16, P(out), P(anc), s) == 0
    assert lib.lca_decode(h, None, *args[1:], 256, 16, 16, P(out), P(anc), s) == 1
    assert lib.lca_decode(h, *args, 256, 0, 16, P(out), P(anc), s) == 1
    assert lib.lca_decode(h, *args, 256, 16, -1, P(out), P(anc), s) == 1
    assert lib.lca_decode(h, *args, 257, 16, 16, P(out), P(anc), s) == 1    # L > max_L
    assert lib.lca_decode(h, *args, 0, 16, 16, P(out), P(anc), s) == 1
    assert lib.lca_decode(h, *args, 256, 16, 16, P(out), None, s) == 1      # n_G > 0 needs anchors
    assert lib.lca_decode(h, *args, 256, 16, 300, P(out), None, s) == 0     # n_G == 0: may be NULL
    assert lib.lca_decode(h, P(d.q_c) + 2, *args[1:], 256, 16, 16, P(out), P(anc), s) == 3
    assert lib.lca_decode(h, *args, 256, 3, 0, P(out), P(anc), s) == 0     # odd g: CUDA-core kernel
    assert plan.kernel(256, 3, 0) == "simt" and plan.kernel(256, 16, 16) == "tcgen05"
    torch.cuda.synchronize()
    assert plan.device_error() == 0
    # a group size with no kernel is refused before anything is launched
    big = kvc.Plan(1, 16, 512, 64, "bf16", 4096)
    c = torch.zeros(1, 4096, 512, dtype=torch.bfloat16, device="cuda")
    k = torch.zeros(1, 4096, 64, dtype=torch.bfloat16, device="cuda")
    assert lib.lca_decode(big.handle, P(d.q_c), P(d.q_r), P(c), P(k), 4096, 2000, 0, P(out), P(anc),
                          s) == 2
    assert lib.lca_plan_set(big.handle, kvc.OPT_NUM_CTAS, 10**6) == 1
    assert lib.lca_plan_set(big.handle, 99, 1) == 1
    big.close()
    # B * L beyond the 32-bit TMA row range is refused before anything is launched
    huge_L = (1 << 30) + 128
    huge = kvc.Plan(2, 16, 512, 64, "bf16", huge_L)
    assert lib.lca_decode(huge.handle, P(d.q_c), P(d.q_r), P(c), P(k), huge_L, 16, 0, P(out),
                          P(anc), s) == 2
    huge.close()
