"""The paged, variable-length decode on the GPU against the oracle.

lca_decode_paged reads each sequence's cache through its block table and its
own length (both on the device); every sequence must come out as the decode
of its own contiguous tokens (oracle.lca_paged, itself pinned against the
torch-built LCA of each prefix).  The pools hold NaN in every row no sequence
owns -- spare pages and the rows past each sequence's last token in its last
page -- and the block tables hold -1 past each sequence's last page, so a
kernel that reads either shows it (NaN outputs, or a device input error).
Bars as for lca_decode: <= 2e-2 (bf16) / 1e-5 (fp32) max relative error,
gated anchors equal, the others in their group within the near-tie gate."""
import numpy as np
import pytest

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

import kv_compression_b200 as kvc  # noqa: E402
import workloads  # noqa: E402
from gpu_helpers import (ANC_SENTINEL, ANCHOR_GAP, BF16_TOL, F32_TOL, OUT_SENTINEL, Guarded,  # noqa: E402
                         group_scores, rel_err, to_device)
from oracle import oracle as orc  # noqa: E402

pytestmark = pytest.mark.gpu

# (H, dtype, lengths, page_size, g, w, seed, kernel)
CASES = [
    (128, "bf16", [1500, 1, 130, 64, 700], 64, 16, 100, 1, "tcgen05_pair"),
    (128, "bf16", [2000, 900, 257], 128, 32, 256, 2, "tcgen05_pair"),
    (128, "bf16", [1000, 1000, 65], 64, 64, 64, 3, "tcgen05_pair"),
    (128, "bf16", [3000, 77, 1], 192, 8, 300, 4, "tcgen05_pair"),
    (16, "bf16", [1500, 1, 130, 64, 700], 64, 16, 100, 5, "tcgen05"),
    (16, "bf16", [2000, 333, 128, 129], 128, 128, 256, 6, "tcgen05"),
    (16, "bf16", [3000, 77, 191], 192, 8, 300, 7, "tcgen05"),
    (4, "f32", [700, 1, 65, 300], 64, 8, 50, 8, "simt"),
]


def _inputs(H, dtype, lengths, g, w, seed):
    kw = dict(d_c=64, d_r=16) if dtype == "f32" else {}
    wl = workloads.small("paged", B=len(lengths), H=H, L=max(lengths), g=g, w=w, dtype=dtype, seed=seed, **kw)
    return wl, workloads.generate(wl)


class PagedDevice:
    def __init__(self, x, cache):
        self.q_c, self.q_r = to_device(x.q_c), to_device(x.q_r)
        self.c_pool, self.k_pool = to_device(cache.c_pool), to_device(cache.k_pool)
        self.table = torch.from_numpy(cache.block_table).cuda()
        self.lens = torch.from_numpy(cache.seq_lens).cuda()


def _run(plan, wl, d, ps, g, w, stride):
    out = Guarded((wl.B, wl.H, wl.d_c), torch.float32, float("nan"), OUT_SENTINEL)
    anc = Guarded((wl.B, wl.H, max(stride, 1)), torch.int32, -7, ANC_SENTINEL)
    plan.decode_paged(d.q_c, d.q_r, d.c_pool, d.k_pool, ps, d.table, d.lens, g, w, out.t,
                      anc.t if stride > 0 else None)
    torch.cuda.synchronize()
    st = plan.device_error()
    out.check()
    anc.check()
    return st, out.t.cpu().numpy().astype(np.float64), anc.t.cpu().numpy()


def _check_sequences(x, ref, got, anc, lengths, g, w, tol, skip=()):
    for b, L in enumerate(lengths):
        if b in skip:
            continue
        assert np.all(np.isfinite(got[b])), b
        err = rel_err(got[b], ref.out[b])
        assert err <= tol, (b, L, err)
        nG = orc.num_groups(L, g, w)
        a, ra = anc[b, :, :nG], ref.anchor[b]
        assert np.all(anc[b, :, nG:] == -7), "anchor written past the sequence's groups"
        if nG == 0:
            continue
        lo = (np.arange(nG) * g)[None, :]
        assert np.all((a >= lo) & (a < lo + g)), "anchor outside its group"
        gate = ref.tie_gap[b] > ANCHOR_GAP * ref.max_abs_s[b][:, None]
        assert np.array_equal(a[gate], ra[gate]), f"sequence {b}: gated anchors differ"
        hh, jj = np.nonzero(~gate)
        if hh.size:
            s = group_scores(x, np.full(hh.size, b), hh, jj, g)
            chosen = s[np.arange(hh.size), a[hh, jj] - jj * g]
            assert np.all(chosen >= s.max(axis=1) - ANCHOR_GAP * ref.max_abs_s[b][hh])


@pytest.mark.parametrize("case", CASES, ids=lambda c: "H{}_{}_L{}_ps{}_g{}_w{}".format(
    c[0], c[1], "-".join(map(str, c[2])), c[3], c[4], c[5]))
def test_paged_matches_oracle(case):
    H, dt, lengths, ps, g, w, seed, kernel = case
    wl, x = _inputs(H, dt, lengths, g, w, seed)
    cache = workloads.paged_layout(x, lengths, ps, seed=seed)
    d = PagedDevice(x, cache)
    plan = kvc.Plan(wl.B, wl.H, wl.d_c, wl.d_r, wl.dtype, wl.L)
    assert plan.kernel(wl.L, g, w) == kernel
    stride = kvc.num_groups(wl.L, g, w)
    st, got, anc = _run(plan, wl, d, ps, g, w, stride)
    assert st == kvc.LCA_OK, f"device error {st} at site {plan.device_error_site():#x}"
    ref = orc.lca_paged(x.q_c, x.q_r, cache.c_pool, cache.k_pool, cache.block_table, cache.seq_lens, ps, g, w)
    _check_sequences(x, ref, got, anc, lengths, g, w, F32_TOL if dt == "f32" else BF16_TOL)


@pytest.mark.parametrize("H,kernel", [(128, "tcgen05_pair"), (16, "tcgen05"), (16, "simt")])
def test_identity_layout_equals_contiguous_decode(H, kernel):
    """Equal lengths and pages in order: the paged decode runs the same tiles
    as lca_decode on the contiguous cache and gives the same bits."""
    wl = workloads.small("paged_id", B=3, H=H, L=1024, g=16, w=100, seed=11)
    x = workloads.generate(wl)
    plan = kvc.Plan(wl.B, wl.H, wl.d_c, wl.d_r, wl.dtype, wl.L)
    if kernel == "simt":
        plan.set(kvc.OPT_FORCE_SIMT, 1)
    assert plan.kernel(wl.L, 16, 100) == kernel
    q_c, q_r = to_device(x.q_c), to_device(x.q_r)
    c, k = to_device(x.c_kv), to_device(x.k_r)
    nG = kvc.num_groups(wl.L, 16, 100)
    out = torch.empty(wl.B, wl.H, wl.d_c, device="cuda")
    anc = torch.empty(wl.B, wl.H, nG, dtype=torch.int32, device="cuda")
    plan.decode(q_c, q_r, c, k, wl.L, 16, 100, out, anc)
    table = torch.arange(wl.B * 16, dtype=torch.int32, device="cuda").view(wl.B, 16)
    lens = torch.full((wl.B,), wl.L, dtype=torch.int32, device="cuda")
    out_p = torch.empty_like(out)
    anc_p = torch.empty_like(anc)
    plan.decode_paged(q_c, q_r, c.view(-1, wl.d_c), k.view(-1, wl.d_r), 64, table, lens, 16, 100, out_p, anc_p)
    torch.cuda.synchronize()
    assert plan.device_error() == kvc.LCA_OK
    assert torch.equal(out, out_p) and torch.equal(anc, anc_p)


def test_ranges_outnumber_tiles():
    """One short sequence: far fewer tiles than tile ranges, so most clusters
    find no work in the metadata and leave."""
    lengths = [100]
    wl, x = _inputs(128, "bf16", lengths, 16, 32, 12)
    cache = workloads.paged_layout(x, lengths, 64, seed=12)
    d = PagedDevice(x, cache)
    plan = kvc.Plan(wl.B, wl.H, wl.d_c, wl.d_r, wl.dtype, 4096)
    stride = kvc.num_groups(4096, 16, 32)
    st, got, anc = _run(plan, wl, d, 64, 16, 32, stride)
    assert st == kvc.LCA_OK
    ref = orc.lca_paged(x.q_c, x.q_r, cache.c_pool, cache.k_pool, cache.block_table, cache.seq_lens, 64, 16, 32)
    _check_sequences(x, ref, got, anc, lengths, 16, 32, BF16_TOL)


@pytest.mark.parametrize("H", [128, 16, 4])
def test_out_of_range_lengths_and_pages_are_reported(H):
    """A length of 0 and one past max_pages * page_size leave those sequences
    NaN and raise LCA_ERR_DEVICE_INPUT; the others decode normally.  A used
    table entry past the pool is read as page 0 and raises the same error."""
    dt = "f32" if H == 4 else "bf16"
    lengths = [600, 300, 300, 200]
    wl, x = _inputs(H, dt, lengths, 8, 64, 13)
    cache = workloads.paged_layout(x, lengths, 64, seed=13)
    d = PagedDevice(x, cache)
    plan = kvc.Plan(wl.B, wl.H, wl.d_c, wl.d_r, wl.dtype, wl.L)
    stride = kvc.num_groups(wl.L, 8, 64)
    bad = torch.tensor([600, 0, 300, cache.block_table.shape[1] * 64 + 1], dtype=torch.int32, device="cuda")
    d.lens = bad
    st, got, anc = _run(plan, wl, d, 64, 8, 64, stride)
    assert st == kvc.LCA_ERR_DEVICE_INPUT
    assert np.all(np.isnan(got[1])) and np.all(np.isnan(got[3]))
    ref = orc.lca_paged(x.q_c, x.q_r, cache.c_pool, cache.k_pool, cache.block_table, cache.seq_lens, 64, 8, 64)
    tol = F32_TOL if dt == "f32" else BF16_TOL
    _check_sequences(x, ref, got, anc, lengths, 8, 64, tol, skip=(1, 3))
    d.lens = torch.from_numpy(cache.seq_lens).cuda()
    d.table = d.table.clone()
    d.table[2, 1] = cache.num_pages + 5
    st, got, anc = _run(plan, wl, d, 64, 8, 64, stride)
    assert st == kvc.LCA_ERR_DEVICE_INPUT
    _check_sequences(x, ref, got, anc, lengths, 8, 64, tol, skip=(2,))


def test_captured_graph_follows_device_lengths():
    """The call reads lengths and tables on the device only: a CUDA graph
    captured once decodes whatever lengths the tensor holds at replay."""
    wl, x = _inputs(128, "bf16", [1200] * 3, 16, 100, 14)
    cache = workloads.paged_layout(x, [1200] * 3, 64, seed=14)   # pages for every length up to 1200
    d = PagedDevice(x, cache)
    d.lens.copy_(torch.tensor([1200, 500, 64], dtype=torch.int32))
    plan = kvc.Plan(wl.B, wl.H, wl.d_c, wl.d_r, wl.dtype, wl.L)
    stride = kvc.num_groups(wl.L, 16, 100)
    out = torch.empty(wl.B, wl.H, wl.d_c, device="cuda")
    anc = torch.full((wl.B, wl.H, stride), -7, dtype=torch.int32, device="cuda")
    args = (d.q_c, d.q_r, d.c_pool, d.k_pool, 64, d.table, d.lens, 16, 100, out, anc)
    plan.decode_paged(*args)          # first call outside the capture (kernel attributes)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        plan.decode_paged(*args)
    for new in ([1200, 500, 64], [700, 1, 1100], [64, 64, 64]):
        d.lens.copy_(torch.tensor(new, dtype=torch.int32))
        anc.fill_(-7)
        graph.replay()
        torch.cuda.synchronize()
        assert plan.device_error() == kvc.LCA_OK
        lens = np.asarray(new, np.int32)
        ref = orc.lca_paged(x.q_c, x.q_r, cache.c_pool, cache.k_pool, cache.block_table, lens, 64, 16, 100)
        _check_sequences(x, ref, out.cpu().numpy().astype(np.float64), anc.cpu().numpy(), new, 16, 100,
                         BF16_TOL)
    del graph


def test_paged_argument_errors():
    wl, x = _inputs(16, "bf16", [256], 16, 16, 15)
    plan = kvc.Plan(wl.B, wl.H, wl.d_c, wl.d_r, wl.dtype, wl.L)
    lib = kvc.load_library()
    buf = torch.zeros(4096, 512, dtype=torch.bfloat16, device="cuda")
    tab = torch.zeros(1, 8, dtype=torch.int32, device="cuda")
    lens = torch.full((1,), 256, dtype=torch.int32, device="cuda")
    out = torch.empty(1, 16, 512, device="cuda")
    anc = torch.empty(1, 16, 16, dtype=torch.int32, device="cuda")
    s = torch.cuda.current_stream().cuda_stream
    P = lambda t: t.data_ptr()  # noqa: E731

    def call(page_size=64, num_pages=8, anchor=P(anc), table=P(tab), g=16):
        return lib.lca_decode_paged(plan.handle, P(buf), P(buf), P(buf), P(buf), num_pages, page_size, table, 8,
                                    P(lens), g, 16, P(out), anchor, 16, s)

    assert call() == kvc.LCA_OK
    assert call(page_size=32) == 1        # not a multiple of 64
    assert call(page_size=0) == 1
    assert call(num_pages=0) == 1
    assert call(g=0) == 1
    assert call(anchor=None) == 1         # groups are possible
    assert call(table=P(tab) + 2) == 3    # misaligned table
    torch.cuda.synchronize()
    assert plan.device_error() == kvc.LCA_OK
