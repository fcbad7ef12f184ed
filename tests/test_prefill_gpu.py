"""LCA prefill (lca_prefill_paged) on the GPU against the oracle.

A chunk of n queries of one paged sequence, query i at position pos0 + i,
each condensing its own causal prefix [0, pos0 + i] (its own groups and
window); the oracle is oracle.lca_prefill, pinned against torch LCA of every
prefix.  The pool holds NaN in every row the sequence does not own, and the
tokens after the chunk's last position are NaN too, so a query that reads past
its own position shows it.  Bars as for lca_decode."""
import numpy as np
import pytest

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

import kv_compression_b200 as kvc  # noqa: E402
import workloads  # noqa: E402
from gpu_helpers import ANC_SENTINEL, BF16_TOL, F32_TOL, OUT_SENTINEL, Guarded, to_device  # noqa: E402
from oracle import oracle as orc  # noqa: E402
from test_paged_gpu import _check_sequences  # noqa: E402

pytestmark = pytest.mark.gpu

# (H, dtype, n queries, pos0, page_size, g, w, seed, kernel)
CASES = [
    (128, "bf16", 40, 1000, 64, 16, 100, 1, "tcgen05_pair"),
    (128, "bf16", 24, 0, 64, 8, 16, 2, "tcgen05_pair"),
    (16, "bf16", 24, 700, 128, 32, 64, 3, "tcgen05"),
    (16, "bf16", 16, 3, 64, 4, 0, 4, "tcgen05"),
    (4, "f32", 10, 200, 64, 8, 20, 5, "simt"),
]


def _chunk(H, dt, n, pos0, ps, g, w, seed, tail=37):
    """The sequence's cache (pos0 + n tokens of it, then `tail` NaN tokens in its
    last pages) and the chunk's n queries."""
    kw = dict(d_c=64, d_r=16) if dt == "f32" else {}
    L = pos0 + n
    seq = workloads.generate(workloads.small("prefill_kv", B=1, H=H, L=L + tail, g=g, w=w, dtype=dt, seed=seed,
                                             **kw))
    nan = workloads.nan_fill(dt)
    seq.c_kv[:, L:] = nan
    seq.k_r[:, L:] = nan
    cache = workloads.paged_layout(seq, [L + tail], ps, seed=seed)
    qs = workloads.generate(workloads.small("prefill_q", B=n, H=H, L=1, g=g, w=w, dtype=dt, seed=seed + 100,
                                            **kw))
    return seq, cache, qs.q_c, qs.q_r


def _run(H, dt, n, pos0, ps, g, w, seed):
    seq, cache, q_c, q_r = _chunk(H, dt, n, pos0, ps, g, w, seed)
    kw = dict(d_c=64, d_r=16) if dt == "f32" else dict(d_c=512, d_r=64)
    plan = kvc.Plan(n, H, kw["d_c"], kw["d_r"], dt, pos0 + n + 64)
    stride = max(kvc.num_groups(pos0 + n, g, w), 1)
    out = Guarded((n, H, kw["d_c"]), torch.float32, float("nan"), OUT_SENTINEL)
    anc = Guarded((n, H, stride), torch.int32, -7, ANC_SENTINEL)
    c_pool, k_pool = to_device(cache.c_pool), to_device(cache.k_pool)
    row = torch.from_numpy(cache.block_table[0].copy()).cuda()
    dq_c, dq_r = to_device(q_c), to_device(q_r)
    plan.prefill_paged(dq_c, dq_r, c_pool, k_pool, ps, row, pos0, g, w, out.t, anc.t)
    torch.cuda.synchronize()
    st = plan.device_error()
    out.check()
    anc.check()
    return plan, seq, cache, q_c, q_r, st, out.t.cpu().numpy().astype(np.float64), anc.t.cpu().numpy(), \
        (dq_c, dq_r, c_pool, k_pool, row, out.t, anc.t)


@pytest.mark.parametrize("case", CASES, ids=lambda c: "H{}_{}_n{}_pos{}_ps{}_g{}_w{}".format(*c[:7]))
def test_prefill_matches_oracle(case):
    H, dt, n, pos0, ps, g, w, seed, kernel = case
    plan, seq, cache, q_c, q_r, st, got, anc, dev = _run(H, dt, n, pos0, ps, g, w, seed)
    assert plan.kernel(pos0 + n + 64, g, w) == kernel
    assert st == kvc.LCA_OK, f"device error {st} at site {plan.device_error_site():#x}"
    ref = orc.lca_prefill(q_c, q_r, cache.c_pool, cache.k_pool, cache.block_table[0], pos0, ps, g, w)
    lengths = list(range(pos0 + 1, pos0 + n + 1))
    # _check_sequences reads each query's group scores from the inputs it is given:
    # the one sequence's cache, with query i's q in row i
    x = workloads.Inputs(seq.wl.with_(B=n), q_c, q_r, np.repeat(seq.c_kv, n, axis=0), np.repeat(seq.k_r, n, axis=0))
    _check_sequences(x, ref, got, anc, lengths, g, w, F32_TOL if dt == "f32" else BF16_TOL)


def test_prefill_equals_paged_decode_of_each_prefix():
    """The prefill chunk is the variable-length paged decode with the row
    repeated and lengths pos0 + 1 .. pos0 + n: the same bits."""
    H, dt, n, pos0, ps, g, w, seed = 128, "bf16", 20, 900, 64, 16, 100, 6
    plan, seq, cache, q_c, q_r, st, got, anc, dev = _run(H, dt, n, pos0, ps, g, w, seed)
    assert st == kvc.LCA_OK
    dq_c, dq_r, c_pool, k_pool, row, _, _ = dev
    table = row[None, :].repeat(n, 1).contiguous()
    lens = torch.arange(pos0 + 1, pos0 + n + 1, dtype=torch.int32, device="cuda")
    out2 = torch.empty(n, H, 512, device="cuda")
    anc2 = torch.full((n, H, anc.shape[2]), -7, dtype=torch.int32, device="cuda")
    plan.decode_paged(dq_c, dq_r, c_pool, k_pool, ps, table, lens, g, w, out2, anc2)
    torch.cuda.synchronize()
    assert plan.device_error() == kvc.LCA_OK
    assert np.array_equal(out2.cpu().numpy().astype(np.float64), got)
    assert np.array_equal(anc2.cpu().numpy(), anc)


def test_prefill_argument_errors():
    H, dt, n, ps = 16, "bf16", 8, 64
    plan = kvc.Plan(n, H, 512, 64, dt, 1024)
    lib = kvc.load_library()
    buf = torch.zeros(4096, 512, dtype=torch.bfloat16, device="cuda")
    row = torch.zeros(16, dtype=torch.int32, device="cuda")
    out = torch.empty(n, H, 512, device="cuda")
    anc = torch.empty(n, H, 64, dtype=torch.int32, device="cuda")
    s = torch.cuda.current_stream().cuda_stream
    P = lambda t: t.data_ptr()  # noqa: E731

    def call(pos0, max_pages=16):
        return lib.lca_prefill_paged(plan.handle, P(buf), P(buf), P(buf), P(buf), 8, ps, P(row), max_pages, pos0,
                                     16, 16, P(out), P(anc), 64, s)

    assert call(0) == kvc.LCA_OK
    assert call(1024 - n) == kvc.LCA_OK
    assert call(1024 - n + 1) == 1        # past max_L
    assert call(-1) == 1
    assert call(100, max_pages=1) == 1    # past max_pages * page_size
    torch.cuda.synchronize()
    assert plan.device_error() == kvc.LCA_OK
