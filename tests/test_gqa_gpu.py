"""GQA LCA decode (lca_decode_gqa) on the GPU against the oracle.

Query heads share KV heads (r = H / H_kv of them); the oracle is
oracle.lca_gqa (values pooled with the group softmax, the top-scoring token's
key kept), pinned against torch and against the MLA oracle with a zero
semantic query.  Bars: <= 2e-2 (bf16) / 1e-5 (fp32) max relative error; fp32
anchors exact, bf16 anchors exact where the oracle's top-2 gap exceeds 1e-3 of
max |s| and otherwise in their group within that gate of the maximum."""
import numpy as np
import pytest

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

import kv_compression_b200 as kvc  # noqa: E402
import workloads  # noqa: E402
from gpu_helpers import (ANC_SENTINEL, ANCHOR_GAP, BF16_TOL, F32_TOL, OUT_SENTINEL, Guarded, rel_err,  # noqa: E402
                         to_device)
from oracle import oracle as orc  # noqa: E402

pytestmark = pytest.mark.gpu

# (B, H, H_kv, d_k, d_v, L, g, w, dtype, seed)
CASES = [
    (2, 28, 4, 128, 128, 2000, 16, 100, "bf16", 1),    # Distill-Qwen-7B-style heads
    (3, 8, 8, 64, 64, 1500, 8, 64, "bf16", 2),         # one query head per KV head
    (2, 32, 2, 128, 128, 1000, 32, 200, "bf16", 3),    # sixteen per KV head
    (1, 4, 2, 64, 32, 700, 4, 0, "f32", 4),            # d_v != d_k, no window
    (2, 8, 4, 128, 128, 64, 16, 100, "bf16", 5),       # L <= w: dense
    (2, 14, 2, 128, 128, 777, 1, 0, "bf16", 6),        # g = 1: dense
    (2, 6, 3, 96, 64, 1100, 64, 130, "f32", 7),        # 64-token groups, odd widths
]


def _wide(a):
    return workloads.bf16_bits_to_f32(a).astype(np.float64) if a.dtype == np.uint16 else a.astype(np.float64)


@pytest.mark.parametrize("case", CASES, ids=lambda c: "B{}_H{}_kv{}_dk{}_dv{}_L{}_g{}_w{}_{}".format(*c[:9]))
def test_gqa_matches_oracle(case):
    B, H, H_kv, d_k, d_v, L, g, w, dt, seed = case
    x = workloads.generate_gqa(B, H, H_kv, d_k, d_v, L, dt, seed)
    plan = kvc.Plan(B, H, d_v, d_k, dt, L)
    nG = kvc.num_groups(L, g, w)
    out = Guarded((B, H, d_v), torch.float32, float("nan"), OUT_SENTINEL)
    anc = Guarded((B, H, max(nG, 1)), torch.int32, -7, ANC_SENTINEL)
    plan.decode_gqa(to_device(x.q), to_device(x.k), to_device(x.v), L, H_kv, g, w, out.t, anc.t if nG else None)
    torch.cuda.synchronize()
    assert plan.device_error() == kvc.LCA_OK
    out.check()
    anc.check()
    got = out.t.cpu().numpy().astype(np.float64)
    ref = orc.lca_gqa(x.q, x.k, x.v, g, w)
    assert np.all(np.isfinite(got))
    err = rel_err(got, ref.out)
    assert err <= (F32_TOL if dt == "f32" else BF16_TOL), err
    if nG == 0:
        return
    a = anc.t.cpu().numpy()[:, :, :nG]
    lo = (np.arange(nG) * g)[None, None, :]
    assert np.all((a >= lo) & (a < lo + g)), "anchor outside its group"
    if dt == "f32":
        assert np.array_equal(a, ref.anchor)
        return
    gate = ref.tie_gap > ANCHOR_GAP * ref.max_abs_s[..., None]
    assert np.array_equal(a[gate], ref.anchor[gate])
    # the others: the chosen token's double score within the gate of the group maximum
    r = H // H_kv
    for b, h, j in np.argwhere(~gate):
        K = _wide(x.k[b, j * g:(j + 1) * g, h // r])
        sc = K @ _wide(x.q[b, h])
        assert sc[a[b, h, j] - j * g] >= sc.max() - ANCHOR_GAP * ref.max_abs_s[b, h]


def test_gqa_argument_errors():
    plan = kvc.Plan(1, 28, 128, 128, "bf16", 256)
    lib = kvc.load_library()
    buf = torch.zeros(1 << 20, dtype=torch.bfloat16, device="cuda")
    out = torch.empty(1, 28, 128, device="cuda")
    anc = torch.empty(1, 28, 16, dtype=torch.int32, device="cuda")
    s = torch.cuda.current_stream().cuda_stream
    P = lambda t: t.data_ptr()  # noqa: E731
    call = lambda kv, L=256, g=16, w=0: lib.lca_decode_gqa(plan.handle, P(buf), P(buf), P(buf), L, kv, g, w,  # noqa: E731
                                                            P(out), P(anc), s)
    assert call(4) == kvc.LCA_OK
    assert call(3) == 1            # 28 query heads do not split over 3 KV heads
    assert call(1) == kvc.LCA_ERR_UNSUPPORTED   # 28 query heads on one KV head: more than 16
    assert call(4, L=257) == 1     # past max_L
    assert call(4, g=0) == 1
    torch.cuda.synchronize()
    assert plan.device_error() == kvc.LCA_OK
