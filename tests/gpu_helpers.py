"""Shared helpers of the GPU tests: upload seeded inputs, run the library,
run the oracle on the same inputs, compare."""
from __future__ import annotations

import numpy as np
import torch

import kv_compression_b200 as kvc
import workloads
from oracle import oracle as orc
from workloads import bf16_bits_to_f32

BF16_TOL = 2e-2      # bf16 latents, fp32 accumulation
F32_TOL = 1e-5       # fp32 latents
ANCHOR_GAP = 1e-3    # bf16 anchors are gated where the oracle's top-2 gap > 1e-3 * max|s|


def to_device(a: np.ndarray) -> torch.Tensor:
    if a.dtype == np.uint16:
        return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).cuda()
    return torch.from_numpy(a).cuda()


class DeviceInputs:
    def __init__(self, x: workloads.Inputs):
        self.x = x
        self.q_c, self.q_r = to_device(x.q_c), to_device(x.q_r)
        self.c_kv, self.k_r = to_device(x.c_kv), to_device(x.k_r)


def make_plan(wl: workloads.Workload, opts: dict | None = None) -> kvc.Plan:
    plan = kvc.Plan(wl.B, wl.H, wl.d_c, wl.d_r, wl.dtype, wl.L)
    for k, v in (opts or {}).items():
        plan.set(k, v)
    return plan


GUARD = 4096                      # guard elements on each side of an output buffer
OUT_SENTINEL = -3.0e38            # exact float32 value no kernel writes
ANC_SENTINEL = -123456789


class Guarded:
    """A device tensor with sentinel-filled guard regions before and after it, so a
    write past either end of an output (there is no sanitizer on the pool) is seen."""

    def __init__(self, shape, dtype, fill, sentinel):
        self.n = int(np.prod(shape))
        self.sentinel = sentinel
        self.buf = torch.full((self.n + 2 * GUARD,), sentinel, dtype=dtype, device="cuda")
        self.t = self.buf[GUARD:GUARD + self.n].view(shape)   # 16 KB in: 16-byte aligned
        self.t.fill_(fill)

    def check(self) -> None:
        head, tail = self.buf[:GUARD], self.buf[GUARD + self.n:]
        assert bool((head == self.sentinel).all()), "write before the start of an output"
        assert bool((tail == self.sentinel).all()), "write past the end of an output"


def run_lca(plan: kvc.Plan, d: DeviceInputs, g: int, w: int):
    wl = d.x.wl
    nG = kvc.num_groups(wl.L, g, w)
    out = Guarded((wl.B, wl.H, wl.d_c), torch.float32, float("nan"), OUT_SENTINEL)
    anc = Guarded((wl.B, wl.H, max(nG, 1)), torch.int32, -7, ANC_SENTINEL)
    plan.decode(d.q_c, d.q_r, d.c_kv, d.k_r, wl.L, g, w, out.t, anc.t if nG > 0 else None)
    torch.cuda.synchronize()
    st = plan.device_error()
    assert st == kvc.LCA_OK, f"device error {st} at wait site {plan.device_error_site():#x}"
    out.check()
    anc.check()
    return out.t.cpu().numpy().astype(np.float64), anc.t.cpu().numpy()[:, :, :nG]


def run_dense(plan: kvc.Plan, d: DeviceInputs):
    wl = d.x.wl
    out = Guarded((wl.B, wl.H, wl.d_c), torch.float32, float("nan"), OUT_SENTINEL)
    plan.dense(d.q_c, d.q_r, d.c_kv, d.k_r, wl.L, out.t)
    torch.cuda.synchronize()
    out.check()
    return out.t.cpu().numpy().astype(np.float64)


def oracle_lca(x: workloads.Inputs, g: int, w: int, rows=None, heads=None):
    qc, qr = x.q_c, x.q_r
    if heads is not None:
        qc, qr = qc[:, heads], qr[:, heads]
    return orc.lca(qc, qr, x.c_kv, x.k_r, g=g, w=w, rows=rows)


def oracle_dense(x: workloads.Inputs, rows=None, heads=None):
    qc, qr = x.q_c, x.q_r
    if heads is not None:
        qc, qr = qc[:, heads], qr[:, heads]
    return orc.mla(qc, qr, x.c_kv, x.k_r, rows=rows)


def rel_err(got: np.ndarray, ref: np.ndarray) -> float:
    """max over (b, h) of ||got - ref||_inf / ||ref||_inf."""
    g = got.reshape(-1, got.shape[-1]); r = ref.reshape(-1, ref.shape[-1])
    return float((np.abs(g - r).max(1) / np.maximum(np.abs(r).max(1), 1e-30)).max())


def group_scores(x: workloads.Inputs, b: np.ndarray, h: np.ndarray, j: np.ndarray, g: int) -> np.ndarray:
    """Full MLA scores s_t = q_c.c_t + q_r.k_t (float64) of the g tokens of group j
    of sequence b, head h, for arrays of (b, h, j); returns [n, g]."""
    def wide(a):
        return bf16_bits_to_f32(a).astype(np.float64) if a.dtype == np.uint16 else a.astype(np.float64)
    t = j[:, None] * g + np.arange(g)[None, :]                     # [n, g] token positions
    qc = wide(x.q_c[b, h])                                          # [n, d_c]
    qr = wide(x.q_r[b, h])
    c = wide(x.c_kv[b[:, None], t])                                 # [n, g, d_c]
    k = wide(x.k_r[b[:, None], t])
    return np.einsum("ngd,nd->ng", c, qc) + np.einsum("ngd,nd->ng", k, qr)


def check_anchor_validity(got_anc, ref, x: workloads.Inputs, g: int, heads=None, mask=None) -> int:
    """Every anchor selected by `mask` lies in its own group and its double
    score is within the near-tie gate (ANCHOR_GAP * max|s|) of the group's
    maximum: where several tokens are that close to the maximum, fp32
    accumulation of bf16 products may legitimately pick any of them.
    Returns the number of anchors checked."""
    nG = got_anc.shape[-1]
    lo = (np.arange(nG) * g)[None, None, :]
    assert np.all((got_anc >= lo) & (got_anc < lo + g)), "anchor outside its group"
    idx = np.argwhere(mask if mask is not None else np.ones(got_anc.shape, bool))
    if idx.size == 0:
        return 0
    rows = np.asarray(ref.rows)[idx[:, 0]]
    hs = idx[:, 1] if heads is None else np.asarray(heads)[idx[:, 1]]
    s = group_scores(x, rows, hs, idx[:, 2], g)
    a = got_anc[idx[:, 0], idx[:, 1], idx[:, 2]] - idx[:, 2] * g
    gate = ANCHOR_GAP * ref.max_abs_s[idx[:, 0], idx[:, 1]]
    chosen = s[np.arange(len(a)), a]
    bad = chosen < s.max(axis=1) - gate
    assert not bad.any(), f"{int(bad.sum())} anchors score more than the gate below their group max"
    return len(a)


def compare(got_out, got_anc, ref, tol: float, exact_anchors: bool, x=None, g=None, heads=None):
    """Check outputs and anchors; returns (rel_err, gated anchor agreement, gated count).

    Gated bf16 anchors (top-2 gap > ANCHOR_GAP * max|s|) must equal the
    oracle's.  With the inputs `x` and group size `g`, every other anchor must
    lie in its group with a score within the gate of the group maximum."""
    assert np.all(np.isfinite(got_out))
    err = rel_err(got_out, ref.out)
    assert err <= tol, f"max relative error {err:.3e} > {tol:.1e}"
    if ref.anchor.size == 0:
        return err, 1.0, 0
    assert got_anc.shape == ref.anchor.shape
    assert np.all((got_anc >= 0)), "anchor not written"
    if exact_anchors:
        thr = 1e-6 * ref.max_abs_s[..., None]
        assert np.all(ref.tie_gap > thr), "near-tie in an exact-anchor case"
        assert np.array_equal(got_anc, ref.anchor)
        return err, 1.0, ref.anchor.size
    gate = ref.tie_gap > ANCHOR_GAP * ref.max_abs_s[..., None]
    agree = got_anc[gate] == ref.anchor[gate]
    assert agree.all(), f"{(~agree).sum()} gated anchors differ"
    if x is not None:
        check_anchor_validity(got_anc, ref, x, g, heads=heads, mask=~gate)
    return err, float(agree.mean()) if agree.size else 1.0, int(gate.sum())
