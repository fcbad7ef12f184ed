"""Pins for the CPU oracle: checks against things other than the oracle itself.

Each pin takes a loaded oracle library and raises AssertionError when the
oracle disagrees with what the page and the mathematics fix.  The sources of
truth used here are independent of ``oracle/lca_oracle.c``:

* torch float64 library routines (softmax, argmax, scaled_dot_product_attention,
  matmul) applied to the condensed set built as the page describes it
  ("Latent-Condensed Transformer for Efficient Long Context Modeling",
  section 2, "O Algoritmo LCA", steps 1-3);
* closed forms: zero query (uniform pooling, anchor = first token of each
  group), groups of identical tokens (LCA = dense attention over one
  representative per group, because no parameter or bias is added --
  section 2, "Vantagens Teoricas"), g = 1 and w >= L (nothing condensed, so
  LCA is dense MLA attention, section 1);
* invariances: permuting tokens inside a group, a constant RoPE key;
* constructed exact ties (lowest index wins);
* brute force over every (g, w) on tiny L.

The same pins are run against deliberately broken copies of the oracle
(tests/test_oracle_mutants.py) to show that each plausible mistake is caught.
"""
from __future__ import annotations

import math

import numpy as np
import torch
import torch.nn.functional as F

from oracle import oracle as orc
import workloads
from workloads import bf16_bits_to_f32, f32_to_bf16_bits

REL_TOL = 1e-10  # double vs double, different summation orders


# ----------------------------------------------------------------------------- helpers
def rand_inputs(rng, B, H, L, d_c, d_r, dtype="f32"):
    s_q = 1.0 / math.sqrt(d_c + d_r)
    q_c = (rng.standard_normal((B, H, d_c)) * s_q).astype(np.float32)
    q_r = (rng.standard_normal((B, H, d_r)) * s_q).astype(np.float32)
    c_kv = rng.standard_normal((B, L, d_c)).astype(np.float32)
    k_r = rng.standard_normal((B, L, d_r)).astype(np.float32)
    if dtype == "bf16":
        return tuple(f32_to_bf16_bits(a) for a in (q_c, q_r, c_kv, k_r))
    return q_c, q_r, c_kv, k_r


def widen(a: np.ndarray) -> np.ndarray:
    if a.dtype == np.uint16:
        return bf16_bits_to_f32(a).astype(np.float64)
    return a.astype(np.float64)


def partition(L: int, g: int, w: int):
    """Groups and window by walking the sequence: the last w tokens are the
    window; full groups of g are then taken from the front while they end
    before the window; any leftover tokens join the window."""
    win_start = max(0, L - w)
    groups, t = [], 0
    while t + g <= win_start:
        groups.append(list(range(t, t + g)))
        t += g
    window = list(range(t, L))
    return groups, window


def rel_err(a: np.ndarray, b: np.ndarray) -> float:
    """max over rows of ||a - b||_inf / ||b||_inf."""
    a = a.reshape(-1, a.shape[-1]); b = b.reshape(-1, b.shape[-1])
    num = np.abs(a - b).max(axis=1)
    den = np.maximum(np.abs(b).max(axis=1), 1e-300)
    return float((num / den).max())


def torch_attention(q: np.ndarray, keys: np.ndarray, vals: np.ndarray) -> np.ndarray:
    """Library softmax attention of one query per head over given rows, scale 1.
    q [H, d], keys [H, n, d] or [n, d], vals [H, n, d_v] or [n, d_v]."""
    H = q.shape[0]
    qt = torch.from_numpy(q)[None, :, None, :]
    kt = torch.from_numpy(keys)
    vt = torch.from_numpy(vals)
    if kt.dim() == 2:
        kt = kt[None].expand(H, -1, -1)
    if vt.dim() == 2:
        vt = vt[None].expand(H, -1, -1)
    o = F.scaled_dot_product_attention(qt, kt[None], vt[None], scale=1.0)
    return o[0, :, 0, :].numpy()


def torch_lca_seq(qc, qr, C, K, g, w, stats=False):
    """LCA for one sequence built from library routines, per the page's steps.
    Returns (out [H, d_c], anchor [H, n_G]); with stats=True also the top-2
    score gap of every group [H, n_G] (torch.topk; +inf for one-token groups)
    and max |s| over the sequence [H] -- the near-tie report the GPU tests use
    to decide which bf16 anchors must match."""
    H = qc.shape[0]
    groups, window = partition(C.shape[0], g, w)
    Ct, Kt = torch.from_numpy(C), torch.from_numpy(K)
    outs, ancs, gaps, amax = [], [], [], []
    for h in range(H):
        qch, qrh = torch.from_numpy(qc[h]), torch.from_numpy(qr[h])
        s = Ct @ qch + Kt @ qrh                     # full MLA score of every token
        amax.append(float(s.abs().max()))
        keys, vals, anc, gap = [], [], [], []
        for G in groups:
            idx = torch.tensor(G)
            wts = torch.softmax(s[idx], dim=0)         # step 2: query-aware pooling weights
            a = G[int(torch.argmax(s[idx]))]           # step 2: highest-scoring token (first max)
            if len(G) >= 2:
                top = torch.topk(s[idx], 2).values
                gap.append(float(top[0] - top[1]))
            else:
                gap.append(math.inf)
            cbar = wts @ Ct[idx]
            keys.append(torch.cat([cbar, Kt[a]]))
            vals.append(cbar)
            anc.append(a)
        for t in window:                                # high-fidelity local window
            keys.append(torch.cat([Ct[t], Kt[t]]))
            vals.append(Ct[t])
        keys_np = torch.stack(keys).numpy()
        vals_np = torch.stack(vals).numpy()
        q = np.concatenate([qc[h], qr[h]])[None]
        outs.append(torch_attention(q, keys_np, vals_np)[0])   # step 3
        ancs.append(anc)
        gaps.append(gap)
    out = np.stack(outs)
    ancs = np.array(ancs, dtype=np.int32).reshape(H, len(groups))
    if stats:
        return out, ancs, np.array(gaps, np.float64).reshape(H, len(groups)), np.array(amax)
    return out, ancs


def torch_dense_seq(qc, qr, C, K):
    q = np.concatenate([qc, qr], axis=1)
    return torch_attention(q, np.concatenate([C, K], axis=1), C)


# ----------------------------------------------------------------------------- pins
def pin_segmentation(lib):
    for g in (1, 2, 3, 4, 8, 16):
        for k in (0, 1, 3):
            for r in (0, 1, g - 1):
                L = g * k + r + 5
                for w in sorted({0, 1, max(g - 1, 0), L - 1, L, L + 5}):
                    groups, _ = partition(L, g, w)
                    assert orc.num_groups(L, g, w, lib) == len(groups), (L, g, w)


def pin_dense_vs_torch(lib):
    rng = np.random.default_rng(11)
    for dtype in ("f32", "bf16"):
        qc, qr, C, K = rand_inputs(rng, 2, 3, 37, 24, 8, dtype)
        got = orc.mla(qc, qr, C, K, lib=lib)
        for b in range(2):
            ref = torch_dense_seq(widen(qc[b]), widen(qr[b]), widen(C[b]), widen(K[b]))
            assert rel_err(got[b], ref) < REL_TOL


def pin_g1_dense(lib):
    rng = np.random.default_rng(12)
    for dtype in ("f32", "bf16"):
        qc, qr, C, K = rand_inputs(rng, 2, 3, 41, 24, 8, dtype)
        for w in (0, 5, 40):
            res = orc.lca(qc, qr, C, K, g=1, w=w, lib=lib)
            nG = orc.num_groups(41, 1, w, lib)
            for b in range(2):
                ref = torch_dense_seq(widen(qc[b]), widen(qr[b]), widen(C[b]), widen(K[b]))
                assert rel_err(res.out[b], ref) < REL_TOL
                # with g = 1 the anchor of group j is token j itself
                assert np.array_equal(res.anchor[b], np.tile(np.arange(nG, dtype=np.int32), (3, 1)))


def pin_window_dense(lib):
    rng = np.random.default_rng(13)
    qc, qr, C, K = rand_inputs(rng, 1, 2, 33, 16, 8)
    for g in (2, 4, 7):
        for w in (33, 34, 100):
            res = orc.lca(qc, qr, C, K, g=g, w=w, lib=lib)
            ref = torch_dense_seq(widen(qc[0]), widen(qr[0]), widen(C[0]), widen(K[0]))
            assert res.anchor.shape[-1] == 0
            assert rel_err(res.out[0], ref) < REL_TOL


def pin_zero_query(lib):
    rng = np.random.default_rng(14)
    _, _, C, K = rand_inputs(rng, 1, 2, 53, 16, 8)
    qc = np.zeros((1, 2, 16), np.float32); qr = np.zeros((1, 2, 8), np.float32)
    for g, w in ((4, 5), (5, 0), (8, 13), (3, 52), (1, 7)):
        res = orc.lca(qc, qr, C, K, g=g, w=w, lib=lib)
        groups, window = partition(53, g, w)
        Cd = widen(C[0])
        # all scores are 0: uniform pooling, every entry weighs the same
        total = sum(Cd[G].mean(axis=0) for G in groups) + Cd[window].sum(axis=0)
        ref = total / (len(groups) + len(window))
        for h in range(2):
            assert rel_err(res.out[0, h], ref) < REL_TOL
            assert list(res.anchor[0, h]) == [G[0] for G in groups]


def pin_constant_groups(lib):
    rng = np.random.default_rng(15)
    L, g, w, d_c, d_r, H = 30, 4, 6, 16, 8, 3
    groups, window = partition(L, g, w)
    qc, qr, C, K = rand_inputs(rng, 1, H, L, d_c, d_r)
    reps = []
    for G in groups:                       # every token of a group is the same token
        C[0, G] = C[0, G[0]]
        K[0, G] = K[0, G[0]]
        reps.append(G[0])
    res = orc.lca(qc, qr, C, K, g=g, w=w, lib=lib)
    keep = reps + window                   # one representative per group, then the window
    ref = torch_dense_seq(widen(qc[0]), widen(qr[0]), widen(C[0][keep]), widen(K[0][keep]))
    assert rel_err(res.out[0], ref) < REL_TOL
    for h in range(H):                     # exact ties inside every group: lowest index
        assert list(res.anchor[0, h]) == reps


def _check_near_tie_report(res, gap, amax, where):
    """The oracle's top-2 gaps and max |s| against torch (float64, another
    summation order: equal to ~1e-15 relative)."""
    tol = 1e-12 * max(float(amax.max()), 1.0)
    assert np.allclose(res.max_abs_s[0], amax, rtol=1e-12, atol=0.0), where
    finite = np.isfinite(gap)
    assert np.array_equal(np.isfinite(res.tie_gap[0]), finite), where
    assert np.all(np.abs(res.tie_gap[0][finite] - gap[finite]) <= tol), where


def pin_brute_force(lib):
    rng = np.random.default_rng(16)
    for dtype in ("f32", "bf16"):
        for L in (1, 2, 5, 9, 16):
            qc, qr, C, K = rand_inputs(rng, 1, 2, L, 8, 4, dtype)
            for g in range(1, L + 2):
                for w in range(0, L + 2):
                    res = orc.lca(qc, qr, C, K, g=g, w=w, lib=lib)
                    ref, anc, gap, amax = torch_lca_seq(widen(qc[0]), widen(qr[0]), widen(C[0]),
                                                        widen(K[0]), g, w, stats=True)
                    assert rel_err(res.out[0], ref) < REL_TOL, (dtype, L, g, w)
                    assert np.array_equal(res.anchor[0], anc), (dtype, L, g, w)
                    _check_near_tie_report(res, gap, amax, (dtype, L, g, w))


def pin_near_tie_report(lib):
    """The near-tie report on longer sequences and several heads, where the
    group maximum sits anywhere in the group and max |s| comes from a
    negative score about half of the time (scores are shifted per head so
    that both signs occur)."""
    rng = np.random.default_rng(22)
    for dtype in ("f32", "bf16"):
        for (L, g, w, shift) in ((96, 8, 5, -3.0), (130, 16, 0, 3.0), (64, 4, 9, -2.0)):
            qc, qr, C, K = rand_inputs(rng, 1, 4, L, 16, 8, dtype)
            # a constant RoPE key component shifts every score of a head by the
            # same amount (here negative or positive), which moves max |s|
            # between the largest and the most negative score
            if dtype == "f32":
                K[0, :, 0] = np.float32(shift / max(abs(float(qr[0, 0, 0])), 1e-3))
            res = orc.lca(qc, qr, C, K, g=g, w=w, lib=lib)
            _, anc, gap, amax = torch_lca_seq(widen(qc[0]), widen(qr[0]), widen(C[0]), widen(K[0]),
                                              g, w, stats=True)
            assert np.array_equal(res.anchor[0], anc), (dtype, L, g, w)
            _check_near_tie_report(res, gap, amax, (dtype, L, g, w))
            # the gap is measured from the anchor: never negative, and zero
            # only at an exact tie
            assert np.all(res.tie_gap[0] >= 0.0)


def pin_ties(lib):
    rng = np.random.default_rng(17)
    L, g, w, d_c, d_r = 40, 8, 8, 16, 8
    qc, qr, C, K = rand_inputs(rng, 1, 1, L, d_c, d_r)
    u = np.concatenate([widen(qc[0, 0]), widen(qr[0, 0])])
    u /= np.linalg.norm(u)
    row = (6.0 * u).astype(np.float32)         # scores far above the N(0,1) background
    planted = {0: (2, 5), 1: (8, 9), 2: (17, 23), 3: (24, 25, 31)}
    for j, ts in planted.items():
        for t in ts:
            C[0, t] = row[:d_c]; K[0, t] = row[d_c:]
    res = orc.lca(qc, qr, C, K, g=g, w=w, lib=lib)
    for j, ts in planted.items():
        assert res.anchor[0, 0, j] == min(ts)
        assert res.tie_gap[0, 0, j] == 0.0


def pin_formulations(lib):
    rng = np.random.default_rng(18)
    for dtype in ("f32", "bf16"):
        for (L, g, w) in ((64, 8, 8), (67, 4, 5), (50, 16, 0), (20, 32, 3)):
            qc, qr, C, K = rand_inputs(rng, 2, 3, L, 32, 8, dtype)
            a = orc.lca(qc, qr, C, K, g=g, w=w, formulation=0, lib=lib)
            b = orc.lca(qc, qr, C, K, g=g, w=w, formulation=1, lib=lib)
            assert rel_err(b.out, a.out) < 1e-12
            assert np.array_equal(a.anchor, b.anchor)


def pin_permutation(lib):
    rng = np.random.default_rng(19)
    L, g, w = 45, 5, 7
    qc, qr, C, K = rand_inputs(rng, 1, 2, L, 16, 8)
    groups, _ = partition(L, g, w)
    base = orc.lca(qc, qr, C, K, g=g, w=w, lib=lib)
    perm = np.arange(L)
    for G in groups:
        perm[G] = rng.permutation(G)
    C2, K2 = C[:, perm].copy(), K[:, perm].copy()   # new position t holds old token perm[t]
    res = orc.lca(qc, qr, C2, K2, g=g, w=w, lib=lib)
    assert rel_err(res.out, base.out) < REL_TOL
    inv = np.argsort(perm)                           # old token -> new position
    assert np.array_equal(res.anchor, inv[base.anchor])


def pin_constant_rope(lib):
    rng = np.random.default_rng(20)
    L, g, w = 48, 4, 6
    qc, qr, C, K = rand_inputs(rng, 1, 3, L, 16, 8)
    k0 = rng.standard_normal(8).astype(np.float32)
    Kc = np.broadcast_to(k0, K.shape).copy()
    Kz = np.zeros_like(K)
    a = orc.lca(qc, qr, C, Kc, g=g, w=w, lib=lib)
    b = orc.lca(qc, qr, C, Kz, g=g, w=w, lib=lib)
    # a constant positional key shifts every score by the same amount per head
    assert rel_err(a.out, b.out) < REL_TOL
    assert np.array_equal(a.anchor, b.anchor)


# ----------------------------------------------------------------------------- stored cache
def torch_stored_seq(qc_cond, qr_cond, C, K, g, w, qc=None, qr=None, bias=0.0):
    """The stored, head-shared condensed cache of one sequence built from
    library routines: head-mean score (torch.mean over heads), group softmax
    and argmax, pooled latent by matmul, then softmax attention with explicit
    logits (the bias added to the condensed entries).  Returns (out [H, d_c],
    anchor [n_G], cbar [n_G, d_c], gap [n_G], max |s_bar|)."""
    groups, window = partition(C.shape[0], g, w)
    Ct, Kt = torch.from_numpy(C), torch.from_numpy(K)
    qcc, qrc = torch.from_numpy(qc_cond), torch.from_numpy(qr_cond)
    s_heads = Ct @ qcc.T + Kt @ qrc.T                  # [L, H]
    sbar = s_heads.mean(dim=1)                         # the head-mean score
    keys, vals, anc, gaps, cbars, is_cond = [], [], [], [], [], []
    amax = 0.0
    for G in groups:
        idx = torch.tensor(G)
        sg = sbar[idx]
        amax = max(amax, float(sg.abs().max()))
        wts = torch.softmax(sg, dim=0)
        a = G[int(torch.argmax(sg))]
        gaps.append(float(torch.topk(sg, 2).values[0] - torch.topk(sg, 2).values[1]) if len(G) > 1
                    else math.inf)
        cbar = wts @ Ct[idx]
        keys.append(torch.cat([cbar, Kt[a]])); vals.append(cbar); anc.append(a); cbars.append(cbar)
        is_cond.append(True)
    for t in window:
        keys.append(torch.cat([Ct[t], Kt[t]])); vals.append(Ct[t]); is_cond.append(False)
    qc = qc_cond if qc is None else qc
    qr = qr_cond if qr is None else qr
    q = torch.from_numpy(np.concatenate([qc, qr], axis=1))          # [H, d]
    Kmat, Vmat = torch.stack(keys), torch.stack(vals)
    logits = q @ Kmat.T + bias * torch.tensor(is_cond, dtype=torch.float64)[None, :]
    out = torch.softmax(logits, dim=1) @ Vmat
    cb = torch.stack(cbars).numpy() if cbars else np.zeros((0, C.shape[1]))
    return out.numpy(), np.array(anc, np.int32), cb, np.array(gaps), amax


def pin_stored_brute_force(lib):
    rng = np.random.default_rng(30)
    for dtype in ("f32", "bf16"):
        for L in (1, 3, 8, 13):
            qc, qr, C, K = rand_inputs(rng, 1, 3, L, 8, 4, dtype)
            qc2, qr2, _, _ = rand_inputs(rng, 1, 3, L, 8, 4, dtype)
            for g in range(1, L + 2):
                for w in range(0, L + 2, 2):
                    for bias in (0.0, math.log(g)):
                        # condense with one query, decode with another
                        res = orc.lca_stored(qc, qr, C, K, g, w, q_c=qc2, q_r=qr2, bias=bias, lib=lib)
                        out, anc, cb, gap, amax = torch_stored_seq(
                            widen(qc[0]), widen(qr[0]), widen(C[0]), widen(K[0]), g, w,
                            widen(qc2[0]), widen(qr2[0]), bias)
                        where = (dtype, L, g, w, bias)
                        assert rel_err(res.out[0], out) < REL_TOL, where
                        assert np.array_equal(res.anchor[0], anc), where
                        if len(anc):
                            assert rel_err(res.cbar[0], cb) < REL_TOL, where
                            assert np.allclose(res.kanc[0], widen(K[0])[anc], rtol=0, atol=0), where
                            fin = np.isfinite(gap)
                            assert np.array_equal(np.isfinite(res.tie_gap[0]), fin), where
                            assert np.all(np.abs(res.tie_gap[0][fin] - gap[fin]) <= 1e-12 * max(amax, 1)), where
                            assert abs(res.max_abs_s[0] - amax) <= 1e-12 * max(amax, 1), where


def pin_stored_g1_dense(lib):
    """g = 1: every stored entry is a token itself, so decode over the stored
    cache is dense MLA attention (torch SDPA)."""
    rng = np.random.default_rng(31)
    qc, qr, C, K = rand_inputs(rng, 2, 3, 29, 16, 8, "bf16")
    for w in (0, 4, 29):
        res = orc.lca_stored(qc, qr, C, K, 1, w, lib=lib)
        for b in range(2):
            ref = torch_dense_seq(widen(qc[b]), widen(qr[b]), widen(C[b]), widen(K[b]))
            assert rel_err(res.out[b], ref) < REL_TOL
            assert list(res.anchor[b]) == list(range(res.anchor.shape[1]))


def pin_stored_single_head(lib):
    """H = 1 and the same query for condensing and decoding: the head mean is
    that head's score, so the stored path is the per-head LCA decode."""
    rng = np.random.default_rng(32)
    for (L, g, w) in ((70, 8, 9), (64, 16, 0), (33, 4, 40)):
        qc, qr, C, K = rand_inputs(rng, 2, 1, L, 16, 8)
        res = orc.lca_stored(qc, qr, C, K, g, w, lib=lib)
        ref = orc.lca(qc, qr, C, K, g=g, w=w, lib=lib)
        assert rel_err(res.out, ref.out) < REL_TOL
        assert np.array_equal(res.anchor, ref.anchor[:, 0])


def pin_stored_constant_groups(lib):
    """Groups of identical tokens: each stored entry is that token.  Without a
    bias the decode is dense attention over one representative per group;
    with bias log g each entry counts as its g tokens, which is exactly dense
    attention over all L tokens."""
    rng = np.random.default_rng(33)
    L, g, w, H = 34, 4, 5, 3
    groups, window = partition(L, g, w)
    qc, qr, C, K = rand_inputs(rng, 1, H, L, 16, 8)
    reps = []
    for G in groups:
        C[0, G] = C[0, G[0]]; K[0, G] = K[0, G[0]]; reps.append(G[0])
    res0 = orc.lca_stored(qc, qr, C, K, g, w, lib=lib)
    keep = reps + window
    ref0 = torch_dense_seq(widen(qc[0]), widen(qr[0]), widen(C[0][keep]), widen(K[0][keep]))
    assert rel_err(res0.out[0], ref0) < REL_TOL
    assert list(res0.anchor[0]) == reps
    res1 = orc.lca_stored(qc, qr, C, K, g, w, bias=math.log(g), lib=lib)
    ref1 = torch_dense_seq(widen(qc[0]), widen(qr[0]), widen(C[0]), widen(K[0]))
    assert rel_err(res1.out[0], ref1) < REL_TOL


def pin_stored_zero_query(lib):
    """A zero condensing query: uniform pooling (c_bar = the group mean) and
    the first token of each group as anchor."""
    rng = np.random.default_rng(34)
    _, _, C, K = rand_inputs(rng, 1, 2, 40, 16, 8)
    qz, qrz = np.zeros((1, 2, 16), np.float32), np.zeros((1, 2, 8), np.float32)
    cb, ka, an, gap, mx = orc.condense_shared(qz, qrz, C, K, 5, 1, 6, lib=lib)
    for jj in range(6):
        j = 1 + jj
        assert rel_err(cb[0, jj][None], widen(C[0, 5 * j:5 * j + 5]).mean(axis=0)[None]) < REL_TOL
        assert an[0, jj] == 5 * j
        assert np.array_equal(ka[0, jj], widen(K[0, 5 * j]))


# ----------------------------------------------------------------------------- paged cache
def _paged_inputs(rng, dtype, B, L, d_c=16, d_r=8, H=2):
    q_c, q_r, c_kv, k_r = rand_inputs(rng, B, H, L, d_c, d_r, dtype)
    wl = workloads.small("paged_pin", B=B, H=H, L=L, g=8, w=20, d_c=d_c, d_r=d_r, dtype=dtype)
    return workloads.Inputs(wl, q_c, q_r, c_kv, k_r)


def _check_paged_against_prefix(lib, x, cache, g, w):
    """Each sequence of the paged decode against the torch-built LCA of its own
    contiguous tokens [0, L_b) (and, exactly, against the oracle's contiguous
    decode of them)."""
    res = orc.lca_paged(x.q_c, x.q_r, cache.c_pool, cache.k_pool, cache.block_table, cache.seq_lens,
                        cache.page_size, g, w, lib=lib)
    assert np.all(np.isfinite(res.out)), "a NaN row outside the sequences was read"
    for b, L in enumerate(cache.seq_lens):
        L = int(L)
        C, K = x.c_kv[b:b + 1, :L], x.k_r[b:b + 1, :L]
        ref, anc = torch_lca_seq(widen(x.q_c[b]), widen(x.q_r[b]), widen(C[0]), widen(K[0]), g, w)
        assert rel_err(res.out[b], ref) < REL_TOL, (b, L)
        assert np.array_equal(res.anchor[b], anc), (b, L)
        whole = orc.lca(x.q_c[b:b + 1], x.q_r[b:b + 1], np.ascontiguousarray(C), np.ascontiguousarray(K),
                        g, w, lib=lib)
        assert np.array_equal(res.out[b], whole.out[0]) and np.array_equal(res.anchor[b], whole.anchor[0])


def pin_paged_vs_prefix(lib):
    """Paged, variable-length decode: sequence b gathered through its block
    table is its own context of L_b tokens (lengths of one token, one page,
    ragged, and longer than the window), for two page sizes and both element
    types; every unowned pool row holds NaN."""
    for dtype, ps, seed in (("f32", 64, 41), ("bf16", 64, 42), ("f32", 128, 43)):
        rng = np.random.default_rng(seed)
        x = _paged_inputs(rng, dtype, B=5, L=300)
        cache = workloads.paged_layout(x, [300, 1, 130, 64, 21], ps, seed=seed)
        _check_paged_against_prefix(lib, x, cache, 8, 20)


def pin_paged_shared_prefix(lib):
    """Two sequences sharing their first pages (a common prompt prefix): the
    second sees the shared tokens as its own first tokens."""
    rng = np.random.default_rng(44)
    x = _paged_inputs(rng, "f32", B=3, L=400)
    x.c_kv[1, :256] = x.c_kv[0, :256]
    x.k_r[1, :256] = x.k_r[0, :256]
    x.c_kv[2, :128] = x.c_kv[0, :128]
    x.k_r[2, :128] = x.k_r[0, :128]
    cache = workloads.paged_layout(x, [300, 400, 150], 64, seed=44, shared_prefix={1: (0, 4), 2: (0, 2)})
    assert np.array_equal(cache.block_table[1, :4], cache.block_table[0, :4])
    assert np.array_equal(cache.block_table[2, :2], cache.block_table[0, :2])
    _check_paged_against_prefix(lib, x, cache, 8, 20)


def pin_prefill_causal_prefixes(lib):
    """Prefill of a chunk of queries at positions pos0 .. pos0 + n - 1 of one
    paged sequence: query i equals the torch-built LCA of tokens [0, pos0 + i]
    with its own segmentation (groups complete and appear as the position
    grows), and tokens after a query's position never change its output."""
    rng = np.random.default_rng(45)
    for dtype, ps in (("f32", 64), ("bf16", 128)):
        n, pos0, g, w = 6, 57, 4, 10
        x = _paged_inputs(rng, dtype, B=1, L=pos0 + n)
        qc, qr, _, _ = rand_inputs(rng, n, 2, 1, 16, 8, dtype)
        cache = workloads.paged_layout(x, [pos0 + n], ps, seed=45)
        res = orc.lca_prefill(qc, qr, cache.c_pool, cache.k_pool, cache.block_table[0], pos0, ps, g, w, lib=lib)
        for i in range(n):
            L = pos0 + i + 1
            ref, anc = torch_lca_seq(widen(qc[i]), widen(qr[i]), widen(x.c_kv[0, :L]), widen(x.k_r[0, :L]), g, w)
            assert rel_err(res.out[i], ref) < REL_TOL, (dtype, i)
            assert np.array_equal(res.anchor[i], anc)
            assert res.anchor[i].shape[1] == max(0, (L - w) // g)
        # causality: overwrite the last token; every earlier query is unchanged
        pool2 = cache.c_pool.copy()
        last = pos0 + n - 1
        pool2[cache.block_table[0, last // ps] * ps + last % ps] = cache.c_pool[0]
        res2 = orc.lca_prefill(qc, qr, pool2, cache.k_pool, cache.block_table[0], pos0, ps, g, w, lib=lib)
        assert np.array_equal(res2.out[:n - 1], res.out[:n - 1])
        assert not np.array_equal(res2.out[n - 1], res.out[n - 1])


# ----------------------------------------------------------------------------- GQA
def _gqa_inputs(rng, B, H, H_kv, L, d_k, d_v, dtype="f32"):
    s = 1.0 / math.sqrt(d_k)
    q = (rng.standard_normal((B, H, d_k)) * s).astype(np.float32)
    k = rng.standard_normal((B, L, H_kv, d_k)).astype(np.float32)
    v = rng.standard_normal((B, L, H_kv, d_v)).astype(np.float32)
    if dtype == "bf16":
        return tuple(f32_to_bf16_bits(a) for a in (q, k, v))
    return q, k, v


def torch_gqa_seq(q, K, V, g, w):
    """GQA LCA for one (sequence, query head) from library routines: the
    condensed set (anchor key, softmax-pooled value) then torch SDPA."""
    groups, window = partition(K.shape[0], g, w)
    Kt, Vt, qt = torch.from_numpy(K), torch.from_numpy(V), torch.from_numpy(q)
    s = Kt @ qt
    keys, vals, anc = [], [], []
    for G in groups:
        idx = torch.tensor(G)
        a = G[int(torch.argmax(s[idx]))]
        vals.append(torch.softmax(s[idx], dim=0) @ Vt[idx])
        keys.append(Kt[a])
        anc.append(a)
    for t in window:
        keys.append(Kt[t])
        vals.append(Vt[t])
    o = torch_attention(q[None], torch.stack(keys).numpy(), torch.stack(vals).numpy())[0]
    return o, anc


def pin_gqa_brute_force(lib):
    """Every (g, w) on short sequences, both element types, 3 query heads per KV
    head: the oracle's GQA LCA against the torch-built condensed set."""
    rng = np.random.default_rng(51)
    for dtype in ("f32", "bf16"):
        q, k, v = _gqa_inputs(rng, 2, 6, 2, 13, 8, 6, dtype)
        for g in (1, 2, 3, 5):
            for w in (0, 1, 4, 13):
                res = orc.lca_gqa(q, k, v, g, w, lib=lib)
                for b in range(2):
                    for h in range(6):
                        o, anc = torch_gqa_seq(widen(q[b, h]), widen(k[b, :, h // 3]), widen(v[b, :, h // 3]), g, w)
                        assert rel_err(res.out[b, h], o) < REL_TOL, (dtype, g, w, b, h)
                        assert list(res.anchor[b, h]) == anc


def pin_gqa_is_mla_lca_with_zero_semantic_query(lib):
    """The reading restated in MLA terms: per KV head, GQA LCA is the MLA LCA
    of that head's query heads with q_c = 0, C_KV = V (pooled) and K_R = K
    (anchored) -- against the pinned MLA oracle."""
    rng = np.random.default_rng(52)
    q, k, v = _gqa_inputs(rng, 2, 8, 2, 300, 16, 12)
    res = orc.lca_gqa(q, k, v, 8, 40, lib=lib)
    for kv in range(2):
        hs = slice(4 * kv, 4 * kv + 4)
        ref = orc.lca(np.zeros((2, 4, 12), np.float32), np.ascontiguousarray(q[:, hs]),
                      np.ascontiguousarray(v[:, :, kv]), np.ascontiguousarray(k[:, :, kv]), 8, 40, lib=lib)
        assert rel_err(res.out[:, hs], ref.out) < REL_TOL
        assert np.array_equal(res.anchor[:, hs], ref.anchor)


def pin_gqa_dense_limits(lib):
    """g = 1 and w >= L: nothing is condensed, so GQA LCA is dense GQA softmax
    attention (torch SDPA over the head's K and V)."""
    rng = np.random.default_rng(53)
    q, k, v = _gqa_inputs(rng, 1, 4, 2, 50, 8, 8)
    for g, w in ((1, 0), (4, 50), (3, 64)):
        res = orc.lca_gqa(q, k, v, g, w, lib=lib)
        for h in range(4):
            o = torch_attention(widen(q[0, h])[None], widen(k[0, :, h // 2]), widen(v[0, :, h // 2]))[0]
            assert rel_err(res.out[0, h], o) < REL_TOL


def pin_gqa_kv_head_sharing(lib):
    """A query head reads only its own KV head: changing another KV head's
    cache leaves it unchanged, and two equal query heads of one KV head agree."""
    rng = np.random.default_rng(54)
    q, k, v = _gqa_inputs(rng, 1, 6, 3, 90, 8, 8)
    q[0, 1] = q[0, 0]
    res = orc.lca_gqa(q, k, v, 4, 10, lib=lib)
    assert np.array_equal(res.out[0, 0], res.out[0, 1])
    k2, v2 = k.copy(), v.copy()
    k2[:, :, 2] += 1.0
    v2[:, :, 2] *= -1.0
    res2 = orc.lca_gqa(q, k2, v2, 4, 10, lib=lib)
    assert np.array_equal(res2.out[0, :4], res.out[0, :4])
    assert not np.allclose(res2.out[0, 4:], res.out[0, 4:])


def pin_gqa_ties(lib):
    """Groups whose keys are identical: every score ties, so the anchor is the
    group's first token and the pooled value is the plain mean of its values."""
    rng = np.random.default_rng(55)
    q, k, v = _gqa_inputs(rng, 1, 2, 1, 40, 8, 8)
    g, w = 5, 10
    for j in range(6):
        k[0, j * g:(j + 1) * g] = k[0, j * g]
    res = orc.lca_gqa(q, k, v, g, w, lib=lib)
    assert np.array_equal(res.anchor[0], np.tile(np.arange(6) * g, (2, 1)))
    assert np.all(res.tie_gap[0] == 0)
    for h in range(2):
        keys = np.concatenate([widen(k[0, 0:30:g, 0]), widen(k[0, 30:, 0])])
        vals = np.concatenate([widen(v[0, :30, 0]).reshape(6, g, 8).mean(axis=1), widen(v[0, 30:, 0])])
        o = torch_attention(widen(q[0, h])[None], keys, vals)[0]
        assert rel_err(res.out[0, h], o) < REL_TOL


GQA_PINS = [pin_gqa_brute_force, pin_gqa_is_mla_lca_with_zero_semantic_query, pin_gqa_dense_limits,
            pin_gqa_kv_head_sharing, pin_gqa_ties]


STORED_PINS = [pin_stored_brute_force, pin_stored_g1_dense, pin_stored_single_head,
               pin_stored_constant_groups, pin_stored_zero_query]

ALL_PINS = [pin_segmentation, pin_dense_vs_torch, pin_g1_dense, pin_window_dense, pin_zero_query,
            pin_constant_groups, pin_brute_force, pin_near_tie_report, pin_ties, pin_formulations,
            pin_permutation, pin_constant_rope] + STORED_PINS + [pin_paged_vs_prefix,
                                                                  pin_paged_shared_prefix,
                                                                  pin_prefill_causal_prefixes] + GQA_PINS
