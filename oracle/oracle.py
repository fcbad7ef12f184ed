"""Python face of the double-precision CPU oracle (``lca_oracle.c``).

TEST INFRASTRUCTURE ONLY: the test suite, the package's smoke entry point and
the benchmark's CPU-baseline leg are the only callers.  Nothing here imports
the CUDA package, and the CUDA package never imports this module.

Inputs are the stored arrays themselves (float32, or bfloat16 carried as
uint16 bit patterns); the C code widens every element exactly to double.
What the oracle computes, and the readings of the page it rests on, are
described at the top of ``lca_oracle.c`` ("Latent-Condensed Transformer for
Efficient Long Context Modeling", section 2, "O Algoritmo LCA").
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import time
from dataclasses import dataclass

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(_HERE, "lca_oracle.c")
LIB = os.path.join(_HERE, "liblca_oracle.so")

F32, BF16 = 0, 1


def build(src: str = SRC, out: str = LIB, extra_cflags: tuple[str, ...] = ()) -> str:
    """Compile the oracle with gcc (-O2, OpenMP, IEEE double: no fast-math)."""
    if (os.path.exists(out) and src == SRC and not extra_cflags
            and os.path.getmtime(out) >= os.path.getmtime(src)):
        return out
    cmd = ["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared", *extra_cflags,
           "-o", out, src, "-lm"]
    subprocess.run(cmd, check=True)
    return out


def _load(path: str) -> ctypes.CDLL:
    lib = ctypes.CDLL(path)
    vp, i32, i64, dp = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_void_p
    lib.lca_oracle_seq.argtypes = [i32, i32, i32, i64, i32, i32, i32, vp, vp, vp, vp, i32,
                                   dp, vp, dp, dp, i32]
    lib.lca_oracle_seq.restype = i32
    lib.mla_oracle_seq.argtypes = [i32, i32, i32, i64, i32, vp, vp, vp, vp, dp, i32]
    lib.mla_oracle_seq.restype = i32
    lib.lca_oracle_num_groups.argtypes = [i64, i32, i32]
    lib.lca_oracle_num_groups.restype = i64
    lib.lca_oracle_condense_shared.argtypes = [i32, i32, i32, i64, i32, i64, i64, i32, vp, vp, vp,
                                               vp, dp, dp, vp, dp, dp]
    lib.lca_oracle_condense_shared.restype = i32
    lib.lca_oracle_decode_stored.argtypes = [i32, i32, i32, i64, i64, i32, vp, vp, dp, dp, vp, vp,
                                             ctypes.c_double, dp]
    lib.lca_oracle_decode_stored.restype = i32
    lib.lca_oracle_partial.argtypes = [i32, i32, i64, i32, i32, i64, i64, i32, vp, vp, vp, vp, dp, dp,
                                       dp, vp]
    lib.lca_oracle_partial.restype = i32
    lib.lca_oracle_merge.argtypes = [i32, i32, dp, dp, dp, dp]
    lib.lca_oracle_merge.restype = None
    return lib


_LIBS: dict[str, ctypes.CDLL] = {}


def load(path: str | None = None) -> ctypes.CDLL:
    path = path or build()
    if path not in _LIBS:
        _LIBS[path] = _load(path)
    return _LIBS[path]


def _dtype_code(a: np.ndarray) -> int:
    if a.dtype == np.float32:
        return F32
    if a.dtype == np.uint16:
        return BF16
    raise TypeError(f"oracle inputs are float32 or bf16-as-uint16, got {a.dtype}")


def _ptr(a: np.ndarray | None) -> int | None:
    return None if a is None else a.ctypes.data


@dataclass
class OracleResult:
    out: np.ndarray          # [nb, H, d_c] float64
    anchor: np.ndarray       # [nb, H, n_G] int32
    tie_gap: np.ndarray      # [nb, H, n_G] float64: top-2 score gap per group
    max_abs_s: np.ndarray    # [nb, H] float64
    rows: list[int]          # which sequences b were computed
    seconds: float           # wall time of the oracle calls
    threads: int


def num_groups(L: int, g: int, w: int, lib: ctypes.CDLL | None = None) -> int:
    return int((lib or load()).lca_oracle_num_groups(L, g, w))


def lca(q_c, q_r, c_kv, k_r, g: int, w: int, rows=None, formulation: int = 0,
        nthreads: int = 0, lib: ctypes.CDLL | None = None) -> OracleResult:
    """LCA decode for the sequences in ``rows`` (default: all).

    q_c [B,H,d_c], q_r [B,H,d_r], c_kv [B,L,d_c], k_r [B,L,d_r]; all float32 or
    all bf16-as-uint16.  formulation 0 = materialised condensed cache (the
    returned definition), 1 = folded form (cross-check).
    """
    lib = lib or load()
    B, H, d_c = q_c.shape
    d_r = q_r.shape[2]
    L = c_kv.shape[1]
    dt = _dtype_code(q_c)
    for a in (q_r, c_kv, k_r):
        assert _dtype_code(a) == dt
    rows = list(range(B)) if rows is None else list(rows)
    nG = num_groups(L, g, w, lib)
    out = np.zeros((len(rows), H, d_c), np.float64)
    anc = np.zeros((len(rows), H, max(nG, 0)), np.int32)
    gap = np.zeros((len(rows), H, max(nG, 0)), np.float64)
    mx = np.zeros((len(rows), H), np.float64)
    t0 = time.perf_counter()
    for i, b in enumerate(rows):
        qc = np.ascontiguousarray(q_c[b]); qr = np.ascontiguousarray(q_r[b])
        ck = np.ascontiguousarray(c_kv[b]); kr = np.ascontiguousarray(k_r[b])
        o = np.zeros((H, d_c), np.float64)
        an = np.zeros((H, max(nG, 1)), np.int32)
        gp = np.zeros((H, max(nG, 1)), np.float64)
        m = np.zeros((H,), np.float64)
        st = lib.lca_oracle_seq(H, d_c, d_r, L, g, w, dt, _ptr(qc), _ptr(qr), _ptr(ck), _ptr(kr),
                                formulation, _ptr(o), _ptr(an), _ptr(gp), _ptr(m), nthreads)
        if st != 0:
            raise RuntimeError(f"lca_oracle_seq failed with status {st}")
        out[i] = o
        anc[i] = an[:, :nG]
        gap[i] = gp[:, :nG]
        mx[i] = m
    secs = time.perf_counter() - t0
    return OracleResult(out, anc, gap, mx, rows, secs, nthreads or (os.cpu_count() or 1))


def mla(q_c, q_r, c_kv, k_r, rows=None, nthreads: int = 0,
        lib: ctypes.CDLL | None = None) -> np.ndarray:
    """Dense MLA decode (softmax over all L tokens) for the sequences in ``rows``."""
    lib = lib or load()
    B, H, d_c = q_c.shape
    d_r = q_r.shape[2]
    L = c_kv.shape[1]
    dt = _dtype_code(q_c)
    rows = list(range(B)) if rows is None else list(rows)
    out = np.zeros((len(rows), H, d_c), np.float64)
    for i, b in enumerate(rows):
        qc = np.ascontiguousarray(q_c[b]); qr = np.ascontiguousarray(q_r[b])
        ck = np.ascontiguousarray(c_kv[b]); kr = np.ascontiguousarray(k_r[b])
        o = np.zeros((H, d_c), np.float64)
        st = lib.mla_oracle_seq(H, d_c, d_r, L, dt, _ptr(qc), _ptr(qr), _ptr(ck), _ptr(kr),
                                _ptr(o), nthreads)
        if st != 0:
            raise RuntimeError(f"mla_oracle_seq failed with status {st}")
        out[i] = o
    return out


@dataclass
class StoredResult:
    """The stored, head-shared condensed cache of one batch and its decode."""
    cbar: np.ndarray         # [nb, n_G, d_c] float64: pooled latents
    kanc: np.ndarray         # [nb, n_G, d_r] float64: the anchors' RoPE keys
    anchor: np.ndarray       # [nb, n_G] int32 absolute positions
    tie_gap: np.ndarray      # [nb, n_G] float64: top-2 gap of the head-mean score
    max_abs_s: np.ndarray    # [nb] float64: max |head-mean score| over condensed tokens
    out: np.ndarray | None   # [nb, H, d_c] float64: decode over [stored || window]
    rows: list[int]


def condense_shared(q_c, q_r, c_kv, k_r, g: int, j0: int, n: int, rows=None,
                    lib: ctypes.CDLL | None = None):
    """Condense groups j0 .. j0+n-1 of every sequence in ``rows`` with the
    head-mean score of q (one entry per group, shared by all heads).
    Returns (cbar [nb,n,d_c], kanc [nb,n,d_r], anchor [nb,n], tie_gap [nb,n], max_abs [nb])."""
    lib = lib or load()
    B, H, d_c = q_c.shape
    d_r = q_r.shape[2]
    L = c_kv.shape[1]
    dt = _dtype_code(q_c)
    rows = list(range(B)) if rows is None else list(rows)
    cb = np.zeros((len(rows), n, d_c), np.float64)
    ka = np.zeros((len(rows), n, d_r), np.float64)
    an = np.zeros((len(rows), max(n, 1)), np.int32)
    gp = np.zeros((len(rows), max(n, 1)), np.float64)
    mx = np.zeros((len(rows),), np.float64)
    for i, b in enumerate(rows):
        qc = np.ascontiguousarray(q_c[b]); qr = np.ascontiguousarray(q_r[b])
        ck = np.ascontiguousarray(c_kv[b]); kr = np.ascontiguousarray(k_r[b])
        c1 = np.zeros((max(n, 1), d_c)); k1 = np.zeros((max(n, 1), max(d_r, 1)))
        a1 = np.zeros((max(n, 1),), np.int32); g1 = np.zeros((max(n, 1),)); m1 = np.zeros((1,))
        st = lib.lca_oracle_condense_shared(H, d_c, d_r, L, g, j0, n, dt, _ptr(qc), _ptr(qr), _ptr(ck),
                                            _ptr(kr), _ptr(c1), _ptr(k1), _ptr(a1), _ptr(g1), _ptr(m1))
        if st != 0:
            raise RuntimeError(f"lca_oracle_condense_shared failed with status {st}")
        cb[i] = c1[:n]; ka[i] = k1[:n, :d_r]; an[i] = a1; gp[i] = g1; mx[i] = m1[0]
    return cb, ka, an[:, :n], gp[:, :n], mx


def decode_stored(q_c, q_r, cbar, kanc, c_win, k_win, bias: float = 0.0, rows=None,
                  lib: ctypes.CDLL | None = None) -> np.ndarray:
    """Softmax attention of q over [stored condensed entries || window tokens].
    q_c [B,H,d_c], q_r [B,H,d_r] stored values; cbar [nb,n,d_c], kanc [nb,n,d_r]
    float64 (one row per sequence in ``rows``); c_win [B,n_win,d_c], k_win
    [B,n_win,d_r] stored values; ``bias`` added to condensed logits."""
    lib = lib or load()
    B, H, d_c = q_c.shape
    d_r = q_r.shape[2]
    dt = _dtype_code(q_c)
    rows = list(range(B)) if rows is None else list(rows)
    n = cbar.shape[1]
    n_win = c_win.shape[1]
    out = np.zeros((len(rows), H, d_c), np.float64)
    for i, b in enumerate(rows):
        qc = np.ascontiguousarray(q_c[b]); qr = np.ascontiguousarray(q_r[b])
        cb = np.ascontiguousarray(cbar[i], dtype=np.float64)
        ka = np.ascontiguousarray(kanc[i], dtype=np.float64)
        cw = np.ascontiguousarray(c_win[b]); kw = np.ascontiguousarray(k_win[b])
        o = np.zeros((H, d_c), np.float64)
        st = lib.lca_oracle_decode_stored(H, d_c, d_r, n, n_win, dt, _ptr(qc), _ptr(qr),
                                          _ptr(cb) if n else None, _ptr(ka) if n else None,
                                          _ptr(cw) if n_win else None, _ptr(kw) if n_win else None,
                                          float(bias), _ptr(o))
        if st != 0:
            raise RuntimeError(f"lca_oracle_decode_stored failed with status {st}")
        out[i] = o
    return out


def lca_stored(q_cond, q_r_cond, c_kv, k_r, g: int, w: int, q_c=None, q_r=None, bias: float = 0.0,
               rows=None, lib: ctypes.CDLL | None = None) -> StoredResult:
    """The whole stored-cache path for one batch: condense every group (n_G of
    them, the section-2 segmentation) with the query (q_cond, q_r_cond), then
    decode the query (q_c, q_r) -- by default the same one -- over [stored ||
    window], the window being tokens [n_G g, L)."""
    lib = lib or load()
    L = c_kv.shape[1]
    nG = num_groups(L, g, w, lib)
    rows = list(range(q_cond.shape[0])) if rows is None else list(rows)
    cb, ka, an, gp, mx = condense_shared(q_cond, q_r_cond, c_kv, k_r, g, 0, nG, rows, lib)
    q_c = q_cond if q_c is None else q_c
    q_r = q_r_cond if q_r is None else q_r
    out = decode_stored(q_c, q_r, cb, ka, c_kv[:, nG * g:], k_r[:, nG * g:], bias, rows, lib)
    return StoredResult(cb, ka, an, gp, mx, out, rows)


def slice_groups(L: int, g: int, w: int, pos0: int, n_tok: int, lib: ctypes.CDLL | None = None) -> int:
    """Condensed groups that lie inside tokens [pos0, pos0 + n_tok)."""
    nG = num_groups(L, g, w, lib)
    win0 = nG * g
    lo = pos0 // g if pos0 < win0 else nG
    hi = (pos0 + n_tok) // g if pos0 + n_tok < win0 else nG
    return max(0, hi - lo)


def partial(q_c, q_r, c_kv, k_r, g: int, w: int, pos0: int, n_tok: int, rows=None,
            lib: ctypes.CDLL | None = None):
    """Partial softmax sums (M, Z, O) of the entries held by tokens [pos0,
    pos0 + n_tok) of the whole context c_kv [B,L,d_c]; returns (m [nb,H],
    z [nb,H], o [nb,H,d_c], anchor [nb,H,n_slice_groups])."""
    lib = lib or load()
    B, H, d_c = q_c.shape
    d_r = q_r.shape[2]
    L = c_kv.shape[1]
    dt = _dtype_code(q_c)
    rows = list(range(B)) if rows is None else list(rows)
    ng = slice_groups(L, g, w, pos0, n_tok, lib)
    m = np.zeros((len(rows), H)); z = np.zeros((len(rows), H)); o = np.zeros((len(rows), H, d_c))
    an = np.zeros((len(rows), H, max(ng, 1)), np.int32)
    esz = 4 if dt == F32 else 2
    for i, b in enumerate(rows):
        ck = np.ascontiguousarray(c_kv[b]); kr = np.ascontiguousarray(k_r[b])
        for h in range(H):
            qc = np.ascontiguousarray(q_c[b, h]); qr = np.ascontiguousarray(q_r[b, h])
            mm = np.zeros(1); zz = np.zeros(1); oo = np.zeros(d_c); aa = np.zeros(max(ng, 1), np.int32)
            st = lib.lca_oracle_partial(d_c, d_r, L, g, w, pos0, n_tok, dt, _ptr(qc), _ptr(qr), _ptr(ck),
                                        _ptr(kr), _ptr(mm), _ptr(zz), _ptr(oo), _ptr(aa))
            if st != 0:
                raise RuntimeError(f"lca_oracle_partial failed with status {st} (slice cuts a group?)")
            m[i, h], z[i, h], o[i, h], an[i, h] = mm[0], zz[0], oo, aa
    del esz
    return m, z, o, an[:, :, :ng]


def merge(ms, zs, os_, lib: ctypes.CDLL | None = None) -> np.ndarray:
    """Merge stacked partials ms [n,nb,H], zs [n,nb,H], os_ [n,nb,H,d_c] -> out [nb,H,d_c]."""
    lib = lib or load()
    ms, zs, os_ = (np.asarray(a, np.float64) for a in (ms, zs, os_))
    n, nb, H, d_c = os_.shape
    out = np.zeros((nb, H, d_c))
    for b in range(nb):
        for h in range(H):
            m = np.ascontiguousarray(ms[:, b, h]); z = np.ascontiguousarray(zs[:, b, h])
            o = np.ascontiguousarray(os_[:, b, h]); r = np.zeros(d_c)
            lib.lca_oracle_merge(n, d_c, _ptr(m), _ptr(z), _ptr(o), _ptr(r))
            out[b, h] = r
    return out


@dataclass
class PagedResult:
    out: np.ndarray            # [B, H, d_c] float64
    anchor: list               # per sequence b: [H, n_G(b)] int32
    tie_gap: list              # per sequence b: [H, n_G(b)] float64
    max_abs_s: np.ndarray      # [B, H] float64


def paged_rows(block_table, b: int, L: int, page_size: int) -> np.ndarray:
    """Pool rows of tokens 0 .. L-1 of sequence b: token t sits in page
    block_table[b, t // page_size], at offset t % page_size in it."""
    t = np.arange(L, dtype=np.int64)
    return block_table[b, t // page_size].astype(np.int64) * page_size + t % page_size


def lca_paged(q_c, q_r, c_pool, k_pool, block_table, seq_lens, page_size: int, g: int, w: int,
              nthreads: int = 0, lib: ctypes.CDLL | None = None) -> PagedResult:
    """LCA decode over a paged cache with a length per sequence.

    q_c [B,H,d_c], q_r [B,H,d_r]; c_pool [P*page_size, d_c], k_pool
    [P*page_size, d_r]; block_table [B, max_pages] int; seq_lens [B].  Sequence
    b is the contiguous context of its seq_lens[b] tokens gathered through its
    block-table row (paged_rows), decoded exactly as ``lca`` decodes a
    contiguous cache of that length: its own segmentation (n_G(b) groups,
    section 2 step 1) and its own window.  No pool row outside those tokens
    is read.
    """
    lib = lib or load()
    B, H, d_c = q_c.shape
    out = np.zeros((B, H, d_c), np.float64)
    mx = np.zeros((B, H), np.float64)
    anchors, gaps = [], []
    for b in range(B):
        L = int(seq_lens[b])
        rows = paged_rows(block_table, b, L, page_size)
        r = lca(q_c[b:b + 1], q_r[b:b + 1], c_pool[rows][None], k_pool[rows][None], g, w,
                nthreads=nthreads, lib=lib)
        out[b] = r.out[0]
        mx[b] = r.max_abs_s[0]
        anchors.append(r.anchor[0])
        gaps.append(r.tie_gap[0])
    return PagedResult(out, anchors, gaps, mx)


def lca_prefill(q_c, q_r, c_pool, k_pool, table_row, pos0: int, page_size: int, g: int, w: int,
                nthreads: int = 0, lib: ctypes.CDLL | None = None) -> PagedResult:
    """LCA prefill of a chunk of n queries of one sequence: query i sits at
    position pos0 + i and attends causally to tokens [0, pos0 + i], which it
    condenses itself (its own n_G = floor((pos0 + i + 1 - w) / g) groups and
    its own window).  The sequence's tokens are paged through the one block-
    table row ``table_row``.  Each query is the decode of its own causal prefix,
    so this is ``lca_paged`` with the row shared by every query and lengths
    pos0 + 1 .. pos0 + n."""
    n = q_c.shape[0]
    table = np.repeat(np.asarray(table_row, np.int32)[None, :], n, axis=0)
    lens = np.arange(pos0 + 1, pos0 + n + 1, dtype=np.int32)
    return lca_paged(q_c, q_r, c_pool, k_pool, table, lens, page_size, g, w, nthreads=nthreads, lib=lib)


def _wide(a: np.ndarray) -> np.ndarray:
    """Stored elements widened exactly to float64 (bf16 carried as uint16 bits)."""
    if a.dtype == np.uint16:
        return (np.ascontiguousarray(a).astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)
    return a.astype(np.float64)


def lca_gqa(q, k_cache, v_cache, g: int, w: int, rows=None, lib: ctypes.CDLL | None = None) -> OracleResult:
    """LCA decode for grouped-query attention (GQA), one query token per sequence.

    q [B,H,d_k]; k_cache [B,L,H_kv,d_k] (keys with RoPE applied); v_cache
    [B,L,H_kv,d_v]; query head h reads KV head h // (H / H_kv).

    The LCA page's dual path ("Latent-Condensed Transformer for Efficient Long
    Context Modeling", section 2, "Condensacao Dual-Path"; section 3, item 3
    extends it to GQA) pools the semantic component with the query-aware group
    softmax and keeps the positional (RoPE) component of the top-scoring token.
    In a GQA cache the key carries the position and the value the content, so
    for each query head and each group G_j of the section-2 segmentation:
      scores   s_t = q . k_t
      weights  w_t = softmax over t in G_j of s_t
      anchor   a_j = the lowest index in G_j with the largest s_t
      entry    key k_{a_j}, value v_bar_j = sum_t w_t v_t, logit q . k_{a_j} = s_{a_j}
    and the window tokens stand for themselves; the output is the softmax
    attention over [condensed || window].  Plain float64 numpy, step by step.
    """
    B, H, d_k = q.shape
    L, H_kv = k_cache.shape[1], k_cache.shape[2]
    d_v = v_cache.shape[3]
    assert H % H_kv == 0 and k_cache.shape[3] == d_k and v_cache.shape[:3] == (B, L, H_kv)
    r = H // H_kv
    rows = list(range(B)) if rows is None else list(rows)
    nG = num_groups(L, g, w, lib)
    win0 = max(nG, 0) * g
    out = np.zeros((len(rows), H, d_v))
    anc = np.zeros((len(rows), H, max(nG, 0)), np.int32)
    gap = np.zeros((len(rows), H, max(nG, 0)))
    mx = np.zeros((len(rows), H))
    t0 = time.perf_counter()
    for i, b in enumerate(rows):
        for h in range(H):
            kv = h // r
            K = _wide(k_cache[b, :, kv])            # [L, d_k]
            V = _wide(v_cache[b, :, kv])            # [L, d_v]
            s = K @ _wide(q[b, h])                  # [L]
            mx[i, h] = np.abs(s).max()
            logits, values = [], []
            for j in range(nG):
                sg = s[j * g:(j + 1) * g]
                a = int(np.argmax(sg))               # first maximum: the lowest index
                e = np.exp(sg - sg[a])
                wt = e / e.sum()
                values.append(wt @ V[j * g:(j + 1) * g])
                logits.append(sg[a])
                anc[i, h, j] = j * g + a
                srt = np.sort(sg)
                gap[i, h, j] = srt[-1] - srt[-2] if g >= 2 else np.inf
            for t in range(win0, L):
                logits.append(s[t])
                values.append(V[t])
            lg = np.asarray(logits)
            p = np.exp(lg - lg.max())
            out[i, h] = (p / p.sum()) @ np.asarray(values)
    return OracleResult(out, anc, gap, mx, rows, time.perf_counter() - t0, 1)
