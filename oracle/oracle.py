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
