"""Seeded synthetic inputs for the LCA decode step.

This module is shared by the oracle-side tests and the GPU-side tests and
benchmark, and holds none of the method's arithmetic: it only draws random
numbers, scales them, rounds them to bfloat16 and plants needle rows.

Recipe (every tensor, every sequence b, is its own counter-seeded stream, so
any subset of sequences can be regenerated bit-identically on its own):

  rng(tensor, b) = numpy.random.default_rng([seed, TENSOR_ID[tensor], b])
  x = rng.standard_normal(shape_of_one_sequence, dtype=float32) * scale

  q_c, q_r : [H, d_c], [H, d_r]      scale = q_scale
  c_kv, k_r: [L, d_c], [L, d_r]      scale = kv_scale

then rounded to bfloat16 with round-to-nearest-even when the workload is
bf16 (the arrays are then carried as uint16 bit patterns).

The needle workload additionally plants, per sequence, 64 identical rows at
positions drawn without replacement from [0, L) (rng tensor "needle_pos",
sorted).  Their [C_KV ; K_R] row is 4 * sqrt(d_c + d_r) * u where u is the unit
vector along the mean over heads of that sequence's [q_c ; q_r] -- four times
the expected norm of an N(0,1) row, pointed along the query direction -- then
rounded to bfloat16.  Identical rows make exact score ties, so groups holding
two needles exercise the lowest-index anchor tie-break.

Shapes follow DeepSeek-V2(-Lite) multi-head latent attention (d_c=512 latent,
d_r=64 RoPE key); no model weights are involved.
"""
from __future__ import annotations

import math
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass, field, replace

import numpy as np

TENSOR_ID = {"q_c": 1, "q_r": 2, "c_kv": 3, "k_r": 4, "needle_pos": 5, "page_order": 6,
             "gqa_q": 7, "gqa_k": 8, "gqa_v": 9}
NEEDLES_PER_SEQ = 64


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    d_c: int
    d_r: int
    L: int
    g: int
    w: int
    dtype: str            # "f32" or "bf16"
    q_scale: float
    kv_scale: float
    needles: bool = False
    seed: int = 0
    sweep: tuple = field(default=())   # extra (g, w) points on the same inputs

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)

    @property
    def n_groups(self) -> int:
        return (self.L - self.w) // self.g if self.L > self.w else 0

    @property
    def elem_bytes(self) -> int:
        return 4 if self.dtype == "f32" else 2


def _v2_q_scale() -> float:
    return 1.0 / math.sqrt(576.0)


WORKLOADS: dict[str, Workload] = {
    # tiny fp32 parity case: everything N(0,1)/sqrt(d_c + d_r)
    "tiny_f32": Workload("tiny_f32", B=1, H=4, d_c=64, d_r=16, L=1024, g=8, w=64, dtype="f32",
                         q_scale=1.0 / math.sqrt(80.0), kv_scale=1.0 / math.sqrt(80.0)),
    # DeepSeek-V2-Lite-shaped decode (the headline throughput workload)
    "v2lite": Workload("v2lite", B=8, H=16, d_c=512, d_r=64, L=32768, g=16, w=1024,
                       dtype="bf16", q_scale=_v2_q_scale(), kv_scale=1.0),
    # DeepSeek-V2-shaped decode, 128 heads sharing one latent
    "v2": Workload("v2", B=32, H=128, d_c=512, d_r=64, L=65536, g=16, w=2048, dtype="bf16",
                   q_scale=_v2_q_scale(), kv_scale=1.0),
    # long-context needle decode
    "needle": Workload("needle", B=4, H=128, d_c=512, d_r=64, L=131072, g=32, w=4096,
                       dtype="bf16", q_scale=_v2_q_scale(), kv_scale=1.0, needles=True),
    # group/window sweep: one input set, ten (g, w) points
    "sweep": Workload("sweep", B=16, H=16, d_c=512, d_r=64, L=65536, g=16, w=512,
                      dtype="bf16", q_scale=_v2_q_scale(), kv_scale=1.0,
                      sweep=tuple((g, w) for g in (4, 8, 16, 32, 64) for w in (512, 4096))),
}


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 to bfloat16 (round to nearest, ties to even); uint16 bits."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    lsb = (u >> np.uint32(16)) & np.uint32(1)
    r = (u + np.uint32(0x7FFF) + lsb) >> np.uint32(16)
    return r.astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """Exact widening of bfloat16 bit patterns to float32."""
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def _rng(seed: int, tensor: str, b: int) -> np.random.Generator:
    return np.random.default_rng([seed, TENSOR_ID[tensor], b])


def _draw(wl: Workload, tensor: str, b: int, shape, scale: float) -> np.ndarray:
    x = _rng(wl.seed, tensor, b).standard_normal(shape, dtype=np.float32)
    if scale != 1.0:
        x *= np.float32(scale)
    return f32_to_bf16_bits(x) if wl.dtype == "bf16" else x


def needle_positions(wl: Workload, b: int) -> np.ndarray:
    n = min(NEEDLES_PER_SEQ, wl.L)
    return np.sort(_rng(wl.seed, "needle_pos", b).choice(wl.L, size=n, replace=False))


def _needle_row(wl: Workload, qc_b: np.ndarray, qr_b: np.ndarray) -> np.ndarray:
    """4 * sqrt(d) * unit(mean over heads of [q_c; q_r]) as stored values."""
    if wl.dtype == "bf16":
        qc = bf16_bits_to_f32(qc_b).astype(np.float64)
        qr = bf16_bits_to_f32(qr_b).astype(np.float64)
    else:
        qc, qr = qc_b.astype(np.float64), qr_b.astype(np.float64)
    u = np.concatenate([qc, qr], axis=1).mean(axis=0)
    u /= np.linalg.norm(u)
    row = (4.0 * math.sqrt(wl.d_c + wl.d_r) * u).astype(np.float32)
    return f32_to_bf16_bits(row) if wl.dtype == "bf16" else row


@dataclass
class Inputs:
    wl: Workload
    q_c: np.ndarray     # [B, H, d_c]
    q_r: np.ndarray     # [B, H, d_r]
    c_kv: np.ndarray    # [B, L, d_c]
    k_r: np.ndarray     # [B, L, d_r]
    needle_pos: list | None = None


def generate(wl: Workload, threads: int = 8) -> Inputs:
    """All B sequences of a workload, drawn per the module recipe."""
    np_dt = np.float32 if wl.dtype == "f32" else np.uint16
    q_c = np.empty((wl.B, wl.H, wl.d_c), np_dt)
    q_r = np.empty((wl.B, wl.H, wl.d_r), np_dt)
    c_kv = np.empty((wl.B, wl.L, wl.d_c), np_dt)
    k_r = np.empty((wl.B, wl.L, wl.d_r), np_dt)
    pos = [None] * wl.B

    def one(b: int) -> None:
        q_c[b] = _draw(wl, "q_c", b, (wl.H, wl.d_c), wl.q_scale)
        q_r[b] = _draw(wl, "q_r", b, (wl.H, wl.d_r), wl.q_scale)
        c_kv[b] = _draw(wl, "c_kv", b, (wl.L, wl.d_c), wl.kv_scale)
        k_r[b] = _draw(wl, "k_r", b, (wl.L, wl.d_r), wl.kv_scale)
        if wl.needles:
            p = needle_positions(wl, b)
            row = _needle_row(wl, q_c[b], q_r[b])
            c_kv[b][p] = row[: wl.d_c]
            k_r[b][p] = row[wl.d_c:]
            pos[b] = p

    with ThreadPoolExecutor(max_workers=max(1, threads)) as ex:
        list(ex.map(one, range(wl.B)))
    return Inputs(wl, q_c, q_r, c_kv, k_r, pos if wl.needles else None)


def small(name: str, B: int, H: int, L: int, g: int, w: int, d_c: int = 512, d_r: int = 64,
          dtype: str = "bf16", seed: int = 0, needles: bool = False) -> Workload:
    """A reduced-size workload with the same distributions as the named families."""
    if dtype == "f32":
        s = 1.0 / math.sqrt(d_c + d_r)
        return Workload(name, B, H, d_c, d_r, L, g, w, "f32", s, s, needles, seed)
    return Workload(name, B, H, d_c, d_r, L, g, w, "bf16", 1.0 / math.sqrt(d_c + d_r), 1.0,
                    needles, seed)


@dataclass
class PagedCache:
    """A batch's caches laid out in pages of a shared pool (input layout only)."""
    c_pool: np.ndarray        # [num_pages * page_size, d_c]
    k_pool: np.ndarray        # [num_pages * page_size, d_r]
    block_table: np.ndarray   # [B, max_pages] int32
    seq_lens: np.ndarray      # [B] int32
    page_size: int

    @property
    def num_pages(self) -> int:
        return self.c_pool.shape[0] // self.page_size


def nan_fill(dtype: str):
    """The value planted in pool rows that no sequence owns: a quiet NaN."""
    return np.uint16(0x7FC0) if dtype == "bf16" else np.float32(np.nan)


def paged_layout(x: Inputs, seq_lens, page_size: int, seed: int = 0, spare_pages: int = 3,
                 shared_prefix: dict | None = None, unused_entry: int = -1) -> PagedCache:
    """Scatter tokens [0, seq_lens[b]) of each sequence of ``x`` into pages of a
    pool, in a seeded random page order (rng tensor "page_order").

    Every pool row that holds none of those tokens -- the spare pages, and the
    rows past a sequence's last token in its last page -- holds NaN, so that a
    kernel that reads one shows it.  Block-table entries past a sequence's last
    page hold ``unused_entry`` (-1 by default: not a page).  ``shared_prefix``
    maps a sequence b to (a, n) with a < b: b's block table starts with a's
    first n pages (prefix sharing; both sequences must own them whole), and
    b's tokens over those pages must equal a's (the caller arranges the inputs
    so).
    """
    wl = x.wl
    seq_lens = np.asarray(seq_lens, np.int32)
    B = wl.B
    assert seq_lens.shape == (B,) and np.all(seq_lens >= 1) and np.all(seq_lens <= wl.L)
    need = [-(-int(n) // page_size) for n in seq_lens]
    shared_prefix = dict(shared_prefix or {})
    own = list(need)
    for b, (a, n) in shared_prefix.items():
        assert a < b and n * page_size <= min(int(seq_lens[a]), int(seq_lens[b]))
        own[b] -= n
    num_pages = sum(own) + spare_pages
    order = np.random.default_rng([seed, TENSOR_ID["page_order"], 0]).permutation(num_pages)
    max_pages = max(need)
    table = np.full((B, max_pages), unused_entry, np.int32)
    fill = nan_fill(wl.dtype)
    c_pool = np.full((num_pages * page_size, wl.d_c), fill, x.c_kv.dtype)
    k_pool = np.full((num_pages * page_size, wl.d_r), fill, x.k_r.dtype)
    nxt = 0
    for b in range(B):
        first = 0
        if b in shared_prefix:
            a, first = shared_prefix[b]
            table[b, :first] = table[a, :first]
        for j in range(first, need[b]):
            table[b, j] = order[nxt]
            nxt += 1
        L = int(seq_lens[b])
        for j in range(first, need[b]):
            t0, t1 = j * page_size, min(L, (j + 1) * page_size)
            r0 = int(table[b, j]) * page_size
            c_pool[r0:r0 + t1 - t0] = x.c_kv[b, t0:t1]
            k_pool[r0:r0 + t1 - t0] = x.k_r[b, t0:t1]
    return PagedCache(c_pool, k_pool, table, seq_lens, page_size)


@dataclass
class GqaInputs:
    q: np.ndarray       # [B, H, d_k]
    k: np.ndarray       # [B, L, H_kv, d_k]
    v: np.ndarray       # [B, L, H_kv, d_v]
    dtype: str


def generate_gqa(B: int, H: int, H_kv: int, d_k: int, d_v: int, L: int, dtype: str = "bf16",
                 seed: int = 0) -> GqaInputs:
    """A grouped-query-attention decode batch: per sequence b, q = N(0,1)/sqrt(d_k)
    [H, d_k], keys and values N(0,1) [L, H_kv, d] (rng tensors "gqa_q", "gqa_k",
    "gqa_v"), rounded to bfloat16 when dtype is bf16.  Shapes follow
    Distill-Qwen-7B-style GQA (28 query heads over 4 KV heads of 128)."""
    np_dt = np.float32 if dtype == "f32" else np.uint16
    q = np.empty((B, H, d_k), np_dt)
    k = np.empty((B, L, H_kv, d_k), np_dt)
    v = np.empty((B, L, H_kv, d_v), np_dt)
    for b in range(B):
        for name, arr, shape, scale in (("gqa_q", q, (H, d_k), 1.0 / math.sqrt(d_k)),
                                        ("gqa_k", k, (L, H_kv, d_k), 1.0), ("gqa_v", v, (L, H_kv, d_v), 1.0)):
            x = _rng(seed, name, b).standard_normal(shape, dtype=np.float32)
            if scale != 1.0:
                x *= np.float32(scale)
            arr[b] = f32_to_bf16_bits(x) if dtype == "bf16" else x
    return GqaInputs(q, k, v, dtype)
