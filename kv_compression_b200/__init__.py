"""LCA decode on B200: Python binding of liblca.so (include/lca.h).

Argument marshalling only: every step of the decode runs in the library's
CUDA kernels.  Tensors are torch CUDA tensors (PyTorch supplies device memory
and streams); there is no CPU fallback -- without the built library, or
without a CUDA device, every call raises.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "liblca.so")
CHECKED_LIB_PATH = os.path.join(HERE, "liblca_checked.so")

LCA_OK = 0
LCA_ERR_UNSUPPORTED = 2
LCA_ERR_DEVICE_TIMEOUT = 5
STATUS = {0: "LCA_OK", 1: "LCA_ERR_INVALID_ARG", 2: "LCA_ERR_UNSUPPORTED", 3: "LCA_ERR_ALIGNMENT",
          4: "LCA_ERR_CUDA", 5: "LCA_ERR_DEVICE_TIMEOUT", 6: "LCA_ERR_PLAN_MISMATCH",
          7: "LCA_ERR_NO_MEMORY", 8: "LCA_ERR_DEVICE_CHECK", 9: "LCA_ERR_DEVICE_INPUT"}
LCA_ERR_DEVICE_INPUT = 9
LCA_F32, LCA_BF16 = 0, 1
OPT_FORCE_SIMT, OPT_NUM_CTAS, OPT_WAIT_TIMEOUT_NS, OPT_DEBUG_SKIP_LOAD, OPT_KERNEL = 1, 2, 3, 4, 5
KERNEL_NAMES = {0: "none", 1: "simt", 2: "tcgen05", 3: "tcgen05_pair"}
KERNEL_CODES = {v: k for k, v in KERNEL_NAMES.items()}

EXPORTS = ["lca_plan_create", "lca_plan_destroy", "lca_plan_set", "lca_decode", "mla_decode",
           "lca_decode_host", "lca_num_groups", "lca_status_string", "lca_get_device_error",
           "lca_plan_kernel", "lca_plan_set_timing_event", "lca_decode_noalloc", "lca_condense",
           "lca_stored_rows", "lca_build_stored", "lca_decode_stored", "lca_slice_groups",
           "lca_decode_partial", "lca_merge_partials", "lca_get_device_error_site", "lca_decode_paged",
           "lca_prefill_paged", "lca_decode_gqa"]


class LcaError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {STATUS.get(status, status)}")


_lib: ctypes.CDLL | None = None


def load_library(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load liblca.so and declare its signatures.  Raises if it is missing."""
    global _lib
    if _lib is not None and path == LIB_PATH:
        return _lib
    if not os.path.exists(path):
        raise ImportError(f"liblca.so not built at {path}; run python -m kv_compression_b200.build")
    lib = ctypes.CDLL(path)
    vp, i32, i64 = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64
    lib.lca_plan_create.argtypes = [i32, i32, i32, i32, i32, i64, ctypes.POINTER(vp)]
    lib.lca_plan_destroy.argtypes = [vp]
    lib.lca_plan_set.argtypes = [vp, i32, i64]
    lib.lca_decode.argtypes = [vp, vp, vp, vp, vp, i64, i32, i32, vp, vp, vp]
    lib.mla_decode.argtypes = [vp, vp, vp, vp, vp, i64, vp, vp]
    lib.lca_decode_host.argtypes = [vp, vp, vp, vp, vp, i64, i32, i32, vp, vp, vp]
    lib.lca_num_groups.argtypes = [i64, i32, i32]
    lib.lca_num_groups.restype = i64
    lib.lca_status_string.argtypes = [i32]
    lib.lca_status_string.restype = ctypes.c_char_p
    lib.lca_get_device_error.argtypes = [vp, vp]
    lib.lca_plan_kernel.argtypes = [vp, i64, i32, i32]
    lib.lca_plan_set_timing_event.argtypes = [vp, vp]
    lib.lca_decode_noalloc.argtypes = [i32, i32, i32, i32, i32, vp, vp, vp, vp, i64, i32, i32, vp,
                                       vp, vp]
    lib.lca_condense.argtypes = [vp, vp, vp, vp, vp, i64, i32, i64, i64, vp, vp, i64, i64, vp, vp]
    lib.lca_stored_rows.argtypes = [i64, i32, i32]
    lib.lca_stored_rows.restype = i64
    lib.lca_build_stored.argtypes = [vp, vp, vp, vp, vp, i64, i32, i32, vp, vp, vp, vp]
    lib.lca_decode_stored.argtypes = [vp, vp, vp, vp, vp, i64, i64, ctypes.c_float, vp, vp]
    lib.lca_slice_groups.argtypes = [i64, i32, i32, i64, i64]
    lib.lca_slice_groups.restype = i64
    lib.lca_decode_partial.argtypes = [vp, vp, vp, vp, vp, i64, i64, i64, i32, i32, vp, vp, vp, vp]
    lib.lca_merge_partials.argtypes = [vp, i32, vp, vp, vp, vp]
    lib.lca_get_device_error_site.argtypes = [vp]
    lib.lca_get_device_error_site.restype = i32
    lib.lca_decode_paged.argtypes = [vp, vp, vp, vp, vp, i64, i32, vp, i64, vp, i32, i32, vp, vp, i64, vp]
    lib.lca_prefill_paged.argtypes = [vp, vp, vp, vp, vp, i64, i32, vp, i64, i64, i32, i32, vp, vp, i64, vp]
    lib.lca_decode_gqa.argtypes = [vp, vp, vp, vp, i64, i32, i32, i32, vp, vp, vp]
    for name in ("lca_plan_create", "lca_plan_destroy", "lca_plan_set", "lca_decode", "mla_decode",
                 "lca_decode_host", "lca_get_device_error", "lca_plan_kernel",
                 "lca_plan_set_timing_event", "lca_decode_noalloc", "lca_condense",
                 "lca_build_stored", "lca_decode_stored", "lca_decode_partial", "lca_merge_partials",
                 "lca_decode_paged", "lca_prefill_paged", "lca_decode_gqa"):
        getattr(lib, name).restype = i32
    if path == LIB_PATH:
        _lib = lib
    return lib


def num_groups(L: int, g: int, w: int) -> int:
    return int(load_library().lca_num_groups(L, g, w))


def _check(status: int, what: str) -> None:
    if status != LCA_OK:
        raise LcaError(status, what)


def _ptr(t) -> int | None:
    return None if t is None else t.data_ptr()


def _stream_handle(stream) -> int | None:
    import torch
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


@dataclass
class Plan:
    """A liblca plan (shapes, kernel choice, split workspace) on the current device."""
    B: int
    H: int
    d_c: int
    d_r: int
    dtype: str
    max_L: int
    lib_path: str | None = None    # another build of the library (the range-checked one)

    def __post_init__(self):
        import torch
        if not torch.cuda.is_available():
            raise RuntimeError("kv_compression_b200 needs a CUDA device (no CPU fallback)")
        self._lib = load_library(self.lib_path or LIB_PATH)
        h = ctypes.c_void_p()
        dt = LCA_BF16 if self.dtype == "bf16" else LCA_F32
        _check(self._lib.lca_plan_create(self.B, self.H, self.d_c, self.d_r, dt, self.max_L,
                                         ctypes.byref(h)), "lca_plan_create")
        self._h = h

    @property
    def handle(self) -> int:
        return self._h.value

    def close(self) -> None:
        if getattr(self, "_h", None) is not None and self._h.value:
            self._lib.lca_plan_destroy(self._h)
            self._h = ctypes.c_void_p()

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def set(self, opt: int, value: int) -> None:
        _check(self._lib.lca_plan_set(self._h, opt, int(value)), "lca_plan_set")

    def set_timing_event(self, event) -> None:
        """Record `event` (a torch.cuda.Event, already created) after the main kernel of
        each later call; None turns it off."""
        handle = None if event is None else event.cuda_event
        _check(self._lib.lca_plan_set_timing_event(self._h, handle), "lca_plan_set_timing_event")

    def kernel(self, L: int, g: int, w: int) -> str:
        return KERNEL_NAMES[self._lib.lca_plan_kernel(self._h, L, g, w)]

    def decode(self, q_c, q_r, c_kv, k_r, L: int, g: int, w: int, out, anchor, stream=None) -> None:
        """lca_decode on torch CUDA tensors (asynchronous on `stream`)."""
        _check(self._lib.lca_decode(self._h, _ptr(q_c), _ptr(q_r), _ptr(c_kv), _ptr(k_r), L, g, w,
                                    _ptr(out), _ptr(anchor), _stream_handle(stream)), "lca_decode")

    def dense(self, q_c, q_r, c_kv, k_r, L: int, out, stream=None) -> None:
        """mla_decode (dense MLA softmax attention over all L tokens)."""
        _check(self._lib.mla_decode(self._h, _ptr(q_c), _ptr(q_r), _ptr(c_kv), _ptr(k_r), L,
                                    _ptr(out), _stream_handle(stream)), "mla_decode")

    def decode_host(self, q_c, q_r, c_kv, k_r, L: int, g: int, w: int, out, anchor,
                    stream=None) -> None:
        """lca_decode_host on host (ideally pinned) torch CPU tensors; synchronous."""
        _check(self._lib.lca_decode_host(self._h, _ptr(q_c), _ptr(q_r), _ptr(c_kv), _ptr(k_r), L,
                                         g, w, _ptr(out), _ptr(anchor), _stream_handle(stream)),
               "lca_decode_host")

    def condense(self, q_c, q_r, c_kv, k_r, L: int, g: int, j0: int, n: int, c_dst, k_dst,
                 dst_rows: int, dst_row0: int, anchor, stream=None) -> None:
        """lca_condense: groups j0 .. j0+n-1 into rows dst_row0.. of [B][dst_rows][d] buffers."""
        _check(self._lib.lca_condense(self._h, _ptr(q_c), _ptr(q_r), _ptr(c_kv), _ptr(k_r), L, g, j0, n,
                                      _ptr(c_dst), _ptr(k_dst), dst_rows, dst_row0, _ptr(anchor),
                                      _stream_handle(stream)), "lca_condense")

    def build_stored(self, q_c, q_r, c_kv, k_r, L: int, g: int, w: int, c_store, k_store, anchor,
                     stream=None) -> None:
        """lca_build_stored: [condensed groups || window tokens] per sequence."""
        _check(self._lib.lca_build_stored(self._h, _ptr(q_c), _ptr(q_r), _ptr(c_kv), _ptr(k_r), L, g, w,
                                          _ptr(c_store), _ptr(k_store), _ptr(anchor),
                                          _stream_handle(stream)), "lca_build_stored")

    def decode_stored(self, q_c, q_r, c_store, k_store, n_rows: int, n_cond: int, bias: float, out,
                      stream=None) -> None:
        """lca_decode_stored: attention over the stored rows, `bias` on the first n_cond."""
        _check(self._lib.lca_decode_stored(self._h, _ptr(q_c), _ptr(q_r), _ptr(c_store), _ptr(k_store),
                                           n_rows, n_cond, float(bias), _ptr(out),
                                           _stream_handle(stream)), "lca_decode_stored")

    def decode_partial(self, q_c, q_r, c_slice, k_slice, n_tok: int, pos0: int, L: int, g: int, w: int,
                       part_mz, part_o, anchor, stream=None) -> None:
        """lca_decode_partial: (M, Z, O) of the entries held by tokens [pos0, pos0 + n_tok)."""
        _check(self._lib.lca_decode_partial(self._h, _ptr(q_c), _ptr(q_r), _ptr(c_slice), _ptr(k_slice),
                                            n_tok, pos0, L, g, w, _ptr(part_mz), _ptr(part_o),
                                            _ptr(anchor), _stream_handle(stream)), "lca_decode_partial")

    def merge_partials(self, n_parts: int, part_mz, part_o, out, stream=None) -> None:
        """lca_merge_partials: out from n_parts stacked partials."""
        _check(self._lib.lca_merge_partials(self._h, n_parts, _ptr(part_mz), _ptr(part_o), _ptr(out),
                                            _stream_handle(stream)), "lca_merge_partials")

    def decode_paged(self, q_c, q_r, c_pool, k_pool, page_size: int, block_table, seq_lens, g: int, w: int,
                     out, anchor, stream=None) -> None:
        """lca_decode_paged: pools [num_pages * page_size, d], block_table [B, max_pages] and
        seq_lens [B] int32 CUDA tensors; anchor [B, H, anchor_stride] int32 or None."""
        num_pages = c_pool.shape[0] // page_size
        stride = 0 if anchor is None else anchor.shape[2]
        _check(self._lib.lca_decode_paged(self._h, _ptr(q_c), _ptr(q_r), _ptr(c_pool), _ptr(k_pool), num_pages,
                                          page_size, _ptr(block_table), block_table.shape[1], _ptr(seq_lens),
                                          g, w, _ptr(out), _ptr(anchor), stride, _stream_handle(stream)),
               "lca_decode_paged")

    def prefill_paged(self, q_c, q_r, c_pool, k_pool, page_size: int, table_row, pos0: int, g: int, w: int,
                      out, anchor, stream=None) -> None:
        """lca_prefill_paged: the plan's B queries at positions pos0 .. pos0 + B - 1 of the one
        sequence paged through table_row [max_pages] int32; anchor [B, H, stride] or None."""
        num_pages = c_pool.shape[0] // page_size
        stride = 0 if anchor is None else anchor.shape[2]
        _check(self._lib.lca_prefill_paged(self._h, _ptr(q_c), _ptr(q_r), _ptr(c_pool), _ptr(k_pool), num_pages,
                                           page_size, _ptr(table_row), table_row.shape[0], pos0, g, w, _ptr(out),
                                           _ptr(anchor), stride, _stream_handle(stream)), "lca_prefill_paged")

    def decode_gqa(self, q, k_cache, v_cache, L: int, n_kv_heads: int, g: int, w: int, out, anchor,
                   stream=None) -> None:
        """lca_decode_gqa: q [B,H,d_k], k_cache [B,L,H_kv,d_k], v_cache [B,L,H_kv,d_v] CUDA tensors."""
        _check(self._lib.lca_decode_gqa(self._h, _ptr(q), _ptr(k_cache), _ptr(v_cache), L, n_kv_heads, g, w,
                                        _ptr(out), _ptr(anchor), _stream_handle(stream)), "lca_decode_gqa")

    def device_error(self, stream=None) -> int:
        return int(self._lib.lca_get_device_error(self._h, _stream_handle(stream)))

    def device_error_site(self) -> int:
        """Where (a per-wait-site code) the last error device_error reported arose."""
        return int(self._lib.lca_get_device_error_site(self._h))


def lca_decode(q_c, q_r, c_kv, k_r, g: int, w: int, plan: Plan | None = None, stream=None):
    """Convenience: allocate outputs and run one LCA decode.

    q_c [B,H,d_c], q_r [B,H,d_r], c_kv [B,L,d_c], k_r [B,L,d_r] CUDA tensors
    (bf16 or fp32, contiguous).  Returns (out [B,H,d_c] fp32, anchor [B,H,n_G] int32).
    """
    import torch
    B, H, d_c = q_c.shape
    d_r = q_r.shape[2]
    L = c_kv.shape[1]
    dt = "bf16" if q_c.dtype == torch.bfloat16 else "f32"
    plan = plan or Plan(B, H, d_c, d_r, dt, L)
    nG = num_groups(L, g, w)
    out = torch.empty(B, H, d_c, dtype=torch.float32, device=q_c.device)
    anchor = torch.empty(B, H, max(nG, 0), dtype=torch.int32, device=q_c.device)
    plan.decode(q_c, q_r, c_kv, k_r, L, g, w, out, anchor if nG > 0 else None, stream)
    return out, anchor


def mla_decode(q_c, q_r, c_kv, k_r, plan: Plan | None = None, stream=None):
    """Convenience: dense MLA decode; returns out [B,H,d_c] fp32."""
    import torch
    B, H, d_c = q_c.shape
    d_r = q_r.shape[2]
    L = c_kv.shape[1]
    dt = "bf16" if q_c.dtype == torch.bfloat16 else "f32"
    plan = plan or Plan(B, H, d_c, d_r, dt, L)
    out = torch.empty(B, H, d_c, dtype=torch.float32, device=q_c.device)
    plan.dense(q_c, q_r, c_kv, k_r, L, out, stream)
    return out


def stored_rows(L: int, g: int, w: int) -> int:
    return int(load_library().lca_stored_rows(L, g, w))


def slice_groups(L: int, g: int, w: int, pos0: int, n_tok: int) -> int:
    return int(load_library().lca_slice_groups(L, g, w, pos0, n_tok))
