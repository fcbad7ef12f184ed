"""The C-ABI library loads and exports what include/lca.h declares (no GPU)."""
import ctypes
import os
import re

import pytest

import kv_compression_b200 as kvc
from kv_compression_b200 import build as kbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    kbuild.build()
    return kvc.load_library()


def declared_functions():
    with open(os.path.join(ROOT, "include", "lca.h")) as f:
        src = f.read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(\w+)\s*\([^;{]*\)\s*;", src)))


def test_header_declares_expected_entry_points():
    names = declared_functions()
    for n in kvc.EXPORTS:
        assert n in names, n
    assert set(names) == set(kvc.EXPORTS), names


def test_library_exports_every_declared_symbol(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name


def test_host_only_helpers(lib):
    assert lib.lca_num_groups(32768, 16, 1024) == 1984
    assert lib.lca_num_groups(65536, 16, 2048) == 3968
    assert lib.lca_num_groups(131072, 32, 4096) == 3968
    assert lib.lca_num_groups(10, 4, 10) == 0
    assert lib.lca_num_groups(11, 4, 2) == 2
    assert lib.lca_num_groups(11, 0, 2) == -1
    assert lib.lca_num_groups(0, 1, 0) == -1
    for s in range(10):
        assert lib.lca_status_string(s) != b"unknown status"
    assert lib.lca_status_string(99) == b"unknown status"


def test_null_arguments_rejected_without_device(lib):
    # argument checks run before any CUDA call
    assert lib.lca_plan_create(1, 1, 8, 8, 0, 16, None) == 1
    assert lib.lca_plan_destroy(None) == 0
    assert lib.lca_plan_set(None, 1, 1) == 1
    assert lib.lca_decode(None, None, None, None, None, 16, 1, 0, None, None, None) == 1
    assert lib.mla_decode(None, None, None, None, None, 16, None, None) == 1
    assert lib.lca_get_device_error(None, None) == 1
    assert lib.lca_plan_kernel(None, 16, 1, 0) == 0
    assert lib.lca_decode_paged(None, None, None, None, None, 1, 64, None, 1, None, 1, 0, None, None, 0,
                                None) == 1
    assert lib.lca_prefill_paged(None, None, None, None, None, 1, 64, None, 1, 0, 1, 0, None, None, 0,
                                 None) == 1
    assert lib.lca_decode_gqa(None, None, None, None, 16, 1, 1, 0, None, None, None) == 1


def test_plan_creation_fails_cleanly_without_gpu(lib):
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    h = ctypes.c_void_p()
    st = lib.lca_plan_create(1, 16, 512, 64, 1, 1024, ctypes.byref(h))
    assert st == 4 and not h.value   # LCA_ERR_CUDA, nothing allocated


def test_binding_refuses_cpu_fallback():
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    with pytest.raises(RuntimeError):
        kvc.Plan(1, 16, 512, 64, "bf16", 1024)
