"""The C-ABI library loads and exports every entry point include/gqe.h declares; argument
checks that need no GPU (CPU only: no kernel is launched)."""
import ctypes
import os
import re

import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_entry_points():
    names = []
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            text = open(os.path.join(ROOT, "include", fn)).read()
            text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
            names += re.findall(r"\b(gqe_[a-z_0-9]+)\s*\(", text)
    return sorted(set(names))


def test_library_exports_every_declared_symbol():
    from moe_query_head_b200 import gqe as G
    names = declared_entry_points()
    assert "gqe_forward" in names and "gqe_create" in names
    for n in names:
        assert hasattr(G.lib, n), f"libgqe.so does not export {n}"
        assert n in G.EXPORTED, f"binding does not wrap {n}"


def test_status_strings():
    from moe_query_head_b200 import gqe as G
    for code in range(6):
        assert G.status_str(code).startswith("GQE_")
    assert "unknown" in G.status_str(99)


def test_workspace_bytes_and_shape_checks():
    from moe_query_head_b200 import gqe as G
    n = G.gqe_workspace_bytes(768, 16, 8, 1, 48, G.GQE_BF16, 16384)
    assert n > 2 * 8 * 16384 * 48 * 2  # at least K and V
    assert G.gqe_workspace_bytes(768, 15, 8, 1, 48, G.GQE_BF16, 16384) == -1  # N % G
    assert G.gqe_workspace_bytes(768, 16, 8, 3, 48, G.GQE_BF16, 16384) == -1  # k > E
    assert G.gqe_workspace_bytes(768, 16, 8, 1, 40, G.GQE_BF16, 16384) == -1  # d_h
    assert G.gqe_workspace_bytes(768, 128, 8, 1, 48, G.GQE_BF16, 16384) == -1  # N > 64


def test_create_rejects_bad_shapes_before_touching_cuda():
    from moe_query_head_b200 import gqe as G
    h = ctypes.c_void_p()
    assert G.lib.gqe_create(ctypes.byref(h), 768, 15, 8, 1, 48, 0, 1024) == G.GQE_ERR_INVALID_ARG
    assert G.lib.gqe_create(ctypes.byref(h), 768, 16, 8, 3, 48, 0, 1024) == G.GQE_ERR_INVALID_ARG
    assert G.lib.gqe_create(ctypes.byref(h), 768, 16, 8, 1, 40, 0, 1024) == G.GQE_ERR_UNSUPPORTED
    assert G.lib.gqe_create(None, 768, 16, 8, 1, 48, 0, 1024) == G.GQE_ERR_INVALID_ARG
    assert h.value is None


def test_null_handle_paths():
    from moe_query_head_b200 import gqe as G
    z = ctypes.c_void_p()
    assert G.lib.gqe_forward(None, z, 1, 1, z, z, z, z, z, z, 16, 8, 1, 48, 0, 1, z, z, z) \
        == G.GQE_ERR_INVALID_ARG
    assert G.lib.gqe_check_device_status(None, None) == G.GQE_ERR_INVALID_ARG
    assert G.lib.gqe_kernel_launches(None) == -1
    assert G.lib.gqe_set_group_range(None, 0, 1) == G.GQE_ERR_INVALID_ARG
    assert G.lib.gqe_enable_backward(None) == G.GQE_ERR_INVALID_ARG
    assert G.lib.gqe_backward(None, z, 1, 1, z, z, z, z, z, z, 16, 8, 1, 48, 0, 1, z, 0.0, z, z,
                              z, z, z, z, z, None) == G.GQE_ERR_INVALID_ARG
    assert G.lib.gqe_backward_launches(None) == -1
    assert G.lib.gqe_backward_begin(None, z, 1, 1, z, z, z, z, z, z, 16, 8, 1, 48, 0, 1, z, z,
                                    None) == G.GQE_ERR_INVALID_ARG
    assert G.lib.gqe_backward_finish(None, z, 1, 1, z, z, z, z, z, z, 16, 8, 1, 48, 0, 1, z,
                                     0.0, z, z, z, z, z, z, z, z, None) == G.GQE_ERR_INVALID_ARG
    assert G.lib.gqe_decode(None, z, 1, z, z, 8, z, z, z, z, z, z, z, 16, 8, 1, 48, 0, z, z,
                            None) == G.GQE_ERR_INVALID_ARG
    G.lib.gqe_destroy(None)


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-GPU error path")
def test_create_without_gpu_reports_cuda_error():
    from moe_query_head_b200 import gqe as G
    h = ctypes.c_void_p()
    assert G.lib.gqe_create(ctypes.byref(h), 768, 16, 8, 1, 48, 0, 1024) == G.GQE_ERR_CUDA
