"""ctypes binding of the GQE C ABI (include/gqe.h): argument marshalling only.

Every function here has the name of the C entry point it calls and passes torch tensors'
device pointers and the current CUDA stream through unchanged; all computation happens in
libgqe.so's kernels. If the library is missing, importing this module raises: there is no
fallback path.
"""
from __future__ import annotations

import ctypes
import os

import torch

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libgqe.so")

GQE_OK, GQE_ERR_INVALID_ARG, GQE_ERR_UNSUPPORTED, GQE_ERR_WORKSPACE, GQE_ERR_CUDA, \
    GQE_ERR_TIMEOUT = range(6)
GQE_BF16, GQE_F32 = 0, 1
VARIANTS = {"gqe": 0, "weighted_concat": 1, "hard_concat": 2}
TENSORS = {"K": 0, "V": 1, "Q": 2, "Z": 3, "PSEL": 4, "W": 5, "LOGITS": 6}

EXPORTED = ("gqe_create", "gqe_forward", "gqe_get_routing", "gqe_get_tensor",
            "gqe_check_device_status", "gqe_set_spin_limit", "gqe_destroy", "gqe_status_str",
            "gqe_workspace_bytes", "gqe_kernel_launches", "gqe_set_stage_events",
            "gqe_stage_name", "gqe_route_static", "gqe_exp2_fma", "gqe_selftest_timeout",
            "gqe_decode", "gqe_enable_backward", "gqe_backward", "gqe_backward_launches",
            "gqe_set_group_range", "gqe_backward_begin", "gqe_backward_finish")
GQE_NUM_STAGES = 6


class GQEError(RuntimeError):
    def __init__(self, status: int, where: str):
        super().__init__(f"{where}: {status_str(status)}")
        self.status = status


def _load() -> ctypes.CDLL:
    if not os.path.exists(_LIB_PATH):
        raise ImportError(
            f"GQE CUDA library not built ({_LIB_PATH} missing); run "
            "`python -m moe_query_head_b200.build`")
    lib = ctypes.CDLL(_LIB_PATH)
    P, I, I64, SZ = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_size_t
    lib.gqe_create.argtypes = [ctypes.POINTER(P), I, I, I, I, I, I, I64]
    lib.gqe_create.restype = I
    lib.gqe_forward.argtypes = [P, P, I, I, P, P, P, P, P, P, I, I, I, I, I, I, P, P, P]
    lib.gqe_forward.restype = I
    lib.gqe_decode.argtypes = [P, P, I, P, P, I, P, P, P, P, P, P, P, I, I, I, I, I, P, P, P]
    lib.gqe_decode.restype = I
    lib.gqe_get_routing.argtypes = [P, P, P, P, P, P]
    lib.gqe_get_routing.restype = I
    lib.gqe_get_tensor.argtypes = [P, I, P, SZ, P]
    lib.gqe_get_tensor.restype = I
    lib.gqe_check_device_status.argtypes = [P, P]
    lib.gqe_check_device_status.restype = I
    lib.gqe_set_spin_limit.argtypes = [P, I64]
    lib.gqe_set_spin_limit.restype = I
    lib.gqe_destroy.argtypes = [P]
    lib.gqe_destroy.restype = None
    lib.gqe_status_str.argtypes = [I]
    lib.gqe_status_str.restype = ctypes.c_char_p
    lib.gqe_workspace_bytes.argtypes = [I, I, I, I, I, I, I64]
    lib.gqe_workspace_bytes.restype = I64
    lib.gqe_kernel_launches.argtypes = [P]
    lib.gqe_kernel_launches.restype = I
    lib.gqe_set_stage_events.argtypes = [P, ctypes.POINTER(P), I]
    lib.gqe_set_stage_events.restype = I
    lib.gqe_stage_name.argtypes = [I]
    lib.gqe_stage_name.restype = ctypes.c_char_p
    lib.gqe_route_static.argtypes = [P, I, I, I, I, P, P, P, P, P, P]
    lib.gqe_route_static.restype = I
    lib.gqe_exp2_fma.argtypes = [P, P, I, P]
    lib.gqe_exp2_fma.restype = I
    lib.gqe_selftest_timeout.argtypes = [P, ctypes.c_int64, P]
    lib.gqe_selftest_timeout.restype = I
    lib.gqe_set_group_range.argtypes = [P, I, I]
    lib.gqe_set_group_range.restype = I
    lib.gqe_enable_backward.argtypes = [P]
    lib.gqe_enable_backward.restype = I
    lib.gqe_backward.argtypes = [P, P, I, I, P, P, P, P, P, P, I, I, I, I, I, I, P,
                                 ctypes.c_float, P, P, P, P, P, P, P, P]
    lib.gqe_backward.restype = I
    lib.gqe_backward_begin.argtypes = [P, P, I, I, P, P, P, P, P, P, I, I, I, I, I, I, P, P, P]
    lib.gqe_backward_begin.restype = I
    lib.gqe_backward_finish.argtypes = [P, P, I, I, P, P, P, P, P, P, I, I, I, I, I, I, P,
                                        ctypes.c_float, P, P, P, P, P, P, P, P, P]
    lib.gqe_backward_finish.restype = I
    lib.gqe_backward_launches.argtypes = [P]
    lib.gqe_backward_launches.restype = I
    return lib


lib = _load()


def status_str(status: int) -> str:
    return lib.gqe_status_str(int(status)).decode()


def _check(status: int, where: str) -> None:
    if status != GQE_OK:
        raise GQEError(status, where)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def gqe_workspace_bytes(dim, N, G, k, d_h, dtype, max_tokens) -> int:
    return int(lib.gqe_workspace_bytes(dim, N, G, k, d_h, dtype, max_tokens))


def gqe_create(dim, N, G, k, d_h, dtype, max_tokens) -> ctypes.c_void_p:
    h = ctypes.c_void_p()
    _check(lib.gqe_create(ctypes.byref(h), dim, N, G, k, d_h, dtype, max_tokens), "gqe_create")
    return h


def gqe_forward(h, x, B, T, W_r, W_q, W_k, W_v, W_shared, W_o, N, G, k, d_h, variant, causal,
                out, aux_loss=None, stream=None) -> None:
    _check(lib.gqe_forward(h, _ptr(x), B, T, _ptr(W_r), _ptr(W_q), _ptr(W_k), _ptr(W_v),
                           _ptr(W_shared), _ptr(W_o), N, G, k, d_h, variant, causal, _ptr(out),
                           _ptr(aux_loss), _stream(stream)), "gqe_forward")


def gqe_decode(h, x, B, k_cache, v_cache, L_max, lengths, W_r, W_q, W_k, W_v, W_shared, W_o,
               N, G, k, d_h, variant, out, aux_loss=None, stream=None) -> None:
    """One generation step with a KV cache (see include/gqe.h); lengths is an int32 device
    tensor and is not modified."""
    _check(lib.gqe_decode(h, _ptr(x), B, _ptr(k_cache), _ptr(v_cache), L_max, _ptr(lengths),
                          _ptr(W_r), _ptr(W_q), _ptr(W_k), _ptr(W_v), _ptr(W_shared), _ptr(W_o),
                          N, G, k, d_h, variant, _ptr(out), _ptr(aux_loss), _stream(stream)),
           "gqe_decode")


def gqe_set_group_range(h, g0: int, g1: int) -> None:
    """Restricts the handle to groups g0 .. g1-1 of the layer (see include/gqe.h)."""
    _check(lib.gqe_set_group_range(h, int(g0), int(g1)), "gqe_set_group_range")


def gqe_enable_backward(h) -> None:
    """Allocates the handle's backward workspace (see include/gqe.h)."""
    _check(lib.gqe_enable_backward(h), "gqe_enable_backward")


def gqe_backward(h, x, B, T, W_r, W_q, W_k, W_v, W_shared, W_o, N, G, k, d_h, variant, causal,
                 dy, aux_grad, dx, dW_r, dW_q, dW_k, dW_v, dW_shared, dW_o, stream=None) -> None:
    """Gradients of <dy, y> + aux_grad * aux_loss of the handle's last gqe_forward (same
    arguments); every gradient is a float32 device tensor (see include/gqe.h)."""
    _check(lib.gqe_backward(h, _ptr(x), B, T, _ptr(W_r), _ptr(W_q), _ptr(W_k), _ptr(W_v),
                            _ptr(W_shared), _ptr(W_o), N, G, k, d_h, variant, causal, _ptr(dy),
                            float(aux_grad), _ptr(dx), _ptr(dW_r), _ptr(dW_q), _ptr(dW_k),
                            _ptr(dW_v), _ptr(dW_shared), _ptr(dW_o), _stream(stream)),
           "gqe_backward")


def gqe_backward_begin(h, x, B, T, W_r, W_q, W_k, W_v, W_shared, W_o, N, G, k, d_h, variant,
                       causal, dy, slot_dot, stream=None) -> None:
    """Phase 1 of the backward of a handle's last gqe_forward: writes this handle's share of
    <dslot, slot> per token to slot_dot (float32 [B*T], device; see include/gqe.h)."""
    _check(lib.gqe_backward_begin(h, _ptr(x), B, T, _ptr(W_r), _ptr(W_q), _ptr(W_k), _ptr(W_v),
                                  _ptr(W_shared), _ptr(W_o), N, G, k, d_h, variant, causal,
                                  _ptr(dy), _ptr(slot_dot), _stream(stream)),
           "gqe_backward_begin")


def gqe_backward_finish(h, x, B, T, W_r, W_q, W_k, W_v, W_shared, W_o, N, G, k, d_h, variant,
                        causal, dy, aux_grad, slot_dot, dx, dW_r, dW_q, dW_k, dW_v, dW_shared,
                        dW_o, stream=None) -> None:
    """Phase 2: the gradients, given <dslot, slot> summed over the layer's group ranges."""
    _check(lib.gqe_backward_finish(h, _ptr(x), B, T, _ptr(W_r), _ptr(W_q), _ptr(W_k),
                                   _ptr(W_v), _ptr(W_shared), _ptr(W_o), N, G, k, d_h, variant,
                                   causal, _ptr(dy), float(aux_grad), _ptr(slot_dot), _ptr(dx),
                                   _ptr(dW_r), _ptr(dW_q), _ptr(dW_k), _ptr(dW_v),
                                   _ptr(dW_shared), _ptr(dW_o), _stream(stream)),
           "gqe_backward_finish")


def gqe_backward_launches(h) -> int:
    return int(lib.gqe_backward_launches(h))


def gqe_get_routing(h, sel=None, gates=None, counts=None, mean_prob=None, stream=None) -> None:
    _check(lib.gqe_get_routing(h, _ptr(sel), _ptr(gates), _ptr(counts), _ptr(mean_prob),
                               _stream(stream)), "gqe_get_routing")


def gqe_get_tensor(h, which: str, dst, stream=None) -> None:
    _check(lib.gqe_get_tensor(h, TENSORS[which], _ptr(dst), dst.numel() * dst.element_size(),
                              _stream(stream)), "gqe_get_tensor")


def gqe_check_device_status(h, stream=None) -> int:
    return int(lib.gqe_check_device_status(h, _stream(stream)))


def gqe_set_spin_limit(h, limit: int) -> None:
    _check(lib.gqe_set_spin_limit(h, int(limit)), "gqe_set_spin_limit")


def gqe_destroy(h) -> None:
    lib.gqe_destroy(h)


def gqe_kernel_launches(h) -> int:
    return int(lib.gqe_kernel_launches(h))


def gqe_route_static(logits, M, N, G, k, sel, gates, counts, mean_prob, aux_loss=None,
                     stream=None) -> None:
    """Routing from precomputed logits with no device allocation (see include/gqe.h)."""
    _check(lib.gqe_route_static(_ptr(logits), M, N, G, k, _ptr(sel), _ptr(gates), _ptr(counts),
                                _ptr(mean_prob), _ptr(aux_loss), _stream(stream)),
           "gqe_route_static")


def gqe_selftest_timeout(h, spin: int, stream=None) -> None:
    """Makes one bounded device wait run out on purpose (see include/gqe.h)."""
    _check(lib.gqe_selftest_timeout(h, spin, _stream(stream)), "gqe_selftest_timeout")


def gqe_exp2_fma(inp, out, stream=None) -> None:
    """Diagnostic: the softmax's FMA-pipe exp2, elementwise (float32 device tensors)."""
    _check(lib.gqe_exp2_fma(_ptr(inp), _ptr(out), inp.numel(), _stream(stream)), "gqe_exp2_fma")


def gqe_stage_name(i: int):
    r = lib.gqe_stage_name(int(i))
    return None if r is None else r.decode()


def gqe_set_stage_events(h, events) -> None:
    """events: GQE_NUM_STAGES + 1 torch.cuda.Event(enable_timing=True) objects, each
    already recorded once (torch creates the underlying cudaEvent_t lazily), or None."""
    if not events:
        _check(lib.gqe_set_stage_events(h, None, 0), "gqe_set_stage_events")
        return
    arr = (ctypes.c_void_p * len(events))(*[ctypes.c_void_p(e.cuda_event) for e in events])
    _check(lib.gqe_set_stage_events(h, arr, len(events)), "gqe_set_stage_events")
