"""ctypes binding of ``include/moe.h`` -- argument marshalling only.

Every function here has the name of the C entry point it calls and forwards
plain pointers and sizes; all work runs in the CUDA library.  Tensors are
torch CUDA tensors (device memory and streams are torch's job); ``None``
passes a NULL pointer.  A non-OK status raises ``MoEError``.
"""

from __future__ import annotations

import ctypes
import math
import os
from typing import Optional

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libmoe_b200.so")

MOE_OK = 0
MOE_ERR_INVALID_ARG = 1
MOE_ERR_UNSUPPORTED = 2
MOE_ERR_WORKSPACE = 3
MOE_ERR_CUDA = 4
MOE_ERR_DEVICE_TIMEOUT = 5

MOE_W_BF16 = 0
MOE_W_INT4_G128 = 1
MOE_W_NVFP4 = 2
MOE_MAX_TOP_K = 16
MOE_MAX_EXPERTS = 1024
MOE_INT4_MAX_SWIGLU_LIMIT = 255.0

EXPORTED = (
    "moe_status_string", "moe_config_validate", "moe_workspace_size", "moe_workspace_init",
    "moe_router_topk", "moe_permute", "moe_grouped_swiglu_ffn", "moe_grouped_swiglu_ffn_gather", "moe_combine",
    "moe_forward", "moe_forward_ep",
    "moe_read_device_error", "moe_permute_no_alloc", "moe_selftest_device_timeout", "moe_selftest_pair_timeout",
)
MOE_NO_ALLOC_MAX_ROWS = 131072
MOE_SELFTEST_SCRATCH_BYTES = 65536
MOE_SELFTEST_PAIR_BF16 = 0
MOE_SELFTEST_PAIR_INT4 = 1


class MoEError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_name(status)}")


class moe_config(ctypes.Structure):
    _fields_ = [
        ("hidden", ctypes.c_int32),
        ("num_experts", ctypes.c_int32),
        ("top_k", ctypes.c_int32),
        ("expert_inter", ctypes.c_int32),
        ("shared_inter", ctypes.c_int32),
        ("swiglu_limit", ctypes.c_float),
        ("routed_scaling_factor", ctypes.c_float),
        ("renormalize", ctypes.c_int32),
        ("expert_format", ctypes.c_int32),
    ]


class moe_weights(ctypes.Structure):
    _fields_ = [
        ("router_w", ctypes.c_void_p),
        ("correction_bias", ctypes.c_void_p),
        ("w_gate_up", ctypes.c_void_p),
        ("s_gate_up", ctypes.c_void_p),
        ("w_down", ctypes.c_void_p),
        ("s_down", ctypes.c_void_p),
        ("shared_w_gate_up", ctypes.c_void_p),
        ("shared_w_down", ctypes.c_void_p),
        ("g_gate_up", ctypes.c_void_p),
        ("g_down", ctypes.c_void_p),
    ]


_lib = None


def load_library(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load the CUDA library; raise loudly when it was not built."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(
            f"CUDA library not found at {path}; build it with "
            "`python -m routed_swiglu_experts_b200.build` (there is no CPU fallback)")
    lib = ctypes.CDLL(path)
    P, I32, SZ = ctypes.c_void_p, ctypes.c_int32, ctypes.c_size_t
    CFG, W = ctypes.POINTER(moe_config), ctypes.POINTER(moe_weights)
    sig = {
        "moe_status_string": (ctypes.c_char_p, [ctypes.c_int]),
        "moe_config_validate": (ctypes.c_int, [CFG]),
        "moe_workspace_size": (ctypes.c_int, [CFG, I32, ctypes.POINTER(SZ)]),
        "moe_workspace_init": (ctypes.c_int, [P, SZ, P]),
        "moe_router_topk": (ctypes.c_int, [CFG, W, P, I32, P, P, P, SZ, P]),
        "moe_permute": (ctypes.c_int, [CFG, P, P, P, I32, P, P, P, P, P, P, SZ, P]),
        "moe_grouped_swiglu_ffn": (ctypes.c_int, [CFG, W, P, P, P, I32, P, P, P, P, SZ, P]),
        "moe_grouped_swiglu_ffn_gather": (ctypes.c_int, [CFG, W, P, I32, P, P, P, P, P, P, SZ, P]),
        "moe_combine": (ctypes.c_int, [CFG, P, P, P, P, I32, P, P]),
        "moe_forward": (ctypes.c_int, [CFG, W, P, I32, P, P, P, P, SZ, P]),
        "moe_forward_ep": (ctypes.c_int, [CFG, W, I32, I32, P, I32, P, P, P, P, SZ, P]),
        "moe_read_device_error": (ctypes.c_int, [P, P, ctypes.POINTER(I32)]),
        "moe_selftest_device_timeout": (ctypes.c_int, [P, SZ, P]),
        "moe_selftest_pair_timeout": (ctypes.c_int, [P, SZ, I32, P]),
        "moe_permute_no_alloc": (ctypes.c_int, [CFG, P, P, P, I32, P, P, P, P, P, P]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib


def status_name(status: int) -> str:
    try:
        return load_library().moe_status_string(int(status)).decode()
    except RuntimeError:
        return f"status {status}"


def _ptr(t) -> Optional[int]:
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream) -> Optional[int]:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(status: int, where: str):
    if status != MOE_OK:
        raise MoEError(status, where)


def make_config(hidden, num_experts, top_k, expert_inter, shared_inter, swiglu_limit,
                routed_scaling_factor=1.0, renormalize=False, expert_format=MOE_W_BF16) -> moe_config:
    return moe_config(int(hidden), int(num_experts), int(top_k), int(expert_inter), int(shared_inter),
                      float(swiglu_limit), float(routed_scaling_factor), int(bool(renormalize)),
                      int(expert_format))


def make_weights(router_w=None, correction_bias=None, w_gate_up=None, s_gate_up=None, w_down=None,
                 s_down=None, shared_w_gate_up=None, shared_w_down=None, g_gate_up=None,
                 g_down=None) -> moe_weights:
    return moe_weights(_ptr(router_w), _ptr(correction_bias), _ptr(w_gate_up), _ptr(s_gate_up),
                       _ptr(w_down), _ptr(s_down), _ptr(shared_w_gate_up), _ptr(shared_w_down),
                       _ptr(g_gate_up), _ptr(g_down))


def weight_format(w_gate_up, g_gate_up=None) -> int:
    """The moe_weight_format of a layer's routed tensors: bf16 weights, or
    uint8 codes -- NVFP4 when the per-expert fp32 tensor scales are given,
    else W4A16."""
    if g_gate_up is not None:
        return MOE_W_NVFP4
    return MOE_W_INT4_G128 if str(w_gate_up.dtype) == "torch.uint8" else MOE_W_BF16


# ------------------------------------------------------- C entry points ----

def moe_config_validate(cfg: moe_config) -> int:
    return load_library().moe_config_validate(ctypes.byref(cfg))


def moe_workspace_size(cfg: moe_config, max_tokens: int) -> int:
    n = ctypes.c_size_t(0)
    _check(load_library().moe_workspace_size(ctypes.byref(cfg), int(max_tokens), ctypes.byref(n)),
           "moe_workspace_size")
    return n.value


def moe_workspace_init(ws, stream=None):
    _check(load_library().moe_workspace_init(_ptr(ws), ws.numel() * ws.element_size(), _stream(stream)),
           "moe_workspace_init")


def moe_router_topk(cfg, w, x, T, topk_ids, topk_w, ws, stream=None):
    _check(load_library().moe_router_topk(ctypes.byref(cfg), ctypes.byref(w), _ptr(x), int(T), _ptr(topk_ids),
                                          _ptr(topk_w), _ptr(ws), ws.numel() * ws.element_size(),
                                          _stream(stream)), "moe_router_topk")


def moe_permute(cfg, topk_ids, topk_w, x, T, expert_offsets, row_of, src, w_perm, x_perm, ws, stream=None):
    _check(load_library().moe_permute(ctypes.byref(cfg), _ptr(topk_ids), _ptr(topk_w), _ptr(x), int(T),
                                      _ptr(expert_offsets), _ptr(row_of), _ptr(src), _ptr(w_perm),
                                      _ptr(x_perm), _ptr(ws), ws.numel() * ws.element_size(),
                                      _stream(stream)), "moe_permute")


def moe_grouped_swiglu_ffn(cfg, w, x_perm, expert_offsets, w_perm, T, y_perm, x_shared, shared_out, ws,
                           stream=None):
    _check(load_library().moe_grouped_swiglu_ffn(
        ctypes.byref(cfg), ctypes.byref(w), _ptr(x_perm), _ptr(expert_offsets), _ptr(w_perm), int(T),
        _ptr(y_perm), _ptr(x_shared), _ptr(shared_out), _ptr(ws), ws.numel() * ws.element_size(),
        _stream(stream)), "moe_grouped_swiglu_ffn")


def moe_grouped_swiglu_ffn_gather(cfg, w, x, T, src, expert_offsets, w_perm, y_perm, shared_out, ws, stream=None):
    _check(load_library().moe_grouped_swiglu_ffn_gather(
        ctypes.byref(cfg), ctypes.byref(w), _ptr(x), int(T), _ptr(src), _ptr(expert_offsets), _ptr(w_perm),
        _ptr(y_perm), _ptr(shared_out), _ptr(ws), ws.numel() * ws.element_size(), _stream(stream)),
        "moe_grouped_swiglu_ffn_gather")


def moe_combine(cfg, y_perm, row_of, topk_w, shared_out, T, out, stream=None):
    _check(load_library().moe_combine(ctypes.byref(cfg), _ptr(y_perm), _ptr(row_of), _ptr(topk_w),
                                      _ptr(shared_out), int(T), _ptr(out), _stream(stream)), "moe_combine")


def moe_forward(cfg, w, x, T, out, topk_ids_opt, topk_w_opt, ws, stream=None):
    _check(load_library().moe_forward(ctypes.byref(cfg), ctypes.byref(w), _ptr(x), int(T), _ptr(out),
                                      _ptr(topk_ids_opt), _ptr(topk_w_opt), _ptr(ws),
                                      ws.numel() * ws.element_size(), _stream(stream)), "moe_forward")


def moe_forward_ep(cfg, w, expert_begin, expert_end, x, T, out_partial, topk_ids_opt, topk_w_opt, ws, stream=None):
    _check(load_library().moe_forward_ep(ctypes.byref(cfg), ctypes.byref(w), int(expert_begin), int(expert_end),
                                         _ptr(x), int(T), _ptr(out_partial), _ptr(topk_ids_opt), _ptr(topk_w_opt),
                                         _ptr(ws), ws.numel() * ws.element_size(), _stream(stream)), "moe_forward_ep")


def moe_permute_no_alloc(cfg, topk_ids, topk_w, x, T, expert_offsets, row_of, src, w_perm, x_perm, stream=None):
    """moe_permute without a workspace (scratch held inside the library)."""
    _check(load_library().moe_permute_no_alloc(ctypes.byref(cfg), _ptr(topk_ids), _ptr(topk_w), _ptr(x), int(T),
                                               _ptr(expert_offsets), _ptr(row_of), _ptr(src), _ptr(w_perm),
                                               _ptr(x_perm), _stream(stream)), "moe_permute_no_alloc")


def moe_read_device_error(ws, stream=None) -> int:
    code = ctypes.c_int32(0)
    _check(load_library().moe_read_device_error(_ptr(ws), _stream(stream), ctypes.byref(code)),
           "moe_read_device_error")
    return code.value


def moe_selftest_device_timeout(scratch, stream=None):
    """Test hook: force the tensor-core kernel's timeout path on a tiny tile
    (the error lands in scratch's error word; read it with
    moe_read_device_error(scratch))."""
    _check(load_library().moe_selftest_device_timeout(_ptr(scratch), scratch.numel() * scratch.element_size(),
                                                      _stream(stream)), "moe_selftest_device_timeout")


def moe_selftest_pair_timeout(scratch, kernel, stream=None):
    """Test hook: force the timeout path of a CTA-pair grouped GEMM
    (MOE_SELFTEST_PAIR_BF16 or MOE_SELFTEST_PAIR_INT4) on a tiny tile; read
    the error with moe_read_device_error(scratch)."""
    _check(load_library().moe_selftest_pair_timeout(_ptr(scratch), scratch.numel() * scratch.element_size(),
                                                    int(kernel), _stream(stream)), "moe_selftest_pair_timeout")


def status_strings():
    lib = load_library()
    return {s: lib.moe_status_string(s).decode() for s in range(6)}


INF = math.inf
