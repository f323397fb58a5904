"""ctypes declarations of the C ABI in ``include/moe_b200.h``.

Loading is lazy and loud: the first call that needs the library raises
``RuntimeError`` if ``libmoe_b200.so`` has not been built. There is no fallback
implementation.
"""
from __future__ import annotations

import ctypes
import os
import threading

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmoe_b200.so")

MOE_OK = 0
MOE_ERR_INVALID_ARG = 1
MOE_ERR_UNSUPPORTED = 2
MOE_ERR_WORKSPACE_TOO_SMALL = 3
MOE_ERR_CUDA = 4
MOE_ERR_DEVICE_TIMEOUT = 5

MOE_ACT_SWIGLU = 0
MOE_ACT_RELU2 = 1
MOE_ACT_GELU_TANH = 2
MOE_ACT_SWIGLUOAI = 3
MOE_DTYPE_FP8_PER_TENSOR = 2
MOE_DTYPE_MXFP8 = 3
MOE_DTYPE_NVFP4 = 4
MOE_DTYPE_BF16 = 0
MOE_DTYPE_FP8_BLOCK128 = 1
MOE_FLAG_PDL = 1


class Problem(ctypes.Structure):
    _fields_ = [
        ("num_tokens", ctypes.c_int32),
        ("hidden", ctypes.c_int32),
        ("num_routed", ctypes.c_int32),
        ("num_shared", ctypes.c_int32),
        ("intermediate", ctypes.c_int32),
        ("topk", ctypes.c_int32),
        ("renormalize", ctypes.c_int32),
        ("activation", ctypes.c_int32),
        ("wdtype", ctypes.c_int32),
        ("block_m", ctypes.c_int32),
        ("flags", ctypes.c_uint32),
        ("input_scale", ctypes.c_float),
        ("activation_scale", ctypes.c_float),
    ]


class Layout(ctypes.Structure):
    _fields_ = [(n, ctypes.c_size_t) for n in (
        "total_bytes", "status", "num_blocks", "topk_ids", "topk_w", "sorted_pair_ids",
        "expert_offsets", "block_expert", "pair_to_row", "chunk_hist", "xq", "xq_scale", "act",
        "actq", "act_scale", "y", "xs", "xs_scale", "group_info", "io_hidden", "io_logits", "io_out")] + [
        ("max_rows", ctypes.c_int64),
        ("num_chunks", ctypes.c_int32),
        ("block_m", ctypes.c_int32),
    ]


class MoeError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)} ({status})")


_P = ctypes.POINTER(Problem)
_V = ctypes.c_void_p
_S = ctypes.c_size_t
_I = ctypes.c_int32

# name -> (restype, argtypes); every function declared in include/moe_b200.h
SIGNATURES = {
    "moe_status_string": (ctypes.c_char_p, [_I]),
    "moe_check_problem": (_I, [_P]),
    "moe_padded_intermediate": (_I, [_I, _I, _I]),
    "moe_workspace_layout": (_I, [_P, ctypes.POINTER(Layout)]),
    "moe_workspace_size": (_S, [_P]),
    "moe_prepare_weights": (_I, [_P, _I, _V, _V, _V, _V, _V]),
    "moe_prepared_weights_bytes": (_S, [_P, _I]),
    "moe_quantize_weights_fp8": (_I, [_V, ctypes.c_int64, _I, _I, _V, _V, _V]),
    "moe_quantize_weights_fp8_per_tensor": (_I, [_V, ctypes.c_int64, _I, _I, _V, _V, _V]),
    "moe_quantize_weights_mxfp8": (_I, [_V, ctypes.c_int64, _I, _I, _V, _V, _V]),
    "moe_prepare_weights_mxfp8": (_I, [_P, _V, _V, _V, _V, _V, _V, _V]),
    "moe_quantize_weights_nvfp4": (_I, [_V, ctypes.c_int64, _I, _I, _V, _V, _V, _V]),
    "moe_prepare_weights_nvfp4": (_I, [_P, _V, _V, _V, _V, _V, _V, _V]),
    "moe_ep_workspace_size": (_S, [_P, _I]),
    "moe_ep_max_send_rows": (ctypes.c_int64, [_P, _I]),
    "moe_ep_dispatch": (_I, [_P, _I, _I, _V, _V, _V, _V, _V, _V, _V, _V, _V, _S, _V]),
    "moe_ep_combine": (_I, [_P, _I, _V, _V, _V, _V]),
    "moe_forward": (_I, [_P, _V, _V, _V, _V, _V, _V, _V, _V, _S, _V]),
    "moe_forward_routed": (_I, [_P, _V, _V, _V, _V, _V, _V, _V, _V, _V, _S, _V]),
    "moe_forward_host": (_I, [_P, _V, _V, _V, _V, _V, _V, _V, _V, _S, _V]),
    "moe_stage_route": (_I, [_P, _V, _V, _S, _V]),
    "moe_stage_align": (_I, [_P, _V, _S, _V]),
    "moe_stage_quant_act": (_I, [_P, _V, _V, _S, _V]),
    "moe_stage_permute": (_I, [_P, _V, _V, _S, _V]),
    "moe_stage_gemm1": (_I, [_P, _V, _V, _V, _V, _S, _V]),
    "moe_stage_gemm2": (_I, [_P, _V, _V, _V, _S, _V]),
    "moe_stage_combine": (_I, [_P, _V, _V, _S, _V]),
    "moe_get_device_status": (_I, [_V, _V, ctypes.POINTER(_I)]),
    "moe_align_noalloc": (_I, [_P, _V, _V, _V, _V, _V, _V, _V]),
    "moe_selftest_bounded_wait": (_I, [_V, ctypes.c_uint32, _I, _V]),
}

_lib = None
_lock = threading.Lock()


def lib() -> ctypes.CDLL:
    """The loaded library; raises RuntimeError if it has not been built."""
    global _lib
    if _lib is not None:
        return _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise RuntimeError(
                    f"{LIB_PATH} is missing: build it with "
                    "`python -m mixture_experts_expert_topk_b200.build` (no CPU fallback exists)")
            h = ctypes.CDLL(LIB_PATH)
            for name, (res, args) in SIGNATURES.items():
                fn = getattr(h, name)
                fn.restype = res
                fn.argtypes = args
            _lib = h
    return _lib


def status_string(status: int) -> str:
    try:
        return lib().moe_status_string(status).decode()
    except RuntimeError:
        return str(status)


def check(status: int, where: str) -> None:
    if status != MOE_OK:
        raise MoeError(status, where)
