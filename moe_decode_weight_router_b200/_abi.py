"""ctypes declarations of the C ABI in include/moe_decode.h (argument marshalling only)."""
from __future__ import annotations

import ctypes
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libmoe_decode.so")

P = ctypes.c_void_p
I = ctypes.c_int
Z = ctypes.c_size_t

STATUS_NAMES = {
    0: "MOE_OK", 1: "MOE_ERR_INVALID_ARG", 2: "MOE_ERR_UNSUPPORTED_SHAPE", 3: "MOE_ERR_ALIGNMENT",
    4: "MOE_ERR_WORKSPACE", 5: "MOE_ERR_DTYPE", 6: "MOE_ERR_CUDA", 7: "MOE_ERR_TIMEOUT",
    8: "MOE_ERR_SELFCHECK",
}

FMT_NONE, FMT_BF16, FMT_MXFP4_CODES, FMT_E8M0_SCALES, FMT_E4M3, FMT_F32 = range(6)


class Buf(ctypes.Structure):
    _fields_ = [("ptr", P), ("fmt", I)]


class Layer(ctypes.Structure):
    _fields_ = [("router", Buf), ("w13_codes", Buf), ("w13_scales", Buf), ("w2_codes", Buf),
                ("w2_scales", Buf), ("shared_w13", Buf), ("shared_w2", Buf)]


class Model(ctypes.Structure):
    _fields_ = [("n_layers", I), ("H", I), ("I", I), ("E", I), ("top_k", I), ("Is", I), ("V", I),
                ("rms_eps", ctypes.c_float), ("layers", ctypes.POINTER(Layer)), ("lm_head", Buf),
                ("lm_scale", Buf), ("step_path", I)]

STEP_AUTO, STEP_PER_LAYER = 0, 1


class Trace(ctypes.Structure):
    _fields_ = [("x", P), ("h", P), ("ids", P), ("w", P), ("events", ctypes.POINTER(P)), ("n_events", I),
                ("timeline", P), ("wait_limit_ns", ctypes.c_ulonglong), ("hold_layer", I)]


# name -> (restype, argtypes); every symbol the header declares
SIGNATURES = {
    "moe_status_string": (ctypes.c_char_p, [I]),
    "moe_abi_version": (I, []),
    "moe_last_cuda_error": (I, []),
    "moe_workspace_status": (I, [P, P]),
    "moe_route_workspace_bytes": (Z, [I, I]),
    "moe_route": (I, [P, I, I, P, I, I, P, P, P, P, Z, P]),
    "moe_experts_workspace_bytes": (Z, [I, I, I, I, I, I]),
    "moe_mxfp4_experts": (I, [P, I, I, I, I, I, P, P, P, P, P, P, P, P, I, P, P, Z, P]),
    "lm_head_fp8_quantize": (I, [P, I, I, P, P, P]),
    "moe_prefill_workspace_bytes": (Z, [I, I, I, I, I, I]),
    "moe_prefill_layer": (I, [P, I, I, I, I, I, P, P, P, P, P, P, P, I, P, P, P, P, P, Z, P]),
    "moe_mxfp8_quantize": (I, [P, I, I, P, P, P]),
    "lm_head_workspace_bytes": (Z, [I, I, I]),
    "lm_head_fp8_gemv": (I, [P, I, I, I, P, P, P, P, P, Z, P]),
    "lm_head_fp8_verify": (I, [P, I, I, I, P, P, P, P, P, P, P, Z, P]),
    "lm_head_bf16_gemv": (I, [P, I, I, I, P, P, P, P, Z, P]),
    "moe_sample": (I, [P, I, I, ctypes.c_float, I, ctypes.c_float, P, P, P]),
    "lm_head_fp8_gemv_noalloc": (I, [P, I, I, I, P, P, P, P, P]),
    "moe_selfcheck_workspace_bytes": (Z, []),
    "moe_selfcheck": (I, [P, Z, P, ctypes.POINTER(I), ctypes.POINTER(ctypes.c_float)]),
    "decode_step_workspace_bytes": (Z, [ctypes.POINTER(Model), I]),
    "decode_step_launch_names": (I, [ctypes.POINTER(Model), I, ctypes.POINTER(ctypes.c_char_p), I]),
    "decode_step": (I, [ctypes.POINTER(Model), P, I, P, P, ctypes.POINTER(Trace), P, Z, P]),
    "decode_step_graph_create": (I, [ctypes.POINTER(Model), P, I, P, P, ctypes.POINTER(Trace), P, Z,
                                     ctypes.POINTER(P)]),
    "decode_step_graph_launch": (I, [P, P]),
    "decode_step_graph_destroy": (None, [P]),
}

_lib = None


def load(path: str = LIB_PATH):
    """Load libmoe_decode.so; raises if it is missing (no fallback exists)."""
    global _lib
    if _lib is None:
        if not os.path.exists(path):
            raise ImportError(
                f"{path} is missing: build the CUDA library first "
                "(python -m moe_decode_weight_router_b200.build)")
        lib = ctypes.CDLL(path)
        for name, (res, args) in SIGNATURES.items():
            f = getattr(lib, name)
            f.restype = res
            f.argtypes = args
        _lib = lib
    return _lib
