"""ctypes declarations of librglru.so (include/rglru.h). No arithmetic happens here."""
from __future__ import annotations

import ctypes
import os

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "librglru.so")

RGLRU_F32 = 0
RGLRU_BF16 = 1

STATUS = {
    0: "RGLRU_OK", -1: "RGLRU_ERR_NULL", -2: "RGLRU_ERR_SHAPE", -3: "RGLRU_ERR_ALIGN", -4: "RGLRU_ERR_DTYPE",
    -5: "RGLRU_ERR_WORKSPACE", -6: "RGLRU_ERR_CUDA", -7: "RGLRU_ERR_TIMEOUT", -8: "RGLRU_ERR_DEVICE",
}

STATUS_CODE = {v: k for k, v in STATUS.items()}

# Every function the header declares, with (restype, argtypes).
_P = ctypes.c_void_p
_I = ctypes.c_int
_L = ctypes.c_int64
_S = ctypes.c_size_t


class RGLRUParams(ctypes.Structure):
    _fields_ = [("conv_w", _P), ("conv_b", _P), ("W_a", _P), ("b_a", _P), ("W_x", _P), ("b_x", _P),
                ("Lambda", _P)]


_PP = ctypes.POINTER(RGLRUParams)


class RGLRUGrads(ctypes.Structure):
    _fields_ = [("dx", _P), ("dconv_state0", _P), ("dconv_w", _P), ("dconv_b", _P), ("dW_a", _P), ("db_a", _P),
                ("dW_x", _P), ("db_x", _P), ("dLambda", _P), ("dh0", _P)]


_GP = ctypes.POINTER(RGLRUGrads)


class RGLRULayerWeights(ctypes.Structure):
    _fields_ = [("norm1_scale", _P), ("W_1", _P), ("W_2", _P), ("W_o", _P), ("norm2_scale", _P), ("W_gate", _P),
                ("W_up", _P), ("W_down", _P)]


_LWP = ctypes.POINTER(RGLRULayerWeights)


class RGLRUAttentionWeights(ctypes.Structure):
    _fields_ = [("W_qkv", _P), ("W_o", _P)]


_AWP = ctypes.POINTER(RGLRUAttentionWeights)


class RGLRUAttentionLayerWeights(ctypes.Structure):
    _fields_ = [("norm1_scale", _P), ("W_qkv", _P), ("W_o", _P), ("norm2_scale", _P), ("W_gate", _P), ("W_up", _P),
                ("W_down", _P)]


_ALWP = ctypes.POINTER(RGLRUAttentionLayerWeights)

SIGNATURES = {
    "rglru_forward_workspace_bytes": (_S, [_I, _I, _I, _I]),
    "rglru_forward": (_I, [_PP, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _P, _S, _P]),
    "rglru_step_workspace_bytes": (_S, [_I, _I, _I]),
    "rglru_step": (_I, [_PP, _P, _P, _P, _P, _I, _I, _L, _I, _P, _S, _P]),
    "rglru_block_workspace_bytes": (_S, [_I, _I, _I, _I, _I]),
    "rglru_block_forward": (_I, [_PP, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _P, _S, _P]),
    "rglru_layer_workspace_bytes": (_S, [_I, _I, _I, _I, _I, _I]),
    "rglru_layer_forward": (_I, [_PP, _LWP, _P, _P, _P, _P, _I, _I, _I, _I, _I, ctypes.c_float, _I, _P, _S, _P]),
    "rglru_layer_step_workspace_bytes": (_S, [_I, _I, _I, _I, _I]),
    "rglru_layer_step": (_I, [_PP, _LWP, _P, _P, _P, _P, _I, _I, _I, _I, _L, ctypes.c_float, _I, _P, _S, _P]),
    "rglru_attention_step_workspace_bytes": (_S, [_I, _I, _I]),
    "rglru_attention_step": (_I, [_AWP, _P, _P, _P, _P, _I, _I, _I, _L, _P, _S, _P]),
    "rglru_attention_layer_step_workspace_bytes": (_S, [_I, _I, _I, _I]),
    "rglru_attention_layer_step": (_I, [_ALWP, _P, _P, _P, _P, _I, _I, _I, _I, _L, ctypes.c_float, _P, _S, _P]),
    "rglru_conv1d": (_I, [_P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _P]),
    "rglru_gate_pitch": (_L, [_I]),
    "rglru_gate_proj": (_I, [_P, _P, _P, _P, _P, _P, _L, _I, _I, _P]),
    "rglru_scan_workspace_bytes": (_S, [_I, _I, _I, _I]),
    "rglru_scan": (_I, [_PP, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _P, _S, _P]),
    "rglru_gate_coeffs": (_I, [_PP, _P, _P, _L, _I, _P]),
    "rglru_scan_coeffs": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _P, _S, _P]),
    "rglru_scan_noalloc": (_I, [_PP, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _P]),
    "rglru_scan_noalloc_status": (_I, [_P]),
    "rglru_gemm_bf16": (_I, [_P, _P, _P, _L, _I, _I, _P]),
    "rglru_backward_workspace_bytes": (_S, [_I, _I, _I]),
    "rglru_backward": (_I, [_PP, _P, _P, _P, _P, _P, _P, _GP, _I, _I, _I, _P, _S, _P]),
    "rglru_saved_bytes": (_S, [_I, _I, _I]),
    "rglru_forward_kernels": (_I, [_I, _I, _I, _I]),
    "rglru_forward_train": (_I, [_PP, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _P, _S, _P]),
    "rglru_backward_saved": (_I, [_PP, _P, _P, _P, _P, _P, _P, _P, _GP, _I, _I, _I, _P, _S, _P]),
    "rglru_gate_scan_workspace_bytes": (_S, [_I, _I, _I, _I]),
    "rglru_gate_scan": (_I, [_PP, _P, _P, _P, _P, _I, _I, _I, _I, _P, _S, _P]),
    "rglru_workspace_status": (_I, [_P, _P]),
    "rglru_strerror": (ctypes.c_char_p, [_I]),
    "rglru_last_cuda_error": (_I, []),
    "rglru_version": (_I, []),
    "rglru_debug_scan_stall": (_I, [_L]),
}

_lib = None


class RGLRUError(RuntimeError):
    def __init__(self, fn: str, code: int, detail: str = ""):
        self.code = code
        super().__init__(f"{fn} failed: {STATUS.get(code, code)} ({detail})")


def load() -> ctypes.CDLL:
    """Loads librglru.so; raises if it has not been built (there is no fallback)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"{LIB_PATH} is missing: build it with `python -m gated_linear_rnn_conv1d_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    for name, (res, args) in SIGNATURES.items():
        f = getattr(lib, name)
        f.restype = res
        f.argtypes = args
    _lib = lib
    return lib


def check(fn: str, code: int) -> None:
    if code != 0:
        lib = load()
        detail = lib.rglru_strerror(code).decode()
        if code == -6:
            detail += f"; cudaError={lib.rglru_last_cuda_error()}"
        raise RGLRUError(fn, code, detail)
