"""ctypes declarations of include/svla.h (libsvla.so, built in-tree).

Loading fails loudly when the library is missing: there is no fallback path.
"""
from __future__ import annotations

import ctypes
import os

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libsvla.so")

SVLA_OK = 0
STATUS = {
    0: "SVLA_OK", -1: "SVLA_ERR_ARG", -2: "SVLA_ERR_SHAPE", -3: "SVLA_ERR_BLOB_SIZE",
    -4: "SVLA_ERR_EMPTY_PREFIX", -5: "SVLA_ERR_CUDA", -6: "SVLA_ERR_OOM",
    -7: "SVLA_ERR_TIMEOUT", -8: "SVLA_ERR_UNSUPPORTED",
}
SVLA_ERR_ARG, SVLA_ERR_SHAPE, SVLA_ERR_BLOB_SIZE = -1, -2, -3
SVLA_ERR_EMPTY_PREFIX, SVLA_ERR_CUDA, SVLA_ERR_OOM = -4, -5, -6
SVLA_ERR_TIMEOUT, SVLA_ERR_UNSUPPORTED = -7, -8

EPI_F32, EPI_BF16, EPI_ADD_F32, EPI_SILU_BF16 = 0, 1, 2, 3


class SvlaConfig(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int) for n in (
        "p_layers", "p_width", "p_heads", "p_kv_heads", "head_dim", "p_ffn",
        "e_layers", "e_width", "e_heads", "e_kv_heads", "e_ffn", "action_dim")] + \
        [(n, ctypes.c_float) for n in ("rope_base", "rms_eps", "t_min_period", "t_max_period")] + \
        [(n, ctypes.c_int) for n in ("max_batch", "max_prefix", "max_chunk")]


_P = ctypes.c_void_p
_I = ctypes.c_int
_S = ctypes.c_size_t

# name -> (restype, argtypes)
SIGNATURES = {
    "svla_create": (_I, [ctypes.POINTER(SvlaConfig), _P, _S, _I, ctypes.POINTER(_P)]),
    "svla_create_ex": (_I, [ctypes.POINTER(SvlaConfig), _P, _S, _I, ctypes.c_uint, ctypes.POINTER(_P)]),
    "svla_set_prefix_weights": (_I, [_P, _I]),
    "svla_prefix_weights": (_I, [_P]),
    "svla_set_expert_weights": (_I, [_P, _I]),
    "svla_expert_weights": (_I, [_P]),
    "svla_train_step": (_I, [_P, _P, _P, _I, _I, _P, _P, _P, _I, _P, _P, _P]),
    "svla_train_grad_elems": (_S, [_P]),
    "svla_destroy": (_I, [_P]),
    "svla_kv_cache_bytes": (_S, [_P, _I, _I]),
    "svla_blob_bytes": (_S, [ctypes.POINTER(SvlaConfig)]),
    "svla_prefill": (_I, [_P, _P, _P, _I, _I, _P, _P]),
    "svla_denoise": (_I, [_P, _P, _P, _I, _I, _P, _I, _I, _P, _P, _P]),
    "svla_denoise_prefix": (_I, [_P, _P, _P, _I, _I, _P, _I, _I, _P, _I, _P, _P, _P]),
    "svla_sample": (_I, [_P, _P, _P, _I, _I, ctypes.c_uint64, _I, _I, _P, _P, _P, _P]),
    "svla_device_status": (_I, [_P, _P]),
    "svla_last_error": (ctypes.c_char_p, [_P]),
    "svla_status_string": (ctypes.c_char_p, [_I]),
    "svla_op_gemm": (_I, [_I, _P, _I, _P, _I, _I, _I, _I, _P, _I, _P, _I, _P, _S, _P, _P]),
    "svla_op_gemm_noalloc": (_I, [_I, _P, _I, _P, _I, _I, _I, _I, _P, _I, _P, _I, _P, _P]),
    "svla_op_gemm_workspace_bytes": (_S, [_I, _I, _I, _I]),
    "svla_op_gemm_splits": (_I, [_I, _I, _I]),
    "svla_op_attention": (_I, [_P, _I, _P, _P, _I, _P, _I, _I, _I, _I, _I, _I, _I, _P, _I, _P]),
    "svla_op_rmsnorm": (_I, [_P, _P, _I, _I, ctypes.c_float, _P, _P]),
    "svla_set_wait_limit_ns": (None, [ctypes.c_uint64]),
    "svla_set_denoise_path": (_I, [_P, _I]),
    "svla_assembly_blob_bytes": (ctypes.c_size_t, [_I, _I, _I, _I]),
    "svla_set_assembly": (_I, [_P, _P, ctypes.c_size_t, _I, _I, _I, _I, _I]),
    "svla_assemble_prefix": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _P, _P, _P]),
    "svla_denoise_fused_supported": (_I, [_P, _I, _I]),
    "svla_op_quantize_affine8": (_I, [_P, _I, _I, _I, _P, _I, _P, _P]),
    "svla_op_gemm_w8": (_I, [_I, _P, _I, _P, _I, _P, _P, _I, _I, _I, _P, _I, _P, _I, _P, _P]),
    "svla_op_gemm_w8_splits": (_I, [_I, _I, _I]),
    "svla_op_gemm_w8_tile_n": (_I, [_I, _I, _I]),
}

DENOISE_AUTO, DENOISE_GRAPH, DENOISE_FUSED = 0, 1, 2
CREATE_PREFIX_INT8 = 1
CREATE_TRAIN = 2
CREATE_EXPERT_INT8 = 4

_lib = None


def load() -> ctypes.CDLL:
    """Load libsvla.so and declare its signatures (once)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"libsvla.so not found at {LIB_PATH}; build it with "
                "`python -m vision_language_action_b200.build` (needs nvcc)")
        lib = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _lib = lib
    return _lib


class SvlaError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"{STATUS.get(status, status)}: {msg}")
        self.status = status


def check(status: int, handle=None) -> None:
    if status != SVLA_OK:
        lib = load()
        msg = lib.svla_last_error(handle)
        raise SvlaError(status, msg.decode() if msg else "")
