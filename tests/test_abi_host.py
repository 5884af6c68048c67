"""C-ABI checks that need no GPU: the library loads, exports every symbol the
header declares, and rejects bad arguments on the host before any CUDA work."""
import ctypes
import os
import re

import numpy as np
import pytest

import synth
from vision_language_action_b200 import _abi
from vision_language_action_b200.runtime import config_from_shape

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_symbols():
    src = open(os.path.join(ROOT, "include", "svla.h")).read()
    return sorted(set(re.findall(r"SVLA_API\s+[\w\s\*]+?\b(svla_\w+)\s*\(", src)))


def test_library_exports_every_declared_symbol():
    lib = _abi.load()
    declared = _declared_symbols()
    assert len(declared) >= 16
    for name in declared:
        assert hasattr(lib, name), name
        assert name in _abi.SIGNATURES, f"binding lacks {name}"


def test_status_strings():
    lib = _abi.load()
    for code, name in _abi.STATUS.items():
        assert lib.svla_status_string(code).decode() == name


@pytest.mark.parametrize("shape", ["tiny", "smolvla"])
def test_blob_bytes_matches_manifest(shape):
    lib = _abi.load()
    s = synth.SHAPES[shape]
    cfg = config_from_shape(s, 1, 8, 8)
    n = sum(int(np.prod(shp)) for _, shp in synth.manifest(s))
    assert lib.svla_blob_bytes(ctypes.byref(cfg)) == 2 * n


def test_create_rejects_wrong_blob_size_before_touching_the_gpu():
    lib = _abi.load()
    s = synth.SHAPES["tiny"]
    cfg = config_from_shape(s, 1, 24, 8)
    n = lib.svla_blob_bytes(ctypes.byref(cfg))
    blob = np.zeros(n // 2 + 4, np.uint16)
    h = ctypes.c_void_p()
    for nbytes in (n - 2, n + 2, 0):
        st = lib.svla_create(ctypes.byref(cfg), ctypes.c_void_p(blob.ctypes.data), nbytes, 0, ctypes.byref(h))
        assert st == _abi.SVLA_ERR_BLOB_SIZE
        assert h.value is None
        assert b"manifest" in lib.svla_last_error(None)


def test_create_rejects_bad_config():
    lib = _abi.load()
    s = synth.SHAPES["tiny"]
    blob = np.zeros(16, np.uint16)
    h = ctypes.c_void_p()
    for bad in (dict(head_dim=48), dict(p_kv_heads=3), dict(action_dim=100), dict(e_layers=3),
                dict(p_ffn=100), dict(rms_eps=0.0)):
        cfg = config_from_shape(s.replace(**bad), 1, 24, 8)
        st = lib.svla_create(ctypes.byref(cfg), ctypes.c_void_p(blob.ctypes.data), 32, 0, ctypes.byref(h))
        assert st == _abi.SVLA_ERR_SHAPE, bad
    cfg = config_from_shape(s, 0, 24, 8)
    assert lib.svla_create(ctypes.byref(cfg), ctypes.c_void_p(blob.ctypes.data), 32, 0,
                           ctypes.byref(h)) == _abi.SVLA_ERR_SHAPE
    assert lib.svla_create(None, None, 0, 0, ctypes.byref(h)) == _abi.SVLA_ERR_ARG


def test_null_handle_calls_fail_cleanly():
    lib = _abi.load()
    assert lib.svla_prefill(None, None, None, 1, 1, None, None) == _abi.SVLA_ERR_ARG
    assert lib.svla_denoise(None, None, None, 1, 1, None, 1, 1, None, None, None) == _abi.SVLA_ERR_ARG
    assert lib.svla_device_status(None, None) == _abi.SVLA_ERR_ARG
    assert lib.svla_kv_cache_bytes(None, 1, 1) == 0
    assert lib.svla_destroy(None) == _abi.SVLA_OK


def test_op_argument_checks():
    lib = _abi.load()
    p = ctypes.c_void_p(16)
    # unknown epilogue, bad strides, misaligned pointers: rejected before any launch
    assert lib.svla_op_gemm(9, p, 64, p, 64, 4, 4, 64, p, 4, None, 0, None, 0, None, None) == _abi.SVLA_ERR_ARG
    assert lib.svla_op_gemm(0, p, 60, p, 64, 4, 4, 64, p, 4, None, 0, None, 0, None, None) == _abi.SVLA_ERR_SHAPE
    assert lib.svla_op_gemm(0, ctypes.c_void_p(18), 64, p, 64, 4, 4, 64, p, 4, None, 0, None, 0, None,
                            None) == _abi.SVLA_ERR_ARG
    assert lib.svla_op_attention(p, 64, p, p, 64, None, 1, 3, 2, 64, 1, 1, 0, p, 64, None) == _abi.SVLA_ERR_SHAPE
    assert lib.svla_op_attention(p, 64, p, p, 64, None, 1, 1, 1, 48, 1, 1, 0, p, 64, None) == _abi.SVLA_ERR_SHAPE
    assert lib.svla_op_rmsnorm(ctypes.c_void_p(16), p, 1, 6, 1e-5, p, None) == _abi.SVLA_ERR_SHAPE


def test_gemm_plan_workspace_rules():
    lib = _abi.load()
    # large M: one split, no workspace
    assert lib.svla_op_gemm_splits(12800, 4096, 720) == 1
    assert lib.svla_op_gemm_workspace_bytes(12800, 4096, 720, 0) == 0
    # batch-1 shapes split K over a cluster of at most 8 CTAs to cover the SMs,
    # never more splits than K blocks; cluster reductions need no workspace
    for (M, N, K) in [(50, 720, 2048), (50, 4096, 720), (50, 1600, 720), (1, 320, 64), (177, 960, 960)]:
        sp = lib.svla_op_gemm_splits(M, N, K)
        assert 1 <= sp <= min(8, (K + 63) // 64)
        assert lib.svla_op_gemm_workspace_bytes(M, N, K, 0) == 0
    assert lib.svla_op_gemm_splits(50, 720, 2048) > 1
    assert lib.svla_op_gemm_workspace_bytes(50, 720, 2048, 1) == 0
    # more than 8 forced splits reduce through a global workspace
    assert lib.svla_op_gemm_workspace_bytes(50, 720, 2048, 16) > 0


@pytest.mark.parametrize("shape", ["tiny", "smolvla"])
def test_assembly_blob_bytes_and_null_handle(shape):
    lib = _abi.load()
    s = synth.SHAPES[shape]
    a = synth.ASSEMBLY_SHAPES[shape]
    n = sum(int(np.prod(shp)) for _, shp in synth.assembly_manifest(a, s.p_width))
    assert lib.svla_assembly_blob_bytes(s.p_width, a.vis_width, a.shuffle, a.state_dim) == 2 * n
    assert lib.svla_assembly_blob_bytes(0, a.vis_width, a.shuffle, a.state_dim) == 0
    assert lib.svla_set_assembly(None, None, 0, 8, 8, 2, 8, 1) == _abi.SVLA_ERR_ARG
    assert lib.svla_assemble_prefix(None, None, None, None, None, 1, 1, 0, None, None, None) == _abi.SVLA_ERR_ARG


def test_int8_argument_checks_and_plan():
    lib = _abi.load()
    p = ctypes.c_void_p(16)
    s = synth.SHAPES["tiny"]
    blob = np.zeros(16, np.uint16)
    h = ctypes.c_void_p()
    cfg = config_from_shape(s, 1, 24, 8)
    assert lib.svla_create_ex(ctypes.byref(cfg), ctypes.c_void_p(blob.ctypes.data), 32, 0, 8,
                              ctypes.byref(h)) == _abi.SVLA_ERR_ARG
    cfg = config_from_shape(s.replace(p_heads=3, p_kv_heads=1), 1, 24, 8)  # O projection K = 96
    assert lib.svla_create_ex(ctypes.byref(cfg), ctypes.c_void_p(blob.ctypes.data), 32, 0,
                              _abi.CREATE_PREFIX_INT8, ctypes.byref(h)) == _abi.SVLA_ERR_SHAPE
    assert lib.svla_set_prefix_weights(None, 8) == _abi.SVLA_ERR_ARG
    assert lib.svla_prefix_weights(None) == 0
    assert lib.svla_set_expert_weights(None, 8) == _abi.SVLA_ERR_ARG
    assert lib.svla_expert_weights(None) == 0
    # quantiser: K a multiple of 16 (a ragged last group of K mod 64 inputs), aligned pointers
    assert lib.svla_op_quantize_affine8(p, 88, 4, 88, p, 88, p, None) == _abi.SVLA_ERR_SHAPE
    assert lib.svla_op_quantize_affine8(p, 8, 4, 8, p, 8, p, None) == _abi.SVLA_ERR_SHAPE
    assert lib.svla_op_quantize_affine8(None, 64, 4, 64, p, 64, p, None) == _abi.SVLA_ERR_ARG
    assert lib.svla_op_quantize_affine8(ctypes.c_void_p(18), 64, 4, 64, p, 64, p, None) == _abi.SVLA_ERR_ARG
    # int8 GEMM: epilogue, K % 16, N % 8, splits <= 8, 16-byte alignment
    args = lambda **kw: dict(dict(epi=0, lda=64, ldq=64, g=None, M=4, N=8, K=64, ldc=8, sp=0), **kw)
    def call(a):
        return lib.svla_op_gemm_w8(a["epi"], p, a["lda"], p, a["ldq"], p, a["g"], a["M"], a["N"], a["K"], p,
                                   a["ldc"], None, a["sp"], None, None)
    assert call(args(epi=9)) == _abi.SVLA_ERR_ARG
    assert call(args(K=40, lda=40, ldq=48)) == _abi.SVLA_ERR_SHAPE
    assert call(args(N=12, ldc=12)) == _abi.SVLA_ERR_SHAPE
    assert call(args(sp=9)) == _abi.SVLA_ERR_SHAPE
    assert call(args(ldq=72)) == _abi.SVLA_ERR_SHAPE
    assert call(args(g=ctypes.c_void_p(24))) == _abi.SVLA_ERR_ARG
    # at the batch-1 prefill's shapes the int8 plan splits K like the dense plan
    # (same partial-sum order); large M takes 128-wide tiles without a split
    for (M, N, K) in [(177, 1600, 960), (177, 960, 960), (177, 5120, 960), (177, 960, 2560), (354, 960, 2560)]:
        assert lib.svla_op_gemm_w8_splits(M, N, K) == lib.svla_op_gemm_splits(M, N, K), (M, N, K)
    assert lib.svla_op_gemm_w8_splits(5664, 5120, 960) == 1
    # ragged K (the expert's 720 = 11 x 64 + 16) plans like any other width
    assert lib.svla_op_gemm_w8_splits(1600, 4096, 720) == 1
    assert lib.svla_op_gemm_w8_splits(50, 1600, 720) >= 1
    assert lib.svla_op_gemm_w8_splits(50, 1600, 40) == 0
    assert lib.svla_op_gemm_w8_tile_n(5664, 5120, 960) == 128
    assert lib.svla_op_gemm_w8_splits(177, 1600, 100) == 0


def test_train_argument_checks():
    lib = _abi.load()
    assert lib.svla_train_grad_elems(None) == 0
    p = ctypes.c_void_p(16)
    assert lib.svla_train_step(None, p, p, 1, 1, p, p, p, 1, p, p, None) == _abi.SVLA_ERR_ARG
    s = synth.SHAPES["tiny"]
    blob = np.zeros(16, np.uint16)
    h = ctypes.c_void_p()
    cfg = config_from_shape(s, 1, 24, 8)
    # unknown flag bits are rejected before the blob size
    assert lib.svla_create_ex(ctypes.byref(cfg), ctypes.c_void_p(blob.ctypes.data), 32, 0, 8,
                              ctypes.byref(h)) == _abi.SVLA_ERR_ARG
    assert lib.svla_create_ex(ctypes.byref(cfg), ctypes.c_void_p(blob.ctypes.data), 32, 0, _abi.CREATE_TRAIN,
                              ctypes.byref(h)) == _abi.SVLA_ERR_BLOB_SIZE


def test_op_wrappers_refuse_host_tensors():
    """The kernel-level wrappers marshal device tensors only: host tensors fail loudly
    (there is no CPU fallback)."""
    import torch
    from vision_language_action_b200 import runtime as rt
    A = torch.zeros(4, 64, dtype=torch.bfloat16)
    W = torch.zeros(8, 64, dtype=torch.bfloat16)
    C = torch.zeros(4, 8)
    with pytest.raises(ValueError):
        rt.op_gemm("f32", A, W, C)
    with pytest.raises(ValueError):
        rt.op_quantize_affine8(W)
    with pytest.raises(ValueError):
        rt.op_rmsnorm(C, torch.zeros(8, dtype=torch.bfloat16), torch.zeros(4, 8, dtype=torch.bfloat16))
