"""svla_op_gemm_noalloc: the GEMM entry point for callers that cannot allocate
GPU memory (a control loop that forbids cudaMalloc after start-up, a host that
owns all device memory through its own pool, a plain-C caller without an
allocator). It must give the same result as svla_op_gemm with a caller-owned
workspace, call after call, since every call reuses the library's one static
scratch array.

This file is named so that pytest collects it last.
"""
import ctypes

import pytest

torch = pytest.importorskip("torch")

from vision_language_action_b200 import _abi  # noqa: E402

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

DEV = "cuda:0"


def P(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else None


def S():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def with_workspace(epi, A, W, C, bias, splits):
    lib = _abi.load()
    M, K = A.shape
    N = W.shape[0]
    nbytes = lib.svla_op_gemm_workspace_bytes(M, N, K, splits)
    ws = torch.zeros(max(nbytes, 16), dtype=torch.uint8, device=DEV)
    _abi.check(lib.svla_op_gemm(epi, P(A), K, P(W), K, M, N, K, P(C), C.stride(0), P(bias), splits, P(ws), nbytes,
                                None, S()))
    torch.cuda.synchronize()


def without_workspace(epi, A, W, C, bias, splits, status):
    lib = _abi.load()
    M, K = A.shape
    N = W.shape[0]
    _abi.check(lib.svla_op_gemm_noalloc(epi, P(A), K, P(W), K, M, N, K, P(C), C.stride(0), P(bias), splits,
                                        P(status), S()))
    torch.cuda.synchronize()


# batch-1 shapes of the path with more K splits than one cluster holds: the
# partial tiles go through the scratch (global-memory reduction)
@pytest.mark.parametrize("M,N,K,splits", [(50, 720, 2048, 16), (50, 960, 720, 12), (64, 320, 2048, 16),
                                          (50, 1600, 720, 9)])
@pytest.mark.parametrize("epi", [_abi.EPI_F32, _abi.EPI_ADD_F32, _abi.EPI_BF16])
def test_noalloc_matches_workspace_entry_point_twice(M, N, K, splits, epi):
    lib = _abi.load()
    assert 0 < lib.svla_op_gemm_workspace_bytes(M, N, K, splits) <= 8 << 20
    g = torch.Generator(device="cpu").manual_seed(M + N + K + epi)
    A = torch.randn(M, K, generator=g).to(torch.bfloat16).to(DEV)
    W = (0.05 * torch.randn(N, K, generator=g)).to(torch.bfloat16).to(DEV)
    bias = torch.randn(N, generator=g).to(DEV)
    dt = torch.bfloat16 if epi == _abi.EPI_BF16 else torch.float32
    R0 = torch.randn(M, N, generator=g).to(DEV).to(dt)
    ref = R0.clone()
    with_workspace(epi, A, W, ref, bias, splits)
    scale = (A.double().abs() @ W.double().abs().T) + bias.double().abs() + R0.double().abs()
    tol = 1e-5 * scale + 1e-6 if epi != _abi.EPI_BF16 else 2 ** -8 * scale + 1e-4
    # float64 reference of the same contraction (fp32 accumulation of K products)
    exact = A.double() @ W.double().T + bias.double()
    if epi == _abi.EPI_ADD_F32:
        exact = exact + R0.double()
    assert ((ref.double() - exact).abs() <= tol).all()
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    for _ in range(2):   # two calls in a row share (and must re-arm) the static scratch
        out = R0.clone()
        without_workspace(epi, A, W, out, bias, splits, status)
        assert status.item() == 0
        # same plan, same split order: the partial sums are added in the same
        # order as with a caller-owned workspace, so the result is bit for bit equal
        assert torch.equal(out, ref)
        assert ((out.double() - exact).abs() <= tol).all()


def test_noalloc_rejects_plans_larger_than_its_scratch():
    lib = _abi.load()
    M, N, K, splits = 1600, 4096, 720, 8
    assert lib.svla_op_gemm_workspace_bytes(M, N, K, splits) > 8 << 20
    p = ctypes.c_void_p(256)
    st = lib.svla_op_gemm_noalloc(_abi.EPI_F32, p, K, p, K, M, N, K, p, N, None, splits, None, None)
    assert st == _abi.SVLA_ERR_SHAPE
    assert b"scratch" in lib.svla_last_error(None)
