"""Single kernels of the path through the C ABI, against float64 references of
the same operation at awkward shapes (ragged tiles, tiny and large M, masks)."""
import ctypes

import numpy as np
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


def gemm(epi, A, W, C, bias=None, splits=0, status=None):
    lib = _abi.load()
    M, K = A.shape
    N = W.shape[0]
    ws_bytes = lib.svla_op_gemm_workspace_bytes(M, N, K, splits)
    ws = torch.zeros(max(ws_bytes, 16), dtype=torch.uint8, device=DEV)
    st = lib.svla_op_gemm(epi, P(A), A.stride(0), P(W), W.stride(0), M, N, K, P(C), C.stride(0), P(bias),
                          splits, P(ws), ws_bytes, P(status), S())
    _abi.check(st)
    return ws


SHAPES = [
    (1, 320, 64), (50, 720, 960), (50, 1600, 720), (63, 960, 720), (64, 320, 320), (65, 720, 2048),
    (177, 1600, 960), (177, 960, 2560), (1600, 4096, 720), (1600, 720, 2048), (300, 96, 128),
    (513, 720, 960), (2568, 1600, 960), (5664, 5120, 960),
]


@pytest.mark.parametrize("M,N,K", SHAPES)
@pytest.mark.parametrize("splits", [0, 1, 3])
def test_gemm_f32_matches_fp64(M, N, K, splits):
    g = torch.Generator(device="cpu").manual_seed(M * 7 + N * 3 + K)
    A = torch.randn(M, K, generator=g).to(torch.bfloat16).to(DEV)
    W = (0.05 * torch.randn(N, K, generator=g)).to(torch.bfloat16).to(DEV)
    bias = torch.randn(N, generator=g).to(DEV)
    C = torch.full((M, N), float("nan"), device=DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    gemm(_abi.EPI_F32, A, W, C, bias, splits, status)
    torch.cuda.synchronize()
    ref = A.double() @ W.double().T + bias.double()
    scale = A.double().abs() @ W.double().abs().T
    err = (C.double() - ref).abs()
    assert status.item() == 0
    assert torch.isfinite(C).all()
    assert (err <= 1e-5 * scale + 1e-6).all(), float((err / (scale + 1e-9)).max())


@pytest.mark.parametrize("M,N,K", [(50, 720, 2048), (1600, 4096, 720), (177, 1600, 960)])
def test_gemm_epilogues(M, N, K):
    g = torch.Generator(device="cpu").manual_seed(3)
    A = torch.randn(M, K, generator=g).to(torch.bfloat16).to(DEV)
    W = (0.05 * torch.randn(N, K, generator=g)).to(torch.bfloat16).to(DEV)
    bias = torch.randn(N, generator=g).to(DEV)
    acc = A.double() @ W.double().T + bias.double()
    # bf16 store
    Cb = torch.empty(M, N, dtype=torch.bfloat16, device=DEV)
    gemm(_abi.EPI_BF16, A, W, Cb, bias)
    # residual add
    R0 = torch.randn(M, N, generator=g).to(DEV)
    R = R0.clone()
    gemm(_abi.EPI_ADD_F32, A, W, R, bias)
    # silu
    Cs = torch.empty(M, N, dtype=torch.bfloat16, device=DEV)
    gemm(_abi.EPI_SILU_BF16, A, W, Cs, bias)
    torch.cuda.synchronize()
    assert ((Cb.double() - acc).abs() <= 2 ** -8 * acc.abs() + 1e-4).all()
    np.testing.assert_allclose(R.double().cpu(), (R0.double() + acc).cpu(), rtol=1e-5, atol=1e-4)
    silu = acc * torch.sigmoid(acc)
    assert ((Cs.double() - silu).abs() <= 2 ** -7 * silu.abs() + 1e-3).all()


def _offset(shape, dtype, elems, fill):
    """A contiguous [M, N] view whose first element sits `elems` elements past a fresh allocation."""
    M, N = shape
    store = torch.full((M * N + elems,), fill, dtype=dtype, device=DEV)
    return store[elems:].view(M, N)


@pytest.mark.parametrize("M,N,K", [(50, 720, 2048), (177, 960, 720), (1600, 720, 960), (4096, 720, 2048),
                                   (1600, 4096, 720), (300, 96, 128)])
def test_gemm_outputs_at_16_byte_offsets_match_aligned(M, N, K):
    """The epilogue moves 32 bytes per access where the address allows it and 16 otherwise: outputs
    (and residuals) that start 16 bytes past a 32-byte boundary give the same bits."""
    g = torch.Generator(device="cpu").manual_seed(M + N + K)
    A = torch.randn(M, K, generator=g).to(torch.bfloat16).to(DEV)
    W = (0.05 * torch.randn(N, K, generator=g)).to(torch.bfloat16).to(DEV)
    bias = torch.randn(N, generator=g).to(DEV)
    R0 = torch.randn(M, N, generator=g).to(DEV)
    out = {}
    for off in (0, 1):
        Cf = _offset((M, N), torch.float32, 4 * off, float("nan"))
        Cb = _offset((M, N), torch.bfloat16, 8 * off, float("nan"))
        R = _offset((M, N), torch.float32, 4 * off, 0.0)
        R.copy_(R0)
        assert Cf.data_ptr() % 32 == 16 * off and Cb.data_ptr() % 32 == 16 * off and R.data_ptr() % 32 == 16 * off
        gemm(_abi.EPI_F32, A, W, Cf, bias)
        gemm(_abi.EPI_BF16, A, W, Cb, bias)
        gemm(_abi.EPI_ADD_F32, A, W, R, bias)
        torch.cuda.synchronize()
        out[off] = (Cf.clone(), Cb.clone(), R.clone())
    for a, b in zip(out[0], out[1]):
        assert torch.equal(a.view(torch.int16) if a.dtype == torch.bfloat16 else a.view(torch.int32),
                           b.view(torch.int16) if b.dtype == torch.bfloat16 else b.view(torch.int32))
    ref = A.double() @ W.double().T + bias.double()
    np.testing.assert_allclose(out[1][2].double().cpu(), (R0.double() + ref).cpu(), rtol=1e-5, atol=1e-4)


@pytest.mark.parametrize("splits", [2, 5, 8, 16])
def test_gemm_split_k_is_deterministic(splits):
    """<= 8 splits reduce across a thread-block cluster, more through the global
    workspace; both sum the splits in a fixed order."""
    g = torch.Generator(device="cpu").manual_seed(11)
    A = torch.randn(50, 2048, generator=g).to(torch.bfloat16).to(DEV)
    W = (0.05 * torch.randn(720, 2048, generator=g)).to(torch.bfloat16).to(DEV)
    outs = []
    for _ in range(3):
        C = torch.empty(50, 720, device=DEV)
        gemm(_abi.EPI_F32, A, W, C, None, splits)
        outs.append(C)
    torch.cuda.synchronize()
    assert torch.equal(outs[0], outs[1]) and torch.equal(outs[0], outs[2])
    ref = A.double() @ W.double().T
    assert ((outs[0].double() - ref).abs() <= 1e-5 * (A.double().abs() @ W.double().abs().T) + 1e-6).all()


@pytest.mark.parametrize("M,splits", [(256, 1), (50, 4), (50, 12)])
def test_gemm_timeout_path_reports_and_recovers(M, splits):
    """A wait limit of 0 makes the first unsatisfied wait give up: the kernel
    records SVLA_ERR_TIMEOUT, drains its copies, still meets every cluster
    barrier, frees its tensor memory and returns; the context stays usable."""
    lib = _abi.load()
    g = torch.Generator(device="cpu").manual_seed(5)
    A = torch.randn(M, 960, generator=g).to(torch.bfloat16).to(DEV)
    W = (0.05 * torch.randn(960, 960, generator=g)).to(torch.bfloat16).to(DEV)
    C = torch.zeros(M, 960, device=DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    try:
        lib.svla_set_wait_limit_ns(0)
        gemm(_abi.EPI_F32, A, W, C, None, splits, status)
        torch.cuda.synchronize()
    finally:
        lib.svla_set_wait_limit_ns(1_000_000_000)
    assert status.item() == _abi.SVLA_ERR_TIMEOUT
    status.zero_()
    gemm(_abi.EPI_F32, A, W, C, None, splits, status)
    torch.cuda.synchronize()
    assert status.item() == 0
    ref = A.double() @ W.double().T
    assert torch.allclose(C.double(), ref, rtol=1e-4, atol=1e-4)


@pytest.mark.parametrize("splits", [12, 16])
def test_gemm_timeout_leaves_the_global_counters_zeroed(splits):
    """More than 8 splits reduce through the caller's workspace with one arrival
    counter per tile. A CTA aborted by a wait that ran out still takes its turn
    on that counter, so after the failed launch every counter is back at zero
    and the next launch on the same workspace is correct."""
    lib = _abi.load()
    g = torch.Generator(device="cpu").manual_seed(9)
    M, N, K = 50, 720, 2048
    A = torch.randn(M, K, generator=g).to(torch.bfloat16).to(DEV)
    W = (0.05 * torch.randn(N, K, generator=g)).to(torch.bfloat16).to(DEV)
    ws_bytes = lib.svla_op_gemm_workspace_bytes(M, N, K, splits)
    assert ws_bytes > 0
    ws = torch.zeros(ws_bytes, dtype=torch.uint8, device=DEV)
    # the workspace starts with one int counter per output tile, padded to 256
    # bytes: M = 50 and N = 720 give fewer than 64 tiles at any tile width

    def run(C, status):
        _abi.check(lib.svla_op_gemm(_abi.EPI_F32, P(A), K, P(W), K, M, N, K, P(C), N, None, splits, P(ws),
                                    ws_bytes, P(status), S()))

    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    C = torch.zeros(M, N, device=DEV)
    try:
        lib.svla_set_wait_limit_ns(0)
        run(C, status)
        torch.cuda.synchronize()
    finally:
        lib.svla_set_wait_limit_ns(1_000_000_000)
    assert status.item() == _abi.SVLA_ERR_TIMEOUT
    assert int(ws[:256].view(torch.int32).abs().sum().item()) == 0
    status.zero_()
    run(C, status)
    torch.cuda.synchronize()
    assert status.item() == 0
    ref = A.double() @ W.double().T
    assert ((C.double() - ref).abs() <= 1e-5 * (A.double().abs() @ W.double().abs().T) + 1e-6).all()


# ---------------------------------------------------------------------------
# attention
# ---------------------------------------------------------------------------
def attn_ref(q, k, v, valid, nq, nkv, hd, causal):
    B, Lq, _ = q.shape
    Lk = k.shape[1]
    qd = q.double().view(B, Lq, nq, hd).transpose(1, 2)
    kd = k.double().view(B, Lk, nkv, hd).transpose(1, 2).repeat_interleave(nq // nkv, dim=1)
    vd = v.double().view(B, Lk, nkv, hd).transpose(1, 2).repeat_interleave(nq // nkv, dim=1)
    s = qd @ kd.transpose(-1, -2) / hd ** 0.5
    mask = torch.ones(B, 1, Lq, Lk, dtype=torch.bool, device=q.device)
    if valid is not None:
        mask &= valid.bool()[:, None, None, :]
    if causal:
        mask &= torch.ones(Lq, Lk, dtype=torch.bool, device=q.device).tril()[None, None]
    s = s.masked_fill(~mask, float("-inf"))
    o = torch.softmax(s, -1) @ vd
    return o.transpose(1, 2).reshape(B, Lq, nq * hd)


def run_attn(q, k, v, valid, nq, nkv, hd, causal):
    lib = _abi.load()
    B, Lq, _ = q.shape
    Lk = k.shape[1]
    out = torch.full((B, Lq, nq * hd), float("nan"), dtype=torch.bfloat16, device=DEV)
    st = lib.svla_op_attention(P(q), q.stride(1), P(k), P(v), k.stride(1), P(valid), B, nq, nkv, hd, Lq, Lk,
                               int(causal), P(out), out.stride(1), S())
    _abi.check(st)
    torch.cuda.synchronize()
    return out


@pytest.mark.parametrize("hd,nq,nkv", [(64, 15, 5), (32, 4, 2)])
@pytest.mark.parametrize("Lq,Lk,causal,maskkind", [
    (50, 50, True, None), (1, 1, False, None), (7, 2, False, None), (50, 177, False, "holes"),
    (177, 177, False, "holes"), (50, 321, False, "tail"), (130, 145, False, "one"), (100, 100, True, None),
    (64, 65, False, "one_last"),
])
def test_attention_matches_fp64(hd, nq, nkv, Lq, Lk, causal, maskkind):
    g = torch.Generator(device="cpu").manual_seed(Lq * 1000 + Lk)
    B = 3
    # sharpened q/k so a wrong mask or an off-by-one key shows up well above tolerance
    q = (3 * torch.randn(B, Lq, nq * hd, generator=g)).to(torch.bfloat16).to(DEV)
    k = (3 * torch.randn(B, Lk, nkv * hd, generator=g) / hd ** 0.25).to(torch.bfloat16).to(DEV)
    v = torch.randn(B, Lk, nkv * hd, generator=g).to(torch.bfloat16).to(DEV)
    valid = None
    if maskkind is not None:
        vm = torch.ones(B, Lk, dtype=torch.uint8)
        if maskkind == "holes":
            vm[:, 3:9] = 0
            vm[1, Lk // 2:Lk // 2 + 20] = 0
            vm[2, :Lk - 5] = 0
        elif maskkind == "tail":
            vm[0, Lk - 31:] = 0
            vm[2, Lk - 1:] = 0
        elif maskkind == "one":
            vm[:] = 0
            vm[:, 17] = 1
        elif maskkind == "one_last":
            vm[:] = 0
            vm[:, Lk - 1] = 1
        valid = vm.to(DEV)
    out = run_attn(q, k, v, valid, nq, nkv, hd, causal)
    ref = attn_ref(q, k, v, valid, nq, nkv, hd, causal)
    err = (out.double() - ref).abs().max().item()
    assert err < 2e-2, err
    if maskkind in ("one", "one_last"):
        # a single visible key: the output is that key's v (bf16 exact up to p = 1 rounding)
        j = 17 if maskkind == "one" else Lk - 1
        vv = v.view(B, Lk, nkv, hd)[:, j].repeat_interleave(nq // nkv, dim=1).reshape(B, nq * hd)
        assert torch.equal(out, vv[:, None, :].expand_as(out))


def test_attention_first_causal_row_returns_own_v():
    g = torch.Generator(device="cpu").manual_seed(9)
    q = (3 * torch.randn(2, 50, 960, generator=g)).to(torch.bfloat16).to(DEV)
    k = torch.randn(2, 50, 320, generator=g).to(torch.bfloat16).to(DEV)
    v = torch.randn(2, 50, 320, generator=g).to(torch.bfloat16).to(DEV)
    out = run_attn(q, k, v, None, 15, 5, 64, True)
    v0 = v.view(2, 50, 5, 64)[:, 0].repeat_interleave(3, dim=1).reshape(2, 960)
    assert torch.equal(out[:, 0], v0)


@pytest.mark.parametrize("M,D", [(1, 960), (50, 720), (177, 960), (1000, 128), (3, 96)])
def test_rmsnorm(M, D):
    lib = _abi.load()
    g = torch.Generator(device="cpu").manual_seed(M + D)
    x = torch.randn(M, D, generator=g).to(DEV) * 3
    w = (1 + 0.1 * torch.randn(D, generator=g)).to(torch.bfloat16).to(DEV)
    y = torch.empty(M, D, dtype=torch.bfloat16, device=DEV)
    _abi.check(lib.svla_op_rmsnorm(P(x), P(w), M, D, 1e-5, P(y), S()))
    torch.cuda.synchronize()
    xd = x.double()
    ref = xd / torch.sqrt((xd * xd).mean(-1, keepdim=True) + 1e-5) * w.double()
    assert ((y.double() - ref).abs() <= 2 ** -8 * ref.abs() + 1e-6).all()
