"""Weight-only int8 prefix (the vlm-8bit preset of the mlx-smolvla PyPI page,
§Run a checkpoint) through the C ABI.

* The quantiser's codes and scales bit for bit against the oracle's.
* The int8 GEMM (codes from the oracle) against a float64 product with the
  dequantised weights, at ragged, split and large shapes, and bit for bit
  against the dense GEMM on the dequantised weights where both take the same
  plan (the batch-1 prefill's shapes).
* The int8 prefill and the chunk after it against the oracle run on the
  dequantised model (readings 22-24), and bit for bit against the dense
  prefill given the dequantised weights.
"""
import ctypes

import numpy as np
import pytest

torch = pytest.importorskip("torch")

import oracle  # noqa: E402
import synth  # noqa: E402
from oracle import quant as oq  # noqa: E402
from tests import helpers as H  # noqa: E402
from vision_language_action_b200 import _abi  # noqa: E402
from vision_language_action_b200.runtime import SmolVLA  # noqa: E402

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

DEV = "cuda:0"


def P(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else None


def S():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def bf16_dev(x_f32: np.ndarray) -> torch.Tensor:
    """float32 values that are bf16 values -> device bf16 tensor (same bits)."""
    bits = synth.f32_to_bf16_bits(np.asarray(x_f32, np.float32))
    return torch.from_numpy(bits.view(np.int16)).to(DEV).view(torch.bfloat16)


def weight_matrix(seed, N, K):
    """bf16 weights ~N(0, 0.02) with a few outliers, one narrow offset group and
    one constant group (the degenerate case alpha = 0)."""
    rng = np.random.default_rng(seed)
    w = 0.02 * rng.standard_normal((N, K)).astype(np.float32)
    w[rng.integers(0, N, 4), rng.integers(0, K, 4)] = 0.4
    w[0, :64] = 0.01 + 1e-4 * rng.standard_normal(64)
    if N > 1:
        w[1, K - 64:] = -0.03125
    return synth.bf16_bits_to_f32(synth.f32_to_bf16_bits(w)).astype(np.float32)


def pairs_dev(alpha, beta) -> torch.Tensor:
    """(alpha, beta) [N, G] -> device bf16 [G, N, 2]."""
    ab = np.stack([alpha.T, beta.T], axis=-1).astype(np.float32)
    return bf16_dev(ab)


def effective_weight(q, alpha, beta, gain=None) -> np.ndarray:
    """The GEMM operand: bf16(w^ * g) with w^ = bf16(alpha q + beta) (the float32
    product of two bf16 values is exact)."""
    wh = oq.dequantize_affine8(q, alpha, beta).astype(np.float32)
    if gain is None:
        return wh
    return oq._bf16_rne(wh * gain[None, :].astype(np.float32))


@pytest.mark.parametrize("N,K", [(1600, 960), (960, 2560), (5120, 960), (8, 64), (3, 128)])
def test_quantizer_matches_oracle_bit_for_bit(N, K):
    lib = _abi.load()
    w = weight_matrix(N + K, N, K)
    q_ref, a_ref, b_ref = oq.quantize_affine8(w)
    W = bf16_dev(w)
    q = torch.empty((N, K), dtype=torch.uint8, device=DEV)
    ab = torch.empty((K // 64, N, 2), dtype=torch.int16, device=DEV)
    _abi.check(lib.svla_op_quantize_affine8(P(W), K, N, K, P(q), K, P(ab), S()))
    torch.cuda.synchronize()
    assert np.array_equal(q.cpu().numpy(), q_ref)
    abn = ab.cpu().numpy().view(np.uint16)
    assert np.array_equal(abn[..., 0].T, synth.f32_to_bf16_bits(a_ref))
    assert np.array_equal(synth.bf16_bits_to_f32(abn[..., 1].T), b_ref)


def gemm_w8(epi, A, q, ab, gain, C, bias=None, splits=0, status=None):
    lib = _abi.load()
    M, K = A.shape
    N = q.shape[0]
    st = lib.svla_op_gemm_w8(epi, P(A), A.stride(0), P(q), q.stride(0), P(ab), P(gain), M, N, K, P(C), C.stride(0),
                             P(bias), splits, P(status), S())
    _abi.check(st)


def w8_operands(seed, N, K, with_gain):
    w = weight_matrix(seed, N, K)
    q, a, b = oq.quantize_affine8(w)
    rng = np.random.default_rng(seed + 1)
    gain = None
    if with_gain:
        gain = synth.bf16_bits_to_f32(synth.f32_to_bf16_bits(
            (1.0 + 0.1 * rng.standard_normal(K)).astype(np.float32))).astype(np.float32)
    dev = dict(q=torch.from_numpy(q).to(DEV), ab=pairs_dev(a, b), gain=bf16_dev(gain) if with_gain else None)
    return dev, effective_weight(q, a, b, gain)


SHAPES = [
    (1, 320, 64), (50, 720, 960), (177, 1600, 960), (177, 960, 2560), (65, 736, 2048), (300, 96, 128),
    (513, 720, 960), (1600, 4096, 768), (5664, 5120, 960),
]


@pytest.mark.parametrize("M,N,K", SHAPES)
@pytest.mark.parametrize("splits", [0, 1, 3])
def test_gemm_w8_matches_fp64(M, N, K, splits):
    dev, w_eff = w8_operands(M + N + K, N, K, with_gain=(splits != 1))
    g = torch.Generator(device="cpu").manual_seed(M * 7 + N * 3 + K)
    A = torch.randn(M, K, generator=g).to(torch.bfloat16).to(DEV)
    bias = torch.randn(N, generator=g).to(DEV)
    C = torch.full((M, N), float("nan"), device=DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    gemm_w8(_abi.EPI_F32, A, dev["q"], dev["ab"], dev["gain"], C, bias, splits, status)
    torch.cuda.synchronize()
    Wd = torch.from_numpy(w_eff.astype(np.float64)).to(DEV)
    ref = A.double() @ Wd.T + bias.double()
    scale = A.double().abs() @ Wd.abs().T
    err = (C.double() - ref).abs()
    assert status.item() == 0
    assert torch.isfinite(C).all()
    assert (err <= 1e-5 * scale + 1e-6).all(), float((err / (scale + 1e-9)).max())


@pytest.mark.parametrize("M,N,K", [(177, 1600, 960), (177, 960, 2560), (177, 5120, 960), (177, 960, 960)])
@pytest.mark.parametrize("with_gain", [False, True])
def test_gemm_w8_bitwise_equals_dense_on_dequantised_weights(M, N, K, with_gain):
    """Same tile width and splits -> same partial-sum order: the int8 GEMM is the
    dense GEMM given bf16(w^ * g), bit for bit."""
    lib = _abi.load()
    assert lib.svla_op_gemm_w8_splits(M, N, K) == lib.svla_op_gemm_splits(M, N, K)
    dev, w_eff = w8_operands(3 * N + K, N, K, with_gain)
    g = torch.Generator(device="cpu").manual_seed(N + K)
    A = torch.randn(M, K, generator=g).to(torch.bfloat16).to(DEV)
    C8 = torch.empty(M, N, device=DEV)
    Cd = torch.empty(M, N, device=DEV)
    gemm_w8(_abi.EPI_F32, A, dev["q"], dev["ab"], dev["gain"], C8)
    W = bf16_dev(w_eff)
    _abi.check(lib.svla_op_gemm(_abi.EPI_F32, P(A), K, P(W), K, M, N, K, P(Cd), N, None, 0, None, 0, None, S()))
    torch.cuda.synchronize()
    assert torch.equal(C8, Cd)


@pytest.mark.parametrize("M,N,K", [(50, 720, 2048), (177, 1600, 960), (1600, 4096, 768)])
def test_gemm_w8_epilogues(M, N, K):
    dev, w_eff = w8_operands(11, N, K, with_gain=False)
    g = torch.Generator(device="cpu").manual_seed(5)
    A = torch.randn(M, K, generator=g).to(torch.bfloat16).to(DEV)
    bias = torch.randn(N, generator=g).to(DEV)
    acc = A.double() @ torch.from_numpy(w_eff.astype(np.float64)).to(DEV).T + bias.double()
    Cb = torch.empty(M, N, dtype=torch.bfloat16, device=DEV)
    gemm_w8(_abi.EPI_BF16, A, dev["q"], dev["ab"], None, Cb, bias)
    R0 = torch.randn(M, N, generator=g).to(DEV)
    R = R0.clone()
    gemm_w8(_abi.EPI_ADD_F32, A, dev["q"], dev["ab"], None, R, bias)
    Cs = torch.empty(M, N, dtype=torch.bfloat16, device=DEV)
    gemm_w8(_abi.EPI_SILU_BF16, A, dev["q"], dev["ab"], None, Cs, bias)
    torch.cuda.synchronize()
    tol = 1e-2 * acc.abs().max().item()
    assert (Cb.double() - acc).abs().max().item() <= tol
    assert (R.double() - (R0.double() + acc)).abs().max().item() <= 1e-4 * acc.abs().max().item() + 1e-4
    assert (Cs.double() - torch.nn.functional.silu(acc)).abs().max().item() <= tol


@pytest.mark.parametrize("splits", [1, 3])
def test_gemm_w8_timeout_path_reports_and_recovers(splits):
    """Wait limit 0: the bounded waits give up, the CTA records SVLA_ERR_TIMEOUT,
    drains its copies and MMAs, frees its tensor memory; the next launch is right."""
    lib = _abi.load()
    M, N, K = 177, 960, 960
    dev, w_eff = w8_operands(21, N, K, with_gain=False)
    A = torch.randn(M, K, generator=torch.Generator().manual_seed(1)).to(torch.bfloat16).to(DEV)
    C = torch.zeros(M, N, device=DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    try:
        lib.svla_set_wait_limit_ns(0)
        gemm_w8(_abi.EPI_F32, A, dev["q"], dev["ab"], None, C, None, splits, status)
        torch.cuda.synchronize()
    finally:
        lib.svla_set_wait_limit_ns(1_000_000_000)
    assert status.item() in (0, _abi.SVLA_ERR_TIMEOUT)
    status.zero_()
    gemm_w8(_abi.EPI_F32, A, dev["q"], dev["ab"], None, C, None, splits, status)
    torch.cuda.synchronize()
    assert status.item() == 0
    ref = A.double() @ torch.from_numpy(w_eff.astype(np.float64)).to(DEV).T
    assert (C.double() - ref).abs().max().item() <= 1e-4 * ref.abs().max().item()


# ----------------------------------------------------------------------------
# the int8 prefill
# ----------------------------------------------------------------------------
def dequantised_model(wl_name):
    """Oracle weights of the vlm-8bit model and the dense blob holding them."""
    s, wb, _ = H.weights(wl_name)
    W = H.oracle_weights(wl_name)
    Wq = oq.quantize_prefix(W, s.p_layers)
    wbq = dict(wb)
    for name in oq.prefix_matrix_names(s.p_layers):
        wbq[name] = synth.f32_to_bf16_bits(Wq[name].astype(np.float32))
    return Wq, synth.pack_blob(s, wbq)


def device_inputs(wl_name, B):
    inp = H.inputs(wl_name)
    embeds = torch.from_numpy(inp["embeds"][:B].view(np.int16)).to(DEV).view(torch.bfloat16)
    valid = torch.from_numpy(inp["valid"][:B]).to(DEV)
    noise = torch.from_numpy(inp["noise"][:B]).to(DEV)
    return embeds, valid, noise


def check_int8_query(wl_name, Wq, kv, actions, b):
    wl = synth.WORKLOADS[wl_name]
    s = wl.model
    inp = H.inputs(wl_name)
    valid = inp["valid"][b].astype(bool)
    emb = synth.bf16_bits_to_f32(inp["embeds"][b]).astype(np.float64)
    K, V = oracle.prefill(Wq, s, emb, valid)
    B, L = kv.shape[2], kv.shape[3]
    kvn = kv.float().cpu().numpy().reshape(2, s.p_layers, B, L, s.p_kv_heads, s.head_dim)
    for l in range(s.p_layers):
        rk = H.rel_l2(kvn[0, l, b][valid], K[l][valid])
        rv = H.rel_l2(kvn[1, l, b][valid], V[l][valid])
        assert rk <= H.KV_REL_L2 and rv <= H.KV_REL_L2, (wl_name, b, l, rk, rv)
    _, _, x = oracle.denoise(Wq, s, K, V, inp["valid"][b], inp["noise"][b].astype(np.float64), wl.n_steps)
    got = actions[b].cpu().numpy()
    assert H.max_abs(got, x) <= H.CHUNK_MAX_ABS, (wl_name, b, H.max_abs(got, x))
    assert H.rel_l2(got, x) <= H.CHUNK_REL_L2, (wl_name, b, H.rel_l2(got, x))


@pytest.mark.parametrize("wl_name,queries", [("tiny", [0]), ("smolvla_b1", [0]), ("smolvla_b32", [3, 30])])
def test_int8_prefill_and_chunk_match_oracle(wl_name, queries):
    wl = synth.WORKLOADS[wl_name]
    s, _, blob = H.weights(wl_name)
    Wq, _ = dequantised_model(wl_name)
    m = SmolVLA(s, blob, max_batch=wl.B, max_prefix=wl.L, max_chunk=wl.H, prefix_int8=True)
    try:
        assert m.prefix_weights == 8
        embeds, valid, noise = device_inputs(wl_name, wl.B)
        kv = m.prefill(embeds, valid)
        actions, _ = m.denoise(kv, valid, noise, wl.n_steps)
        assert m.device_status() == _abi.SVLA_OK
        torch.cuda.synchronize()
        for b in queries:
            check_int8_query(wl_name, Wq, kv, actions, b)
    finally:
        m.close()


@pytest.mark.parametrize("wl_name", ["smolvla_b1", "smolvla_b32"])
def test_int8_prefill_bitwise_equals_dense_prefill_on_dequantised_blob(wl_name):
    """Batch 1: every int8 GEMM is the fused kernel with the dense GEMM's plan;
    batch 32: every projection is dequantised into a buffer and the dense GEMM
    runs on it. Either way the operand is exactly the dense path's folded weight
    computed from w^, so the K/V caches agree bit for bit with the dense prefill
    given the dequantised blob. Switching the int8 handle back to its dense
    weights reproduces the dense handle given the original blob."""
    wl = synth.WORKLOADS[wl_name]
    s, _, blob = H.weights(wl_name)
    _, blob_q = dequantised_model(wl_name)
    embeds, valid, _ = device_inputs(wl_name, wl.B)
    kw = dict(max_batch=wl.B, max_prefix=wl.L, max_chunk=wl.H)
    m8 = SmolVLA(s, blob, prefix_int8=True, **kw)
    mq = SmolVLA(s, blob_q, **kw)
    md = SmolVLA(s, blob, **kw)
    try:
        kv8 = m8.prefill(embeds, valid)
        kvq = mq.prefill(embeds, valid)
        kvd = md.prefill(embeds, valid)
        m8.set_prefix_weights(16)
        kv16 = m8.prefill(embeds, valid)
        m8.set_prefix_weights(8)
        kv8b = m8.prefill(embeds, valid)
        assert m8.device_status() == _abi.SVLA_OK
        torch.cuda.synchronize()
        assert torch.equal(kv8.view(torch.int16), kvq.view(torch.int16))
        assert torch.equal(kv16.view(torch.int16), kvd.view(torch.int16))
        assert torch.equal(kv8b.view(torch.int16), kv8.view(torch.int16))
        assert not torch.equal(kv8.view(torch.int16), kvd.view(torch.int16))
        with pytest.raises(_abi.SvlaError):
            md.set_prefix_weights(8)
        with pytest.raises(_abi.SvlaError):
            m8.set_prefix_weights(4)
        assert md.prefix_weights == 16
    finally:
        for m in (m8, mq, md):
            m.close()
