"""Weight-only int8 action expert (reading 29: the vlm-8bit scheme of the
mlx-smolvla PyPI page, §Run a checkpoint, applied to the expert's layer
matrices, a row's last group holding its K mod 64 remaining inputs) through
the C ABI.

* The quantiser's codes and scales bit for bit against the oracle's at the
  expert's ragged widths (K = 720 = 11 * 64 + 16, and small ragged cases).
* The int8 GEMM at ragged K against a float64 product with the dequantised
  weights.
* The chunk of an int8-expert handle (dense prefix) against the oracle run on
  the dequantised expert, on the persistent kernel (batch 1) and on the
  multi-kernel path (batch 1, batch 32, batch 8 with prefix 321 and chunk 100).
* Bit for bit against a dense handle given the dequantised blob where both
  take the same partial-sum order: the persistent kernel's in-shared-memory
  dequantisation and the many-tile path's dequantise-then-dense GEMM produce
  exactly the dense path's folded weights.
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

import oracle  # noqa: E402
import synth  # noqa: E402
from oracle import quant as oq  # noqa: E402
from tests import helpers as H  # noqa: E402
from tests.test_gpu_int8 import P, S, bf16_dev, gemm_w8  # noqa: E402
from vision_language_action_b200 import _abi  # noqa: E402
from vision_language_action_b200.runtime import SmolVLA  # noqa: E402

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

DEV = "cuda:0"


def groups(K):
    return (K + 63) // 64


def ragged_matrix(seed, N, K):
    """bf16 weights ~N(0, 0.02) with a few outliers, a narrow offset first group
    and a constant last group (alpha = 0), at any K (a multiple of 16)."""
    rng = np.random.default_rng(seed)
    w = 0.02 * rng.standard_normal((N, K)).astype(np.float32)
    w[rng.integers(0, N, 4), rng.integers(0, K, 4)] = 0.4
    k1 = min(64, K)
    w[0, :k1] = 0.01 + 1e-4 * rng.standard_normal(k1)
    if N > 1:
        w[1, 64 * ((K - 1) // 64):] = -0.03125
    return synth.bf16_bits_to_f32(synth.f32_to_bf16_bits(w)).astype(np.float32)


@pytest.mark.parametrize("N,K", [(1600, 720), (4096, 720), (960, 720), (7, 80), (5, 16), (3, 208)])
def test_quantizer_ragged_groups_match_oracle_bit_for_bit(N, K):
    lib = _abi.load()
    w = ragged_matrix(N * 3 + K, N, K)
    q_ref, a_ref, b_ref = oq.quantize_affine8(w)
    W = bf16_dev(w)
    q = torch.empty((N, K), dtype=torch.uint8, device=DEV)
    ab = torch.empty((groups(K), N, 2), dtype=torch.int16, device=DEV)
    _abi.check(lib.svla_op_quantize_affine8(P(W), K, N, K, P(q), K, P(ab), S()))
    torch.cuda.synchronize()
    assert np.array_equal(q.cpu().numpy(), q_ref)
    abn = ab.cpu().numpy().view(np.uint16)
    assert np.array_equal(abn[..., 0].T, synth.f32_to_bf16_bits(a_ref))
    assert np.array_equal(synth.bf16_bits_to_f32(abn[..., 1].T), b_ref)


@pytest.mark.parametrize("N,K", [(960, 720), (7, 80), (64, 960)])
def test_python_binding_sizes_the_scale_pairs_for_ragged_k(N, K):
    """runtime.op_quantize_affine8 allocates ceil(K/64) (alpha, beta) groups,
    the number the kernel writes, and returns the oracle's codes and pairs."""
    from vision_language_action_b200 import runtime

    w = ragged_matrix(N + K, N, K)
    q_ref, a_ref, b_ref = oq.quantize_affine8(w)
    q, ab = runtime.op_quantize_affine8(bf16_dev(w))
    torch.cuda.synchronize()
    assert tuple(ab.shape) == (groups(K), N, 2)
    assert np.array_equal(q.cpu().numpy(), q_ref)
    abn = ab.view(torch.int16).cpu().numpy().view(np.uint16)
    assert np.array_equal(abn[..., 0].T, synth.f32_to_bf16_bits(a_ref))
    assert np.array_equal(synth.bf16_bits_to_f32(abn[..., 1].T), b_ref)


@pytest.mark.parametrize("M,N,K", [(50, 1600, 720), (50, 4096, 720), (177, 960, 720), (1600, 4096, 720),
                                   (3, 64, 80)])
@pytest.mark.parametrize("with_gain", [False, True])
def test_gemm_w8_ragged_k_matches_fp64(M, N, K, with_gain):
    w = ragged_matrix(M + 2 * N + K, N, K)
    q, a, b = oq.quantize_affine8(w)
    gain = None
    if with_gain:
        rng = np.random.default_rng(K)
        gain = synth.bf16_bits_to_f32(synth.f32_to_bf16_bits(
            (1.0 + 0.1 * rng.standard_normal(K)).astype(np.float32))).astype(np.float32)
    wh = oq.dequantize_affine8(q, a, b).astype(np.float32)
    w_eff = wh if gain is None else oq._bf16_rne(wh * gain[None, :])
    qd = torch.from_numpy(q).to(DEV)
    abd = bf16_dev(np.stack([a.T, b.T], axis=-1).astype(np.float32))
    g = torch.Generator(device="cpu").manual_seed(M + N)
    A = torch.randn(M, K, generator=g).to(torch.bfloat16).to(DEV)
    C = torch.full((M, N), float("nan"), device=DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    gemm_w8(_abi.EPI_F32, A, qd, abd, bf16_dev(gain) if with_gain else None, C, None, 0, status)
    torch.cuda.synchronize()
    Wd = torch.from_numpy(w_eff.astype(np.float64)).to(DEV)
    ref = A.double() @ Wd.T
    scale = A.double().abs() @ Wd.abs().T
    assert status.item() == 0
    assert torch.isfinite(C).all()
    assert ((C.double() - ref).abs() <= 1e-5 * scale + 1e-6).all()


# ----------------------------------------------------------------------------
# the int8-expert denoise
# ----------------------------------------------------------------------------
def dequantised_expert(wl_name):
    """Oracle weights of the int8-expert model and the dense blob holding them."""
    s, wb, _ = H.weights(wl_name)
    W = H.oracle_weights(wl_name)
    Wq = oq.quantize_expert(W, s.e_layers)
    wbq = dict(wb)
    for name in oq.expert_matrix_names(s.e_layers):
        wbq[name] = synth.f32_to_bf16_bits(Wq[name].astype(np.float32))
    return W, Wq, synth.pack_blob(s, wbq)


def inputs(wl_name):
    wl = synth.WORKLOADS[wl_name]
    inp = H.inputs(wl_name)
    embeds = torch.from_numpy(inp["embeds"][:wl.B].view(np.int16)).to(DEV).view(torch.bfloat16)
    valid = torch.from_numpy(inp["valid"][:wl.B]).to(DEV)
    noise = torch.from_numpy(inp["noise"][:wl.B]).to(DEV)
    return embeds, valid, noise


CASES = [("tiny", _abi.DENOISE_FUSED, [0]), ("tiny", _abi.DENOISE_GRAPH, [0]),
         ("smolvla_b1", _abi.DENOISE_FUSED, [0]), ("smolvla_b1", _abi.DENOISE_GRAPH, [0]),
         ("smolvla_b32", _abi.DENOISE_AUTO, [5, 31]), ("long_prefix_b8", _abi.DENOISE_AUTO, [0, 7])]


@pytest.mark.parametrize("wl_name,path,queries", CASES, ids=[f"{c[0]}-{c[1]}" for c in CASES])
def test_int8_expert_chunk_matches_oracle(wl_name, path, queries):
    wl = synth.WORKLOADS[wl_name]
    s, _, blob = H.weights(wl_name)
    W, Wq, _ = dequantised_expert(wl_name)
    m = SmolVLA(s, blob, max_batch=wl.B, max_prefix=wl.L, max_chunk=wl.H, expert_int8=True)
    try:
        assert m.expert_weights == 8 and m.prefix_weights == 16
        m.set_denoise_path(path)
        embeds, valid, noise = inputs(wl_name)
        kv = m.prefill(embeds, valid)
        actions, _ = m.denoise(kv, valid, noise, wl.n_steps)
        assert m.device_status() == _abi.SVLA_OK
        torch.cuda.synchronize()
        inp = H.inputs(wl_name)
        for b in queries:
            v = inp["valid"][b].astype(bool)
            emb = synth.bf16_bits_to_f32(inp["embeds"][b]).astype(np.float64)
            K, V = oracle.prefill(W, s, emb, v)  # the prefix stays dense
            _, _, x = oracle.denoise(Wq, s, K, V, inp["valid"][b], inp["noise"][b].astype(np.float64), wl.n_steps)
            got = actions[b].cpu().numpy()
            assert H.max_abs(got, x) <= H.CHUNK_MAX_ABS, (wl_name, b, H.max_abs(got, x))
            assert H.rel_l2(got, x) <= H.CHUNK_REL_L2, (wl_name, b, H.rel_l2(got, x))
            # the int8 expert is a different model: its chunk moves away from the dense one
            _, _, xd = oracle.denoise(W, s, K, V, inp["valid"][b], inp["noise"][b].astype(np.float64), wl.n_steps)
            assert H.max_abs(x, xd) > 0.0
    finally:
        m.close()


BITWISE = [("smolvla_b1", _abi.DENOISE_FUSED), ("tiny", _abi.DENOISE_FUSED), ("smolvla_b32", _abi.DENOISE_AUTO)]


@pytest.mark.parametrize("wl_name,path", BITWISE, ids=[f"{c[0]}-{c[1]}" for c in BITWISE])
def test_int8_expert_bitwise_equals_dense_on_dequantised_blob(wl_name, path):
    """The persistent kernel dequantises each job's int8 rows into exactly the
    dense copy's folded bf16 rows; the many-tile graph path dequantises a matrix
    and runs the dense GEMM's plan on it; the hoisted cross K/V GEMMs take one
    split on both sides. So the chunk equals the dense handle's given the
    dequantised blob, bit for bit. Switching back to 16 bits reproduces the
    dense handle given the original blob."""
    wl = synth.WORKLOADS[wl_name]
    s, _, blob = H.weights(wl_name)
    _, _, blob_q = dequantised_expert(wl_name)
    kw = dict(max_batch=wl.B, max_prefix=wl.L, max_chunk=wl.H)
    m8 = SmolVLA(s, blob, expert_int8=True, **kw)
    mq = SmolVLA(s, blob_q, **kw)
    md = SmolVLA(s, blob, **kw)
    try:
        for m in (m8, mq, md):
            m.set_denoise_path(path)
        embeds, valid, noise = inputs(wl_name)
        kv = md.prefill(embeds, valid)
        a8, _ = m8.denoise(kv, valid, noise, wl.n_steps)
        aq, _ = mq.denoise(kv, valid, noise, wl.n_steps)
        ad, _ = md.denoise(kv, valid, noise, wl.n_steps)
        m8.set_expert_weights(16)
        a16, _ = m8.denoise(kv, valid, noise, wl.n_steps)
        m8.set_expert_weights(8)
        a8b, _ = m8.denoise(kv, valid, noise, wl.n_steps)
        assert m8.device_status() == _abi.SVLA_OK
        torch.cuda.synchronize()
        assert torch.equal(a8, aq)
        assert torch.equal(a16, ad)
        assert torch.equal(a8b, a8)
        assert not torch.equal(a8, ad)
        with pytest.raises(_abi.SvlaError):
            md.set_expert_weights(8)
        with pytest.raises(_abi.SvlaError):
            m8.set_expert_weights(4)
        assert md.expert_weights == 16
    finally:
        for m in (m8, mq, md):
            m.close()


def test_int8_expert_trace_and_prefix_overwrite_on_both_paths():
    """The traced run and the prefix overwrite (a chunk junction) take the same
    int8 weights: the traced chunk equals the untraced one, the last trace row
    is the chunk, and the overwritten rows land on the given actions."""
    wl_name = "smolvla_b1"
    wl = synth.WORKLOADS[wl_name]
    s, _, blob = H.weights(wl_name)
    m = SmolVLA(s, blob, max_batch=wl.B, max_prefix=wl.L, max_chunk=wl.H, expert_int8=True)
    try:
        embeds, valid, noise = inputs(wl_name)
        kv = m.prefill(embeds, valid)
        d = 7
        prev = torch.randn(wl.B, d, s.action_dim, generator=torch.Generator().manual_seed(3)).to(DEV)
        for path in (_abi.DENOISE_FUSED, _abi.DENOISE_GRAPH):
            m.set_denoise_path(path)
            a0, _ = m.denoise(kv, valid, noise, wl.n_steps)
            a1, tr = m.denoise(kv, valid, noise, wl.n_steps, trace=True)
            ap, _ = m.denoise_prefix(kv, valid, noise, wl.n_steps, prev)
            assert m.device_status() == _abi.SVLA_OK
            torch.cuda.synchronize()
            assert torch.equal(a0, a1)
            assert torch.equal(tr[-1, 1], a1)
            assert torch.equal(ap[:, :d], prev)
    finally:
        m.close()


def test_int8_expert_persistent_timeout_reports_and_recovers():
    """Wait limit 0 on the int8 persistent kernel: the first unsatisfied wait
    (a grid barrier, a weight slot awaited for its dequantisation) gives up, the
    kernel records SVLA_ERR_TIMEOUT and drains; the next launch is exact."""
    wl_name = "tiny"
    wl = synth.WORKLOADS[wl_name]
    s, _, blob = H.weights(wl_name)
    m = SmolVLA(s, blob, max_batch=wl.B, max_prefix=wl.L, max_chunk=wl.H, expert_int8=True)
    lib = _abi.load()
    try:
        m.set_denoise_path(_abi.DENOISE_FUSED)
        embeds, valid, noise = inputs(wl_name)
        kv = m.prefill(embeds, valid)
        ref, _ = m.denoise(kv, valid, noise, wl.n_steps)
        assert m.device_status() == _abi.SVLA_OK
        lib.svla_set_wait_limit_ns(0)
        try:
            m.denoise(kv, valid, noise, wl.n_steps)
            st = m.device_status()
        finally:
            lib.svla_set_wait_limit_ns(1_000_000_000)
        assert st == _abi.SVLA_ERR_TIMEOUT
        again, _ = m.denoise(kv, valid, noise, wl.n_steps)
        assert m.device_status() == _abi.SVLA_OK
        assert torch.equal(again, ref)
    finally:
        m.close()
