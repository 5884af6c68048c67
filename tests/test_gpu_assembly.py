"""Parity of svla_assemble_prefix (connector pixel shuffle + linear on the
tcgen05 GEMM, state token, prefix layout) with the assembly oracle, and of the
chain assembly -> prefill -> denoise with the oracle fed the oracle's own
assembled prefix.

Gates: text rows and the pad mask bitwise; connector rows and the state token
within bf16 output rounding of an fp32-accumulated product
(|diff| <= 2^-7 |ref| + 2^-10 max|ref|); the chain within the gates of the
denoise parity tests.
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

import synth  # noqa: E402
from tests import helpers as H  # noqa: E402
from vision_language_action_b200 import _abi  # noqa: E402
from vision_language_action_b200.runtime import SmolVLA  # noqa: E402

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

DEV = "cuda:0"


def _setup(shape_name, B, seed):
    import oracle
    s = synth.SHAPES[shape_name]
    a = synth.ASSEMBLY_SHAPES[shape_name]
    wbits = synth.gen_assembly_weights(a, s.p_width, seed)
    inp = synth.gen_assembly_inputs(a, s.p_width, B, seed)
    L = a.n_img * a.tokens_per_image + a.text_len + 1
    _, wb, blob = H.weights({"tiny": "tiny", "smolvla": "smolvla_b1"}[shape_name])
    m = SmolVLA(s, blob, max_batch=B, max_prefix=L, max_chunk=50)
    m.set_assembly(synth.pack_assembly_blob(a, s.p_width, wbits), a.vis_width, a.grid, a.shuffle, a.state_dim,
                   a.n_img)
    w = {k: synth.bf16_bits_to_f32(v).astype(np.float64) for k, v in wbits.items()}
    refs = []
    for b in range(B):
        emb, valid = oracle.assemble_prefix(w["w_conn"], w["w_state"], w["b_state"],
                                            synth.bf16_bits_to_f32(inp["vis"][b]).astype(np.float64),
                                            synth.bf16_bits_to_f32(inp["text"][b]).astype(np.float64),
                                            inp["text_valid"][b], inp["state"][b], a.grid, a.shuffle)
        refs.append((emb, valid))
    dev = {
        "vis": torch.from_numpy(inp["vis"].view(np.int16)).to(DEV).view(torch.bfloat16),
        "text": torch.from_numpy(inp["text"].view(np.int16)).to(DEV).view(torch.bfloat16),
        "text_valid": torch.from_numpy(inp["text_valid"]).to(DEV),
        "state": torch.from_numpy(inp["state"]).to(DEV),
    }
    return s, a, m, inp, refs, dev, wb


def _check_rows(got, ref):
    tol = 2.0 ** -7 * np.abs(ref) + 2.0 ** -10 * np.abs(ref).max()
    assert np.all(np.abs(got - ref) <= tol), float(np.max(np.abs(got - ref) - tol))


@pytest.mark.parametrize("shape_name,B", [("tiny", 3), ("smolvla", 2)])
def test_assemble_prefix_parity(shape_name, B):
    s, a, m, inp, refs, dev, _ = _setup(shape_name, B, seed=11)
    try:
        emb, pad = m.assemble_prefix(dev["vis"], dev["text"], dev["text_valid"], dev["state"])
        torch.cuda.synchronize()
        got = emb.float().cpu().numpy()
        padn = pad.cpu().numpy()
        n_vis = a.n_img * a.tokens_per_image
        for b in range(B):
            ref, valid = refs[b]
            assert np.array_equal(padn[b], valid)
            _check_rows(got[b, :n_vis], ref[:n_vis])
            assert np.array_equal(emb[b, n_vis:-1].view(torch.int16).cpu().numpy(), inp["text"][b].view(np.int16))
            _check_rows(got[b, -1:], ref[-1:])
        # run-to-run bitwise deterministic; B = 1 gives query 0's rows within rounding
        # (the connector GEMM's split-K plan depends on the row count, so the fp32
        # summation order, not the result beyond rounding, changes with B)
        emb2, _ = m.assemble_prefix(dev["vis"], dev["text"], dev["text_valid"], dev["state"])
        e1, _ = m.assemble_prefix(dev["vis"][:1].contiguous(), dev["text"][:1].contiguous(),
                                  dev["text_valid"][:1].contiguous(), dev["state"][:1].contiguous())
        torch.cuda.synchronize()
        assert torch.equal(emb2, emb)
        _check_rows(e1[0].float().cpu().numpy(), refs[0][0])
    finally:
        m.close()


def test_assembly_then_prefill_and_denoise_parity():
    """The whole chain on the tiny model against the oracle fed its own assembled prefix."""
    import oracle
    s, a, m, inp, refs, dev, wb = _setup("tiny", 1, seed=12)
    try:
        emb, pad = m.assemble_prefix(dev["vis"], dev["text"], dev["text_valid"], dev["state"])
        noise = torch.from_numpy(np.random.default_rng(12).standard_normal((1, 8, s.action_dim), dtype=np.float32)).to(DEV)
        kv = m.prefill(emb, pad)
        x, _ = m.denoise(kv, pad, noise, 3)
        assert m.device_status() == _abi.SVLA_OK
        ref, valid = refs[0]
        ref_bf16 = synth.bf16_bits_to_f32(synth.f32_to_bf16_bits(ref.astype(np.float32))).astype(np.float64)
        W = oracle.load_weights(wb)
        K, V, _, _, xo = oracle.sample(W, s, ref_bf16, valid, noise[0].cpu().numpy().astype(np.float64), 3)
        L = ref.shape[0]
        kvn = kv.float().cpu().numpy().reshape(2, s.p_layers, 1, L, s.p_kv_heads, s.head_dim)
        ok = valid.astype(bool)
        for l in range(s.p_layers):
            assert H.rel_l2(kvn[0, l, 0][ok], K[l][ok]) <= H.KV_REL_L2
            assert H.rel_l2(kvn[1, l, 0][ok], V[l][ok]) <= H.KV_REL_L2
        got = x[0].cpu().numpy()
        assert H.max_abs(got, xo) <= H.CHUNK_MAX_ABS
        assert H.rel_l2(got, xo) <= H.CHUNK_REL_L2
    finally:
        m.close()


def test_assembly_argument_errors():
    s = synth.SHAPES["tiny"]
    a = synth.ASSEMBLY_SHAPES["tiny"]
    _, _, blob = H.weights("tiny")
    m = SmolVLA(s, blob, max_batch=1, max_prefix=64, max_chunk=8)
    try:
        vis = torch.zeros(1, a.n_img, a.grid * a.grid, a.vis_width, dtype=torch.bfloat16, device=DEV)
        state = torch.zeros(1, a.state_dim, device=DEV)
        emb = torch.empty(1, 64, s.p_width, dtype=torch.bfloat16, device=DEV)
        pad = torch.empty(1, 64, dtype=torch.uint8, device=DEV)
        lib = _abi.load()
        P = lambda t: __import__("ctypes").c_void_p(t.data_ptr())  # noqa: E731
        st = lib.svla_assemble_prefix(m.h, P(vis), None, None, P(state), 1, a.n_img, 0, P(emb), P(pad), None)
        assert st == _abi.SVLA_ERR_ARG  # no weights yet
        bad = np.zeros(10, np.uint16)
        with pytest.raises(_abi.SvlaError) as e:
            m.set_assembly(bad, a.vis_width, a.grid, a.shuffle, a.state_dim, a.n_img)
        assert e.value.status == _abi.SVLA_ERR_BLOB_SIZE
    finally:
        m.close()
