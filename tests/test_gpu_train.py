"""The training step of the expert (the flow-matching fine-tune; readings 25-27
in ``oracle/train.py``) through the C ABI against the oracle: the loss and the
gradient of every trainable tensor, on the tiny shape and on the SmolVLA shape
(two queries with padded prefixes, chunk 50, prefix 177), plus bitwise
reproducibility and the handle flag.

Gates, derived from the arithmetic of the step: the forward keeps bf16
activations and the backward rounds every GEMM operand (the residual's
gradient, dgu, dq/dk/dv, the transposed activations) to bf16 once per layer,
each rounding a relative 2^-9; sixteen layers of such roundings stay well
inside 3e-2 relative L2 per gradient tensor. The loss is dominated by the
target eps - a and is held to 1e-3 relative.

Inputs: W_in is drawn 10x wider than the other synthetic weights. With
N(0, 0.02) the action embedding is ~100x smaller than the time embedding, which
is the same for every row of a query, so a chunk's rows, and its values v_j,
are nearly equal. The softmax gradient ds_j = p_j (dp_j - sum p dp) then
cancels, and the bf16 storage of q/k/v alone moves the self-attention layers'
W_q / W_k gradients by ~5e-2 (measured on the oracle by rounding only those
storage points). With the wider W_in that effect is ~8e-3
(``tests/test_oracle_train.py::test_inputs_are_well_conditioned_for_bf16``).
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

import oracle  # noqa: E402
import synth  # noqa: E402
from oracle import train as ot  # noqa: E402
from tests import helpers as H  # noqa: E402
from vision_language_action_b200 import _abi  # noqa: E402
from vision_language_action_b200.runtime import SmolVLA  # noqa: E402

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

DEV = "cuda:0"
GRAD_REL_L2 = 3e-2
ROUNDED_GRAD_REL_L2 = 1e-2
LOSS_REL = 1e-3


def make_case(shape, B, L, Hc, seed, workload_weights=False):
    """workload_weights: the synthetic workloads' own weights (N(0, 0.02),
    gains 1, biases 0, W_in not widened); else random gains and biases and
    W_in drawn 10x wider (see the module docstring)."""
    s = synth.SHAPES[shape]
    wb = dict(synth.gen_weights(s, seed, random_affine=not workload_weights))
    if not workload_weights:
        wb["w_in"] = synth.f32_to_bf16_bits(10.0 * synth.bf16_bits_to_f32(wb["w_in"]))
    rng = np.random.default_rng([seed, 31])
    kv_bits = synth.f32_to_bf16_bits(rng.standard_normal((2, s.p_layers, B, L, s.p_kv_width)).astype(np.float32))
    valid = np.ones((B, L), np.uint8)
    valid[0, 1] = 0
    if B > 1:
        valid[1, L - 3:] = 0
    a = (0.5 * rng.standard_normal((B, Hc, s.action_dim))).astype(np.float32)
    eps = rng.standard_normal((B, Hc, s.action_dim)).astype(np.float32)
    t = rng.uniform(0.05, 0.95, B).astype(np.float32)
    return s, wb, kv_bits, valid, a, eps, t


def oracle_step(s, wb, kv_bits, valid, a, eps, t, bf16_storage=False):
    W = oracle.load_weights(wb)
    B, L = valid.shape
    kv = synth.bf16_bits_to_f32(kv_bits).astype(np.float64)          # [2, layers, B, L, kv*hd]
    K = kv[0].transpose(1, 0, 2, 3).reshape(B, s.p_layers, L, s.p_kv_heads, s.head_dim)
    V = kv[1].transpose(1, 0, 2, 3).reshape(B, s.p_layers, L, s.p_kv_heads, s.head_dim)
    return ot.train_step(W, s, K, V, valid, a.astype(np.float64), eps.astype(np.float64), t.astype(np.float64),
                         bf16_storage=bf16_storage)


def gpu_step(m, kv_bits, valid, a, eps, t):
    kv = torch.from_numpy(kv_bits.view(np.int16)).to(DEV).view(torch.bfloat16)
    loss, grads = m.train_step(kv, torch.from_numpy(valid).to(DEV), torch.from_numpy(a).to(DEV),
                               torch.from_numpy(eps).to(DEV), torch.from_numpy(t).to(DEV))
    assert m.device_status() == _abi.SVLA_OK
    torch.cuda.synchronize()
    return float(loss.item()), grads.cpu().numpy()


def split_grads(s, g):
    out, off = {}, 0
    for name, shp in synth.manifest(s):
        if name.startswith("p"):
            continue
        n = int(np.prod(shp))
        out[name] = g[off:off + n].reshape(shp)
        off += n
    assert off == g.size
    return out


# the last case spans several key tiles (prefix 321) and two row tiles of the
# attention backward's key pass (chunk 100), the long-prefix workload's shape
@pytest.mark.parametrize("shape,B,L,Hc", [("tiny", 2, 24, 8), ("smolvla", 2, 177, 50), ("smolvla", 1, 321, 100)])
def test_train_step_matches_oracle(shape, B, L, Hc):
    s, wb, kv_bits, valid, a, eps, t = make_case(shape, B, L, Hc, 7)
    m = SmolVLA(s, synth.pack_blob(s, wb), max_batch=B, max_prefix=L, max_chunk=Hc, train=True)
    try:
        assert int(m.lib.svla_train_grad_elems(m.h)) == synth.param_count(s, "expert")
        loss, g = gpu_step(m, kv_bits, valid, a, eps, t)
        loss2, g2 = gpu_step(m, kv_bits, valid, a, eps, t)
    finally:
        m.close()
    assert loss == loss2 and np.array_equal(g, g2), "training step is not bitwise reproducible"
    ref_loss, ref = oracle_step(s, wb, kv_bits, valid, a, eps, t)
    got = split_grads(s, g)
    errs = {n: H.rel_l2(got[n], ref[n]) for n in ot.trainable_names(s)}
    worst = sorted(errs.items(), key=lambda kv: -kv[1])
    print(f"\n{shape}: loss {loss:.6f} oracle {ref_loss:.6f}; worst gradient rel L2:",
          ", ".join(f"{n} {e:.2e}" for n, e in worst[:8]))
    assert abs(loss - ref_loss) <= LOSS_REL * ref_loss, (loss, ref_loss)
    bad = [(n, e) for n, e in worst if not e <= GRAD_REL_L2]
    assert not bad, bad


def rounding_spread(s, wb, kv_bits, valid, a, eps, t):
    """How well the storage-rounded oracle itself fixes each gradient: the
    largest relative L2 distance between two of its realizations whose values
    before every bf16 rounding differ by one or two float32 ulps (k = +-1,
    +-2), as another summation order gives. A well-conditioned tensor barely
    moves; one set by individual rounding decisions moves by percents."""
    orig = ot.bf16_round
    runs = {}
    for k in (1, -1, 2, -2):
        ot.bf16_round = (lambda kk: (lambda x: orig(x * (1 + kk * 2.0 ** -23))))(k)
        try:
            runs[k] = oracle_step(s, wb, kv_bits, valid, a, eps, t, bf16_storage=True)[1]
        finally:
            ot.bf16_round = orig
    return {n: max(H.rel_l2(runs[1][n], runs[-1][n]), H.rel_l2(runs[2][n], runs[-2][n])) for n in runs[1]}


# a tensor the rounded oracle fixes to better than the gate itself is held to it
WELL_CONDITIONED = ROUNDED_GRAD_REL_L2
# an ill-conditioned one: the GPU is one more realization of the rounding policy
SPREAD_FACTOR = 2.5


def self_attention_q_k(s):
    return {f"e{l}.{w}" for l in range(0, s.e_layers, 2) for w in ("wq", "wk")}


@pytest.mark.parametrize("shape,B,L,Hc", [("tiny", 2, 24, 8), ("smolvla", 2, 177, 50)])
def test_train_step_at_workload_weights_matches_storage_rounded_oracle(shape, B, L, Hc):
    """At the workloads' own weights (W_in not widened) a chunk's rows are nearly
    equal and the softmax gradient cancels, so the GPU's bf16 storage moves
    the self-attention W_q / W_k gradients by several percent away from the
    unrounded oracle. The oracle with its forward rounded at the same storage
    points (reading 28 in ``oracle/train.py``) takes that precision effect
    out; what is left is the GPU's own arithmetic (fp32 sums in another
    order, the backward's bf16 operands), held to 1e-2 per gradient tensor.

    At the SmolVLA shape the self-attention W_q / W_k gradients are set by
    individual rounding decisions: realizations of the rounded oracle one or
    two float32 ulps apart before each rounding already disagree on them by
    2-6 % (``rounding_spread``; pinned on the CPU by
    ``tests/test_oracle_train.py::test_workload_self_attention_gradients_are_rounding_bound``).
    No oracle fixes them better, so for a tensor the rounded oracle fixes
    only to d > 1e-2 the GPU is held to 2.5 d; every other tensor (d of at
    most a few 1e-3) to 1e-2."""
    s, wb, kv_bits, valid, a, eps, t = make_case(shape, B, L, Hc, 7, workload_weights=True)
    m = SmolVLA(s, synth.pack_blob(s, wb), max_batch=B, max_prefix=L, max_chunk=Hc, train=True)
    try:
        loss, g = gpu_step(m, kv_bits, valid, a, eps, t)
    finally:
        m.close()
    got = split_grads(s, g)
    ref_loss, ref = oracle_step(s, wb, kv_bits, valid, a, eps, t, bf16_storage=True)
    spread = rounding_spread(s, wb, kv_bits, valid, a, eps, t)
    ill = {n for n, d in spread.items() if d > WELL_CONDITIONED}
    assert ill <= self_attention_q_k(s), sorted(ill - self_attention_q_k(s))
    errs = {n: H.rel_l2(got[n], ref[n]) for n in ot.trainable_names(s)}
    gate = {n: SPREAD_FACTOR * spread[n] if n in ill else ROUNDED_GRAD_REL_L2 for n in errs}
    worst = sorted(errs.items(), key=lambda kv: -kv[1] / gate[kv[0]])
    print(f"\n{shape} (workload weights): loss {loss:.6f} rounded oracle {ref_loss:.6f}; "
          f"{len(ill)} rounding-bound tensors; worst gradient rel L2 (gate):",
          ", ".join(f"{n} {e:.2e} ({gate[n]:.1e})" for n, e in worst[:8]))
    assert abs(loss - ref_loss) <= LOSS_REL * ref_loss, (loss, ref_loss)
    bad = [(n, e, gate[n]) for n, e in worst if not e <= gate[n]]
    assert not bad, bad


def test_train_step_needs_the_flag():
    s, wb, kv_bits, valid, a, eps, t = make_case("tiny", 1, 24, 8, 3)
    m = SmolVLA(s, synth.pack_blob(s, wb), max_batch=1, max_prefix=24, max_chunk=8)
    try:
        assert int(m.lib.svla_train_grad_elems(m.h)) == 0
        with pytest.raises(_abi.SvlaError):
            gpu_step(m, kv_bits, valid, a, eps, t)
    finally:
        m.close()
