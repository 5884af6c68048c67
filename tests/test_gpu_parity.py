"""End-to-end parity of the CUDA path (through the C ABI) with the CPU oracle on
the five synthetic workloads, plus determinism, batch/padding invariance, the
empty-prefix error and svla_sample's noise.

Gates (bf16 storage, fp32 accumulation): per-layer K/V relative L2 <= 5e-3 over
valid positions; final chunk max|diff| <= 2e-2 and relative L2 <= 1e-2. The
per-step trace (velocity and state of every Euler step) is held to the same
chunk gates. Large batches are checked on a seeded subset of queries: queries
are independent, so the oracle runs them one by one.
"""
import gc

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


class Run:
    """GPU run of a workload: handle, device inputs, K/V, chunk and trace."""

    def __init__(self, wl_name, random_affine=False, B=None, path=_abi.DENOISE_AUTO):
        wl = synth.WORKLOADS[wl_name]
        s, _, blob = H.weights(wl_name, random_affine)
        inp = H.inputs(wl_name)
        self.wl, self.s = wl, s
        self.B = wl.B if B is None else B
        self.m = SmolVLA(s, blob, max_batch=self.B, max_prefix=wl.L, max_chunk=wl.H)
        self.m.set_denoise_path(path)
        self.valid = torch.from_numpy(inp["valid"][:self.B]).to(DEV)
        self.noise = torch.from_numpy(inp["noise"][:self.B]).to(DEV)
        if wl.prefix_kind == "kv_given":
            kv = np.stack([inp["k"][:, :self.B], inp["v"][:, :self.B]])
            self.kv = torch.from_numpy(kv.reshape(2, s.p_layers, self.B, wl.L, -1).view(np.int16)).to(DEV)
            self.kv = self.kv.view(torch.bfloat16)
        else:
            self.embeds = torch.from_numpy(inp["embeds"][:self.B].view(np.int16)).to(DEV).view(torch.bfloat16)
            self.kv = self.m.prefill(self.embeds, self.valid)
        self.actions, self.trace = self.m.denoise(self.kv, self.valid, self.noise, wl.n_steps, trace=True)
        assert self.m.device_status() == _abi.SVLA_OK
        torch.cuda.synchronize()

    def kv_np(self):
        L, s = self.wl.L, self.s
        kv = self.kv.float().cpu().numpy().reshape(2, s.p_layers, self.B, L, s.p_kv_heads, s.head_dim)
        return kv[0], kv[1]

    def close(self):
        self.m.close()


def check_query(run: Run, b: int, random_affine=False):
    wl, s = run.wl, run.s
    K, V, vs, xs, x = H.oracle_query(wl.name, b, random_affine)
    valid = H.inputs(wl.name)["valid"][b].astype(bool)
    if wl.prefix_kind != "kv_given":
        Kg, Vg = run.kv_np()
        for l in range(s.p_layers):
            rk = H.rel_l2(Kg[l, b][valid], K[l][valid])
            rv = H.rel_l2(Vg[l, b][valid], V[l][valid])
            assert rk <= H.KV_REL_L2 and rv <= H.KV_REL_L2, (wl.name, b, l, rk, rv)
    tr = run.trace.cpu().numpy()
    for k in range(wl.n_steps):
        assert H.max_abs(tr[k, 1, b], xs[k]) <= H.CHUNK_MAX_ABS, (wl.name, b, "step", k)
        assert H.rel_l2(tr[k, 0, b], vs[k]) <= H.CHUNK_REL_L2, (wl.name, b, "velocity", k)
    got = run.actions[b].cpu().numpy()
    assert np.array_equal(got, tr[-1, 1, b])
    assert H.max_abs(got, x) <= H.CHUNK_MAX_ABS, (wl.name, b, H.max_abs(got, x))
    assert H.rel_l2(got, x) <= H.CHUNK_REL_L2, (wl.name, b, H.rel_l2(got, x))


PATHS = {"graph": _abi.DENOISE_GRAPH, "fused": _abi.DENOISE_FUSED}


@pytest.fixture(scope="module")
def tiny():
    r = Run("tiny")
    yield r
    r.close()


@pytest.mark.parametrize("path", sorted(PATHS))
def test_tiny_parity(path):
    r = Run("tiny", path=PATHS[path])
    try:
        check_query(r, 0)
    finally:
        r.close()


@pytest.mark.parametrize("path", sorted(PATHS))
def test_tiny_random_affine_parity(path):
    r = Run("tiny", random_affine=True, path=PATHS[path])
    try:
        check_query(r, 0, random_affine=True)
    finally:
        r.close()


@pytest.mark.parametrize("path", sorted(PATHS))
def test_smolvla_b1_parity(path):
    r = Run("smolvla_b1", path=PATHS[path])
    try:
        assert r.m.fused_supported(1, r.wl.H)
        check_query(r, 0)
        # run-to-run bitwise determinism of prefill and denoise
        kv2 = r.m.prefill(r.embeds, r.valid)
        a2, t2 = r.m.denoise(kv2, r.valid, r.noise, r.wl.n_steps, trace=True)
        torch.cuda.synchronize()
        assert torch.equal(kv2, r.kv)
        assert torch.equal(a2, r.actions) and torch.equal(t2, r.trace)
    finally:
        r.close()
        gc.collect()


def test_smolvla_b32_parity_and_batch_invariance():
    # batch invariance of one implementation: the graph path at B = 32 and B = 1
    r = Run("smolvla_b32", path=_abi.DENOISE_GRAPH)
    try:
        for b in (0, 13, 31):
            check_query(r, b)
        # query 13 alone gives the same chunk as inside the batch (within tolerance)
        e1 = r.embeds[13:14].contiguous()
        v1 = r.valid[13:14].contiguous()
        n1 = r.noise[13:14].contiguous()
        kv1 = r.m.prefill(e1, v1)
        a1, _ = r.m.denoise(kv1, v1, n1, r.wl.n_steps)
        torch.cuda.synchronize()
        assert H.max_abs(a1[0].cpu().numpy(), r.actions[13].cpu().numpy()) <= 5e-3
        # padding invariance: the same query with its pads removed
        keep = torch.nonzero(r.valid[13]).flatten()
        ec = r.embeds[13:14, keep].contiguous()
        vc = torch.ones(1, keep.numel(), dtype=torch.uint8, device=DEV)
        kvc = r.m.prefill(ec, vc)
        ac, _ = r.m.denoise(kvc, vc, n1, r.wl.n_steps)
        torch.cuda.synchronize()
        assert H.max_abs(ac[0].cpu().numpy(), r.actions[13].cpu().numpy()) <= 5e-3
    finally:
        r.close()
        gc.collect()


def test_long_prefix_b8_parity():
    r = Run("long_prefix_b8")
    try:
        for b in (0, 7):
            check_query(r, b)
    finally:
        r.close()
        gc.collect()


def test_denoise_b256_parity():
    r = Run("denoise_b256")
    try:
        for b in (0, 101, 255):
            check_query(r, b)
    finally:
        r.close()
        gc.collect()


def test_empty_prefix_sets_device_status(tiny):
    v0 = tiny.valid.clone()
    v0[0] = 0
    tiny.m.prefill(tiny.embeds, v0)
    assert tiny.m.device_status() == _abi.SVLA_ERR_EMPTY_PREFIX
    assert tiny.m.device_status() == _abi.SVLA_OK  # cleared on read


def test_host_shape_errors(tiny):
    with pytest.raises(_abi.SvlaError) as e:
        tiny.m.denoise(tiny.kv, tiny.valid, tiny.noise, 0)
    assert e.value.status == _abi.SVLA_ERR_SHAPE
    big = torch.zeros(1, tiny.wl.L + 1, dtype=torch.uint8, device=DEV)
    with pytest.raises(_abi.SvlaError) as e:
        tiny.m.prefill(tiny.embeds, big)
    assert e.value.status == _abi.SVLA_ERR_SHAPE


def test_sample_noise_matches_philox_and_denoise(tiny):
    import oracle
    seed = 0x1234_5678_9ABC
    actions, kv, noise = tiny.m.sample(tiny.embeds, tiny.valid, seed, tiny.wl.H, tiny.wl.n_steps,
                                       return_noise=True)
    torch.cuda.synchronize()
    want = oracle.gaussian_noise(seed, 1, tiny.wl.H, tiny.s.action_dim)
    assert H.max_abs(noise.cpu().numpy(), want) <= 2e-5
    a2, _ = tiny.m.denoise(kv, tiny.valid, noise, tiny.wl.n_steps)
    torch.cuda.synchronize()
    assert torch.equal(a2, actions)


# ---------------------------------------------------------------------------
# prefix overwrite at a chunk junction (reading 17)
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("wl_name,d,queries,path", [
    ("tiny", 3, (0,), "graph"), ("tiny", 3, (0,), "fused"), ("smolvla_b1", 7, (0,), "graph"),
    ("smolvla_b1", 7, (0,), "fused"), ("smolvla_b32", 7, (5, 31), "graph")])
def test_prefix_overwrite_parity(wl_name, d, queries, path):
    import oracle
    r = Run(wl_name, path=PATHS[path])
    try:
        wl, s = r.wl, r.s
        g = torch.Generator(device="cpu").manual_seed(17)
        prefix = torch.randn(r.B, d, s.action_dim, generator=g).to(DEV)
        a, tr = r.m.denoise_prefix(r.kv, r.valid, r.noise, wl.n_steps, prefix, trace=True)
        a0, _ = r.m.denoise_prefix(r.kv, r.valid, r.noise, wl.n_steps, prefix[:, :0].contiguous())
        torch.cuda.synchronize()
        assert torch.equal(a0, r.actions)                       # d = 0 is plain denoise
        assert torch.equal(a[:, :d], prefix)                     # the chunk starts with the given actions
        W = H.oracle_weights(wl_name)
        inp = H.inputs(wl_name)
        trn = tr.cpu().numpy()
        for b in queries:
            emb = synth.bf16_bits_to_f32(inp["embeds"][b]).astype(np.float64)
            K, V = oracle.prefill(W, s, emb, inp["valid"][b])
            vs, xs, x = oracle.denoise_prefix_overwrite(W, s, K, V, inp["valid"][b],
                                                        inp["noise"][b].astype(np.float64), wl.n_steps,
                                                        prefix[b].cpu().numpy().astype(np.float64))
            got = a[b].cpu().numpy()
            assert H.max_abs(got, x) <= H.CHUNK_MAX_ABS and H.rel_l2(got, x) <= H.CHUNK_REL_L2, (b, H.max_abs(got, x))
            for k in range(wl.n_steps):
                assert H.max_abs(trn[k, 1, b], xs[k]) <= H.CHUNK_MAX_ABS, (b, k)
    finally:
        r.close()
        gc.collect()


def test_prefix_overwrite_argument_errors(tiny):
    p = torch.zeros(1, tiny.wl.H + 1, tiny.s.action_dim, device=DEV)
    with pytest.raises(_abi.SvlaError) as e:
        tiny.m.denoise_prefix(tiny.kv, tiny.valid, tiny.noise, 2, p)
    assert e.value.status == _abi.SVLA_ERR_SHAPE
    x = tiny.noise.clone()
    with pytest.raises(_abi.SvlaError) as e:
        tiny.m.denoise_prefix(tiny.kv, tiny.valid, x, 2, p[:, :2].contiguous(), actions=x)
    assert e.value.status == _abi.SVLA_ERR_ARG


# ---------------------------------------------------------------------------
# edge cases on the tiny model: degenerate and ragged sizes
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("path", sorted(PATHS))
@pytest.mark.parametrize("B,L,Hc,n_steps,mask", [
    (1, 1, 1, 1, "all"),          # one prefix token, one action row, one Euler step
    (2, 9, 3, 2, "one_middle"),   # a single valid token amid padding
    (3, 65, 17, 4, "ragged"),     # ragged tiles in every dimension, per-query pad patterns
    (1, 130, 64, 3, "lead_pad"),  # leading padding (positions start at the first valid token)
])
def test_tiny_edge_cases(B, L, Hc, n_steps, mask, path):
    import oracle
    s = synth.SHAPES["tiny"]
    _, wb, blob = H_weights_tiny()
    rng = np.random.default_rng(B * 1000 + L * 10 + Hc)
    emb_bits = synth.f32_to_bf16_bits(rng.standard_normal((B, L, s.p_width), dtype=np.float32))
    noise = rng.standard_normal((B, Hc, s.action_dim), dtype=np.float32)
    valid = np.ones((B, L), np.uint8)
    if mask == "one_middle":
        valid[:] = 0
        valid[:, L // 2] = 1
    elif mask == "ragged":
        valid[0, 60:] = 0
        valid[1, 3:20] = 0
        valid[2, ::3] = 0
    elif mask == "lead_pad":
        valid[0, :40] = 0
    m = SmolVLA(s, blob, max_batch=B, max_prefix=L, max_chunk=Hc)
    try:
        assert m.fused_supported(B, Hc)  # every case here has B * H <= 64
        m.set_denoise_path(PATHS[path])
        e = torch.from_numpy(emb_bits.view(np.int16)).to(DEV).view(torch.bfloat16)
        v = torch.from_numpy(valid).to(DEV)
        n = torch.from_numpy(noise).to(DEV)
        kv = m.prefill(e, v)
        a, _ = m.denoise(kv, v, n, n_steps)
        assert m.device_status() == _abi.SVLA_OK
        kvn = kv.float().cpu().numpy().reshape(2, s.p_layers, B, L, s.p_kv_heads, s.head_dim)
        W = oracle.load_weights(wb)
        for b in range(B):
            emb = synth.bf16_bits_to_f32(emb_bits[b]).astype(np.float64)
            K, V, _, _, x = oracle.sample(W, s, emb, valid[b], noise[b].astype(np.float64), n_steps)
            ok = valid[b].astype(bool)
            for l in range(s.p_layers):
                assert H.rel_l2(kvn[0, l, b][ok], K[l][ok]) <= H.KV_REL_L2
                assert H.rel_l2(kvn[1, l, b][ok], V[l][ok]) <= H.KV_REL_L2
            got = a[b].cpu().numpy()
            assert H.max_abs(got, x) <= H.CHUNK_MAX_ABS and H.rel_l2(got, x) <= H.CHUNK_REL_L2, (b, H.max_abs(got, x))
    finally:
        m.close()


def H_weights_tiny():
    return H.weights("tiny")


# ---------------------------------------------------------------------------
# the persistent denoise kernel: selection rules and its bounded waits
# ---------------------------------------------------------------------------
def test_fused_path_selection(tiny):
    m = tiny.m
    assert m.fused_supported(1, tiny.wl.H)
    assert not m.fused_supported(1, 65)            # more than 64 chunk rows of one query
    with pytest.raises(_abi.SvlaError) as e:
        m.set_denoise_path(7)
    assert e.value.status == _abi.SVLA_ERR_ARG


def test_fused_unsupported_shape_is_rejected():
    s, _, blob = H.weights("tiny")
    m = SmolVLA(s, blob, max_batch=9, max_prefix=24, max_chunk=8)
    try:
        assert not m.fused_supported(9, 8)          # 72 rows
        m.set_denoise_path(_abi.DENOISE_FUSED)
        kv = m.new_kv_cache(9, 24)
        kv.zero_()
        v = torch.ones(9, 24, dtype=torch.uint8, device=DEV)
        n = torch.zeros(9, 8, s.action_dim, device=DEV)
        with pytest.raises(_abi.SvlaError) as e:
            m.denoise(kv, v, n, 2)
        assert e.value.status == _abi.SVLA_ERR_UNSUPPORTED
    finally:
        m.close()


def test_fused_timeout_reports_and_recovers(tiny):
    """A wait limit of 0 makes the first unsatisfied wait (a grid barrier or a
    weight slot) give up: the kernel records SVLA_ERR_TIMEOUT, every CTA leaves
    through the abort word, and the next launch with the normal limit is exact."""
    m = tiny.m
    m.set_denoise_path(_abi.DENOISE_FUSED)
    try:
        ref, _ = m.denoise(tiny.kv, tiny.valid, tiny.noise, tiny.wl.n_steps)
        assert m.device_status() == _abi.SVLA_OK
        lib = _abi.load()
        lib.svla_set_wait_limit_ns(0)
        try:
            m.denoise(tiny.kv, tiny.valid, tiny.noise, tiny.wl.n_steps)
            st = m.device_status()
        finally:
            lib.svla_set_wait_limit_ns(1_000_000_000)
        assert st == _abi.SVLA_ERR_TIMEOUT
        again, _ = m.denoise(tiny.kv, tiny.valid, tiny.noise, tiny.wl.n_steps)
        assert m.device_status() == _abi.SVLA_OK
        assert torch.equal(again, ref)
    finally:
        m.set_denoise_path(_abi.DENOISE_AUTO)
