"""Host-side checks of the figures bench.py reports: the algorithmic work of the
int8 prefill and of the training step counted independently from the
manifest, and the chunk delta summary on a constructed difference."""
import numpy as np

import bench
import synth

S = synth.SHAPES["smolvla"]


def test_prefix_projection_bytes_from_the_manifest():
    man = dict(synth.manifest(S))
    dense = 0
    for l in range(S.p_layers):
        names = ("wq", "wk", "wv") if l == S.p_layers - 1 else ("wq", "wk", "wv", "wo", "wg", "wu", "wd")
        dense += sum(2 * int(np.prod(man[f"p{l}.{n}"])) for n in names)
    assert bench.prefix_projection_bytes(S, 16) == dense
    # int8: one byte per weight plus a bf16 (alpha, beta) pair per 64 weights
    assert bench.prefix_projection_bytes(S, 8) == dense // 2 + dense // 2 // 64 * 4


def test_expert_projection_bytes_from_the_manifest():
    """Every expert layer's seven projections (the odd layers' cross K / V act on
    the 320-wide cache); int8: one byte per weight plus a bf16 (alpha, beta) pair
    per group, 720-wide rows having 12 groups (11 of 64 and one of 16)."""
    man = dict(synth.manifest(S))
    dense = int8 = 0
    for l in range(S.e_layers):
        for n in ("wq", "wk", "wv", "wo", "wg", "wu", "wd"):
            N, K = man[f"e{l}.{n}"]
            dense += 2 * N * K
            int8 += N * K + N * {720: 12, 960: 15, 2048: 32, 320: 5}[K] * 4
    assert bench.expert_projection_bytes(S, 16) == dense
    assert bench.expert_projection_bytes(S, 8) == int8
    assert 0.5 < int8 / dense < 0.54
    for bits in (8, 16):  # per-step projections + the hoisted cross K / V ones
        assert bench.expert_projection_bytes(S, bits, False) + bench.expert_projection_bytes(S, bits, True) == \
            bench.expert_projection_bytes(S, bits)
    cross = sum(2 * int(np.prod(man[f"e{l}.{n}"])) for l in range(1, S.e_layers, 2) for n in ("wk", "wv"))
    assert bench.expert_projection_bytes(S, 16, True) == cross


def test_train_flops_counts_three_products_per_weight_gemm():
    B, L, H = 2, 177, 50
    M, E = B * H, S.e_width
    expert_mats = 0
    for l in range(S.e_layers):
        for n in ("wq", "wo", "wg", "wu", "wd") + (("wk", "wv") if l % 2 == 0 else ()):
            expert_mats += int(np.prod(dict(synth.manifest(S))[f"e{l}.{n}"]))
    gemm = 3 * 2 * M * expert_mats                                   # forward, dX, dW
    gemm += 2 * 2 * (2 * B * L * S.p_kv_width * S.e_kv_width) * (S.e_layers // 2)  # cross K/V: forward, dW
    gemm += 2 * 2 * M * E * 2 * E + 2 * M * E * E + 3 * 2 * M * E * E  # time MLP
    att = sum(7 * 2 * B * S.e_heads * H * (H if l % 2 == 0 else L) * S.head_dim for l in range(S.e_layers))
    assert bench.train_flops(S, B, L, H) == gemm + att


def test_chunk_delta_summary():
    ref = np.zeros((50, 32))
    gpu = ref.copy()
    gpu[:, 3] = np.linspace(0, 1e-2, 50)
    gpu[7, 5] = 3e-2
    d = bench.chunk_delta(gpu, ref)
    assert d["max"] == 3e-2 and not d["pass"]
    assert d["per_dim_max"][5] == 3e-2 and abs(d["per_dim_max"][3] - 1e-2) < 1e-12
    assert d["median"] == 0.0
    assert bench.chunk_delta(ref, ref)["pass"]


def test_oracle_subsets_are_the_batched_workloads_query_subsets():
    """The CPU baseline times the oracle on 4 of 32, 2 of 8 and 4 of 256 queries
    of the batched workloads; each subset is a proper prefix of the batch."""
    assert bench.ORACLE_SUBSETS == {"smolvla_b32": 4, "long_prefix_b8": 2, "denoise_b256": 4}
    for name, n in bench.ORACLE_SUBSETS.items():
        assert 0 < n < synth.WORKLOADS[name].B


def test_traffic_figures_follow_the_sources_they_were_captured_on(tmp_path, monkeypatch):
    """A recorded ncu traffic figure is reported only while the CUDA sources
    hash to the value recorded with it."""
    import json
    f = tmp_path / "t.json"
    f.write_text(json.dumps({"kernels": {"k": {"dram_bytes_per_launch": 123.0,
                                               "sources_sha16": bench.sources_sha16()}}}))
    monkeypatch.setattr(bench, "TRAFFIC_FILE", str(f))
    assert bench.ncu_traffic("k") == 123.0
    assert bench.ncu_traffic("absent") is None
    f.write_text(json.dumps({"kernels": {"k": {"dram_bytes_per_launch": 123.0, "sources_sha16": "0" * 16}}}))
    assert bench.ncu_traffic("k") is None


def test_clock_summary_decodes_the_event_reasons():
    """The sampler keeps (SM MHz, max SM MHz, NVML clock-event reason bits); the
    summary reports the median, the maximum and the throttle reasons seen."""
    assert bench.summarize_clocks([]) is None
    s = bench.summarize_clocks([(1965.0, 1965.0, 0x0), (1950.0, 1965.0, 0x4), (1965.0, 1965.0, 0x1)])
    assert s == {"sm_mhz": 1965.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"], "samples": 3}
    s = bench.summarize_clocks([(1200.0, 1965.0, 0x8 | 0x40), (1100.0, 1965.0, 0x20)])
    assert s["reasons"] == ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown"]
    assert s["sm_mhz"] == 1150.0
    # without a GPU the sampler reports nothing rather than failing
    c = bench.Clocks(0)
    c.start()
    r = c.stop()
    assert r is None or isinstance(r, dict)
