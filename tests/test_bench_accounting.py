"""The bench's algorithmic work counts (CPU only)."""
import math

import bench


def test_update_term_matches_pages_hand_count():
    # page "线性注意力与 SSM", §02: N=32768, dphi=128, dv=64 -> about 2.684e8 MACs per head
    m = bench.update_macs(32768, 128, 64)
    assert m == 268_435_456
    assert abs(m - 2.684e8) / 2.684e8 < 1e-3


def test_algorithmic_bytes_of_the_workloads():
    mb = lambda b: round(b / 1e6, 1)
    assert mb(bench.prefill_bytes("gdn", 2, 8192, 16, 128, 128)) == 272.6
    assert mb(bench.prefill_bytes("gla", 2, 8192, 16, 128, 128)) == 404.8
    assert mb(bench.prefill_bytes("elu", 1, 32768, 16, 128, 64, with_S0=True, with_z=True)) == 403.7
    assert mb(bench.decode_bytes("gla", 256, 16, 128, 128)) == 543.2
    assert mb(bench.decode_bytes("gdn", 256, 16, 128, 128)) == 541.1


def test_macs_per_token_head():
    # C=64: causal pairs P = 2080; GLA = P(dk+dv)/C + 2 dk dv
    assert bench.macs_per_token_head("gla", 128, 128) == 2080 * 256 / 64 + 2 * 128 * 128
    assert math.isclose(bench.macs_per_token_head("gdn", 128, 128),
                        41088 + 31.5 * 128 + 31.5 * 256 + 128 * 128)
    assert math.isclose(bench.macs_per_token_head("elu", 128, 64), 22912.5)


def test_reference_arm_sample_runs():
    dt, tokens = bench.oracle_sample(16)
    assert tokens == 32 and dt > 0


def test_traffic_record_is_valid_per_leg(tmp_path, monkeypatch):
    """A leg's committed DRAM traffic stays valid while the csrc files behind its
    kernels are unchanged; editing one file voids exactly the legs that list it."""
    import json
    csrc = tmp_path / "gated_delta_rule_attn_b200" / "csrc"
    csrc.mkdir(parents=True)
    files = sorted({f for fs in bench.LEG_SOURCES.values() for f in fs})
    for f in files:
        (csrc / f).write_text(f"// {f}\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    legs = {leg: {"bytes_per_launch": 1000 + i, "source_hash": bench.kernel_source_hash(fs)}
            for i, (leg, fs) in enumerate(bench.LEG_SOURCES.items())}
    (tmp_path / "profiles").mkdir()
    (tmp_path / "profiles" / "traffic.json").write_text(json.dumps({"legs": legs}))
    assert set(bench.load_traffic()) == set(bench.LEG_SOURCES)
    (csrc / "chunk_ge.cuh").write_text("// edited\n")
    valid = bench.load_traffic()
    for leg, fs in bench.LEG_SOURCES.items():
        assert (leg in valid) == ("chunk_ge.cuh" not in fs), leg
    assert valid["gdn_prefill"] == legs["gdn_prefill"]["bytes_per_launch"]


def test_cpu_baseline_records_its_host():
    """The oracle baseline says where it ran: the cores this process may use, the
    CPU model and the OpenMP threads, and the single-sequence fp32 time."""
    h = bench.host_cpu()
    assert h["affinity_cores"] >= 1 and h["omp_threads"] >= 1
    assert "cpu_model" in h
    assert bench.oracle_elu_small_ms(reps=1) > 0
