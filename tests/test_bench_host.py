"""Host-side logic of the bench and the build (no GPU): FLOP count, traffic bookkeeping, the
register check that guards the setmaxnreg split, and the JSON config."""
import bench
from w4a4_rank_absorbed_b200 import build
from w4a4_rank_absorbed_b200.synth import make_workload


def test_layer_flops_counts_gemm_and_both_projections():
    M, K, N, r = 4608, 3072, 9216, 32
    assert bench.layer_flops(M, K, N, r) == 2.0 * M * N * K + 2.0 * M * r * K + 2.0 * M * r * N
    assert bench.layer_flops(M, K, N, 0) == 2.0 * M * N * K


def test_traffic_is_reported_only_for_the_profiled_sources(monkeypatch):
    h = bench.linear_sources_hash()
    assert len(h) == 16
    monkeypatch.setattr(bench, "LINEAR_TRAFFIC", {"qkv": {"bytes": 123.0, "sources": h}})
    assert bench.linear_traffic("qkv") == 123.0
    assert bench.linear_traffic("large") is None
    monkeypatch.setattr(bench, "LINEAR_TRAFFIC", {"qkv": {"bytes": 123.0, "sources": "0" * 16}})
    assert bench.linear_traffic("qkv") is None


def test_entry_register_parser():
    log = "\n".join([
        "ptxas info    : Compiling entry function '_ZN4svdq13k_linear_pairE14CUtensorMap_st' for 'sm_100a'",
        "ptxas info    : Function properties for _ZN4svdq13k_linear_pairE14CUtensorMap_st",
        "    8 bytes stack frame, 4 bytes spill stores, 8 bytes spill loads",
        "ptxas info    : Used 128 registers, used 0 barriers",
        "ptxas info    : Compiling entry function '_ZN4svdq8k_linearE14CUtensorMap_st' for 'sm_100a'",
        "ptxas info    : Used 120 registers, used 1 barriers",
    ])
    assert build.entry_registers(log, "13k_linear_pairE") == 128
    assert build.entry_registers(log, "8k_linearE") == 120
    assert build.entry_registers(log, "k_missing") is None


def test_workload_config_names_the_workload_and_sizes():
    wl = make_workload("tiny")
    cfg = bench.workload_config(wl)
    assert cfg["workload"].startswith("tiny")
    assert (cfg["M"], cfg["K"], cfg["N"], cfg["r"]) == (wl.M, wl.K, wl.N, wl.r_eff)
    assert "L2" in cfg["l2"] and "graph" in cfg["launch"]


def test_row_blocks_partition_the_batch():
    for M in (1, 7, 4608, 18432):
        for world in (1, 2, 3, 8):
            blocks = [bench.row_block(M, r, world) for r in range(world)]
            assert blocks[0][0] == 0 and blocks[-1][1] == M
            assert all(a[1] == b[0] for a, b in zip(blocks, blocks[1:]))
            sizes = [hi - lo for lo, hi in blocks]
            assert max(sizes) - min(sizes) <= 1


def test_stats_median_and_percentiles():
    st = bench.stats([5.0, 1.0, 3.0, 2.0, 4.0])
    assert st["median"] == 3.0 and st["n"] == 5
    assert 1.0 <= st["p10"] <= 2.0 and 4.0 <= st["p90"] <= 5.0


def test_byte_counts():
    M, K, N, r = 4608, 3072, 9216, 32
    assert bench.quantize_bytes(M, K, r) == 2 * M * K + M * K / 2 + M * K / 16 + 2 * M * r
    assert bench.linear_flops(M, K, N, r) == 2.0 * M * N * K + 2.0 * M * N * r
    assert bench.unfused_extra_bytes(M, K, N, r) == 2.0 * M * K + 4.0 * M * N


def test_clock_summary_flags_throttle_reasons():
    rows = [["0", "1965", "1965", "900", "0x0", "Not Active", "Not Active", "Not Active", "Active"],
            ["0", "1900", "1965", "950", "0x4", "Not Active", "Not Active", "Not Active", "Not Active"]]
    got = bench.ClockSampler.summarize(rows)
    assert got["sm_max_mhz"] == 1965.0 and got["reasons"] == ["sw_power_cap"] and got["samples"] == 2
