"""The benchmark's accounting on the host: kept-tile counts and FLOPs for
every workload against hand-derived totals, the weak-scaling aggregate, and
when the stored ncu traffic figure applies."""
import os
import sys

import pytest

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
import bench  # noqa: E402
from gen import config, derived_sizes  # noqa: E402
import block_sparse_attention_47_b200 as bsa  # noqa: E402


def keep_of(cfg):
    # the library's closed form; the oracle pins cover the same function
    return bsa.keep_count(derived_sizes(cfg)["nbv"], cfg["keep_ratio"])


@pytest.mark.parametrize("name,over,tiles", [
    # video query blocks x (prefix blocks + keep) + prefix query blocks x all blocks
    ("tiny", {}, 1 * 2 * 32 * 8),                              # 512
    ("lowres", {}, 24 * 504 * 126),                            # 1,524,096
    ("720p", {}, 2 * 24 * 1920 * 480),                         # 44,236,800
    ("720p", {"keep_ratio": 0.0625}, 2 * 24 * 1920 * 120),     # 11,059,200
    ("ref_prefix", {}, 24 * (2016 * (44 + 504) + 44 * 2060)),  # 28,689,792
    ("sweep", {"keep_ratio": 0.01}, 24 * 1440 * 15),           # 34,560 * 15
])
def test_kept_tiles(name, over, tiles):
    cfg = config(name, **over)
    assert bench.kept_tiles(cfg, keep_of(cfg)) == tiles


def test_tile_flops_and_720p_total():
    cfg = config("720p")
    assert bench.tile_flops(cfg) == 4 * 64 * 64 * 128 == 2_097_152
    total = bench.kept_tiles(cfg, keep_of(cfg)) * bench.tile_flops(cfg)
    assert total == pytest.approx(92.77e12, rel=1e-3)
    assert bench.dense_tiles(cfg) * bench.tile_flops(cfg) == pytest.approx(371.1e12, rel=1e-3)
    assert bench.tile_flops(config("tiny")) == 1_048_576


def test_whole_job_aggregate():
    # weak scaling: N ranks' work over the slowest rank's time
    assert bench.whole_job_tflops(1, 92.8e12, 116.0) == pytest.approx(800.0, rel=1e-3)
    assert bench.whole_job_tflops(8, 92.8e12, 116.0) == pytest.approx(6400.0, rel=1e-3)


def test_traffic_figure_only_for_its_workload(monkeypatch):
    cfg = config("720p")
    have = bench.attn_traffic(cfg, 0.25)
    if have is not None:  # the stored capture matches today's kernel source
        assert have == pytest.approx(bench.ATTN_TRAFFIC["bytes_per_bh"] * 2 * 24)
    # other workloads never borrow the figure
    assert bench.attn_traffic(config("720p"), 0.0625) is None
    assert bench.attn_traffic(config("720p_dyn"), 0.25) is None
    assert bench.attn_traffic(config("lowres"), 0.25) is None
    # a changed kernel source voids it
    monkeypatch.setitem(bench.ATTN_TRAFFIC, "sha256", "0" * 64)
    assert bench.attn_traffic(cfg, 0.25) is None


def test_stage_bandwidth(monkeypatch):
    cfg = config("720p")
    R = 2 * 122880 * 24 * 128 * 2                      # one raster tensor, 1.51 GB
    # permuted path: permute (pooling fused in) moves Q, K, V; no pool stage
    gbs = bench.stage_bandwidth(cfg, {"permute": 1.4, "pool": 0.003, "unpermute": 0.65,
                                      "layout": 0.009, "select": 2.9})
    assert gbs["permute"] == pytest.approx(6 * R / 1.4e-3 / 1e9, rel=1e-3)
    assert gbs["unpermute"] == pytest.approx(2 * R / 0.65e-3 / 1e9, rel=1e-3)
    assert set(gbs) == {"permute", "unpermute"}  # fixed layout reads nothing
    dyn = bench.stage_bandwidth(config("720p_dyn"), {"layout": 1.2, "permute": 1.9})
    assert dyn["layout"] == pytest.approx(R / 1.2e-3 / 1e9, rel=1e-3)
    assert bench.stage_bandwidth(cfg, {}) == {}
    # permute-free path: pool_raster reads raster Q and K
    monkeypatch.setitem(bench.PATH, "path", "raster")
    gbs = bench.stage_bandwidth(cfg, {"permute": 0.0, "pool": 0.6, "unpermute": 0.0})
    assert set(gbs) == {"pool"}
    assert gbs["pool"] == pytest.approx(2 * R / 0.6e-3 / 1e9, rel=1e-3)


def test_mma_rate_fraction_at_clock():
    # 148 SMs x 8,192 FLOP per clock at 1,000 MHz is 1,212.4 TFLOP/s
    assert bench.mma_rate_frac(1212.416, {"sm_mhz": 1000.0}) == pytest.approx(1.0)
    assert bench.mma_rate_frac(606.208, {"sm_mhz": 1000.0}) == pytest.approx(0.5)
    assert bench.mma_rate_frac(500.0, None) is None
    assert bench.mma_rate_frac(500.0, {"sm_mhz": None}) is None


def test_peaks_fall_back_per_missing_number(tmp_path, monkeypatch):
    """The generated peaks file: each number it gives is used, each one it
    lacks (or gives in an unusable form) comes from the fallback figures."""
    import json
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    p, kind = bench.peaks()
    assert kind == "fallback" and p == bench.FALLBACK_PEAKS
    (tmp_path / "MEASURED_PEAKS.json").write_text(json.dumps(
        {"hbm_gbs": 6464.9, "bf16_tflops": "n/a", "clocks": {"sm": 1965}}))
    p, kind = bench.peaks()
    assert kind == "fallback"
    assert p["hbm_gbs"] == 6464.9 and p["bf16_tflops"] == bench.FALLBACK_PEAKS["bf16_tflops"]
    (tmp_path / "MEASURED_PEAKS.json").write_text(json.dumps(
        {"hbm_gbs": 6464.9, "bf16_tflops": 1641.7, "bf16_tflops_sustained": 1368.0}))
    p, kind = bench.peaks()
    assert kind == "measured" and p["bf16_tflops_sustained"] == 1368.0
    (tmp_path / "MEASURED_PEAKS.json").write_text("[1, 2]")
    assert bench.peaks() == (bench.FALLBACK_PEAKS, "fallback")
