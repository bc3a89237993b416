"""Host-side helpers of bench.py that turn event times into reported rates (CPU only)."""
import bench
import linear_global_attention_b200 as zb


def test_stage_rates_arithmetic():
    g = zb.geom(2, 16, 16, 2)          # T = 8 tiles, 512 patches, no partial tiles
    kern = {"pool_pack": (4, 8.0), "tile_scores": (8, 4.0), "tile_select": (8, 2.0)}
    r = bench.stage_rates(kern, g, 1000.0)
    T, t_pad, H, patches = 8, 64, 2, 512
    nbytes = 3 * patches * H * 64 * 2 + 3 * H * T * 64 * 64 * 2 + 3 * H * T * 64 * 4 + 2 * H * t_pad * 64 * 2
    assert r["pool_pack"]["bytes_per_layer"] == nbytes
    assert r["pool_pack"]["ms_per_layer"] == 2.0           # 8 ms over 4 layers
    assert abs(r["pool_pack"]["gbs"] - round(nbytes / 2e-3 / 1e9, 1)) < 1e-9
    assert r["tile_scores"]["ms_per_layer"] == 1.0
    assert abs(r["tile_scores"]["fp32_score_tflops"] - round(2 * 64 * T * T * H / 1e-3 / 1e12, 2)) < 1e-9
    assert abs(r["tile_scores"]["bf16_gemm_tflops"] - round(2 * 384 * T * T * H / 1e-3 / 1e12, 1)) < 1e-9
    assert bench.stage_rates({}, g, 1000.0) == {}


def test_stage_rates_dense_kv_rows():
    """13 x 11 grid: tiles 8x8, 8x3, 5x8 and the 5x3 corner, whose 15 rows take 16 in the
    dense K/V layout: 64 + 24 + 40 + 16 = 144 rows per view instead of 4 x 64."""
    g = zb.geom(3, 13, 11, 2)
    r = bench.stage_rates({"pool_pack": (1, 1.0)}, g, 1000.0)
    T, t_pad, H, patches = 12, 64, 2, 3 * 143
    nbytes = (3 * patches * H * 128 + H * T * 64 * 128 + 2 * H * 3 * 144 * 128
              + 3 * H * T * 64 * 4 + 2 * H * t_pad * 128)
    assert r["pool_pack"]["bytes_per_layer"] == nbytes


def test_sparse_traffic_is_null_for_other_sources(monkeypatch):
    monkeypatch.setattr(bench, "SPARSE_TRAFFIC", {"bytes_per_item": 100.0, "sources_sha1": "0" * 40})
    assert bench.sparse_traffic_per_launch(592) is None
    monkeypatch.setattr(bench, "SPARSE_TRAFFIC", {"bytes_per_item": 100.0, "sources_sha1": bench.sparse_sources_sha1()})
    assert bench.sparse_traffic_per_launch(592) == 59200
