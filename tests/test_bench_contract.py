"""The bench's roofline arithmetic on the CPU: the algorithmic bytes each row
is divided by, against the per-call figures worked out from the formats
(nibbles, one E4M3 scale per 16 or one UE8M0 per 32, BF16 activations and
outputs, one fp32 tensor scale), and the source lists that key the committed
DRAM-traffic figures."""
import json
import os

import bench

N, K = bench.MLP, bench.HIDDEN  # the 27B-class MLP layer: 17408 x 5120


def test_layer_shape():
    assert (N, K) == (17408, 5120)


def test_gemv_bytes():
    # 44 564 480 nibble bytes + 5 570 560 scale bytes + x 10 240 + y 34 816 + g 4
    assert bench.gemv_bytes(N, K) == 44_564_480 + 5_570_560 + 10_240 + 34_816 + 4 == 50_180_100


def test_gemm_bytes():
    # weights + X [M, K] + Y [M, N] (BF16) + g
    assert bench.gemm_bytes(32, N, K) == 50_135_040 + 327_680 + 1_114_112 + 4
    assert bench.gemm_bytes(512, N, K) == 50_135_040 + 5_242_880 + 17_825_792 + 4 == 73_203_716


def test_quantize_bytes():
    # amax pass (read W) + quantize pass (read W, write q and s)
    w = 2 * N * K
    assert bench.quantize_bytes(N, K) == 2 * w + 44_564_480 + 5_570_560 == 406_650_880


def test_mxfp4_bytes():
    # one UE8M0 byte per 32 elements, no tensor scale
    assert bench.mx_gemv_bytes(N, K) == 44_564_480 + 2_785_280 + 10_240 + 34_816 == 47_394_816
    assert bench.mx_quantize_bytes(N, K) == 2 * N * K + 44_564_480 + 2_785_280


def test_w4a4_gemm_bytes():
    # weights, FP4 activations + their E4M3 scales, Y, g and x_amax
    assert bench.w4a4_gemm_bytes(512, N, K) == 50_135_040 + 1_310_720 + 163_840 + 17_825_792 + 8 == 69_435_400


def test_moe_bytes():
    # 8 experts of [1536, 2048]: codes + scales + y rows + ids and g, plus x
    e = 1536 * 2048 // 2 + 1536 * 2048 // 16
    assert bench.moe_bytes(8, 1536, 2048) == 8 * (e + 2 * 1536 + 8 + 4) + 2 * 2048


def test_fp4_peak_ratio():
    # NVIDIA's dense figures for B200: 9 PFLOP/s FP4 and 2.25 PFLOP/s BF16
    assert bench.FP4_PER_BF16 == 9 / 2.25


def test_traffic_rows_name_existing_sources():
    for row, files in bench.KERNEL_SOURCES.items():
        for f in files:
            assert os.path.exists(os.path.join(bench.ROOT, f)), (row, f)


def test_down_projection_bytes():
    # the MLP down projection W [5120, 17408]: nibbles + scales + x [17408] + y [5120] + g
    assert bench.gemv_bytes(5120, 17408) == 44_564_480 + 5_570_560 + 34_816 + 10_240 + 4 == 50_180_100


def test_dram_attested_fraction():
    # measured DRAM bytes per call over the event time, against the HBM peak:
    # 363.2 MB of quantizer traffic in 66.46 us at a 6542.4 GB/s peak
    d = bench.dram_attested(363_160_613, 66.46, 6542.4)
    assert abs(d["GB/s_dram"] - 363_160_613 / 66.46e-6 / 1e9) < 1e-6
    assert abs(d["frac_hbm_dram"] - d["GB/s_dram"] / 6542.4) < 1e-12
    assert 0.83 < d["frac_hbm_dram"] < 0.84
    assert bench.dram_attested(None, 66.46, 6542.4) == {"GB/s_dram": None, "frac_hbm_dram": None}


def test_moe_multi_token_bytes():
    # 4 tokens x top-8: 32 problems' expert weights + y rows + ids and g, and the 4 token rows of x
    P = bench.MOE_T * bench.MOE["top"]
    e = 1536 * 2048 // 2 + 1536 * 2048 // 16
    assert bench.moe_bytes(P, 1536, 2048) + 2 * 2048 * (bench.MOE_T - 1) == P * (e + 2 * 1536 + 8 + 4) + 2 * 2048 * bench.MOE_T


def test_traffic_only_for_the_source_it_was_taken_on(tmp_path, monkeypatch):
    # a committed DRAM figure is reported while the row's kernel sources are
    # unchanged, and becomes None (reported as null) once any of them changes
    src = tmp_path / "k.cu"
    src.write_text("kernel v1\n")
    (tmp_path / "profiles").mkdir()
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setitem(bench.KERNEL_SOURCES, "gemv", ["k.cu"])
    table = {"gemv": {"dram_bytes_per_call": 123, "source_hash": bench.kernel_source_hash(["k.cu"])}}
    (tmp_path / "profiles" / "traffic.json").write_text(json.dumps(table))
    assert bench.traffic_from_profiles("gemv") == 123
    src.write_text("kernel v2\n")
    assert bench.traffic_from_profiles("gemv") is None
    assert bench.traffic_from_profiles("gemm_m32") is None  # no entry for the row
