"""Host-side arithmetic of bench.py: the algorithmic flop counts behind the
TFLOP/s figures, checked against counts written out from the iteration's
structure (one GEMM per product, symmetric Gram products at n(n+1)K)."""
import bench


def test_coupled_gemm_count_per_pass():
    # k updates: the first step (R_0 formed elementwise, Z_1 = g) costs the
    # R^2 and Y g products; each later step R = I - Z Y, R^2, Y g, g Z; plus
    # the final residual: 2 + 4 (k - 1) + 1 = 4k - 1
    for k in range(1, 12):
        assert bench.gemm_count([k]) == 2 + 4 * (k - 1) + 1
    assert bench.gemm_count([0]) == 0
    assert bench.gemm_count([10, 6]) == 62


def test_config3_block_flops():
    # 10 + 6 iterations at n = 1024: 62 products of 2 n^3 = 133.1 GFLOP per block
    f = bench.block_flops([10, 6], 1024)
    assert f == 62 * 2 * 1024 ** 3
    assert abs(f / 1e9 - 133.1) < 0.1


def test_polar_flops_per_matrix():
    # 4096 x 1024: per update X^T X on the upper triangle n(n+1)m, R^2
    # n(n+1)n, X Delta 2mn^2; plus the final X^T X.  13 updates: 185.8 GFLOP
    m, n, k = 4096, 1024, 13
    want = k * (n * (n + 1) * m + n * (n + 1) * n + 2 * m * n * n) + n * (n + 1) * m
    assert bench.polar_flops(k) == want
    assert abs(bench.polar_flops(k) / 1e9 - 185.8) < 0.1


def test_workload_config_names_the_workload():
    cfg = bench.workload_config(1)
    assert cfg["workload"].startswith("inv4_root_64x1024sq")
    assert "l2" in cfg and cfg["parallelism"] == "replicas x1"
