"""Host arithmetic of bench.py's roofline: the algorithmic FLOPs and bytes of
the grouped GEMM, checked against the counts written out by hand."""
import bench
import workloads


def test_layer_flops_prefill():
    cfg = workloads.CONFIGS["prefill"]
    # 6 d I per (token, expert) pair: 8192 tokens x (8 routed + 1 shared)
    assert bench.layer_flops(cfg) == 6 * 7168 * 2048 * (8192 * 8 + 8192)
    assert abs(bench.layer_flops(cfg) / 1e12 - 6.494) < 1e-3


def test_gemm_algorithmic_bytes_terms():
    cfg = workloads.CONFIGS["prefill"]
    d, I, rows = 7168, 2048, 8192 * 9
    expert = 3 * d * I + 3 * (d // 128) * (I // 128) * 4      # E4M3 codes + FP32 block scales
    acts = rows * (d + (d // 128) * 4)
    inter = 2 * rows * (I + (I // 128) * 4)                    # H written, then read
    outs = rows * d * 4                                         # FP32 expert outputs
    assert bench.gemm_algorithmic_bytes(cfg, 256) == 257 * expert + acts + inter + outs
    # only the shared expert's weights when no routed expert is touched
    assert bench.gemm_algorithmic_bytes(cfg, 0) == expert + acts + inter + outs
    assert abs(bench.gemm_algorithmic_bytes(cfg, 256) / 1e9 - 14.29) < 0.01


def test_prefill_is_tensor_bound_and_decode_hbm_bound():
    peaks = bench._peaks()
    ridge = 2 * peaks["bf16_sustained"] * 1e12 / (peaks["hbm_gbs"] * 1e9)
    pre, dec = workloads.CONFIGS["prefill"], workloads.CONFIGS["decode"]
    assert bench.layer_flops(pre) / bench.gemm_algorithmic_bytes(pre, 256) > ridge
    assert bench.layer_flops(dec) / bench.gemm_algorithmic_bytes(dec, 256) < ridge
