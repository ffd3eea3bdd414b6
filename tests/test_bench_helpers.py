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
    outs = rows * d * 2                                         # bf16 expert outputs
    assert bench.gemm_algorithmic_bytes(cfg, 256) == 257 * expert + acts + inter + outs
    # only the shared expert's weights when no routed expert is touched
    assert bench.gemm_algorithmic_bytes(cfg, 0) == expert + acts + inter + outs
    assert abs(bench.gemm_algorithmic_bytes(cfg, 256) / 1e9 - 13.234) < 0.001


def test_roofline_bound_is_the_slower_ideal_time():
    peaks = dict(hbm_gbs=6540.0, bf16=1631.7, bf16_sustained=1358.8, source="measured")
    pre, dec = workloads.CONFIGS["prefill"], workloads.CONFIGS["decode"]
    # prefill: 6.494 TFLOP at 3263.4 TF/s = 1.990 ms; 13.234 GB at 6540 GB/s = 2.024 ms
    r = bench.roofline(pre, 5.917e-3, 256, peaks)
    assert abs(r["ideal_ms_tensor"] - 1.990) < 1e-3 and abs(r["ideal_ms_hbm"] - 2.024) < 1e-3
    assert r["bound"] == "hbm" and r["unit"] == "GB/s" and r["peak"] == 6540.0
    assert r["frac"] == r["achieved"] / 6540.0 == r["frac_of_hbm"]
    assert r["gemm_tflops"] == bench.layer_flops(pre) / 5.917e-3 / 1e12
    assert abs(r["frac_of_fp8_burst"] - 0.3363) < 1e-3           # 1097.5 / 3263.4
    assert abs(r["frac_of_fp8_sustained"] - 0.4038) < 1e-3
    assert abs(r["frac_of_fp8_nominal"] - 1097.5 / 4500) < 1e-3
    # with a faster copy the same call is tensor-bound, against the burst peak
    t = bench.roofline(pre, 5.917e-3, 256, dict(peaks, hbm_gbs=8000.0))
    assert t["bound"] == "tensor" and t["peak"] == 2 * 1631.7 and t["frac"] == t["frac_of_fp8_burst"]
    d = bench.roofline(dec, 1.9e-3, 256, peaks)
    assert d["bound"] == "hbm" and d["ideal_ms_hbm"] > 10 * d["ideal_ms_tensor"]


def test_clock_samples_inside_the_region_only():
    import datetime
    t0 = datetime.datetime(2026, 1, 2, 3, 4, 5).timestamp()

    def line(dt, mhz, cap="Not Active"):
        ts = datetime.datetime.fromtimestamp(t0 + dt).strftime("%Y/%m/%d %H:%M:%S.%f")[:-3]
        return f"{ts}, 0, {mhz}, 1965, 900.0, 0x0, Not Active, Not Active, Not Active, {cap}"

    lines = [line(-1.0, 300), line(0.05, 1900), line(0.1, 1500, "Active"), line(0.15, 1700),
             line(2.0, 300)]
    s = bench.ClockSampler.parse(lines, t0, t0 + 0.2)
    assert s["samples"] == 3 and s["sm_mhz"] == 1700 and s["sm_max_mhz"] == 1965
    assert s["reasons"] == ["sw_power_cap"]
    assert bench.ClockSampler.parse([], t0, t0 + 1)["reasons"] == ["unsampled"]


def test_gemm_traffic_only_for_the_source_it_was_taken_on(tmp_path, monkeypatch):
    """The bench reports a committed DRAM-traffic figure only while the GEMM
    source hashes to the value recorded beside it."""
    import shutil
    cfg = workloads.CONFIGS["prefill"]
    root = tmp_path / "repo"
    (root / "profiles").mkdir(parents=True)
    csrc = root / "fine_grained_fp8_sigmoid_b200" / "csrc"
    csrc.mkdir(parents=True)
    shutil.copy(bench.os.path.join(bench.ROOT, "fine_grained_fp8_sigmoid_b200", "csrc", "gemm.cu"), csrc / "gemm.cu")
    sha = bench.gemm_source_sha256(str(csrc))
    prof = root / "profiles" / "grouped_gemm_prefill_traffic.md"
    prof.write_text(f"gemm_cu_sha256: {sha}\ndram_bytes_per_call: 123456789\n")
    monkeypatch.setattr(bench, "ROOT", str(root))
    assert bench.gemm_traffic(cfg) == 123456789.0
    (csrc / "gemm.cu").write_text((csrc / "gemm.cu").read_text() + "// changed\n")
    assert bench.gemm_traffic(cfg) is None
    assert bench.gemm_traffic(workloads.CONFIGS["decode"]) is None     # no profile for it
