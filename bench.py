"""Benchmark of the DeepSeekMoE FP8 layer forward pass on B200.

One step = the whole layer on one batch: route -> quant_1x128 -> permute ->
grouped FP8 GEMM (256 routed experts top-8 + 1 shared, SwiGLU, requant,
down) -> combine -> bias update. The workload is the full DeepSeek-V3 layer
shape at prefill (T=8192 tokens, d=7168, 256 routed top-8 + 1 shared,
I=2048), synthetic seeded inputs already resident in HBM.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

With N > 1 (torchrun), every rank runs its own replica on its own batch
(weak scaling; the layer needs no exchange between replicas); the time is the
max over ranks. Rank 0 prints one JSON line.

--impl reference times the CPU oracle (the plain float64 reference of the
same layer) on the host cores, on a bounded sample of tokens per step.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "DeepSeekMoE FP8 layer tokens/s + TFLOP/s, % FP8 tensor peak (1×B200)"
CONFIG_NAME = "prefill"


def _peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return dict(hbm_gbs=float(p["hbm_gbs"]), bf16=float(p["bf16_tflops"]),
                    bf16_sustained=float(p.get("bf16_tflops_sustained", p["bf16_tflops"])),
                    source="measured")
    except Exception:
        return dict(hbm_gbs=6650.0, bf16=1590.0, bf16_sustained=1400.0, source="fallback")


def gemm_source_sha256(csrc):
    """sha256 of the grouped GEMM's source (gemm.cu)."""
    import hashlib
    h = hashlib.sha256()
    for name in ("gemm.cu",):
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def gemm_traffic(cfg):
    """DRAM bytes per moe_grouped_gemm_fp8 call from the committed ncu summary,
    if it was taken on this workload with the current GEMM source; else None."""
    import hashlib
    import re
    csrc = os.path.join(ROOT, "fine_grained_fp8_sigmoid_b200", "csrc")
    prof = os.path.join(ROOT, "profiles", f"grouped_gemm_{cfg.name}_traffic.md")
    try:
        sha = gemm_source_sha256(csrc)
        txt = open(prof).read()
        if re.search(r"gemm_cu_sha256:\s*" + sha, txt) is None:
            return None
        m = re.search(r"dram_bytes_per_call:\s*([0-9.eE+]+)", txt)
        return float(m.group(1)) if m else None
    except OSError:
        return None


def max_over_ranks(value: float, device=None) -> float:
    """The slowest rank's value (every rank calls this at the same point)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_tokens_per_s(tokens_per_rank: int, world: int, ms_per_step: float) -> float:
    """Tokens of all replicas per second, timed by the slowest rank."""
    return world * tokens_per_rank / (ms_per_step / 1e3)


def layer_flops(cfg, rows_routed=None):
    """Algorithmic FLOPs of the expert GEMMs: 6*d*I per (token, expert) pair
    (gate, up, down), routed pairs plus the shared expert on every token."""
    P = cfg.T * cfg.K_r if rows_routed is None else rows_routed
    return 6.0 * cfg.d * cfg.I * (P + cfg.T)


def weight_bytes(cfg):
    """E4M3 codes plus FP32 block scales of all N_r + 1 experts."""
    per = 3 * cfg.d * cfg.I + 3 * (cfg.d // 128) * (cfg.I // 128) * 4
    return (cfg.N_r + 1) * per


def gemm_algorithmic_bytes(cfg, touched_routed):
    """Bytes one moe_grouped_gemm_fp8 call must move at least: the weights of
    the touched routed experts and the shared one, read once; the permuted
    and shared activations with their scales; the intermediate H written and
    read back; the bf16 outputs written."""
    per_expert = 3 * cfg.d * cfg.I + 3 * (cfg.d // 128) * (cfg.I // 128) * 4
    rows = cfg.T * cfg.K_r + cfg.T
    acts = rows * (cfg.d + cfg.d // 128 * 4)
    inter = 2 * rows * (cfg.I + cfg.I // 128 * 4)
    outs = rows * cfg.d * 2
    return (touched_routed + 1) * per_expert + acts + inter + outs


def workload_desc(cfg):
    return (f"DeepSeek-V3 MoE layer, {cfg.name}: T={cfg.T}, d={cfg.d}, {cfg.N_r} routed experts "
            f"top-{cfg.K_r} + 1 shared, SwiGLU I={cfg.I}, E4M3 1x128/128x128 scales")


class ClockSampler:
    """Samples SM clocks and throttle reasons with nvidia-smi (every 20 ms)
    around a region; summary() keeps the samples taken between mark_start()
    and mark_end() (nvidia-smi stamps each sample with the wall clock)."""

    FIELDS = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    REASONS = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]

    def __init__(self, index: int, period_ms: int = 20):
        self.index = index
        self.period_ms = period_ms
        self.proc = None
        self.lines = []
        self.t0 = self.t1 = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", str(self.period_ms)],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True, bufsize=1)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
            deadline = time.time() + 10.0        # nvidia-smi takes a moment to start
            while not self.lines and time.time() < deadline and self.proc.poll() is None:
                time.sleep(0.01)
        except Exception:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def mark_start(self):
        self.t0 = time.time()

    def mark_end(self):
        self.t1 = time.time()

    def __exit__(self, *a):
        if self.proc is not None:
            time.sleep(2.5 * self.period_ms / 1e3)   # the samples of the region's last moments
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    @staticmethod
    def parse(lines, t0=None, t1=None):
        """Median SM clock, max clock and throttle reasons of the samples whose
        timestamp lies in [t0, t1] (epoch seconds; None: no bound)."""
        import datetime
        sm, mx, reasons = [], None, set()
        for ln in lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 10:
                continue
            try:
                ts = datetime.datetime.strptime(parts[0], "%Y/%m/%d %H:%M:%S.%f").timestamp()
                clk, cmax = float(parts[2]), float(parts[3])
            except ValueError:
                continue
            if (t0 is not None and ts < t0 - 0.02) or (t1 is not None and ts > t1 + 0.02):
                continue
            sm.append(clk)
            mx = cmax
            for n, v in zip(ClockSampler.REASONS, parts[6:10]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}

    def summary(self):
        return self.parse(self.lines, self.t0, self.t1)


# ---------------------------------------------------------------- CPU oracle

def _oracle_sample_setup(cfg, tokens, device="cuda"):
    """Inputs of a small token sample and the oracle-quantised weights of the
    experts it touches (untimed preparation)."""
    from concurrent.futures import ThreadPoolExecutor

    import numpy as np

    import workloads
    from oracle import moe as O
    u = workloads.activations(cfg, device=device)[tokens].cpu().double().numpy()
    e = workloads.centroids(cfg, device=device).cpu().double().numpy()
    b = workloads.bias(cfg, device=device).cpu().double().numpy()
    _, _, idx, _ = O.route(u, e, b, cfg.K_r)
    slots = sorted(set(idx.reshape(-1).tolist()) | {cfg.N_r})
    raw = {s: [x.cpu().double().numpy() for x in workloads.expert_weights(cfg, s, device=device)]
           for s in slots}
    with ThreadPoolExecutor(max_workers=os.cpu_count() or 8) as ex:
        quant = dict(zip(slots, ex.map(lambda s: O.quantise_expert(*raw[s]), slots)))
    return u, e, b, quant


def _blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:
        return 1


def time_oracle(cfg, n_tokens, steps, device="cuda"):
    """Times the oracle forward on a sample of n_tokens tokens per step (the
    same sample every step). Returns (tokens/s, seconds per step, sample desc)."""
    import numpy as np

    from oracle import moe as O
    tokens = np.arange(n_tokens)
    u, e, b, quant = _oracle_sample_setup(cfg, tokens, device)
    t0 = time.perf_counter()
    for _ in range(steps):
        O.moe_forward(u, e, b, cfg.K_r, quant.__getitem__)
    dt = (time.perf_counter() - t0) / steps
    desc = (f"oracle forward (route, quant, permute, {len(quant)} expert FFNs incl. shared, "
            f"combine, bias update) on tokens 0..{n_tokens - 1} of the {cfg.name} batch, "
            f"weights pre-quantised by the oracle; {steps} steps")
    return n_tokens / dt, dt, desc


# ---------------------------------------------------------------- GPU arm

NOMINAL_FP8_TFLOPS = 4500.0     # dense FP8 on B200 (NVIDIA's figure without sparsity)
NOMINAL_HBM_GBS = 8000.0


def roofline(cfg, gemm_s, touched, peaks):
    """Roofline of the grouped GEMM (one moe_grouped_gemm_fp8 call, 2 launches)
    from its average device time. The roof is the slower of the two ideal
    times: algorithmic FLOPs at the dense FP8 peak, and algorithmic bytes at
    the measured copy bandwidth; "bound" names it, and "frac" is the achieved
    rate over it. The FP8 peak is the measured burst figure (dense FP8 = 2 x
    the measured BF16 GEMM rate, the nominal ratio): the timed regions are
    well under a second of back-to-back steps, not the seconds-long
    power-capped loop of the sustained figure. Fractions of the FP8 peak
    (burst, sustained, nominal) and of the HBM bandwidth are reported beside
    it whichever bound applies."""
    flops = layer_flops(cfg)
    nbytes = gemm_algorithmic_bytes(cfg, touched)
    fp8_burst = 2.0 * peaks["bf16"]
    fp8_sust = 2.0 * peaks["bf16_sustained"]
    tf = flops / gemm_s / 1e12
    gbs = nbytes / gemm_s / 1e9
    t_tensor = flops / (fp8_burst * 1e12)
    t_hbm = nbytes / (peaks["hbm_gbs"] * 1e9)
    common = {"gemm_ms": gemm_s * 1e3, "gemm_tflops": tf, "gemm_gbs": gbs,
              "algorithmic_flops": flops, "algorithmic_bytes": nbytes,
              "ideal_ms_tensor": t_tensor * 1e3, "ideal_ms_hbm": t_hbm * 1e3,
              "frac_of_fp8_burst": tf / fp8_burst, "frac_of_fp8_sustained": tf / fp8_sust,
              "frac_of_fp8_nominal": tf / NOMINAL_FP8_TFLOPS,
              "frac_of_hbm": gbs / peaks["hbm_gbs"], "frac_of_hbm_nominal": gbs / NOMINAL_HBM_GBS,
              "experts_touched": touched + 1}
    if t_tensor >= t_hbm:
        return dict({"bound": "tensor", "achieved": tf, "peak": fp8_burst, "unit": "TFLOP/s",
                     "frac": tf / fp8_burst,
                     "peak_source": f"bf16 burst {peaks['bf16']} TF/s x2 (of {peaks['source']})"},
                    **common)
    return dict({"bound": "hbm", "achieved": gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                 "frac": gbs / peaks["hbm_gbs"],
                 "peak_source": f"copy bandwidth {peaks['hbm_gbs']} GB/s (of {peaks['source']})"},
                **common)


def build_layer(cfg, dev):
    import workloads
    from fine_grained_fp8_sigmoid_b200 import MoELayerFP8
    layer = MoELayerFP8(cfg.T, cfg.d, cfg.N_r, cfg.K_r, cfg.I, device=dev)
    for slot in range(cfg.N_r + 1):
        w = workloads.expert_weights(cfg, slot, device=dev)
        layer.load_expert(slot, *w)
        del w
    u = workloads.activations(cfg, device=dev)
    e = workloads.centroids(cfg, device=dev)
    b0 = workloads.bias(cfg, device=dev)
    return layer, u, e, b0


def time_layer(layer, u, e, b, steps, warmup, dev, world, local_rank):
    """Times `steps` layer steps (after `warmup`), CUDA events on the launching
    stream, a barrier and a synchronize on both sides. Returns (ms per step,
    max over ranks; mean GEMM ms; clock summary)."""
    import numpy as np
    import torch
    import torch.distributed as dist

    from fine_grained_fp8_sigmoid_b200 import binding as B
    stream = torch.cuda.current_stream(dev)
    for _ in range(warmup):
        layer.forward(u, e, b, update_bias=True)
    torch.cuda.synchronize(dev)
    if B.moe_get_error() != 0:
        raise RuntimeError("device error word set during warm-up")
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(steps)]
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local_rank) as clk:
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize(dev)
        clk.mark_start()
        start.record(stream)
        for i in range(steps):
            layer.route(u, e, b)
            layer.quant(u)
            layer.permute()
            ev[i][0].record(stream)
            layer.experts()
            ev[i][1].record(stream)
            layer.combine(u)
            layer.bias_update(b)
        stop.record(stream)
        torch.cuda.synchronize(dev)
        clk.mark_end()
        if world > 1:
            dist.barrier()
    ms_total = max_over_ranks(start.elapsed_time(stop), dev)
    gemm_ms = float(np.mean([a.elapsed_time(z) for a, z in ev]))
    if B.moe_get_error() != 0:
        raise RuntimeError("device error word set during the timed region")
    return ms_total / steps, gemm_ms, clk.summary()


def balance_run(layer, u, e, b, b0, steps=100):
    """The auxiliary-loss-free balancing run: `steps` steps of route ->
    experts -> bias update from the initial bias; max/mean expert load of
    every step (read back once at the end)."""
    import torch
    b.copy_(b0)
    ratios = torch.zeros(steps, device=u.device)
    for i in range(steps):
        layer.forward(u, e, b, update_bias=True)
        ratios[i].copy_(layer.max_over_mean[0])
    r = ratios.cpu().tolist()
    return {"steps": steps, "gamma": 0.001, "max_over_mean_first": r[0],
            "max_over_mean_last": r[-1], "max_over_mean_min": min(r),
            "max_over_mean_every_10": r[::10], "max_over_mean_per_step": r}


def e2e_run(layer, u, e, b, b0, steps, dev, world, cfg):
    """End to end through the public API: every step copies its u from pinned
    host memory in and its h' out. The pipelined form overlaps those copies
    with the kernels (a copy stream, two device input buffers); it is first
    checked bit for bit against the plain form, which is the fallback."""
    import torch
    stream = torch.cuda.current_stream(dev)
    u_host = u.cpu().pin_memory()
    out_host = torch.empty(cfg.T, cfg.d, dtype=torch.bfloat16).pin_memory()
    u_dev = torch.empty_like(u)
    mode = "copies overlapped with the kernels (copy stream, double-buffered input)"
    try:
        u_devs = [torch.empty_like(u), torch.empty_like(u)]
        u_host2 = torch.roll(u, shifts=1, dims=0).cpu().pin_memory()
        outs = [torch.empty_like(out_host).pin_memory() for _ in range(2)]
        refs = [torch.empty_like(out_host).pin_memory() for _ in range(2)]
        b.copy_(b0)
        layer.forward_host_pipelined([u_host, u_host2], e, b, outs, u_devs, update_bias=False)
        torch.cuda.synchronize(dev)
        for src, ref in zip([u_host, u_host2], refs):
            layer.forward_host(src, e, b, ref, u_dev, update_bias=False)
            torch.cuda.synchronize(dev)
        if not all(torch.equal(o, r) for o, r in zip(outs, refs)):
            raise RuntimeError("pipelined end-to-end output differs from the plain path")
        b.copy_(b0)
        layer.forward_host_pipelined([u_host] * 2, e, b, [out_host] * 2, u_devs)
        torch.cuda.synchronize(dev)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        layer.forward_host_pipelined([u_host] * steps, e, b, [out_host] * steps, u_devs)
        e1.record(stream)
        torch.cuda.synchronize(dev)
    except Exception as exc:   # the plain, serialised form
        mode = f"serialised copies (pipelined form unavailable: {exc})"
        b.copy_(b0)
        for _ in range(2):
            layer.forward_host(u_host, e, b, out_host, u_dev)
        torch.cuda.synchronize(dev)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(steps):
            layer.forward_host(u_host, e, b, out_host, u_dev)
        e1.record(stream)
        torch.cuda.synchronize(dev)
    ms = max_over_ranks(e0.elapsed_time(e1) / steps, dev)
    return {"value": whole_job_tokens_per_s(cfg.T, world, ms), "unit": "tokens/s",
            "h2d_bytes_per_step": cfg.T * cfg.d * 2, "d2h_bytes_per_step": cfg.T * cfg.d * 2,
            "steps": steps, "mode": mode}


def backward_run(layer, u, e, b, b0, cfg, dev, peaks, steps=3):
    """The expert FFNs' FP8 backward on the same layer after one forward, with
    a seeded BF16 gradient of the expert outputs: dgrad (G and U recomputed,
    dH, SwiGLU backward, dX; 4 grouped GEMMs) and wgrad (three weight
    gradients per expert, one K-grouped launch per weight) timed apart with
    CUDA events, `steps` each."""
    import torch

    from fine_grained_fp8_sigmoid_b200 import binding as B
    from fine_grained_fp8_sigmoid_b200.backward import ExpertFFNBackward
    b.copy_(b0)
    layer.forward(u, e, b, update_bias=False)
    R = cfg.T * cfg.K_r + cfg.T
    g = torch.Generator(device=dev)
    g.manual_seed(cfg.seed + 1000)
    dy = torch.randn(R, cfg.d, generator=g, device=dev).to(torch.bfloat16)
    bw = ExpertFFNBackward(layer)
    r = bw.backward(dy)                      # warm-up, both halves
    idx = torch.cat([layer.sorted_token, torch.arange(cfg.T, dtype=torch.int32, device=dev)])
    xq = torch.empty(R, cfg.d, dtype=torch.uint8, device=dev)
    xs = torch.empty(R, cfg.d // 128, dtype=torch.float32, device=dev)
    B.moe_gather_rows(layer.xq, idx, xq)
    B.moe_gather_rows(layer.xs, idx, xs)
    torch.cuda.synchronize(dev)
    stream = torch.cuda.current_stream(dev)
    e0, e1, e2 = (torch.cuda.Event(enable_timing=True) for _ in range(3))
    e0.record(stream)
    for _ in range(steps):
        r = bw.backward(dy, wgrad=False)
    e1.record(stream)
    for _ in range(steps):
        bw._wgrad(dy, r["dgu"], xq, xs)
    e2.record(stream)
    torch.cuda.synchronize(dev)
    if B.moe_get_error() != 0:
        raise RuntimeError("device error word set in the backward")
    dg_ms, wg_ms = e0.elapsed_time(e1) / steps, e1.elapsed_time(e2) / steps
    pairs = R                                # (token, expert) rows incl. the shared expert's
    fl_dg = 2.0 * pairs * cfg.d * cfg.I * 5  # G, U recomputed, dH, and dX (K = 2I: twice)
    fl_wg = 2.0 * pairs * cfg.d * cfg.I * 3
    fp8 = 2.0 * peaks["bf16"]
    grad_bytes = 4.0 * (cfg.N_r + 1) * 3 * cfg.d * cfg.I
    del bw, r, dy, xq, xs
    torch.cuda.empty_cache()
    return {"what": "expert FFN FP8 backward after one forward, BF16 dY of all routed and shared rows",
            "steps": steps,
            "dgrad": {"ms": dg_ms, "tflops": fl_dg / (dg_ms / 1e3) / 1e12,
                      "frac_of_fp8_burst": fl_dg / (dg_ms / 1e3) / 1e12 / fp8, "gemms": 4},
            "wgrad": {"ms": wg_ms, "tflops": fl_wg / (wg_ms / 1e3) / 1e12,
                      "frac_of_fp8_burst": fl_wg / (wg_ms / 1e3) / 1e12 / fp8,
                      # bound by writing the FP32 gradients of every expert
                      "gradient_bytes": grad_bytes, "gbs": grad_bytes / (wg_ms / 1e3) / 1e9,
                      "frac_of_hbm": grad_bytes / (wg_ms / 1e3) / 1e9 / peaks["hbm_gbs"],
                      "gemms": 3, "note": "one K-grouped GEMM launch per weight, every expert over its own tokens; "
                                          "plus five transposed quantisations"}}


def sub_workload(name, args, dev, world, local_rank, peaks):
    """One more workload of the same layer shape, measured in the same run:
    decode (the HBM-bound weight stream) or skew (with its balancing run)."""
    import torch

    import workloads
    cfg = workloads.CONFIGS[name]
    layer, u, e, b0 = build_layer(cfg, dev)
    b = b0.clone()
    ms_step, gemm_ms, clocks = time_layer(layer, u, e, b, args.steps, args.warmup, dev, world,
                                          local_rank)
    touched = int((layer.counts > 0).sum().item())
    roof = roofline(cfg, gemm_ms / 1e3, touched, peaks)
    res = {"workload": workload_desc(cfg), "T": cfg.T, "steps": args.steps,
           "value": whole_job_tokens_per_s(cfg.T, world, ms_step), "unit": "tokens/s",
           "ms_per_step": ms_step, "tflops": layer_flops(cfg) / (ms_step / 1e3) / 1e12,
           "roofline": roof, "clocks": clocks}
    if name == "decode":
        res["gemm_weight_stream"] = {"gb_per_call": roof["algorithmic_bytes"] / 1e9,
                                     "gbs": roof["gemm_gbs"],
                                     "frac_of_measured_hbm": roof["gemm_gbs"] / peaks["hbm_gbs"],
                                     "frac_of_8tbs": roof["gemm_gbs"] / NOMINAL_HBM_GBS}
    if name == "skew":
        res["balance"] = balance_run(layer, u, e, b, b0)
    del layer, u, e, b, b0
    torch.cuda.empty_cache()
    return res


def workload_config(args):
    """The named workload, with the profiling overrides of --experts/--tokens
    (a smaller layer whose kernels see the same shapes per token)."""
    import dataclasses

    import workloads
    cfg = workloads.CONFIGS[args.workload]
    if args.experts is not None:
        cfg = dataclasses.replace(cfg, name=f"{cfg.name}_e{args.experts}", N_r=args.experts)
    if args.tokens is not None:
        cfg = dataclasses.replace(cfg, name=f"{cfg.name}_t{args.tokens}", T=args.tokens)
    return cfg


def run_ours(args, rank, world, local_rank):
    import torch

    import workloads
    from fine_grained_fp8_sigmoid_b200 import binding as B

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    cfg = workload_config(args)
    peaks = _peaks()

    layer, u, e, b0 = build_layer(cfg, dev)
    b = b0.clone()
    torch.cuda.synchronize(dev)
    gemm_launches = B.moe_grouped_gemm_fp8_launches(cfg.d, cfg.I)
    launches_per_step = layer.launches_per_step()
    K = args.steps
    ms_step, gemm_ms, clocks = time_layer(layer, u, e, b, K, args.warmup, dev, world, local_rank)
    tokens_per_s = whole_job_tokens_per_s(cfg.T, world, ms_step)
    touched = int((layer.counts > 0).sum().item())
    roof = roofline(cfg, gemm_ms / 1e3, touched, peaks)
    layer_tf = layer_flops(cfg) / (ms_step / 1e3) / 1e12
    balance = balance_run(layer, u, e, b, b0) if cfg.name == "skew" else None
    e2e = e2e_run(layer, u, e, b, b0, max(3, K // 2), dev, world, cfg)
    backward = None
    if cfg == workloads.CONFIGS[CONFIG_NAME] and not args.no_sub_workloads:
        backward = backward_run(layer, u, e, b, b0, cfg, dev, peaks)
    del layer, u, e, b, b0
    torch.cuda.empty_cache()

    # the decode and skew workloads of the same layer shape, as sub-results
    extra = {}
    if cfg == workloads.CONFIGS[CONFIG_NAME] and not args.no_sub_workloads:
        for name in ("decode", "skew"):
            extra[name] = sub_workload(name, args, dev, world, local_rank, peaks)

    result = None
    if rank == 0:
        cpu = None
        if world == 1 and not args.no_cpu_baseline:
            tps, dt, desc = time_oracle(cfg, n_tokens=1, steps=3, device=dev)
            cpu = {"value": tps, "unit": "tokens/s", "cores": os.cpu_count(),
                   "blas_threads": _blas_threads(), "kind": "oracle", "sample": desc,
                   "seconds_per_step": dt}
        result = {
            "metric": METRIC,
            "value": tokens_per_s,
            "unit": "tokens/s",
            "n_gpus": world,
            "steps": K,
            "warmup": args.warmup,
            "ms_per_step": ms_step,
            "higher_is_better": True,
            "scaling": "weak",
            "vs_baseline": None,
            "dtype": "e4m3 (fp32 accumulate)",
            "data": "synthetic",
            "config": {"workload": workload_desc(cfg), "T": cfg.T, "d": cfg.d, "N_r": cfg.N_r,
                       "K_r": cfg.K_r, "I": cfg.I, "N_s": 1, "seed": cfg.seed,
                       "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
                       "l2": f"inputs larger than L2: {weight_bytes(cfg) / 1e9:.2f} GB of expert "
                             "weights stream every step"},
            "tflops": layer_tf,
            "pct_fp8_peak": layer_tf / (2.0 * peaks["bf16"]),
            "roofline": dict(roof, kernel=f"moe_grouped_gemm_fp8 ({gemm_launches} launches)",
                             traffic=gemm_traffic(cfg)),
            "cpu_baseline": cpu,
            "e2e": e2e,
            # router, quant, permute (count, scan, scatter, and the row gather
            # unless fused into the GEMM), the GEMM's launches, combine, bias update
            "gpu_launches": launches_per_step * K,
            "balance": balance,
            "clocks": clocks,
        }
        if backward is not None:
            result["backward"] = backward
        result.update(extra)
    return result


def run_reference(args, rank, world):
    """The CPU oracle as the reference arm: rank 0 only."""
    if rank != 0:
        return None
    import workloads
    cfg = workloads.CONFIGS[CONFIG_NAME]
    n_tokens = 1
    dev = "cpu"
    # warm-up steps are part of the same timing helper's preparation
    from oracle import moe as O
    import numpy as np
    tokens = np.arange(n_tokens)
    u, e, b, quant = _oracle_sample_setup(cfg, tokens, device=dev)
    t0 = time.perf_counter()
    for _ in range(max(1, args.warmup)):
        O.moe_forward(u, e, b, cfg.K_r, quant.__getitem__)
    one = (time.perf_counter() - t0) / max(1, args.warmup)
    # the oracle is slow: run the requested steps, but no more than ~60 s of them
    steps = max(1, min(args.steps, int(60.0 / max(one, 1e-3))))
    t0 = time.perf_counter()
    for _ in range(steps):
        O.moe_forward(u, e, b, cfg.K_r, quant.__getitem__)
    dt = (time.perf_counter() - t0) / steps
    tps = n_tokens / dt
    desc = (f"oracle forward on token 0 of the {cfg.name} batch per step ({len(quant)} expert "
            f"FFNs incl. shared), weights pre-quantised by the oracle (inputs drawn on the CPU)")
    return {
        "impl": "reference", "metric": METRIC, "value": tps, "unit": "tokens/s",
        "n_gpus": world, "steps": steps, "steps_requested": args.steps, "warmup": args.warmup,
        "ms_per_step": dt * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": {"workload": workload_desc(cfg), "T": cfg.T, "d": cfg.d, "N_r": cfg.N_r,
                   "K_r": cfg.K_r, "I": cfg.I, "N_s": 1, "sample_tokens": n_tokens},
        "cpu_baseline": {"value": tps, "unit": "tokens/s", "cores": os.cpu_count(),
                         "blas_threads": _blas_threads(), "kind": "oracle", "sample": desc},
        "e2e": {"value": tps, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def free_port() -> int:
    import socket
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        return sk.getsockname()[1]


def launch_ranks(nproc: int, script: str, argv) -> int:
    """Runs `script argv` as nproc ranks on this node under torch.distributed.run
    (rendezvous on 127.0.0.1), bounded by a timeout; returns its exit status."""
    cmd = ["timeout", "-k", "60", "1800", sys.executable, "-m", "torch.distributed.run",
           "--nnodes=1", f"--nproc-per-node={nproc}", "--master-addr", "127.0.0.1",
           "--master-port", str(free_port()), script, *argv]
    return subprocess.call(cmd)


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-sub-workloads", action="store_true",
                    help="measure only the main workload (not decode and skew beside prefill)")
    ap.add_argument("--workload", default=CONFIG_NAME,
                    help="prefill (the benchmark) or a smaller layer for profiling: mid, decode, tiny")
    ap.add_argument("--experts", type=int, default=None,
                    help="profiling only: the workload with this many routed experts")
    ap.add_argument("--tokens", type=int, default=None,
                    help="profiling only: the workload with this many tokens")
    argv = sys.argv[1:] if argv is None else argv
    args = ap.parse_args(argv)
    if args.warmup < 3 and args.impl == "ours":
        args.warmup = 3
    if "WORLD_SIZE" not in os.environ and args.gpus > 1:
        # one process per GPU: re-run this script as args.gpus ranks
        sys.exit(launch_ranks(args.gpus, os.path.abspath(sys.argv[0]), argv))
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE={world}")

    if args.impl == "reference":
        res = run_reference(args, rank, world)
        if res is not None:
            print(json.dumps(res), flush=True)
        return

    if world > 1:
        import datetime

        import torch
        import torch.distributed as dist
        if torch.cuda.is_available():
            torch.cuda.set_device(local_rank)
            dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                    device_id=torch.device("cuda", local_rank))
        else:   # the rank plumbing on CPU (tests)
            dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=300))
    try:
        res = run_ours(args, rank, world, local_rank)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
    if res is not None:
        print(json.dumps(res), flush=True)


if __name__ == "__main__":
    main()
