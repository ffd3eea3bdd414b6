"""Kernel-by-kernel parity of the CUDA path (through the C ABI) with the CPU
oracle, on seeded inputs that span several tiles and ragged tails.

Exactness rules: FP8 codes and scales of the quantisers, top-K from given
scores, the permutation, and the bias update are bit-exact; floating-point
outputs meet |gpu - ref| <= 8e-3 |ref| + 1e-3 rms(ref).
"""
import numpy as np
import pytest
import torch

import workloads
from oracle import moe as O
from oracle.e4m3 import round_fp32

pytestmark = pytest.mark.gpu

from tests.parity import (accumulation_bound, assert_bf16_rounding, assert_close, down_bound,  # noqa: F401
                          f64, near_tie_rows)


# ---------------------------------------------------------------- quantisers

def _activation_rows(rows, cols, seed):
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(rows, cols, generator=g)
    x *= torch.exp2(torch.randint(-30, 30, (rows, 1), generator=g).float())
    if rows >= 4 and cols >= 256:
        x[0, :128] = 0.0                         # all-zero tile
        x[1, 128:256] = -0.0                     # negative zeros
        x[2, :128] = torch.randn(128, generator=g) * 2.0 ** -130   # bf16 subnormals
        x[3, :128] = 448.0 * torch.sign(torch.randn(128, generator=g))
    return x.to(torch.bfloat16)


@pytest.mark.parametrize("rows,cols", [(1, 128), (37, 256), (300, 2048), (1000, 7168)])
def test_quant_1x128_bit_exact(lib, rows, cols):
    from fine_grained_fp8_sigmoid_b200 import binding as B
    x = _activation_rows(rows, cols, seed=rows)
    xd = x.cuda()
    q = torch.empty(rows, cols, dtype=torch.uint8, device="cuda")
    s = torch.empty(rows, cols // 128, dtype=torch.float32, device="cuda")
    B.moe_quant_1x128(xd, q, s)
    torch.cuda.synchronize()
    rq, rs = O.quant_1x128(x.double().numpy())
    assert np.array_equal(s.cpu().double().numpy(), rs)
    assert np.array_equal(q.cpu().numpy(), rq)


@pytest.mark.parametrize("rows,cols", [(128, 128), (256, 384), (2048, 7168)])
def test_quant_128x128_bit_exact(lib, rows, cols):
    from fine_grained_fp8_sigmoid_b200 import binding as B
    g = torch.Generator().manual_seed(cols)
    w = torch.randn(rows, cols, generator=g) * 0.02
    w[:128, :128] = 0.0
    if cols >= 256:
        w[:128, 128:256] *= 1e5
    wd = w.cuda()
    q = torch.empty(rows, cols, dtype=torch.uint8, device="cuda")
    s = torch.empty(rows // 128, cols // 128, dtype=torch.float32, device="cuda")
    B.moe_quant_128x128(wd, q, s)
    torch.cuda.synchronize()
    rq, rs = O.quant_128x128(w.double().numpy())
    assert np.array_equal(s.cpu().double().numpy(), rs)
    assert np.array_equal(q.cpu().numpy(), rq)


# ---------------------------------------------------------------- router

@pytest.mark.parametrize("T,N,K,ties", [(1000, 8, 2, False), (1000, 64, 6, False),
                                        (777, 256, 8, False), (500, 256, 8, True),
                                        (300, 64, 16, False), (64, 16, 16, True)])
def test_topk_from_scores_bit_exact(lib, T, N, K, ties):
    from fine_grained_fp8_sigmoid_b200 import binding as B
    s = workloads.scores(T, N, seed=T + N, ties=ties)
    b = torch.zeros(N) if ties else (torch.rand(N, generator=torch.Generator().manual_seed(N)) - 0.5) * 0.02
    idx = torch.empty(T, K, dtype=torch.int32, device="cuda")
    gates = torch.empty(T, K, dtype=torch.float32, device="cuda")
    B.moe_route(None, None, b.cuda(), K, idx, gates, scores_in=s.cuda())
    torch.cuda.synchronize()
    ref = O.select_topk(s.double().numpy(), b.double().numpy(), K)
    assert np.array_equal(idx.cpu().numpy(), ref)
    rg = O.gates_from(s.double().numpy(), ref)
    assert np.allclose(gates.cpu().double().numpy(), rg, rtol=2e-6, atol=0)


def _check_routing(gpu_idx, s64, b, K, margin=1e-5):
    """Selections equal, except tokens whose K-th and (K+1)-th oracle keys are
    closer than `margin`. Returns the tokens that differ."""
    key = s64 + b[None, :]
    ref = np.argsort(-round_fp32(key), axis=1, kind="stable")
    diff = []
    for t in range(gpu_idx.shape[0]):
        if set(gpu_idx[t]) != set(ref[t, :K]):
            srt = np.sort(key[t])[::-1]
            m = srt[K - 1] - srt[K] if K < key.shape[1] else np.inf
            assert m < margin, f"token {t}: selection differs with margin {m}"
            diff.append(t)
    return diff


@pytest.mark.parametrize("name,T,K", [("tiny", None, None), ("mid", None, None), ("mid", 1000, None),
                                      ("mid", 5000, None), ("prefill", 1500, None), ("decode", None, None),
                                      # top-K lists of 16 (K_r > 8): one tile (cluster of 8), and 40 tiles
                                      ("mid", 128, 12), ("mid", 5000, 16)])
def test_router_tensor_cores(lib, name, T, K):
    import dataclasses
    from fine_grained_fp8_sigmoid_b200 import binding as B
    cfg = workloads.CONFIGS[name]
    if T is not None:
        cfg = cfg.with_tokens(T)
    if K is not None:
        cfg = dataclasses.replace(cfg, K_r=K)
    u, e, b = workloads.activations(cfg), workloads.centroids(cfg), workloads.bias(cfg)
    idx = torch.empty(cfg.T, cfg.K_r, dtype=torch.int32, device="cuda")
    gates = torch.empty(cfg.T, cfg.K_r, dtype=torch.float32, device="cuda")
    sc = torch.empty(cfg.T, cfg.N_r, dtype=torch.float32, device="cuda")
    B.moe_route(u.cuda(), e.cuda(), b.cuda(), cfg.K_r, idx, gates, scores_out=sc)
    torch.cuda.synchronize()
    s64 = O.router_scores(u.double().numpy(), e.double().numpy())
    assert np.abs(sc.cpu().double().numpy() - s64).max() < 1e-5
    gi = idx.cpu().numpy()
    diff = _check_routing(gi, s64, b.double().numpy(), cfg.K_r)
    assert len(diff) <= max(2, cfg.T // 200)
    rg = O.gates_from(s64, gi.astype(np.int64))
    assert np.allclose(gates.cpu().double().numpy(), rg, rtol=1e-4, atol=1e-6)


@pytest.mark.parametrize("name,T,K", [("tiny", None, None), ("mid", 1000, None), ("prefill", 1500, None),
                                      ("prefill", 1, None), ("decode", None, None), ("mid", 5000, 16)])
def test_route_quant_fused(lib, name, T, K):
    """moe_route_quant: the router's own outputs equal moe_route's bit for
    bit, and its xq/xs equal the oracle's 1x128 quantisation of u bit for bit
    (incl. a ragged last token tile, one token, and the cluster-split decode
    launch where each rank quantises its share of the channels)."""
    import dataclasses
    from fine_grained_fp8_sigmoid_b200 import binding as B
    cfg = workloads.CONFIGS[name]
    if T is not None:
        cfg = cfg.with_tokens(T)
    if K is not None:
        cfg = dataclasses.replace(cfg, K_r=K)
    u, e, b = workloads.activations(cfg), workloads.centroids(cfg), workloads.bias(cfg)
    if cfg.T >= 4 and cfg.d >= 256:   # special tiles: zero, -0, bf16 subnormal, +-448
        u = u.clone()
        u[0, :128] = 0.0
        u[1, 128:256] = -0.0
        u[2, :128] = (torch.randn(128, generator=torch.Generator().manual_seed(5)) * 2.0 ** -130).to(u.dtype)
        u[3, :128] = 448.0
    ud, ed, bd = u.cuda(), e.cuda(), b.cuda()
    out = lambda: (torch.empty(cfg.T, cfg.K_r, dtype=torch.int32, device="cuda"),
                   torch.empty(cfg.T, cfg.K_r, dtype=torch.float32, device="cuda"))
    idx0, g0 = out()
    idx1, g1 = out()
    xq = torch.full((cfg.T, cfg.d), 0x55, dtype=torch.uint8, device="cuda")
    xs = torch.full((cfg.T, cfg.d // 128), -1.0, device="cuda")
    B.moe_route(ud, ed, bd, cfg.K_r, idx0, g0)
    B.moe_route_quant(ud, ed, bd, cfg.K_r, idx1, g1, xq, xs)
    torch.cuda.synchronize()
    assert B.moe_get_error() == 0
    assert torch.equal(idx0, idx1) and torch.equal(g0, g1)
    rq, rs = O.quant_1x128(u.double().numpy())
    assert np.array_equal(xq.cpu().numpy(), rq)
    assert np.array_equal(xs.cpu().double().numpy(), rs)


def _tied_centroids(cfg, mode):
    """Centroids with exactly repeated rows, so that logits (and with equal
    bias, keys) tie bit for bit. mode "pairs": a few expert pairs share a
    row, chosen to fall in different threads, warps and column halves of
    the fused router; mode "groups": only 4 distinct rows, each repeated
    N_r/4 times, so every selection breaks ties."""
    e = workloads.centroids(cfg).clone()
    b = workloads.bias(cfg).clone()
    N = cfg.N_r
    if mode == "pairs":
        pairs = [(0, N - 1), (2, 3), (5, N // 2), (7, N // 2 + 7), (N // 4, N // 4 + 4), (1, N - 2)]
        for lo, hi in pairs:
            e[hi] = e[lo]
            b[hi] = b[lo]
        return e, b, pairs
    e = e[torch.arange(N) % 4].clone()
    b = torch.zeros(N) if cfg.bias == "zero" else b[torch.arange(N) % 4].clone()
    return e, b, [(i, j) for i in range(4) for j in range(i + 4, N, 4)]


@pytest.mark.parametrize("name,T,K,mode", [("mid", 4096, None, "pairs"), ("mid", 333, 12, "groups"),
                                           ("prefill", 8192, None, "pairs"), ("prefill", 1500, None, "groups"),
                                           ("decode", 128, None, "pairs"), ("decode", 128, None, "groups")])
def test_router_ties_and_order_through_the_fused_path(lib, name, T, K, mode):
    """The fused router (tensor-core logits, cluster split, insertion lists
    and butterfly merge) returns exactly the top-K of its own FP32 keys
    fl32(s + b): ties go to the lower index and the list is ordered by key
    descending, then index ascending. Checked bit for bit against the
    oracle's top-K applied to the kernel's own affinities (scores_out), on
    centroids with repeated rows so that equal keys really occur."""
    import dataclasses
    from fine_grained_fp8_sigmoid_b200 import binding as B
    cfg = workloads.CONFIGS[name].with_tokens(T)
    if K is not None:
        cfg = dataclasses.replace(cfg, K_r=K)
    u = workloads.activations(cfg)
    e, b, tied = _tied_centroids(cfg, mode)
    idx = torch.empty(cfg.T, cfg.K_r, dtype=torch.int32, device="cuda")
    gates = torch.empty(cfg.T, cfg.K_r, dtype=torch.float32, device="cuda")
    sc = torch.empty(cfg.T, cfg.N_r, dtype=torch.float32, device="cuda")
    B.moe_route(u.cuda(), e.cuda(), b.cuda(), cfg.K_r, idx, gates, scores_out=sc)
    torch.cuda.synchronize()
    s_gpu = sc.cpu().double().numpy()
    gi = idx.cpu().numpy().astype(np.int64)
    bn = b.double().numpy()
    # repeated centroid rows give bit-identical affinities
    for lo, hi in tied:
        assert np.array_equal(s_gpu[:, lo], s_gpu[:, hi]), (lo, hi)
    # the selection and its order are the top-K of the kernel's own keys
    ref = O.select_topk(s_gpu, bn, cfg.K_r)
    bad = np.nonzero((gi != ref).any(axis=1))[0]
    assert bad.size == 0, f"{bad.size} tokens differ, first {bad[:5]}: gpu {gi[bad[0]]} ref {ref[bad[0]]}"
    # ties decided the selection somewhere: a tied partner left out at the
    # K-th place, or two tied experts both selected
    key = round_fp32(s_gpu + bn[None, :])
    kth = np.take_along_axis(key, ref[:, -1:], axis=1)[:, 0]
    outside = np.ones_like(key, dtype=bool)
    np.put_along_axis(outside, ref, False, axis=1)
    assert ((key == kth[:, None]) & outside).any(), "no tie at the selection boundary"
    # gates are the selected affinities normalised in FP32
    assert np.allclose(gates.cpu().double().numpy(), O.gates_from(s_gpu, ref), rtol=2e-6, atol=0)
    # and the oracle's own routing agrees up to the 1e-5 margin rule
    s64 = O.router_scores(u.double().numpy(), e.double().numpy())
    assert np.abs(s_gpu - s64).max() < 1e-5
    _check_routing(gi, s64, bn, cfg.K_r)


# ---------------------------------------------------------------- permutation

@pytest.mark.parametrize("T,N,K,pattern", [(1, 8, 2, "uniform"), (255, 8, 2, "uniform"),
                                           (257, 256, 8, "uniform"), (5000, 64, 6, "uniform"),
                                           (3000, 256, 8, "one_hot_expert"), (600, 1024, 16, "uniform"),
                                           (1000, 16, 16, "first_k"), (100, 4, 1, "uniform")])
def test_permute_bit_exact(lib, T, N, K, pattern):
    from fine_grained_fp8_sigmoid_b200 import binding as B
    idx = workloads.topk_indices(T, N, K, seed=T * 7 + N, pattern=pattern)
    d = 256
    g = torch.Generator().manual_seed(T)
    xq = torch.randint(0, 256, (T, d), generator=g, dtype=torch.uint8)
    xs = torch.rand(T, d // 128, generator=g)
    dev = dict(device="cuda")
    counts = torch.empty(N, dtype=torch.int32, **dev)
    offsets = torch.empty(N + 1, dtype=torch.int32, **dev)
    st = torch.empty(T * K, dtype=torch.int32, **dev)
    inv = torch.empty(T, K, dtype=torch.int32, **dev)
    xqp = torch.empty(T * K, d, dtype=torch.uint8, **dev)
    xsp = torch.empty(T * K, d // 128, dtype=torch.float32, **dev)
    ws = torch.empty(max(B.moe_permute_workspace(T, N), 16), dtype=torch.uint8, **dev)
    B.moe_permute(idx.cuda(), N, counts, offsets, st, inv, ws, xq.cuda(), xs.cuda(), xqp, xsp)
    torch.cuda.synchronize()
    rc, ro, rst, rinv = O.permute(idx.numpy(), N)
    assert np.array_equal(counts.cpu().numpy(), rc)
    assert np.array_equal(offsets.cpu().numpy(), ro)
    assert np.array_equal(st.cpu().numpy(), rst)
    assert np.array_equal(inv.cpu().numpy(), rinv)
    assert np.array_equal(xqp.cpu().numpy(), xq.numpy()[rst])
    assert np.array_equal(xsp.cpu().numpy(), xs.numpy()[rst])


# ---------------------------------------------------------------- combine, bias

@pytest.mark.parametrize("T,K,d", [(1, 1, 8), (333, 2, 256), (1000, 8, 7168)])
@pytest.mark.parametrize("ydt", [torch.bfloat16, torch.float32])
def test_combine(lib, T, K, d, ydt):
    """moe_combine on the layer's bf16 expert rows, and moe_combine_fp32 on
    FP32 rows (the backward's). The kernel's FP32 sum of K + 2 terms is within
    (K + 2) roundings of 2^-24 |term| of the float64 sum, so h' is at most one
    bf16 step plus that from the oracle's value."""
    from fine_grained_fp8_sigmoid_b200 import binding as B
    g = torch.Generator().manual_seed(T + d)
    u = torch.randn(T, d, generator=g).to(torch.bfloat16)
    ysh = (torch.randn(T, d, generator=g) * 3.0).to(ydt)
    yp = (torch.randn(T * K, d, generator=g) * 3.0).to(ydt)
    inv = torch.randperm(T * K, generator=g).reshape(T, K).to(torch.int32)
    gt = torch.rand(T, K, generator=g)
    gt = gt / gt.sum(dim=1, keepdim=True)
    out = torch.empty(T, d, dtype=torch.bfloat16, device="cuda")
    B.moe_combine(u.cuda(), yp.cuda(), ysh.cuda(), inv.cuda(), gt.cuda(), out)
    torch.cuda.synchronize()
    ref = O.combine(u.double().numpy(), yp.double().numpy(), ysh.double().numpy(),
                    inv.numpy(), gt.double().numpy())
    assert_close(f64(out), ref, "combine")
    g64, inv_ = gt.double().numpy(), inv.numpy()
    yp64 = yp.double().numpy()
    terms = np.abs(u.double().numpy()) + np.abs(ysh.double().numpy())
    for k in range(K):
        terms += np.abs(g64[:, k:k + 1] * yp64[inv_[:, k]])
    step = np.ldexp(1.0, np.frexp(np.abs(ref))[1] - 8)
    off = np.abs(f64(out) - ref)
    assert np.all(off <= step + 2 * (K + 2) * 2.0 ** -24 * terms), \
        "combine: more than one bf16 step plus the FP32 sum's rounding from the float64 sum"


@pytest.mark.parametrize("N,T,K", [(8, 64, 2), (256, 8192, 8), (64, 4095, 6), (256, 0, 8)])
def test_bias_update_bit_exact(lib, N, T, K):
    from fine_grained_fp8_sigmoid_b200 import binding as B
    g = torch.Generator().manual_seed(N + T)
    b = (torch.rand(N, generator=g) - 0.5) * 0.02
    if T:
        idx = workloads.topk_indices(T, N, K, seed=N)
        counts = torch.bincount(idx.reshape(-1).long(), minlength=N).to(torch.int32)
        counts[0] = (T * K) // N if (T * K) % N == 0 else counts[0]
    else:
        counts = torch.zeros(N, dtype=torch.int32)
    bd = b.cuda()
    mom = torch.zeros(1, device="cuda")
    B.moe_bias_update(bd, counts.cuda(), T, K, 0.001, mom)
    torch.cuda.synchronize()
    rb, ratio = O.bias_update(b.double().numpy(), counts.numpy(), T, K)
    assert np.array_equal(bd.cpu().double().numpy(), rb)
    assert abs(mom.item() - ratio) <= 1e-6 * max(ratio, 1.0)


# ---------------------------------------------------------------- grouped GEMM

def _gemm_case(d, I, counts, T, seed):
    """Oracle-quantised inputs for the grouped GEMM alone."""
    rng = np.random.default_rng(seed)
    N_r = len(counts)
    P = int(sum(counts))
    xp = round_fp32(rng.standard_normal((P, d)) * np.exp2(rng.integers(-3, 3, (P, 1))))
    xsh = round_fp32(rng.standard_normal((T, d)))
    xq_p, xs_p = O.quant_1x128(xp)
    xq, xs = O.quant_1x128(xsh)
    experts = []
    for _ in range(N_r + 1):
        w = [round_fp32(rng.standard_normal(sh) * 0.02) for sh in [(I, d), (I, d), (d, I)]]
        experts.append(O.quantise_expert(*w))
    offsets = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    return xq_p, xs_p, xq, xs, experts, offsets


@pytest.mark.parametrize("d,I,counts,T", [
    (256, 128, [0, 1, 130, 257], 100),
    (512, 256, [3, 0, 128, 64, 200], 129),
    (2048, 1024, [384, 200], 256),
    (7168, 2048, [5, 300], 130),
    # groups of at most 64 rows run as narrow tiles: every token-width class
    # (N = 16, 32, 48, 64) and its edges, next to wide groups; T = 40 makes
    # the shared expert narrow too
    (512, 256, [16, 17, 33, 48, 49, 63, 64, 65, 0, 1], 40),
])
def test_grouped_gemm_fp8(lib, d, I, counts, T):
    from fine_grained_fp8_sigmoid_b200 import binding as B
    xq_p, xs_p, xq, xs, experts, offsets = _gemm_case(d, I, counts, T, seed=d + I)
    N_r = len(counts)
    P = int(offsets[-1])
    K_r = P // T if P % T == 0 else None
    # the C ABI sizes y_perm as T*K_r rows; pad the routed rows to that
    K_r = -(-P // T)
    Ppad = T * K_r
    dev = dict(device="cuda")
    cu = lambda a, dt: torch.from_numpy(np.ascontiguousarray(a)).to(dt).cuda()
    xq_pd = torch.zeros(Ppad, d, dtype=torch.uint8, **dev)
    xs_pd = torch.ones(Ppad, d // 128, dtype=torch.float32, **dev)
    xq_pd[:P] = cu(xq_p, torch.uint8)
    xs_pd[:P] = cu(xs_p, torch.float32)
    stack = lambda key, dt: cu(np.stack([e[key] for e in experts]), dt)
    wg, wu, wd = stack("gate_q", torch.uint8), stack("up_q", torch.uint8), stack("down_q", torch.uint8)
    sg, su, sd = stack("gate_s", torch.float32), stack("up_s", torch.float32), stack("down_s", torch.float32)
    off = torch.from_numpy(offsets).cuda()
    y_perm = torch.empty(Ppad, d, dtype=torch.bfloat16, **dev)
    y_sh = torch.empty(T, d, dtype=torch.bfloat16, **dev)
    ws = torch.empty(B.moe_grouped_gemm_fp8_workspace(T, K_r, d, I), dtype=torch.uint8, **dev)
    B.moe_grouped_gemm_fp8(xq_pd, xs_pd, off, cu(xq, torch.uint8), cu(xs, torch.float32),
                           wg, wu, wd, sg, su, sd, y_perm, y_sh, ws)
    torch.cuda.synchronize()
    assert B.moe_get_error() == 0
    yp = f64(y_perm)
    rows = Ppad + T
    hq_g = ws[:rows * I].view(rows, I).cpu().numpy()
    off = (rows * I + 255) // 256 * 256
    hs_g = ws[off:off + rows * (I // 128) * 4].view(torch.float32).view(rows, I // 128).cpu().double().numpy()
    groups = [(i, offsets[i], offsets[i + 1], xq_p, xs_p) for i in range(N_r)] + [(N_r, 0, T, xq, xs)]
    for i, a, b_, xq_i, xs_i in groups:
        if b_ <= a:
            continue
        p = O.expert_ffn_parts(xq_i[a:b_], xs_i[a:b_], experts[i])
        g0 = a if i < N_r else Ppad                 # the group's first row in H
        da = accumulation_bound(xq_i[a:b_], xs_i[a:b_], experts[i], p["G"], p["U"])
        flip, _ = near_tie_rows(hq_g[g0:g0 + b_ - a], hs_g[g0:g0 + b_ - a], p["a32"], da, p["hq"], p["hs"],
                                f"expert {i} intermediate")
        ref = p["y"]
        if flip.size:
            ref = ref.copy()
            ref[flip] = O.expert_down(hq_g[g0 + flip], hs_g[g0 + flip], experts[i])
        got = yp[a:b_] if i < N_r else f64(y_sh)
        assert_close(got, ref, f"expert {i}")
        # bf16 outputs: the rounding of the kernel's FP32 sums (near-ties either way)
        assert_bf16_rounding(got, ref, down_bound(hq_g[g0:g0 + b_ - a], hs_g[g0:g0 + b_ - a], experts[i]),
                             f"expert {i} bf16 rounding")


@pytest.mark.parametrize("d,I,T,K,N_r", [(512, 256, 300, 3, 7), (2048, 1024, 700, 6, 16),
                                         (7168, 2048, 200, 8, 12),
                                         # average group <= 64 rows: narrow tiles
                                         (512, 256, 90, 4, 16)])
def test_grouped_gemm_gather_matches_materialised(lib, d, I, T, K, N_r):
    """moe_grouped_gemm_fp8_gather (routed rows gathered from xq by the GEMM's
    loads) gives bit for bit what moe_grouped_gemm_fp8 gives on the
    materialised xq_perm, intermediate included, and matches the oracle."""
    from fine_grained_fp8_sigmoid_b200 import binding as B
    rng = np.random.default_rng(d + T)
    x = round_fp32(rng.standard_normal((T, d)) * np.exp2(rng.integers(-3, 3, (T, 1))))
    xq, xs = O.quant_1x128(x)
    idx = workloads.topk_indices(T, N_r, K, seed=T + K).numpy()
    counts, offsets, sorted_token, _ = O.permute(idx, N_r)
    experts = []
    for _ in range(N_r + 1):
        w = [round_fp32(rng.standard_normal(sh) * 0.02) for sh in [(I, d), (I, d), (d, I)]]
        experts.append(O.quantise_expert(*w))
    dev = dict(device="cuda")
    cu = lambda a, dt: torch.from_numpy(np.ascontiguousarray(a)).to(dt).cuda()
    P = T * K
    stack = lambda key, dt: cu(np.stack([e[key] for e in experts]), dt)
    W = [stack(k, torch.uint8) for k in ("gate_q", "up_q", "down_q")] + \
        [stack(k, torch.float32) for k in ("gate_s", "up_s", "down_s")]
    xq_d, xs_d = cu(xq, torch.uint8), cu(xs, torch.float32)
    st_d, off_d = cu(sorted_token, torch.int32), cu(offsets, torch.int32)
    outs = []
    for gathered in (False, True):
        y_perm = torch.full((P, d), float("nan"), dtype=torch.bfloat16, **dev)
        y_sh = torch.full((T, d), float("nan"), dtype=torch.bfloat16, **dev)
        ws = torch.zeros(B.moe_grouped_gemm_fp8_workspace(T, K, d, I), dtype=torch.uint8, **dev)
        if gathered:
            B.moe_grouped_gemm_fp8_gather(st_d, off_d, xq_d, xs_d, *W, y_perm, y_sh, ws)
        else:
            B.moe_grouped_gemm_fp8(xq_d[st_d.long()].contiguous(), xs_d[st_d.long()].contiguous(), off_d,
                                   xq_d, xs_d, *W, y_perm, y_sh, ws)
        torch.cuda.synchronize()
        assert B.moe_get_error() == 0
        rows = P + T
        outs.append((y_perm.cpu(), y_sh.cpu(), ws[:rows * I].cpu()))
    for a_, b_ in zip(*outs):
        assert torch.equal(a_, b_)
    # and the oracle, on every routed group and the shared expert, under the
    # intermediate's near-tie rule (tests/parity.py)
    yp, ysh = outs[1][0].double().numpy(), outs[1][1].double().numpy()
    hq_g = outs[1][2].view(P + T, I).numpy()
    off_s = (((P + T) * I + 255) // 256) * 256
    hs_g = ws[off_s:off_s + (P + T) * (I // 128) * 4].view(torch.float32).view(P + T, I // 128).cpu().double().numpy()
    for i in range(N_r + 1):
        rows_i = sorted_token[offsets[i]:offsets[i + 1]] if i < N_r else np.arange(T)
        if rows_i.size == 0:
            continue
        h0 = offsets[i] if i < N_r else P           # the group's first row in H
        n = rows_i.size
        p = O.expert_ffn_parts(xq[rows_i], xs[rows_i], experts[i])
        da = accumulation_bound(xq[rows_i], xs[rows_i], experts[i], p["G"], p["U"])
        flip, _ = near_tie_rows(hq_g[h0:h0 + n], hs_g[h0:h0 + n], p["a32"], da, p["hq"], p["hs"],
                                f"expert {i} intermediate")
        ref = p["y"]
        if flip.size:
            ref = ref.copy()
            ref[flip] = O.expert_down(hq_g[h0 + flip], hs_g[h0 + flip], experts[i])
        got = yp[offsets[i]:offsets[i + 1]] if i < N_r else ysh
        assert_close(got, ref, f"expert {i}")
        assert_bf16_rounding(got, ref, down_bound(hq_g[h0:h0 + n], hs_g[h0:h0 + n], experts[i]),
                             f"expert {i} bf16 rounding")


# ---------------------------------------------------------------- failure path

def test_wait_timeout_sets_error_word(lib):
    from fine_grained_fp8_sigmoid_b200 import binding as B
    assert B.moe_get_error() == 0
    B.moe_debug_wait_timeout(2000)           # a 2 ms wait on a barrier nothing signals
    assert B.moe_get_error() == 4            # MOE_ERR_TIMEOUT, read and cleared
    assert B.moe_get_error() == 0
    x = torch.zeros(4, 128, dtype=torch.bfloat16, device="cuda")   # the context still works
    q = torch.empty(4, 128, dtype=torch.uint8, device="cuda")
    s = torch.empty(4, 1, dtype=torch.float32, device="cuda")
    B.moe_quant_1x128(x, q, s)
    torch.cuda.synchronize()
    assert s.cpu().eq(1.0).all()
