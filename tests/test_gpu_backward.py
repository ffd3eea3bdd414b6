"""The expert FFN's FP8 backward on the GPU (fine_grained_fp8_sigmoid_b200/
backward.py over the C ABI) against the oracle's expert_ffn_backward.

Bit-exact where the inputs fix the result: the weight transposes, the
transposed 1x128 quantisation of a BF16 gradient, the transposed 128x128
requantisation of the forward's FP8 rows. Floating-point results: the GPU
accumulates in FP32 (per 128-wide K block, promoted) and the oracle in
float64, and the backward quantises values it computes (dG and dU, along I
for dgrad and along the tokens for wgrad), where an element on an E4M3
rounding boundary may take the neighbouring code on either side; each such
code moves its row of dX (or its wgrad product) by one E4M3 step of one term.
The check is therefore on norms: relative L2 error <= 1e-2 for every row of
dX and every expert's weight gradients, <= 2e-3 over all of them (FP32
rounding alone stays below 1e-5; a wrong scale, operand or transpose gives
errors of order one).
"""

import numpy as np
import pytest
import torch

import workloads
from oracle import moe as O
from oracle.e4m3 import round_bf16, round_fp32

pytestmark = pytest.mark.gpu


def _rel(a, b):
    n = np.linalg.norm(b)
    return np.linalg.norm(a - b) / (n if n > 0 else 1.0)


def test_transpose_bit_exact(lib):
    from fine_grained_fp8_sigmoid_b200 import binding as B
    g = torch.Generator().manual_seed(0)
    x8 = torch.randint(0, 256, (3, 70, 45), generator=g, dtype=torch.uint8).cuda()
    x32 = torch.randn(3, 33, 65, generator=g).cuda()
    d8 = torch.zeros(3, 45, 100, dtype=torch.uint8, device="cuda")
    d32 = torch.zeros(3, 65, 40, device="cuda")
    B.moe_transpose(x8, d8, 20)
    B.moe_transpose(x32, d32, 7)
    torch.cuda.synchronize()
    assert torch.equal(d8[:, :, 20:90], x8.transpose(1, 2))
    assert torch.equal(d8[:, :, :20], torch.zeros_like(d8[:, :, :20]))
    assert torch.equal(d32[:, :, 7:40], x32.transpose(1, 2))


def _groups(rows):
    src = np.concatenate([[0], np.cumsum(rows)])
    dst = np.concatenate([[0], np.cumsum((np.asarray(rows) + 127) // 128 * 128)])
    return src, dst


def _pad(x, m):
    return np.concatenate([x, np.zeros((m - x.shape[0],) + x.shape[1:])]) if m > x.shape[0] else x


@pytest.mark.parametrize("rows,cols", [([5, 0, 130, 256, 1], 256), ([300, 77], 512)])
def test_transposed_quantisation_bit_exact(lib, rows, cols):
    from fine_grained_fp8_sigmoid_b200 import binding as B
    src, dst = _groups(rows)
    R, Kt = int(src[-1]), int(dst[-1])
    rng = np.random.default_rng(R + cols)
    x = round_bf16(rng.standard_normal((R, cols)) * np.exp2(rng.integers(-4, 4, (R, 1))))
    xb = torch.from_numpy(x).to(torch.bfloat16).cuda()
    sd = torch.from_numpy(src.astype(np.int32)).cuda()
    dd = torch.from_numpy(dst.astype(np.int32)).cuda()
    q = torch.empty(cols * Kt, dtype=torch.uint8, device="cuda")
    s = torch.empty(cols * Kt // 128, device="cuda")
    B.moe_quant_1x128_t(xb, sd, dd, q, s)
    # the forward's FP8 rows of the same values, requantised in blocks
    xq, xs = O.quant_1x128(x)
    qb = torch.empty(cols * Kt, dtype=torch.uint8, device="cuda")
    sb = torch.empty((cols // 128) * (Kt // 128), device="cuda")
    B.moe_quant_128x128_t(torch.from_numpy(xq).cuda(), torch.from_numpy(xs).float().cuda(), sd, dd, qb, sb)
    torch.cuda.synchronize()
    # layout [cols][Kt]: group g in columns dst[g]..dst[g+1] of every row
    q, s = q.cpu().numpy().reshape(cols, Kt), s.cpu().double().numpy().reshape(cols, Kt // 128)
    qb, sb = qb.cpu().numpy().reshape(cols, Kt), sb.cpu().double().numpy().reshape(cols // 128, Kt // 128)
    for g in range(len(rows)):
        K = int(dst[g + 1] - dst[g])
        if K == 0:
            continue
        o = int(dst[g])
        xg = _pad(x[src[g]:src[g + 1]], K).T
        rq, rs = O.quant_1x128(xg)
        assert np.array_equal(q[:, o:o + K], rq), g
        assert np.array_equal(s[:, o // 128:(o + K) // 128], rs), g
        hg = _pad(O.dequant_1x128(xq, xs)[src[g]:src[g + 1]], K).T
        bq, bs = O.quant_128x128(round_fp32(hg))
        assert np.array_equal(qb[:, o:o + K], bq), g
        assert np.array_equal(sb[:, o // 128:(o + K) // 128], bs), g


def test_swiglu_backward_quant(lib):
    from fine_grained_fp8_sigmoid_b200 import binding as B
    rng = np.random.default_rng(9)
    R, I = 300, 256
    G, U, D = (round_fp32(rng.standard_normal((R, I)) * sc) for sc in (2.0, 1.0, 0.01))
    dev = lambda a: torch.from_numpy(a).float().cuda()
    dgu = torch.empty(R, 2 * I, device="cuda")
    q = torch.empty(R, 2 * I, dtype=torch.uint8, device="cuda")
    qs = torch.empty(R, 2 * I // 128, device="cuda")
    B.moe_swiglu_backward_quant(dev(G), dev(U), dev(D), dgu, q, qs)
    torch.cuda.synchronize()
    ref = np.concatenate([D * U * O.dsilu(G), D * O.silu(G)], axis=1)
    got = dgu.cpu().double().numpy()
    # FP32 arithmetic: a few roundings per value; silu' has a zero near
    # x = -1.28, where the error is absolute (relative to the tile's scale)
    assert np.allclose(got, ref, rtol=2e-6, atol=2e-6 * np.abs(ref).max())
    rq, rs = O.quant_1x128(round_fp32(got))      # the quantisation of the kernel's own FP32 values
    assert np.array_equal(q.cpu().numpy(), rq)
    assert np.array_equal(qs.cpu().double().numpy(), rs)


@pytest.mark.parametrize("d,I,Kt,groups", [(512, 256, 384, [100, 0, 28]), (1024, 512, 256, [])])
def test_grouped_scaled_gemm(lib, d, I, Kt, groups):
    """c = a b_g^T for grouped rows (and for one group only, as wgrad uses it)."""
    from fine_grained_fp8_sigmoid_b200 import binding as B
    rng = np.random.default_rng(d + Kt)
    P = int(sum(groups))
    T = 70
    R = P + T
    a = round_fp32(rng.standard_normal((R, Kt)))
    aq, as_ = O.quant_1x128(a)
    G = len(groups) + 1
    bs = [O.quant_128x128(round_fp32(rng.standard_normal((d, Kt)) * 0.05)) for _ in range(G)]
    off = np.concatenate([[0], np.cumsum(groups)]).astype(np.int32) if groups else np.zeros(1, np.int32)
    cu = lambda x, dt: torch.from_numpy(np.ascontiguousarray(x)).to(dt).cuda()
    c = torch.empty(R, d, device="cuda")
    ws = torch.empty(B.moe_grouped_scaled_gemm_fp8_workspace(), dtype=torch.uint8, device="cuda")
    B.moe_grouped_scaled_gemm_fp8(cu(aq, torch.uint8), cu(as_, torch.float32), cu(off, torch.int32), P,
                                  cu(np.stack([b[0] for b in bs]), torch.uint8),
                                  cu(np.stack([b[1] for b in bs]), torch.float32), c, ws)
    torch.cuda.synchronize()
    assert B.moe_get_error() == 0
    got = c.cpu().double().numpy()
    bounds = list(off) + [R]
    for gi in range(G):
        lo, hi = bounds[gi], bounds[gi + 1]
        if hi > lo:
            ref = O.scaled_gemm(aq[lo:hi], as_[lo:hi], *bs[gi])
            assert np.allclose(got[lo:hi], ref, rtol=1e-5, atol=1e-6 * np.abs(ref).max()), gi


@pytest.mark.parametrize("M,N,ranges", [(256, 512, [(0, 128), (128, 128), (128, 512), (512, 640)]),
                                         (128, 256, [(0, 0), (0, 0)]),
                                         (384, 768, [(0, 1024)])])
def test_kgrouped_gemm(lib, M, N, ranges):
    """c[g] = a[:, K_g] b[:, K_g]^T over each group's own K range (wgrad's
    form), empty ranges giving zero, against the oracle's scaled GEMM."""
    from fine_grained_fp8_sigmoid_b200 import binding as B
    K = max(hi for _, hi in ranges)
    rng = np.random.default_rng(M + N + K)
    Kp = max(K, 128)
    a = round_fp32(rng.standard_normal((M, Kp)) * np.exp2(rng.integers(-3, 3, (M, 1))))
    b = round_fp32(rng.standard_normal((N, Kp)) * 0.05)
    aq, as_ = O.quant_1x128(a)
    bq, bs = O.quant_128x128(b)
    kofs = np.array([lo for lo, _ in ranges] + [ranges[-1][1]], np.int32)
    cu = lambda x, dt: torch.from_numpy(np.ascontiguousarray(x)).to(dt).cuda()
    G = len(ranges)
    c = torch.full((G, M, N), float("nan"), device="cuda")
    ws = torch.empty(B.moe_kgrouped_gemm_fp8_workspace(), dtype=torch.uint8, device="cuda")
    # K = 0 (every group empty) passes empty operands
    B.moe_kgrouped_gemm_fp8(cu(aq[:, :K], torch.uint8), cu(as_[:, :K // 128], torch.float32),
                            cu(bq[:, :K], torch.uint8), cu(bs[:, :K // 128], torch.float32),
                            cu(kofs, torch.int32), c, ws)
    torch.cuda.synchronize()
    assert B.moe_get_error() == 0
    got = c.cpu().double().numpy()
    for g, (lo, hi) in enumerate(ranges):
        if hi == lo:
            assert np.array_equal(got[g], np.zeros((M, N))), g
            continue
        ref = O.scaled_gemm(aq[:, lo:hi], as_[:, lo // 128:hi // 128], bq[:, lo:hi], bs[:, lo // 128:hi // 128])
        assert np.allclose(got[g], ref, rtol=1e-5, atol=1e-6 * np.abs(ref).max()), g


@pytest.mark.parametrize("cfg", [workloads.MoEConfig("bwd_small", T=150, d=512, N_r=4, K_r=2, I=256, seed=21),
                                 workloads.MoEConfig("bwd_mid", T=400, d=2048, N_r=8, K_r=3, I=1024, seed=22)],
                         ids=lambda c: c.name)
def test_expert_backward_matches_oracle(lib, cfg):
    from fine_grained_fp8_sigmoid_b200 import MoELayerFP8
    from fine_grained_fp8_sigmoid_b200 import binding as B
    from fine_grained_fp8_sigmoid_b200.backward import ExpertFFNBackward
    layer = MoELayerFP8(cfg.T, cfg.d, cfg.N_r, cfg.K_r, cfg.I)
    host_w = {}
    for slot in range(cfg.N_r + 1):
        w = workloads.expert_weights(cfg, slot)
        host_w[slot] = O.quantise_expert(*[t.double().numpy() for t in w])
        layer.load_expert(slot, *[t.cuda() for t in w])
    u, e, b = workloads.activations(cfg), workloads.centroids(cfg), workloads.bias(cfg)
    layer.forward(u.cuda(), e.cuda(), b.cuda())
    R = cfg.T * cfg.K_r + cfg.T
    dy = torch.randn(R, cfg.d, generator=torch.Generator().manual_seed(cfg.seed)).to(torch.bfloat16)
    bwd = ExpertFFNBackward(layer)
    r = bwd.backward(dy.cuda())
    torch.cuda.synchronize()
    assert B.moe_get_error() == 0
    # per expert (and the shared one), the oracle on the same rows
    off = list(layer.offsets.cpu().numpy()) + [R]
    st = np.concatenate([layer.sorted_token.cpu().numpy(), np.arange(cfg.T)])
    xq, xs = O.quant_1x128(u.double().numpy())
    dY = dy.double().numpy()
    dX = r["dX"].cpu().double().numpy()
    errs = []
    for gi in range(cfg.N_r + 1):
        lo, hi = off[gi], off[gi + 1]
        if hi == lo:
            assert r["dw_down"][gi].abs().max().item() == 0.0
            continue
        ref = O.expert_ffn_backward(xq[st[lo:hi]], xs[st[lo:hi]], host_w[gi], dY[lo:hi])
        for row in range(hi - lo):
            assert _rel(dX[lo + row], ref["dx"][row]) <= 1e-2, (gi, row)
        errs.append(_rel(dX[lo:hi], ref["dx"]))
        for k in ("dw_gate", "dw_up", "dw_down"):
            e_ = _rel(r[k][gi].cpu().double().numpy(), ref[k])
            assert e_ <= 1e-2, (gi, k, e_)
            errs.append(e_)
    assert max(errs) <= 2e-3 or np.mean(errs) <= 2e-3, errs
    # dx per token: the shared row plus its routed rows (moe_combine, gates 1)
    inv = layer.inv.cpu().numpy()
    P = cfg.T * cfg.K_r
    tok = dX[P:] + dX[inv].sum(axis=1)
    assert _rel(r["dx"].cpu().double().numpy(), round_bf16(tok)) <= 5e-3
