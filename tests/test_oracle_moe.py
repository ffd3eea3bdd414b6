"""Pins for the oracle's layer steps, CPU only.

Each test fixes a result by something other than the oracle itself: a closed
form, a brute-force algorithm written here, an invariant the equations imply,
or a special case that reduces the layer to something simpler.
"""
import itertools
import math

import numpy as np
import pytest
import torch

import workloads
from oracle import moe
from oracle.e4m3 import decode, encode, round_bf16, round_fp32

GAMMA = 0.001


# ---------------------------------------------------------------- quantisers

def test_quant_1x128_scale_per_tile_closed_form():
    # row r, tile j: all entries +-448 * 2^(r - j)  ->  scale exactly 2^(r - j)
    rows, tiles = 3, 4
    x = np.empty((rows, tiles * 128))
    signs = np.where(np.arange(128) % 3 == 0, -1.0, 1.0)
    for r in range(rows):
        for j in range(tiles):
            x[r, j * 128:(j + 1) * 128] = signs * 448.0 * 2.0 ** (r - j)
    q, s = moe.quant_1x128(x)
    assert np.array_equal(s, 2.0 ** (np.arange(rows)[:, None] - np.arange(tiles)[None, :]))
    assert np.all((q == 0x7E) | (q == 0xFE))
    assert np.array_equal(moe.dequant_1x128(q, s), x)


def test_quant_1x128_error_bound_and_amax_code():
    rng = np.random.default_rng(0)
    x = round_fp32(rng.standard_normal((16, 512)) * np.exp2(rng.integers(-20, 20, (16, 1))))
    x[3, 5] = 0.0
    q, s = moe.quant_1x128(x)
    dq = moe.dequant_1x128(q, s)
    S = np.repeat(s, 128, axis=1)
    normal = np.abs(x / S) >= 2.0 ** -6
    err = np.abs(x - dq)
    assert np.all(err[normal] <= 2.0 ** -4 * np.abs(x[normal]))
    assert np.all(err[~normal] <= 2.0 ** -10 * S[~normal])
    # the element of largest magnitude in each tile encodes to +-448
    t = np.abs(x).reshape(16, 4, 128)
    am = t.argmax(axis=2)
    for r in range(16):
        for j in range(4):
            assert q[r, j * 128 + am[r, j]] in (0x7E, 0xFE)


def test_quant_1x128_zero_tile():
    x = np.zeros((2, 256))
    x[1, 200] = 3.0
    x[0, :128] = -0.0
    q, s = moe.quant_1x128(x)
    assert s[0, 0] == 1.0 and s[0, 1] == 1.0 and s[1, 0] == 1.0
    assert np.all(moe.dequant_1x128(q, s)[0] == 0.0)
    assert np.all(q[0, :128] == 0x80) and np.all(q[0, 128:] == 0x00)
    assert s[1, 1] == float(np.float32(3.0 / 448.0))


def test_quant_128x128_block_scales_closed_form():
    R, C = 256, 384
    w = np.zeros((R, C))
    for i in range(2):
        for j in range(3):
            blk = np.full((128, 128), 448.0 * 2.0 ** (i + 2 * j))
            blk[::2, ::3] *= -0.5
            w[i * 128:(i + 1) * 128, j * 128:(j + 1) * 128] = blk
    q, s = moe.quant_128x128(w)
    expect = np.array([[2.0 ** (i + 2 * j) for j in range(3)] for i in range(2)])
    assert np.array_equal(s, expect)
    assert np.array_equal(moe.dequant_128x128(q, s), w)


def test_quant_128x128_error_bound():
    rng = np.random.default_rng(1)
    w = round_fp32(rng.standard_normal((256, 256)) * 0.02)
    q, s = moe.quant_128x128(w)
    dq = moe.dequant_128x128(q, s)
    S = np.repeat(np.repeat(s, 128, 0), 128, 1)
    normal = np.abs(w / S) >= 2.0 ** -6
    assert np.all(np.abs(w - dq)[normal] <= 2.0 ** -4 * np.abs(w[normal]))
    assert np.all(np.abs(w - dq)[~normal] <= 2.0 ** -10 * S[~normal])


# ---------------------------------------------------------------- router

def test_router_zero_centroids_give_one_half():
    u = np.random.default_rng(0).standard_normal((5, 256))
    s = moe.router_scores(u, np.zeros((8, 256)))
    assert np.all(s == 0.5)


def test_router_one_hot_tokens_read_one_centroid_column():
    rng = np.random.default_rng(1)
    e = rng.standard_normal((6, 16))
    cols = np.array([0, 3, 15, 7])
    u = np.zeros((4, 16))
    u[np.arange(4), cols] = 1.0
    s = moe.router_scores(u, e)
    expect = 1.0 / (1.0 + np.exp(-e[:, cols].T))
    assert np.allclose(s, expect, rtol=0, atol=1e-15)


def _check_topk_definition(key, idx):
    T, N = key.shape
    K = idx.shape[1]
    for t in range(T):
        sel = list(idx[t])
        assert len(set(sel)) == K
        rest = [j for j in range(N) if j not in sel]
        for i in sel:
            for j in rest:
                assert key[t, i] > key[t, j] or (key[t, i] == key[t, j] and i < j)
        for a, b in zip(sel[:-1], sel[1:]):
            assert key[t, a] > key[t, b] or (key[t, a] == key[t, b] and a < b)


@pytest.mark.parametrize("ties", [False, True])
@pytest.mark.parametrize("N,K", [(8, 2), (16, 6), (32, 8), (5, 5)])
def test_select_topk_definition(ties, N, K):
    s = workloads.scores(40, N, seed=N + K, ties=ties).double().numpy()
    b = np.zeros(N) if ties else round_fp32(np.random.default_rng(N).uniform(-0.01, 0.01, N))
    idx = moe.select_topk(s, b, K)
    key = round_fp32(s + b[None, :])
    _check_topk_definition(key, idx)


def test_select_topk_all_equal_keys_take_lowest_indices():
    s = np.full((3, 10), 0.25)
    idx = moe.select_topk(s, np.zeros(10), 4)
    assert np.array_equal(idx, np.tile(np.arange(4), (3, 1)))


def test_bias_changes_selection_not_gates():
    s = np.array([[0.9, 0.8, 0.7, 0.1]])
    b = np.array([0.0, 0.0, 0.0, 1.0])
    idx = moe.select_topk(s, b, 2)
    assert list(idx[0]) == [3, 0]
    g = moe.gates_from(s, idx)
    assert np.allclose(g, [[0.1 / 1.0, 0.9 / 1.0]], rtol=0, atol=1e-15)


def test_gates_sum_to_one_and_follow_scores():
    cfg = workloads.CONFIGS["tiny"]
    u = workloads.activations(cfg).double().numpy()
    e = workloads.centroids(cfg).double().numpy()
    b = workloads.bias(cfg).double().numpy()
    s, s32, idx, g = moe.route(u, e, b, cfg.K_r)
    assert np.allclose(g.sum(axis=1), 1.0, rtol=0, atol=1e-12)
    assert np.all((g > 0) & (g <= 1))
    sel = np.take_along_axis(s, idx, axis=1)
    assert np.allclose(g * sel.sum(axis=1, keepdims=True), sel, rtol=1e-14)


# ---------------------------------------------------------------- permutation

def _counting_sort_bruteforce(idx, N_r):
    """Histogram, exclusive prefix sum, then a scatter in token order."""
    T, K = len(idx), (len(idx[0]) if idx else 0)
    counts = [0] * N_r
    for t in range(T):
        for k in range(K):
            counts[idx[t][k]] += 1
    offsets = [0] * (N_r + 1)
    for i in range(N_r):
        offsets[i + 1] = offsets[i] + counts[i]
    cursor = offsets[:-1].copy()
    sorted_token = [None] * (T * K)
    inv = [[None] * K for _ in range(T)]
    for t in range(T):
        for k in sorted(range(K), key=lambda kk: idx[t][kk]):
            i = idx[t][k]
            sorted_token[cursor[i]] = t
            inv[t][k] = cursor[i]
            cursor[i] += 1
    return counts, offsets, sorted_token, inv


@pytest.mark.parametrize("pattern", ["uniform", "first_k", "one_hot_expert"])
@pytest.mark.parametrize("T,N,K", [(1, 4, 2), (37, 8, 2), (100, 16, 6), (64, 6, 6)])
def test_permute_matches_counting_sort(pattern, T, N, K):
    idx = workloads.topk_indices(T, N, K, seed=T + N, pattern=pattern).numpy()
    counts, offsets, st, inv = moe.permute(idx, N)
    c2, o2, st2, inv2 = _counting_sort_bruteforce(idx.tolist(), N)
    assert list(counts) == c2 and list(offsets) == o2
    assert list(st) == st2
    assert inv.tolist() == inv2


def test_permute_invariants_and_empty():
    idx = workloads.topk_indices(500, 32, 8, seed=5).numpy()
    counts, offsets, st, inv = moe.permute(idx, 32)
    assert counts.sum() == 500 * 8 and offsets[-1] == 4000
    for i in range(32):
        seg = st[offsets[i]:offsets[i + 1]]
        assert np.all(np.diff(seg) > 0)
    T = np.repeat(np.arange(500), 8).reshape(500, 8)
    assert np.array_equal(st[inv], T)
    c0, o0, s0, i0 = moe.permute(np.zeros((0, 4), np.int64), 8)
    assert c0.sum() == 0 and o0.tolist() == [0] * 9 and s0.size == 0


# ---------------------------------------------------------------- GEMM / FFN

def test_scaled_gemm_closed_form_scales():
    # A = 1 everywhere with row/K-block scale 2^-m * 2^kb,
    # W = 1 everywhere with block scale 2^(nb - kb):
    # C[m, n] = sum_kb 128 * 2^-m * 2^kb * 2^(n/128 - kb) = KB * 128 * 2^(n/128 - m)
    M, N, KB = 4, 256, 3
    aq = np.full((M, KB * 128), 0x38, np.uint8)           # 1.0
    a_s = np.array([[2.0 ** (-m + kb) for kb in range(KB)] for m in range(M)])
    wq = np.full((N, KB * 128), 0x38, np.uint8)
    w_s = np.array([[2.0 ** (nb - kb) for kb in range(KB)] for nb in range(N // 128)])
    C = moe.scaled_gemm(aq, a_s, wq, w_s)
    expect = np.array([[KB * 128 * 2.0 ** (n // 128 - m) for n in range(N)] for m in range(M)])
    assert np.array_equal(C, expect)


def test_scaled_gemm_integer_matrices_exact():
    rng = np.random.default_rng(4)
    # E4M3 represents every integer in [-16, 16]
    A = rng.integers(-16, 17, (5, 256))
    W = rng.integers(-16, 17, (128, 256))
    aq, wq = encode(A.astype(np.float64)), encode(W.astype(np.float64))
    C = moe.scaled_gemm(aq, np.ones((5, 2)), wq, np.ones((1, 2)))
    exact = [[sum(int(A[m, k]) * int(W[n, k]) for k in range(256)) for n in range(128)]
             for m in range(5)]
    assert np.array_equal(C, np.array(exact, dtype=np.float64))


def test_silu_special_values():
    assert moe.silu(np.array([0.0]))[0] == 0.0
    assert abs(moe.silu(np.array([40.0]))[0] - 40.0) < 1e-15
    assert abs(moe.silu(np.array([-40.0]))[0]) < 1e-15
    x = np.linspace(-5, 5, 11)
    assert np.allclose(moe.silu(x), x * (1 / (1 + np.exp(-x))), rtol=1e-15)


def _const_expert(d, I, gate_code, up_code, down_code):
    return dict(gate_q=np.full((I, d), gate_code, np.uint8), gate_s=np.ones((I // 128, d // 128)),
                up_q=np.full((I, d), up_code, np.uint8), up_s=np.ones((I // 128, d // 128)),
                down_q=np.full((d, I), down_code, np.uint8), down_s=np.ones((d // 128, I // 128)))


def test_expert_ffn_closed_form():
    # x = 1 (code 0x38, scale 1), all weights 2^-7 (code 0x04):
    # G = U = d * 2^-7 = 1 for d = 128, a = silu(1), requant maps a to 448 * scale,
    # y = I * 2^-7 * 448 * scale = 448 * scale for I = 128 (exact: y is not rounded).
    d = I = 128
    xq = np.full((3, d), 0x38, np.uint8)
    xs = np.ones((3, 1))
    y, h = moe.expert_ffn(xq, xs, _const_expert(d, I, 0x04, 0x04, 0x04))
    a = float(np.float32(1.0 / (1.0 + math.exp(-1.0))))
    scale = float(np.float32(a / 448.0))
    assert np.all(h == 448.0 * scale)
    assert np.all(y == 448.0 * scale)


def test_expert_ffn_gate_and_up_roles():
    # SwiGLU is silu(G) * U with G from W_gate and U from W_up, not the other
    # way round. d = 256, I = 128; row 0 is x = 1, row 1 is x = 1/2 (code 0x38
    # with scales 1 and 0.5). W_gate = 2^-7 (code 0x04) and W_up = 2^-8 (code
    # 0x02) everywhere, so row 0 has G = 2, U = 1 and row 1 has G = 1, U = 1/2.
    # A negative up weight (code 0x82) flips U. Each intermediate tile holds
    # one value a, requantised to +-448 with scale fl32(|a|/448); W_down =
    # 2^-7 (code 0x04) sums I = 128 of them: y = +-448 * scale (exact).
    d, I = 256, 128
    xq = np.full((2, d), 0x38, np.uint8)
    xs = np.array([[1.0, 1.0], [0.5, 0.5]])
    sig = lambda v: 1.0 / (1.0 + math.exp(-v))
    for up_code, sign in [(0x02, 1.0), (0x82, -1.0)]:
        y, h = moe.expert_ffn(xq, xs, _const_expert(d, I, 0x04, up_code, 0x04))
        for row, (G, U) in enumerate([(2.0, 1.0), (1.0, 0.5)]):
            a = float(np.float32(G * sig(G) * U * sign))
            swapped = float(np.float32(U * sig(U) * G * sign))
            assert a != swapped
            scale = float(np.float32(abs(a) / 448.0))
            assert np.all(h[row] == math.copysign(448.0 * scale, a)), row
            assert np.all(y[row] == math.copysign(448.0 * scale, a)), row
            assert y.shape == (2, d) and h.shape == (2, I)


def test_expert_ffn_zero_gate_gives_zero():
    xq = encode(np.random.default_rng(0).standard_normal((4, 256)))
    y, h = moe.expert_ffn(xq, np.ones((4, 2)), _const_expert(256, 128, 0x00, 0x38, 0x38))
    assert np.all(y == 0.0) and np.all(h == 0.0)


# ---------------------------------------------------------------- combine, bias

def test_combine_hand_example():
    u = np.array([[1.0, 2.0], [3.0, 4.0]])
    ysh = np.array([[0.5, 0.5], [0.0, 1.0]])
    yp = np.array([[10.0, 0.0], [0.0, 10.0], [1.0, 1.0], [2.0, 2.0]])
    inv = np.array([[0, 2], [1, 3]])
    g = np.array([[0.75, 0.25], [0.5, 0.5]])
    out = moe.combine(u, yp, ysh, inv, g)
    expect = np.array([[1 + 0.5 + 7.5 + 0.25, 2 + 0.5 + 0 + 0.25],
                       [3 + 0 + 0 + 1.0, 4 + 1 + 5 + 1.0]])
    assert np.array_equal(out, expect)


def test_bias_update_sign_rule():
    b = np.array([0.5, -0.25, 0.0, 0.125], dtype=np.float64)
    counts = np.array([3, 2, 1, 2])          # T*K = 8, N_r = 4 -> mean load 2
    nb, ratio = moe.bias_update(b, counts, T=4, K=2)
    g = np.float32(GAMMA)
    assert nb[0] == np.float32(np.float32(0.5) - g)
    assert nb[1] == -0.25 and nb[3] == 0.125
    assert nb[2] == np.float32(np.float32(0.0) + g)
    assert ratio == 1.5


def test_bias_update_non_integer_mean():
    # mean load 7*3/4 = 5.25: 5 is under, 6 is over
    nb, _ = moe.bias_update(np.zeros(4), np.array([5, 6, 5, 5]), T=7, K=3)
    g = float(np.float32(GAMMA))
    assert list(nb) == [g, -g, g, g]


# ---------------------------------------------------------------- whole layer

def _quantised_provider(cfg):
    cache = {}

    def get(slot):
        if slot not in cache:
            w = [t.double().numpy() for t in workloads.expert_weights(cfg, slot)]
            cache[slot] = moe.quantise_expert(*w)
        return cache[slot]
    return get


def test_single_expert_zero_weights_returns_residual():
    u = workloads.activations(workloads.MoEConfig("t", 9, 256, 1, 1, 128, 3)).double().numpy()
    zero = _const_expert(256, 128, 0, 0, 0)
    r = moe.moe_forward(u, np.zeros((1, 256)), np.zeros(1), 1, lambda s: zero)
    assert np.array_equal(r["out"], u)
    assert np.all(r["gates"] == 1.0)


def test_all_experts_selected_equals_dense_gated_sum():
    cfg = workloads.MoEConfig("dense", T=20, d=256, N_r=4, K_r=4, I=128, seed=11)
    u = workloads.activations(cfg).double().numpy()
    e = workloads.centroids(cfg).double().numpy()
    b = np.zeros(4)
    prov = _quantised_provider(cfg)
    zero = _const_expert(256, 128, 0, 0, 0)
    get = lambda s: zero if s == cfg.N_r else prov(s)
    r = moe.moe_forward(u, e, b, cfg.K_r, get)
    # dense: every expert on every token, gate s_i / sum_j s_j, each expert's
    # output taken as bf16 (the layer's expert-output type)
    s = moe.router_scores(u, e)
    xq, xs = moe.quant_1x128(u)
    acc = u.copy()
    for i in range(4):
        y, _ = moe.expert_ffn(xq, xs, prov(i))
        acc += (s[:, i] / s.sum(axis=1))[:, None] * round_bf16(y)
    # equal bit for bit (the float64 sums differ only in order, far below a
    # bf16 step); unrounded expert outputs would move a few dozen of these
    # 5120 outputs by one bf16 step
    assert np.array_equal(r["out"], round_bf16(acc))


def test_token_sample_matches_full_forward():
    cfg = workloads.CONFIGS["tiny"]
    u = workloads.activations(cfg).double().numpy()
    e = workloads.centroids(cfg).double().numpy()
    b = workloads.bias(cfg).double().numpy()
    prov = _quantised_provider(cfg)
    full = moe.moe_forward(u, e, b, cfg.K_r, prov)
    tok = np.array([0, 5, 17, 63])
    part = moe.moe_forward(u, e, b, cfg.K_r, prov, tokens=tok)
    assert np.array_equal(part["out"], full["out"][tok])
    # up to float64 rounding order (the matmul blocks differently per batch size)
    assert np.allclose(part["y_shared"], full["y_shared"][tok], rtol=1e-12, atol=1e-12)
    assert np.array_equal(part["bias_new"], full["bias_new"])
    # routed outputs sit where the permutation says
    assert full["counts"].sum() == cfg.T * cfg.K_r


def test_tiny_forward_is_finite_and_near_residual_scale():
    cfg = workloads.CONFIGS["tiny"]
    u = workloads.activations(cfg).double().numpy()
    e = workloads.centroids(cfg).double().numpy()
    b = workloads.bias(cfg).double().numpy()
    r = moe.moe_forward(u, e, b, cfg.K_r, _quantised_provider(cfg))
    assert np.all(np.isfinite(r["out"]))
    assert r["out"].shape == (cfg.T, cfg.d)
    # the expert contribution is small next to the N(0,1) residual
    assert np.abs(r["out"] - u).max() < 1.0


# ---------------------------------------------------------------- backward

def test_dsilu_against_autograd():
    x = np.linspace(-30, 30, 601)
    t = torch.tensor(x, dtype=torch.float64, requires_grad=True)
    torch.nn.functional.silu(t).sum().backward()
    assert np.allclose(moe.dsilu(x), t.grad.numpy(), rtol=1e-13, atol=1e-15)
    assert moe.dsilu(np.array([0.0]))[0] == 0.5


def _bwd_case(m=37, d=256, I=128, seed=3):
    rng = np.random.default_rng(seed)
    xq, xs = moe.quant_1x128(rng.standard_normal((m, d)))
    w = moe.quantise_expert(rng.standard_normal((I, d)) * 0.05, rng.standard_normal((I, d)) * 0.05,
                            rng.standard_normal((d, I)) * 0.05)
    dy = round_bf16(rng.standard_normal((m, d)))
    return xq, xs, w, dy


def test_expert_backward_without_quantisation_is_the_autograd_derivative():
    # the wiring (transposes, operand roles, the SwiGLU derivative, the
    # requantisation passed through) against torch float64 autograd of the
    # forward as executed: the same dequantised operands, H = a + (q(a) - a)
    xq, xs, w, dy = _bwd_case()
    r = moe.expert_ffn_backward(xq, xs, w, dy, quantize=False)
    T = lambda a: torch.tensor(a, dtype=torch.float64, requires_grad=True)
    X = T(moe.dequant_1x128(xq, xs))
    Wg, Wu, Wd = (T(moe.dequant_128x128(w[k + "_q"], w[k + "_s"])) for k in ("gate", "up", "down"))
    a = torch.nn.functional.silu(X @ Wg.T) * (X @ Wu.T)
    hq, hs = moe.quant_1x128(round_fp32(a.detach().numpy()))
    H = a + torch.tensor(moe.dequant_1x128(hq, hs) - a.detach().numpy())   # the cast, as a constant shift
    Y = H @ Wd.T
    Y.backward(torch.tensor(dy))
    for got, t in [(r["dx"], X), (r["dw_gate"], Wg), (r["dw_up"], Wu), (r["dw_down"], Wd)]:
        assert np.allclose(got, t.grad.numpy(), rtol=1e-10, atol=1e-12)


def test_expert_backward_quantised_operands_stay_within_the_fp8_error():
    # with the backward's own FP8 quantisations the gradients move by about
    # the E4M3 step (2^-4 relative per operand), not more
    xq, xs, w, dy = _bwd_case(m=300, d=512, I=256, seed=5)
    q = moe.expert_ffn_backward(xq, xs, w, dy)
    e = moe.expert_ffn_backward(xq, xs, w, dy, quantize=False)
    for k in ("dx", "dw_gate", "dw_up", "dw_down"):
        rel = np.linalg.norm(q[k] - e[k]) / np.linalg.norm(e[k])
        assert 1e-4 < rel < 0.08, (k, rel)


def test_expert_backward_exact_on_representable_values():
    # one token row: x = 1, weights 2^-7 everywhere, d = I = 128: G = U = 1,
    # a = silu(1); dY = 1 everywhere (one value per tile: code 448, scale
    # fl32(1/448)). dH = 128 * 2^-7 * q(1); dG = dH U dsilu(1), dU = dH silu(1) (each tile one
    # value, so its code is +-448 and the quantisation exact up to the FP32
    # rounding of the scale); dX = 128 * 2^-7 * (dG + dU)
    d = I = 128
    xq = np.full((1, d), 0x38, np.uint8)
    w = dict(gate_q=np.full((I, d), 0x04, np.uint8), gate_s=np.ones((1, 1)),
             up_q=np.full((I, d), 0x04, np.uint8), up_s=np.ones((1, 1)),
             down_q=np.full((d, I), 0x04, np.uint8), down_s=np.ones((1, 1)))
    r = moe.expert_ffn_backward(xq, np.ones((1, 1)), w, np.ones((1, d)))
    sig = 1 / (1 + math.exp(-1.0))
    q = lambda v: 448.0 * float(np.float32(float(np.float32(v)) / 448.0))   # a tile of one value
    dh = q(1.0)                                  # dY = 1 dequantises to 448 * fl32(1/448)
    dg, du = q(dh * sig * (1 + (1 - sig))), q(dh * sig)
    assert np.all(r["dh"] == dh)
    assert np.allclose(r["dx"], dg + du, rtol=0, atol=1e-15)
    # wgrad: one token (padded to 128 with zeros): dW_down[j][i] = dY * H
    h = q(float(np.float32(sig)))
    assert np.allclose(r["dw_down"], h, rtol=2 ** -10)
