"""Every step of the DeepSeekMoE FP8 layer forward pass, in float64 numpy.

Test infrastructure only (see the package docstring). Each function cites the
passage it follows. "[TR]" is the page "DeepSeek-V3 Teknik Raporu"
(xyznot.com/tr/paper/2412.19437); "[FR]" is its French copy "DeepSeek-V3
Technical Report" (xyznot.com/fr/paper/2412.19437). Where the pages leave a
step open, the docstring says which reading is taken.

Conventions
-----------
* Inputs u (tokens x d) and centroids e (N_r x d) hold bf16 values, passed as
  float64 arrays (exact).
* FP8 tensors are uint8 E4M3 codes plus float64 arrays holding FP32 scales.
  Activation scales are row-major [rows, cols/128]; weight scales are
  [rows/128, cols/128].
* The shared expert is expert slot N_r.
"""
from __future__ import annotations

import numpy as np

from .e4m3 import E4M3_MAX, decode, encode, round_bf16, round_fp32

TILE = 128          # 1x128 activation tiles, 128x128 weight blocks ([TR] Temel fikirler, FP8 bullet)
GAMMA = 0.001       # bias update speed ([TR] Yöntem 2, last paragraph)


# --------------------------------------------------------------------------
# Quantisation ([TR] Temel fikirler, "FP8 Karma Duyarlıklı Eğitim": E4M3 on
# all tensors, one scale per 1x128 activation tile and per 128x128 weight
# block). The pages do not print the scale rule; the reading taken is the
# plain max-abs rule: scale = fl32(amax / 448), q = E4M3_RNE(fl32(x / scale)),
# and scale = 1 when fl32(amax / 448) is zero (an all-zero tile).
# fl32(a / b) for FP32 a, b is computed as a float64 division rounded once to
# FP32, which equals the correctly rounded FP32 division (53 >= 2*24 + 2).
# --------------------------------------------------------------------------

def _scale_from_amax(amax: np.ndarray) -> np.ndarray:
    s = round_fp32(amax / E4M3_MAX)
    return np.where(s == 0.0, 1.0, s)


def quant_1x128(x: np.ndarray):
    """Activation quantisation: one FP32 scale per 1x128 tile of a row.

    x: [rows, cols] float64 holding FP32 values, cols % 128 == 0.
    Returns (q uint8 [rows, cols], scale float64 [rows, cols/128]).
    """
    x = np.asarray(x, dtype=np.float64)
    rows, cols = x.shape
    if cols % TILE:
        raise ValueError("cols must be a multiple of 128")
    t = x.reshape(rows, cols // TILE, TILE)
    scale = _scale_from_amax(np.abs(t).max(axis=2)) if rows else np.ones((0, cols // TILE))
    y = round_fp32(t / scale[:, :, None])
    return encode(y).reshape(rows, cols), scale


def quant_128x128(w: np.ndarray):
    """Weight quantisation: one FP32 scale per 128x128 block.

    w: [R, C] float64 holding FP32 values, R and C multiples of 128.
    Returns (q uint8 [R, C], scale float64 [R/128, C/128]).
    """
    w = np.asarray(w, dtype=np.float64)
    R, C = w.shape
    if R % TILE or C % TILE:
        raise ValueError("weight dims must be multiples of 128")
    b = w.reshape(R // TILE, TILE, C // TILE, TILE)
    scale = _scale_from_amax(np.abs(b).max(axis=(1, 3)))
    y = round_fp32(b / scale[:, None, :, None])
    return encode(y).reshape(R, C), scale


def dequant_1x128(q: np.ndarray, scale: np.ndarray) -> np.ndarray:
    return decode(q) * np.repeat(scale, TILE, axis=1)


def dequant_128x128(q: np.ndarray, scale: np.ndarray) -> np.ndarray:
    return decode(q) * np.repeat(np.repeat(scale, TILE, axis=0), TILE, axis=1)


def quantise_expert(w_gate, w_up, w_down) -> dict:
    """Quantise one expert's three FP32 weight matrices block-wise."""
    gq, gs = quant_128x128(w_gate)
    uq, us = quant_128x128(w_up)
    dq, ds = quant_128x128(w_down)
    return dict(gate_q=gq, gate_s=gs, up_q=uq, up_s=us, down_q=dq, down_s=ds)


# --------------------------------------------------------------------------
# Router ([TR] Yöntem 2; [FR] Méthode 2)
# --------------------------------------------------------------------------

def router_scores(u: np.ndarray, e: np.ndarray) -> np.ndarray:
    """s_{i,t} = Sigmoid(u_t^T e_i), float64 [T, N_r]."""
    z = np.asarray(u, np.float64) @ np.asarray(e, np.float64).T
    return 1.0 / (1.0 + np.exp(-z))


def select_topk(s32: np.ndarray, b: np.ndarray, K: int) -> np.ndarray:
    """Top-K_r experts of the biased keys s_{i,t} + b_i ([TR] Yöntem 2, the
    g'_{i,t} equation: the bias enters the selection only).

    The keys are formed in FP32 (s32 and b hold FP32 values; their sum is
    rounded once to FP32), the precision in which the kernel takes the same
    decision. Equal keys go to the lower expert index. The result is ordered
    by key descending, then index ascending.
    """
    key = round_fp32(np.asarray(s32, np.float64) + np.asarray(b, np.float64)[None, :])
    order = np.argsort(-key, axis=1, kind="stable")
    return order[:, :K].astype(np.int64)


def gates_from(s: np.ndarray, idx: np.ndarray) -> np.ndarray:
    """g_{i,t}: the selected affinities normalised to sum to one.

    [TR] Yöntem 2 says g is obtained by normalising g' (g' = s on the selected
    experts, 0 elsewhere); the formula is not printed, the reading taken is
    g = g' / sum_j g'_j, with the bias excluded.
    """
    sel = np.take_along_axis(np.asarray(s, np.float64), idx, axis=1)
    return sel / sel.sum(axis=1, keepdims=True)


def route(u, e, b, K: int):
    """Full router: returns (s float64, s rounded to FP32, topk idx, gates)."""
    s = router_scores(u, e)
    s32 = round_fp32(s)
    idx = select_topk(s32, b, K)
    return s, s32, idx, gates_from(s, idx)


# --------------------------------------------------------------------------
# Permutation. The pages group tokens per expert without printing how; the
# reading taken is a stable counting sort: rows ordered by (expert asc, token
# asc). This function is that order's definition; the histogram / prefix-sum
# / scatter algorithm is pinned against it by brute force in the tests.
# --------------------------------------------------------------------------

def permute(idx: np.ndarray, N_r: int):
    """Returns counts [N_r], offsets [N_r+1], sorted_token [T*K], inv [T, K].

    Row p of the permuted layout holds token sorted_token[p]; the pair
    (t, k) (token t's k-th selected expert) sits at row inv[t, k].
    """
    idx = np.asarray(idx, np.int64)
    T, K = idx.shape
    flat_e = idx.reshape(-1)
    flat_t = np.repeat(np.arange(T, dtype=np.int64), K)
    counts = np.bincount(flat_e, minlength=N_r).astype(np.int64)
    offsets = np.concatenate([[0], np.cumsum(counts)]).astype(np.int64)
    order = np.lexsort((flat_t, flat_e))            # primary: expert, then token
    sorted_token = flat_t[order]
    inv = np.empty(T * K, dtype=np.int64)
    inv[order] = np.arange(T * K, dtype=np.int64)
    return counts, offsets, sorted_token, inv.reshape(T, K)


# --------------------------------------------------------------------------
# Expert FFN: SwiGLU with gate/up and down projections on FP8 operands.
# The pages say "FFN"; the SwiGLU form and sizes come from the workload
# definitions. FP32 promotion every N_c = 128 ([TR] Temel fikirler, FP8
# bullet) fixes how the GPU accumulates; in float64 the dot product of the
# dequantised operands is the exact target of that accumulation.
# --------------------------------------------------------------------------

def scaled_gemm(aq, a_scale, wq, w_scale) -> np.ndarray:
    """C[m, n] = sum_k (q_A[m,k] s_A[m,k/128]) (q_W[n,k] s_W[n/128,k/128])."""
    A = dequant_1x128(aq, a_scale)
    W = dequant_128x128(wq, w_scale)
    return A @ W.T


def silu(x: np.ndarray) -> np.ndarray:
    with np.errstate(over="ignore"):
        return x / (1.0 + np.exp(-x))


def expert_ffn_parts(xq, xs, w: dict) -> dict:
    """One expert on FP8 rows (xq, xs), with its intermediate values.

    a = silu(X W_gate^T) * (X W_up^T); a is rounded to FP32 (the precision
    the kernel holds it in) and requantised per 1x128 tile along I to
    (hq, hs); then Y = H W_down^T, kept in float64 here (the exact value
    that the layer's bf16 expert output rounds; moe_forward rounds it).
    Returns dict(G, U, a32 [m, I], hq uint8 [m, I], hs [m, I/128], y [m, d]).
    """
    G = scaled_gemm(xq, xs, w["gate_q"], w["gate_s"])
    U = scaled_gemm(xq, xs, w["up_q"], w["up_s"])
    a32 = round_fp32(silu(G) * U)
    hq, hs = quant_1x128(a32)
    return dict(G=G, U=U, a32=a32, hq=hq, hs=hs, y=expert_down(hq, hs, w))


def expert_down(hq, hs, w: dict) -> np.ndarray:
    """The down projection Y = H W_down^T of FP8 intermediate rows (hq, hs)."""
    return scaled_gemm(hq, hs, w["down_q"], w["down_s"])


def expert_ffn(xq, xs, w: dict):
    """One expert on FP8 rows: returns (Y float64 [m, d], H dequantised
    float64 [m, I]); see expert_ffn_parts."""
    p = expert_ffn_parts(xq, xs, w)
    return p["y"], dequant_1x128(p["hq"], p["hs"])


# --------------------------------------------------------------------------
# Backward of one expert FFN in the same FP8 scheme. The pages train in FP8
# ([TR] Temel fikirler, FP8 bullet: E4M3 on all tensors, activations in 1x128
# tiles, weights in 128x128 blocks) and print no backward details; the
# readings taken:
#  * every GEMM of the backward has FP8 operands, E4M3 like the forward's;
#  * an operand's granularity follows its role in the product: the operand
#    whose rows are the product's rows (the "activation" role) has one scale
#    per 1x128 tile along the contraction, the other (the "weight" role) one
#    scale per 128x128 block; before quantisation a value is rounded to FP32;
#  * the requantisation of the intermediate is a cast in the backward (its
#    gradient passes through unchanged);
#  * dgrad uses the forward's weight codes and scales (transposed exactly);
#    wgrad contracts over the expert's tokens, zero-padded to a multiple of
#    128, with the forward's FP8 activations (X and H as the forward used
#    them) requantised in 128x128 blocks and the gradients in 1x128 tiles.
# --------------------------------------------------------------------------

def dsilu(x: np.ndarray) -> np.ndarray:
    """d/dx silu(x) = sigma(x) (1 + x (1 - sigma(x)))."""
    with np.errstate(over="ignore"):
        s = 1.0 / (1.0 + np.exp(-x))
    return s * (1.0 + x * (1.0 - s))


def _fp8_act(x, quantize):
    """An operand in the activation role: 1x128 tiles along the rows."""
    return dequant_1x128(*quant_1x128(round_fp32(x))) if quantize else x


def _fp8_blocks(x, quantize):
    """An operand in the weight role: 128x128 blocks."""
    return dequant_128x128(*quant_128x128(round_fp32(x))) if quantize else x


def _pad_rows(x, m):
    return np.concatenate([x, np.zeros((m - x.shape[0],) + x.shape[1:])]) if m > x.shape[0] else x


def expert_ffn_backward(xq, xs, w: dict, dy, quantize: bool = True) -> dict:
    """Gradients of Y = H W_down^T, H = q(silu(X W_gate^T) * (X W_up^T)) for
    one expert's FP8 rows (xq, xs) given dY [m, d].

    Returns dict with dx [m, d], dw_gate [I, d], dw_up [I, d], dw_down [d, I]
    and the intermediates (G, U, dh, dg, du). quantize=False drops every
    backward quantisation (the forward's FP8 operands stay): then the result
    is the plain float64 derivative of the forward as executed.
    """
    X = dequant_1x128(xq, xs)
    Wg = dequant_128x128(w["gate_q"], w["gate_s"])
    Wu = dequant_128x128(w["up_q"], w["up_s"])
    Wd = dequant_128x128(w["down_q"], w["down_s"])
    G, U = X @ Wg.T, X @ Wu.T
    a32 = round_fp32(silu(G) * U)
    H = dequant_1x128(*quant_1x128(a32))
    m = X.shape[0]
    # dgrad: dH = dY W_down, then through SwiGLU, dX = dG W_gate + dU W_up
    dh = _fp8_act(np.asarray(dy, np.float64), quantize) @ Wd
    dg = dh * U * dsilu(G)
    du = dh * silu(G)
    dgu = _fp8_act(np.concatenate([dg, du], axis=1), quantize)
    I = dg.shape[1]
    dx = dgu[:, :I] @ Wg + dgu[:, I:] @ Wu
    # wgrad: contractions over the tokens, padded to a multiple of 128
    mp = -(-m // 128) * 128
    t_act = lambda g: _fp8_act(_pad_rows(g, mp).T, quantize)     # [features, tokens]
    t_blk = lambda v: _fp8_blocks(_pad_rows(v, mp).T, quantize)
    dw_down = t_act(dy) @ t_blk(H).T
    Xt = t_blk(X)
    dw_gate = t_act(dg) @ Xt.T
    dw_up = t_act(du) @ Xt.T
    return dict(dx=dx, dw_gate=dw_gate, dw_up=dw_up, dw_down=dw_down, G=G, U=U, dh=dh, dg=dg, du=du, H=H)


# --------------------------------------------------------------------------
# Combine ([TR] Yöntem 2, h'_t = u_t + sum_s FFN^(s)(u_t) + sum_i g_{i,t} FFN^(r)_i(u_t))
# --------------------------------------------------------------------------

def combine(u, y_perm, y_shared, inv, gates) -> np.ndarray:
    """h'_t = bf16(u_t + y_shared_t + sum_k g_{t,k} y_perm[inv[t,k]])."""
    acc = np.asarray(u, np.float64) + np.asarray(y_shared, np.float64)
    for k in range(inv.shape[1]):
        acc = acc + gates[:, k:k + 1] * y_perm[inv[:, k]]
    return round_bf16(acc)


# --------------------------------------------------------------------------
# Auxiliary-loss-free bias update ([TR] Yöntem 2, last paragraph: at the end
# of the step b_i <- b_i - gamma if expert i is overloaded, b_i + gamma if
# underloaded, gamma = 0.001). "Overloaded" is not defined on the pages; the
# reading taken compares the load c_i with the mean load T*K_r/N_r in
# integers (c_i * N_r vs T * K_r); equal load leaves b_i unchanged. The
# update is FP32 arithmetic on FP32 values.
# --------------------------------------------------------------------------

def bias_update(b, counts, T: int, K: int, gamma: float = GAMMA):
    b = np.asarray(b, np.float64)
    counts = np.asarray(counts, np.int64)
    N_r = counts.shape[0]
    g32 = float(np.float32(gamma))
    load = counts * N_r
    mean = T * K
    out = b.copy()
    over = load > mean
    under = load < mean
    out[over] = round_fp32(b[over] - g32)
    out[under] = round_fp32(b[under] + g32)
    ratio = float(counts.max() * N_r / mean) if mean > 0 else 0.0
    return out, ratio


# --------------------------------------------------------------------------
# Whole layer
# --------------------------------------------------------------------------

def moe_forward(u, e, b, K: int, weights, tokens=None, select=None, map_fn=map) -> dict:
    """The layer's forward pass.

    u [T, d], e [N_r, d] (bf16 values), b [N_r] (FP32 values).
    weights(slot) -> quantised expert dict (slot N_r is the shared expert).
    tokens: optional 1-D array of token indices; routing, permutation and
    the bias update always cover all T tokens, the expert outputs and the
    combine only the listed tokens (tokens are independent given routing).
    select: optional [T, K] expert choice to use instead of the oracle's own
    top-K (to evaluate a token under another, equally valid, selection when
    two keys are closer than the comparison can resolve); gates are still the
    oracle's affinities normalised over that selection.
    map_fn: how the per-expert FFNs are evaluated (the builtin map, or an
    executor's map to run independent experts side by side; the arithmetic
    of each expert is the same either way).
    """
    u = np.asarray(u, np.float64)
    T, d = u.shape
    N_r = e.shape[0]
    s, s32, idx, gates = route(u, e, b, K)
    if select is not None:
        idx = np.asarray(select, np.int64)
        gates = gates_from(s, idx)
    counts, offsets, sorted_token, inv = permute(idx, N_r)
    b_new, ratio = bias_update(b, counts, T, K)

    sample = np.arange(T) if tokens is None else np.asarray(tokens, np.int64)
    S = sample.shape[0]
    xq, xs = quant_1x128(u[sample])
    sel = idx[sample]
    slots = [int(s_) for s_ in np.unique(sel)]
    whos = [np.argwhere(sel == slot) for slot in slots]      # rows (sample i, k)

    def one(j):
        if j == len(slots):
            return expert_ffn_parts(xq, xs, weights(N_r))
        who = whos[j]
        return expert_ffn_parts(xq[who[:, 0]], xs[who[:, 0]], weights(slots[j]))

    results = list(map_fn(one, range(len(slots) + 1)))
    routed = {}
    for who, p in zip(whos, results[:-1]):
        for key, v in p.items():
            if key not in routed:
                routed[key] = np.zeros((S, K) + v.shape[1:], v.dtype)
            routed[key][who[:, 0], who[:, 1]] = v
    if not routed:
        routed = dict(y=np.zeros((S, K, d)))
    shared = results[-1]
    y_routed, y_shared = routed["y"], shared["y"]
    h_routed = (dequant_1x128(routed["hq"].reshape(S * K, -1), routed["hs"].reshape(S * K, -1)).reshape(S, K, -1)
                if "hq" in routed else None)
    h_shared = dequant_1x128(shared["hq"], shared["hs"])

    # the expert outputs cross to the combine as bf16 (reading: the layer's
    # activations are bf16 on both sides of the FFNs, [TR] Yöntem 2 h'_t
    # equation), and h' is rounded to bf16 once more after the sum
    y_routed_bf16, y_shared_bf16 = round_bf16(y_routed), round_bf16(y_shared)
    acc = u[sample] + y_shared_bf16
    for k in range(K):
        acc = acc + gates[sample, k:k + 1] * y_routed_bf16[:, k]
    out = round_bf16(acc)
    return dict(scores=s, scores32=s32, topk_idx=idx, gates=gates,
                counts=counts, offsets=offsets, sorted_token=sorted_token,
                inv=inv, bias_new=b_new, max_over_mean=ratio, tokens=sample,
                xq=xq, xs=xs, y_routed=y_routed, h_routed=h_routed,
                y_shared=y_shared, h_shared=h_shared, out=out,
                y_routed_bf16=y_routed_bf16, y_shared_bf16=y_shared_bf16,
                routed_parts=routed, shared_parts=shared)
