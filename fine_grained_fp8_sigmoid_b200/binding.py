"""Thin Python binding of the C ABI: same names as include/moe_fp8.h, torch
tensors in, status checked, nothing computed here.

Each function takes CUDA tensors (checked for device, dtype, contiguity and
shape), passes their device pointers and the current CUDA stream to the
library, and raises MoEError on a non-OK status. bf16 tensors are passed as
their raw 16-bit patterns; FP8 tensors are torch.uint8 holding E4M3 codes.
"""
from __future__ import annotations

import ctypes

import torch

from . import _lib
from ._lib import MoEError, check  # noqa: F401


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _want(t, dtype, shape, name):
    if t is None:
        raise ValueError(f"{name} is required")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise ValueError(f"{name}: dtype {t.dtype}, expected {dtype}")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name}: shape {tuple(t.shape)}, expected {tuple(shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t


def _opt(t, dtype, shape, name):
    return None if t is None else _want(t, dtype, shape, name)


def moe_quant_1x128(x, q, scale, stream=None):
    rows, cols = x.shape
    _want(x, torch.bfloat16, (rows, cols), "x")
    _want(q, torch.uint8, (rows, cols), "q")
    _want(scale, torch.float32, (rows, cols // 128), "scale")
    check("moe_quant_1x128", _lib.load().moe_quant_1x128(
        _ptr(x), rows, cols, _ptr(q), _ptr(scale), _stream(stream)))


def moe_quant_128x128(w, q, scale, stream=None):
    rows, cols = w.shape
    _want(w, torch.float32, (rows, cols), "w")
    _want(q, torch.uint8, (rows, cols), "q")
    _want(scale, torch.float32, (rows // 128, cols // 128), "scale")
    check("moe_quant_128x128", _lib.load().moe_quant_128x128(
        _ptr(w), rows, cols, _ptr(q), _ptr(scale), _stream(stream)))


def moe_route(u, e, b, K_r, topk_idx, gates, scores_in=None, scores_out=None, stream=None):
    N_r = b.shape[0]
    if scores_in is not None:
        T = scores_in.shape[0]
        d = 0
        _want(scores_in, torch.float32, (T, N_r), "scores_in")
    else:
        T, d = u.shape
        _want(u, torch.bfloat16, (T, d), "u")
        _want(e, torch.bfloat16, (N_r, d), "e")
    _want(b, torch.float32, (N_r,), "b")
    _want(topk_idx, torch.int32, (T, K_r), "topk_idx")
    _want(gates, torch.float32, (T, K_r), "gates")
    _opt(scores_out, torch.float32, (T, N_r), "scores_out")
    check("moe_route", _lib.load().moe_route(
        _ptr(u), _ptr(e), _ptr(b), _ptr(scores_in), T, d, N_r, K_r, _ptr(scores_out),
        _ptr(topk_idx), _ptr(gates), _stream(stream)))


def moe_route_quant(u, e, b, K_r, topk_idx, gates, xq, xs, scores_out=None, stream=None):
    """moe_route from u and e, and in the same kernel moe_quant_1x128 of u
    into xq [T][d] (E4M3) and xs [T][d/128]."""
    N_r = b.shape[0]
    T, d = u.shape
    _want(u, torch.bfloat16, (T, d), "u")
    _want(e, torch.bfloat16, (N_r, d), "e")
    _want(b, torch.float32, (N_r,), "b")
    _want(topk_idx, torch.int32, (T, K_r), "topk_idx")
    _want(gates, torch.float32, (T, K_r), "gates")
    _want(xq, torch.uint8, (T, d), "xq")
    _want(xs, torch.float32, (T, d // 128), "xs")
    _opt(scores_out, torch.float32, (T, N_r), "scores_out")
    check("moe_route_quant", _lib.load().moe_route_quant(
        _ptr(u), _ptr(e), _ptr(b), T, d, N_r, K_r, _ptr(scores_out), _ptr(topk_idx), _ptr(gates),
        _ptr(xq), _ptr(xs), _stream(stream)))


def moe_permute_workspace(T, N_r):
    return int(_lib.load().moe_permute_workspace(T, N_r))


def moe_permute(topk_idx, N_r, counts, offsets, sorted_token, inv, workspace,
                xq=None, xs=None, xq_perm=None, xs_perm=None, stream=None):
    T, K_r = topk_idx.shape
    _want(topk_idx, torch.int32, (T, K_r), "topk_idx")
    _want(counts, torch.int32, (N_r,), "counts")
    _want(offsets, torch.int32, (N_r + 1,), "offsets")
    _want(sorted_token, torch.int32, (T * K_r,), "sorted_token")
    _want(inv, torch.int32, (T, K_r), "inv")
    d = 0
    if xq is not None:
        d = xq.shape[1]
        _want(xq, torch.uint8, (T, d), "xq")
        _want(xs, torch.float32, (T, d // 128), "xs")
        _want(xq_perm, torch.uint8, (T * K_r, d), "xq_perm")
        _want(xs_perm, torch.float32, (T * K_r, d // 128), "xs_perm")
    check("moe_permute", _lib.load().moe_permute(
        _ptr(topk_idx), T, K_r, N_r, _ptr(xq), _ptr(xs), d, _ptr(counts), _ptr(offsets),
        _ptr(sorted_token), _ptr(inv), _ptr(xq_perm), _ptr(xs_perm), _ptr(workspace),
        workspace.numel() * workspace.element_size() if workspace is not None else 0,
        _stream(stream)))


def moe_permute_noalloc(topk_idx, N_r, counts, offsets, sorted_token, inv,
                        xq=None, xs=None, xq_perm=None, xs_perm=None, stream=None):
    """moe_permute without a workspace: the library's static scratch array is
    used instead (for callers that cannot allocate device memory)."""
    T, K_r = topk_idx.shape
    _want(topk_idx, torch.int32, (T, K_r), "topk_idx")
    _want(counts, torch.int32, (N_r,), "counts")
    _want(offsets, torch.int32, (N_r + 1,), "offsets")
    _want(sorted_token, torch.int32, (T * K_r,), "sorted_token")
    _want(inv, torch.int32, (T, K_r), "inv")
    d = 0
    if xq is not None:
        d = xq.shape[1]
        _want(xq, torch.uint8, (T, d), "xq")
        _want(xs, torch.float32, (T, d // 128), "xs")
        _want(xq_perm, torch.uint8, (T * K_r, d), "xq_perm")
        _want(xs_perm, torch.float32, (T * K_r, d // 128), "xs_perm")
    check("moe_permute_noalloc", _lib.load().moe_permute_noalloc(
        _ptr(topk_idx), T, K_r, N_r, _ptr(xq), _ptr(xs), d, _ptr(counts), _ptr(offsets),
        _ptr(sorted_token), _ptr(inv), _ptr(xq_perm), _ptr(xs_perm), _stream(stream)))


def moe_grouped_gemm_fp8_workspace(T, K_r, d, I):
    return int(_lib.load().moe_grouped_gemm_fp8_workspace(T, K_r, d, I))


def moe_grouped_gemm_fp8_launches(d, I):
    return int(_lib.load().moe_grouped_gemm_fp8_launches(d, I))


def moe_grouped_gemm_fp8(xq_perm, xs_perm, offsets, xq, xs, w_gate, w_up, w_down,
                         s_gate, s_up, s_down, y_perm, y_shared, workspace, stream=None):
    T, d = xq.shape
    P = xq_perm.shape[0]
    G, I, _ = w_gate.shape
    N_r = G - 1
    K_r = P // T if T else 0
    _want(xq_perm, torch.uint8, (P, d), "xq_perm")
    _want(xs_perm, torch.float32, (P, d // 128), "xs_perm")
    _want(offsets, torch.int32, (N_r + 1,), "offsets")
    _want(xq, torch.uint8, (T, d), "xq")
    _want(xs, torch.float32, (T, d // 128), "xs")
    _want(w_gate, torch.uint8, (G, I, d), "w_gate")
    _want(w_up, torch.uint8, (G, I, d), "w_up")
    _want(w_down, torch.uint8, (G, d, I), "w_down")
    _want(s_gate, torch.float32, (G, I // 128, d // 128), "s_gate")
    _want(s_up, torch.float32, (G, I // 128, d // 128), "s_up")
    _want(s_down, torch.float32, (G, d // 128, I // 128), "s_down")
    _want(y_perm, torch.bfloat16, (P, d), "y_perm")
    _want(y_shared, torch.bfloat16, (T, d), "y_shared")
    if T and P != T * K_r:
        raise ValueError("xq_perm rows must be T * K_r")
    check("moe_grouped_gemm_fp8", _lib.load().moe_grouped_gemm_fp8(
        _ptr(xq_perm), _ptr(xs_perm), _ptr(offsets), N_r, K_r, _ptr(xq), _ptr(xs), T,
        _ptr(w_gate), _ptr(w_up), _ptr(w_down), _ptr(s_gate), _ptr(s_up), _ptr(s_down),
        d, I, _ptr(y_perm), _ptr(y_shared), _ptr(workspace),
        workspace.numel() * workspace.element_size(), _stream(stream)))


def moe_grouped_gemm_fp8_gather(sorted_token, offsets, xq, xs, w_gate, w_up, w_down,
                                s_gate, s_up, s_down, y_perm, y_shared, workspace, stream=None):
    """moe_grouped_gemm_fp8 with the routed rows read from xq/xs at sorted_token."""
    T, d = xq.shape
    P = sorted_token.shape[0]
    G, I, _ = w_gate.shape
    N_r = G - 1
    K_r = P // T if T else 0
    _want(sorted_token, torch.int32, (P,), "sorted_token")
    _want(offsets, torch.int32, (N_r + 1,), "offsets")
    _want(xq, torch.uint8, (T, d), "xq")
    _want(xs, torch.float32, (T, d // 128), "xs")
    _want(w_gate, torch.uint8, (G, I, d), "w_gate")
    _want(w_up, torch.uint8, (G, I, d), "w_up")
    _want(w_down, torch.uint8, (G, d, I), "w_down")
    _want(s_gate, torch.float32, (G, I // 128, d // 128), "s_gate")
    _want(s_up, torch.float32, (G, I // 128, d // 128), "s_up")
    _want(s_down, torch.float32, (G, d // 128, I // 128), "s_down")
    _want(y_perm, torch.bfloat16, (P, d), "y_perm")
    _want(y_shared, torch.bfloat16, (T, d), "y_shared")
    if T and P != T * K_r:
        raise ValueError("sorted_token must hold T * K_r rows")
    check("moe_grouped_gemm_fp8_gather", _lib.load().moe_grouped_gemm_fp8_gather(
        _ptr(sorted_token), _ptr(offsets), N_r, K_r, _ptr(xq), _ptr(xs), T,
        _ptr(w_gate), _ptr(w_up), _ptr(w_down), _ptr(s_gate), _ptr(s_up), _ptr(s_down),
        d, I, _ptr(y_perm), _ptr(y_shared), _ptr(workspace),
        workspace.numel() * workspace.element_size(), _stream(stream)))


def moe_grouped_gemm_fp8_rows_workspace(P, T, d, I):
    return int(_lib.load().moe_grouped_gemm_fp8_rows_workspace(P, T, d, I))


def moe_grouped_gemm_fp8_rows(xq_perm, xs_perm, offsets, xq, xs, w_gate, w_up, w_down,
                              s_gate, s_up, s_down, y_perm, y_shared, workspace, stream=None):
    """The grouped GEMM on P = xq_perm.shape[0] routed rows in N_groups groups
    (weights stacked over N_groups + 1 slots, the shared expert last)."""
    T, d = xq.shape
    P = xq_perm.shape[0]
    G, I, _ = w_gate.shape
    N = G - 1
    _want(xq_perm, torch.uint8, (P, d), "xq_perm")
    _want(xs_perm, torch.float32, (P, d // 128), "xs_perm")
    _want(offsets, torch.int32, (N + 1,), "offsets")
    _want(xq, torch.uint8, (T, d), "xq")
    _want(xs, torch.float32, (T, d // 128), "xs")
    _want(w_gate, torch.uint8, (G, I, d), "w_gate")
    _want(w_up, torch.uint8, (G, I, d), "w_up")
    _want(w_down, torch.uint8, (G, d, I), "w_down")
    _want(s_gate, torch.float32, (G, I // 128, d // 128), "s_gate")
    _want(s_up, torch.float32, (G, I // 128, d // 128), "s_up")
    _want(s_down, torch.float32, (G, d // 128, I // 128), "s_down")
    _want(y_perm, torch.bfloat16, (P, d), "y_perm")
    _want(y_shared, torch.bfloat16, (T, d), "y_shared")
    check("moe_grouped_gemm_fp8_rows", _lib.load().moe_grouped_gemm_fp8_rows(
        _ptr(xq_perm), _ptr(xs_perm), _ptr(offsets), N, P, _ptr(xq), _ptr(xs), T,
        _ptr(w_gate), _ptr(w_up), _ptr(w_down), _ptr(s_gate), _ptr(s_up), _ptr(s_down),
        d, I, _ptr(y_perm), _ptr(y_shared), _ptr(workspace),
        workspace.numel() * workspace.element_size(), _stream(stream)))


def moe_group_of_rows(offsets, modulo, out, stream=None):
    n_groups = offsets.shape[0] - 1
    _want(offsets, torch.int32, (n_groups + 1,), "offsets")
    n_rows = out.shape[0]
    _want(out, torch.int32, (n_rows,), "out")
    check("moe_group_of_rows", _lib.load().moe_group_of_rows(
        _ptr(offsets), n_groups, modulo, n_rows, _ptr(out), _stream(stream)))


def moe_gather_rows(src, idx, dst, stream=None):
    """dst[i] = src[idx[i]] along the first dimension (rows of any dtype)."""
    n = idx.shape[0]
    _want(idx, torch.int32, (n,), "idx")
    if src.dtype != dst.dtype or src.shape[1:] != dst.shape[1:] or dst.shape[0] != n:
        raise ValueError("src and dst must share dtype and row shape; dst has len(idx) rows")
    for t, name in ((src, "src"), (dst, "dst")):
        if not t.is_cuda or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous CUDA tensor")
    row_bytes = dst[0].numel() * dst.element_size() if n else src[0].numel() * src.element_size()
    check("moe_gather_rows", _lib.load().moe_gather_rows(
        _ptr(src), src.shape[0], _ptr(idx), n, row_bytes, _ptr(dst), _stream(stream)))


def moe_grouped_scaled_gemm_fp8_workspace():
    return int(_lib.load().moe_grouped_scaled_gemm_fp8_workspace())


def moe_grouped_scaled_gemm_fp8(a, a_s, offsets, P, b, b_s, c, workspace, stream=None):
    """c = a b_g^T: a [P+T][K] (1x128 scales a_s), b [N_groups+1][N][K] (128x128
    scales b_s); rows of group g use slot g, the last T rows the last slot."""
    R, K = a.shape
    G, N, _ = b.shape
    T = R - P
    _want(a, torch.uint8, (R, K), "a")
    _want(a_s, torch.float32, (R, K // 128), "a_s")
    _want(offsets, torch.int32, (G,), "offsets")
    _want(b, torch.uint8, (G, N, K), "b")
    _want(b_s, torch.float32, (G, N // 128, K // 128), "b_s")
    _want(c, torch.float32, (R, N), "c")
    check("moe_grouped_scaled_gemm_fp8", _lib.load().moe_grouped_scaled_gemm_fp8(
        _ptr(a), _ptr(a_s), _ptr(offsets), G - 1, P, T, _ptr(b), _ptr(b_s), K, N, _ptr(c),
        _ptr(workspace), workspace.numel() * workspace.element_size(), _stream(stream)))


def moe_kgrouped_gemm_fp8_workspace():
    return int(_lib.load().moe_kgrouped_gemm_fp8_workspace())


def moe_kgrouped_gemm_fp8(a, a_s, b, b_s, kofs, c, workspace, stream=None):
    """c[g] = a[:, K_g] b[:, K_g]^T for K_g = kofs[g]..kofs[g+1]: a [M][K]
    E4M3 (1x128 scales a_s [M][K/128]), b [N][K] E4M3 (128x128 scales b_s
    [N/128][K/128]), kofs [G+1] int32, c [G][M][N] FP32."""
    M, K = a.shape
    N = b.shape[0]
    G = kofs.shape[0] - 1
    _want(a, torch.uint8, (M, K), "a")
    _want(a_s, torch.float32, (M, K // 128), "a_s")
    _want(b, torch.uint8, (N, K), "b")
    _want(b_s, torch.float32, (N // 128, K // 128), "b_s")
    _want(kofs, torch.int32, (G + 1,), "kofs")
    _want(c, torch.float32, (G, M, N), "c")
    check("moe_kgrouped_gemm_fp8", _lib.load().moe_kgrouped_gemm_fp8(
        _ptr(a), _ptr(a_s), _ptr(b), _ptr(b_s), _ptr(kofs), G, M, N, K, _ptr(c),
        _ptr(workspace), workspace.numel() * workspace.element_size(), _stream(stream)))


def moe_swiglu_backward_quant(g, u, dh, dgu, q, qs, stream=None):
    R, I = g.shape
    for t, n in ((g, "g"), (u, "u"), (dh, "dh")):
        _want(t, torch.float32, (R, I), n)
    _opt(dgu, torch.float32, (R, 2 * I), "dgu")
    _want(q, torch.uint8, (R, 2 * I), "q")
    _want(qs, torch.float32, (R, 2 * I // 128), "qs")
    check("moe_swiglu_backward_quant", _lib.load().moe_swiglu_backward_quant(
        _ptr(g), _ptr(u), _ptr(dh), R, I, _ptr(dgu), _ptr(q), _ptr(qs), _stream(stream)))


def _ld(x):
    if not x.is_cuda or x.dim() != 2 or x.stride(1) != 1:
        raise ValueError("x must be a CUDA matrix with unit column stride")
    return x.stride(0)


def moe_quant_1x128_t(x, src_off, dst_off, q, s, stream=None):
    """x [rows][cols] FP32 or BF16 (a column slice of a wider row-major tensor
    is allowed) -> its per-group transpose q [cols][Ktot] (flat, cols * Ktot
    bytes; group g in columns dst_off[g]..dst_off[g+1]) and s [cols][Ktot/128]
    (flat)."""
    if x.dtype not in (torch.float32, torch.bfloat16):
        raise ValueError("x must be FP32 or BF16")
    cols = x.shape[1]
    Ktot = q.numel() // cols
    n = src_off.shape[0] - 1
    _want(src_off, torch.int32, (n + 1,), "src_off")
    _want(dst_off, torch.int32, (n + 1,), "dst_off")
    _want(q, torch.uint8, (cols * Ktot,), "q")
    _want(s, torch.float32, (cols * Ktot // 128,), "s")
    check("moe_quant_1x128_t", _lib.load().moe_quant_1x128_t(
        _ptr(x), int(x.dtype == torch.bfloat16), _ld(x), cols, _ptr(src_off), _ptr(dst_off), n, Ktot,
        _ptr(q), _ptr(s), _stream(stream)))


def moe_quant_128x128_t(xq, xs, src_off, dst_off, q, s, stream=None):
    """xq [rows][cols] E4M3 with 1x128 scales xs -> its per-group transpose
    q [cols][Ktot] (flat) in 128x128 blocks, scales [cols/128][Ktot/128]
    (flat)."""
    rows, cols = xq.shape
    Ktot = q.numel() // cols
    n = src_off.shape[0] - 1
    _want(xq, torch.uint8, (rows, cols), "xq")
    _want(xs, torch.float32, (rows, cols // 128), "xs")
    _want(src_off, torch.int32, (n + 1,), "src_off")
    _want(dst_off, torch.int32, (n + 1,), "dst_off")
    _want(q, torch.uint8, (cols * Ktot,), "q")
    _want(s, torch.float32, ((cols // 128) * (Ktot // 128),), "s")
    check("moe_quant_128x128_t", _lib.load().moe_quant_128x128_t(
        _ptr(xq), _ptr(xs), cols, cols, _ptr(src_off), _ptr(dst_off), n, Ktot, _ptr(q), _ptr(s),
        _stream(stream)))


def moe_transpose(src, dst, dst_col=0, stream=None):
    """dst[b][j][dst_col + i] = src[b][i][j] (uint8 or float32, 3-D, contiguous)."""
    if src.dtype != dst.dtype or src.dtype not in (torch.uint8, torch.float32):
        raise ValueError("src and dst: both uint8 or both float32")
    B, rows, cols = src.shape
    if dst.shape[0] != B or dst.shape[1] != cols or dst.shape[2] < dst_col + rows:
        raise ValueError("dst must be [batch][cols][>= dst_col + rows]")
    for t, n in ((src, "src"), (dst, "dst")):
        if not t.is_cuda or not t.is_contiguous():
            raise ValueError(f"{n} must be a contiguous CUDA tensor")
    check("moe_transpose", _lib.load().moe_transpose(
        _ptr(src), src.element_size(), B, rows, cols, _ptr(dst), dst.shape[2], dst_col, _stream(stream)))


def moe_combine(u, y_perm, y_shared, inv, gates, out, stream=None):
    """h' from bf16 expert rows (moe_combine), or FP32 rows (moe_combine_fp32)."""
    T, d = u.shape
    K_r = inv.shape[1]
    dt = y_perm.dtype
    if dt not in (torch.bfloat16, torch.float32):
        raise ValueError("y_perm must be bf16 or FP32")
    _want(u, torch.bfloat16, (T, d), "u")
    _want(y_perm, dt, (T * K_r, d), "y_perm")
    _want(y_shared, dt, (T, d), "y_shared")
    _want(inv, torch.int32, (T, K_r), "inv")
    _want(gates, torch.float32, (T, K_r), "gates")
    _want(out, torch.bfloat16, (T, d), "out")
    fn = _lib.load().moe_combine if dt == torch.bfloat16 else _lib.load().moe_combine_fp32
    check("moe_combine", fn(
        _ptr(u), _ptr(y_perm), _ptr(y_shared), _ptr(inv), _ptr(gates), T, K_r, d, _ptr(out),
        _stream(stream)))


def moe_bias_update(b, counts, T, K_r, gamma=0.001, max_over_mean=None, stream=None):
    N_r = b.shape[0]
    _want(b, torch.float32, (N_r,), "b")
    _want(counts, torch.int32, (N_r,), "counts")
    _opt(max_over_mean, torch.float32, (1,), "max_over_mean")
    check("moe_bias_update", _lib.load().moe_bias_update(
        _ptr(b), _ptr(counts), N_r, T, K_r, ctypes.c_float(gamma), _ptr(max_over_mean),
        _stream(stream)))


def moe_debug_wait_timeout(timeout_us, stream=None):
    check("moe_debug_wait_timeout", _lib.load().moe_debug_wait_timeout(timeout_us, _stream(stream)))


def moe_get_error() -> int:
    st = ctypes.c_int(0)
    check("moe_get_error", _lib.load().moe_get_error(ctypes.byref(st)))
    return st.value
