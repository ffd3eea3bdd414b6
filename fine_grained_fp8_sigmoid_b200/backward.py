"""The backward of the layer's expert FFNs in the FP8 scheme, on the library's
kernels ("DeepSeek-V3 Teknik Raporu", Temel fikirler, FP8 bullet: the model
trains in FP8, E4M3 on all tensors, activations in 1x128 tiles, weights in
128x128 blocks; the backward's details are not on the pages, the readings are
stated in include/moe_fp8.h).

Given dY for the rows of the forward's grouped layout (the routed rows in the
permuted order, then the shared expert's T rows), one call computes

  dgrad  G, U = X W_gate^T, X W_up^T        (recomputed; grouped FP8 GEMM)
         dH = dY W_down                     (dY in 1x128 tiles, W_down^T)
         dG = dH U silu'(G), dU = dH silu(G), quantised [dG | dU]
         dX = dG W_gate + dU W_up           (one GEMM with K = 2I)
         dx_t = dX_shared[t] + sum_k dX[inv[t][k]]   (moe_combine, gates 1)
  wgrad  per expert, over its tokens padded to a multiple of 128:
         dW_down = dY^T H,  dW_gate = dG^T X,  dW_up = dU^T X
         (the gradient in 1x128 tiles along the tokens, the forward's X and H
         requantised in 128x128 blocks); one K-grouped GEMM launch per weight
         covers every expert

It reads the forward's state from the MoELayerFP8 (xq, xs, the permutation,
the intermediate H in the GEMM workspace), so it runs after that forward and
before the next one.
"""
from __future__ import annotations

import numpy as np
import torch

from . import binding as B


class ExpertFFNBackward:
    def __init__(self, layer):
        self.layer = L = layer
        G, I, d = L.N_r + 1, L.I, L.d
        if d % 256 or I % 256:
            raise ValueError("the backward's GEMMs need d and I multiples of 256")
        dev = dict(device=L.device)
        # dgrad's weights, transposed once: [W_gate^T | W_up^T] [G][d][2I] and W_down^T [G][I][d]
        self.wgu_t = torch.empty(G, d, 2 * I, dtype=torch.uint8, **dev)
        self.sgu_t = torch.empty(G, d // 128, 2 * I // 128, dtype=torch.float32, **dev)
        self.wd_t = torch.empty(G, I, d, dtype=torch.uint8, **dev)
        self.sd_t = torch.empty(G, I // 128, d // 128, dtype=torch.float32, **dev)
        self.ws = torch.empty(B.moe_grouped_scaled_gemm_fp8_workspace(), dtype=torch.uint8, **dev)
        self.kws = torch.empty(B.moe_kgrouped_gemm_fp8_workspace(), dtype=torch.uint8, **dev)
        self.refresh_weights()

    def refresh_weights(self):
        """Re-derive the transposed weights (after the layer's weights change)."""
        L, I = self.layer, self.layer.I
        B.moe_transpose(L.w_gate, self.wgu_t, 0)
        B.moe_transpose(L.w_up, self.wgu_t, I)
        B.moe_transpose(L.s_gate, self.sgu_t, 0)
        B.moe_transpose(L.s_up, self.sgu_t, I // 128)
        B.moe_transpose(L.w_down, self.wd_t, 0)
        B.moe_transpose(L.s_down, self.sd_t, 0)

    def _gemm(self, a, a_s, offsets, P, b, b_s):
        c = torch.empty(a.shape[0], b.shape[1], dtype=torch.float32, device=a.device)
        B.moe_grouped_scaled_gemm_fp8(a, a_s, offsets, P, b, b_s, c, self.ws)
        return c

    def backward(self, dy, wgrad=True):
        """dy: [T*K_r + T][d] bf16, the gradient of the expert outputs (routed
        rows in the permuted order, then the shared rows). Returns dict(dx
        [T][d] bf16, dX [T*K_r + T][d] FP32 per row, and with wgrad
        dw_gate, dw_up [N_r+1][I][d], dw_down [N_r+1][d][I] FP32)."""
        L = self.layer
        T, d, I, N = L.T, L.d, L.I, L.N_r
        P = T * L.K_r
        R = P + T
        dev = L.device
        f32, u8 = torch.float32, torch.uint8
        if tuple(dy.shape) != (R, d) or dy.dtype != torch.bfloat16:
            raise ValueError(f"dy must be bf16 [{R}][{d}]")
        # the forward's FP8 rows in the grouped layout (routed, then shared)
        idx = torch.cat([L.sorted_token, torch.arange(T, dtype=torch.int32, device=dev)])
        xq, xs = torch.empty(R, d, dtype=u8, device=dev), torch.empty(R, d // 128, dtype=f32, device=dev)
        B.moe_gather_rows(L.xq, idx, xq)
        B.moe_gather_rows(L.xs, idx, xs)
        g = self._gemm(xq, xs, L.offsets, P, L.w_gate, L.s_gate)
        u = self._gemm(xq, xs, L.offsets, P, L.w_up, L.s_up)
        dyq, dys = torch.empty(R, d, dtype=u8, device=dev), torch.empty(R, d // 128, dtype=f32, device=dev)
        B.moe_quant_1x128(dy, dyq, dys)
        dh = self._gemm(dyq, dys, L.offsets, P, self.wd_t, self.sd_t)
        dgu = torch.empty(R, 2 * I, dtype=f32, device=dev)
        gq, gs = torch.empty(R, 2 * I, dtype=u8, device=dev), torch.empty(R, 2 * I // 128, dtype=f32, device=dev)
        B.moe_swiglu_backward_quant(g, u, dh, dgu, gq, gs)
        dX = self._gemm(gq, gs, L.offsets, P, self.wgu_t, self.sgu_t)
        dx = torch.empty(T, d, dtype=torch.bfloat16, device=dev)
        B.moe_combine(torch.zeros(T, d, dtype=torch.bfloat16, device=dev), dX[:P], dX[P:], L.inv,
                      torch.ones(T, L.K_r, dtype=f32, device=dev), dx)
        out = dict(dx=dx, dX=dX, g=g, u=u, dh=dh, dgu=dgu)
        if wgrad:
            out.update(self._wgrad(dy, dgu, xq, xs))
        return out

    def _wgrad(self, dy, dgu, xq, xs):
        L = self.layer
        T, d, I, N = L.T, L.d, L.I, L.N_r
        R = T * L.K_r + T
        dev = L.device
        f32, u8 = torch.float32, torch.uint8
        # groups: the routed experts, then the shared one; each group's tokens
        # padded to 128 and laid side by side along K (the transposes are
        # [cols][Kt], group g in columns dst[g]..dst[g+1])
        src = np.concatenate([L.offsets.cpu().numpy().astype(np.int64), [R]])
        rows = np.diff(src)
        dst = np.concatenate([[0], np.cumsum((rows + 127) // 128 * 128)])
        Kt = int(dst[-1])
        src_d = torch.from_numpy(src.astype(np.int32)).to(dev)
        dst_d = torch.from_numpy(dst.astype(np.int32)).to(dev)
        G = N + 1
        dw_down = torch.empty(G, d, I, dtype=f32, device=dev)
        dw_gate = torch.empty(G, I, d, dtype=f32, device=dev)
        dw_up = torch.empty(G, I, d, dtype=f32, device=dev)
        codes = lambda cols: torch.empty(cols * Kt, dtype=u8, device=dev)
        dyt, dyts = codes(d), torch.empty(d * Kt // 128, dtype=f32, device=dev)
        B.moe_quant_1x128_t(dy, src_d, dst_d, dyt, dyts)
        hq, hs = L.intermediate()
        ht, hts = codes(I), torch.empty((I // 128) * (Kt // 128), dtype=f32, device=dev)
        B.moe_quant_128x128_t(hq, hs, src_d, dst_d, ht, hts)
        dgt, dgts = codes(I), torch.empty(I * Kt // 128, dtype=f32, device=dev)
        dut, duts = codes(I), torch.empty(I * Kt // 128, dtype=f32, device=dev)
        B.moe_quant_1x128_t(dgu[:, :I], src_d, dst_d, dgt, dgts)
        B.moe_quant_1x128_t(dgu[:, I:], src_d, dst_d, dut, duts)
        xt, xts = codes(d), torch.empty((d // 128) * (Kt // 128), dtype=f32, device=dev)
        B.moe_quant_128x128_t(xq, xs, src_d, dst_d, xt, xts)
        act = lambda q, s_, cols: (q.view(cols, Kt), s_.view(cols, Kt // 128))
        blk = lambda q, s_, cols: (q.view(cols, Kt), s_.view(cols // 128, Kt // 128))
        # one launch per weight: every expert over its own token range
        B.moe_kgrouped_gemm_fp8(*act(dyt, dyts, d), *blk(ht, hts, I), dst_d, dw_down, self.kws)
        B.moe_kgrouped_gemm_fp8(*act(dgt, dgts, I), *blk(xt, xts, d), dst_d, dw_gate, self.kws)
        B.moe_kgrouped_gemm_fp8(*act(dut, duts, I), *blk(xt, xts, d), dst_d, dw_up, self.kws)
        return dict(dw_gate=dw_gate, dw_up=dw_up, dw_down=dw_down)
