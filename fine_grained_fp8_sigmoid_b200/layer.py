"""MoELayerFP8: owns the device buffers of one DeepSeekMoE FP8 layer and runs
its forward pass through the C ABI, step by step:

  route -> quant_1x128 -> permute -> grouped FP8 GEMM (routed + shared)
        -> combine -> bias update

("DeepSeek-V3 Teknik Raporu", Yöntem 2 for the layer equations; Temel
fikirler, FP8 bullet for the quantisation scheme). PyTorch only allocates
memory and provides the stream; every step runs in the library's kernels.
"""
from __future__ import annotations

import torch

from . import binding as B


class MoELayerFP8:
    """gather=True fuses the permutation's row movement into the grouped
    GEMM's loads (moe_permute without rows, then moe_grouped_gemm_fp8_gather);
    gather=False materialises xq_perm/xs_perm in moe_permute and calls
    moe_grouped_gemm_fp8. Both give the same outputs bit for bit. The default
    (None) fuses for decode-like batches, where the average routed group has
    at most 64 rows and a tile gathers only the rows it holds, and
    materialises otherwise: with full 128-row tiles the 32 four-row TMA
    gathers per K block pace the GEMM's producer (measured at prefill: GEMM
    7.8 ms fused against 5.4 ms materialised; decode: equal).

    fuse_quant=True quantises the activations (1x128 tiles) inside the router
    from the u tiles it already streams (moe_route_quant); False (the
    default) runs moe_route and moe_quant_1x128 apart. Both give the same
    codes and scales bit for bit. Measured at prefill: 169 us fused against
    65 + 53 us apart; the quantisation's 7168 IEEE divisions per token then
    run on the router's eight epilogue warps per SM instead of a full grid."""

    def __init__(self, T: int, d: int, N_r: int, K_r: int, I: int, device="cuda", gather=None,
                 fuse_quant=False):
        self.T, self.d, self.N_r, self.K_r, self.I = T, d, N_r, K_r, I
        self.fuse_quant = bool(fuse_quant)
        self.gather = (T * K_r <= 64 * N_r) if gather is None else bool(gather)
        self.device = torch.device(device)
        G, P = N_r + 1, T * K_r
        dev = dict(device=self.device)
        u8, f32, i32, bf = torch.uint8, torch.float32, torch.int32, torch.bfloat16
        # weights: slot N_r is the shared expert
        self.w_gate = torch.empty(G, I, d, dtype=u8, **dev)
        self.w_up = torch.empty(G, I, d, dtype=u8, **dev)
        self.w_down = torch.empty(G, d, I, dtype=u8, **dev)
        self.s_gate = torch.empty(G, I // 128, d // 128, dtype=f32, **dev)
        self.s_up = torch.empty(G, I // 128, d // 128, dtype=f32, **dev)
        self.s_down = torch.empty(G, d // 128, I // 128, dtype=f32, **dev)
        # activations
        self.topk_idx = torch.empty(T, K_r, dtype=i32, **dev)
        self.gates = torch.empty(T, K_r, dtype=f32, **dev)
        self.xq = torch.empty(T, d, dtype=u8, **dev)
        self.xs = torch.empty(T, d // 128, dtype=f32, **dev)
        self.counts = torch.empty(N_r, dtype=i32, **dev)
        self.offsets = torch.empty(N_r + 1, dtype=i32, **dev)
        self.sorted_token = torch.empty(P, dtype=i32, **dev)
        self.inv = torch.empty(T, K_r, dtype=i32, **dev)
        self.xq_perm = None if gather else torch.empty(P, d, dtype=u8, **dev)
        self.xs_perm = None if gather else torch.empty(P, d // 128, dtype=f32, **dev)
        self.y_perm = torch.empty(P, d, dtype=bf, **dev)
        self.y_shared = torch.empty(T, d, dtype=bf, **dev)
        self.out = torch.empty(T, d, dtype=bf, **dev)
        self.max_over_mean = torch.zeros(1, dtype=f32, **dev)
        self.ws_perm = torch.empty(max(B.moe_permute_workspace(T, N_r), 16), dtype=u8, **dev)
        self.ws_gemm = torch.empty(max(B.moe_grouped_gemm_fp8_workspace(T, K_r, d, I), 256),
                                   dtype=u8, **dev)

    def intermediate(self):
        """Views of the last step's expert intermediate H in the GEMM
        workspace (the layout include/moe_fp8.h gives for
        moe_grouped_gemm_fp8): E4M3 codes [T*K_r + T][I] (routed rows in
        permuted order, then the T shared rows) and their FP32 1x128 scales."""
        rows, I = self.T * self.K_r + self.T, self.I
        off = (rows * I + 255) // 256 * 256
        codes = self.ws_gemm[:rows * I].view(rows, I)
        scales = self.ws_gemm[off:off + rows * (I // 128) * 4].view(torch.float32).view(rows, I // 128)
        return codes, scales

    # ---------------------------------------------------------------- weights
    def load_expert(self, slot: int, w_gate: torch.Tensor, w_up: torch.Tensor,
                    w_down: torch.Tensor, stream=None) -> None:
        """Quantises one expert's FP32 weights (on the device) into slot `slot`."""
        B.moe_quant_128x128(w_gate, self.w_gate[slot], self.s_gate[slot], stream)
        B.moe_quant_128x128(w_up, self.w_up[slot], self.s_up[slot], stream)
        B.moe_quant_128x128(w_down, self.w_down[slot], self.s_down[slot], stream)

    # ---------------------------------------------------------------- steps
    def route(self, u, e, b, scores_out=None, stream=None):
        """Routing; with fuse_quant also the activation quantisation."""
        if self.fuse_quant:
            B.moe_route_quant(u, e, b, self.K_r, self.topk_idx, self.gates, self.xq, self.xs,
                              scores_out=scores_out, stream=stream)
        else:
            B.moe_route(u, e, b, self.K_r, self.topk_idx, self.gates, scores_out=scores_out,
                        stream=stream)

    def quant(self, u, stream=None):
        """The activation quantisation, unless the router already did it."""
        if not self.fuse_quant:
            B.moe_quant_1x128(u, self.xq, self.xs, stream)

    def permute(self, stream=None):
        if self.gather:   # indices only: the GEMM reads the rows from xq/xs
            B.moe_permute(self.topk_idx, self.N_r, self.counts, self.offsets, self.sorted_token,
                          self.inv, self.ws_perm, stream=stream)
        else:
            B.moe_permute(self.topk_idx, self.N_r, self.counts, self.offsets, self.sorted_token,
                          self.inv, self.ws_perm, self.xq, self.xs, self.xq_perm, self.xs_perm,
                          stream=stream)

    def experts(self, stream=None):
        if self.gather:
            B.moe_grouped_gemm_fp8_gather(self.sorted_token, self.offsets, self.xq, self.xs,
                                          self.w_gate, self.w_up, self.w_down, self.s_gate,
                                          self.s_up, self.s_down, self.y_perm, self.y_shared,
                                          self.ws_gemm, stream)
        else:
            B.moe_grouped_gemm_fp8(self.xq_perm, self.xs_perm, self.offsets, self.xq, self.xs,
                                   self.w_gate, self.w_up, self.w_down, self.s_gate, self.s_up,
                                   self.s_down, self.y_perm, self.y_shared, self.ws_gemm, stream)

    def launches_per_step(self, update_bias=True):
        """Kernel launches of one forward: router (with the quantisation
        fused, or apart), permute (count, scan, scatter, and gather unless
        fused), the GEMM's, combine, bias."""
        return ((1 if self.fuse_quant else 2) + (3 if self.gather else 4)
                + B.moe_grouped_gemm_fp8_launches(self.d, self.I) + 1 + int(update_bias))

    def combine(self, u, stream=None):
        B.moe_combine(u, self.y_perm, self.y_shared, self.inv, self.gates, self.out, stream)

    def bias_update(self, b, gamma=0.001, stream=None):
        B.moe_bias_update(b, self.counts, self.T, self.K_r, gamma, self.max_over_mean, stream)

    def forward(self, u, e, b, update_bias=True, stream=None):
        """One pass of the layer on device tensors; returns self.out."""
        self.route(u, e, b, stream=stream)
        self.quant(u, stream)
        self.permute(stream)
        self.experts(stream)
        self.combine(u, stream)
        if update_bias:
            self.bias_update(b, stream=stream)
        return self.out

    def forward_host(self, u_host, e, b, out_host, u_dev, update_bias=True, stream=None):
        """End to end from pinned host memory: copy u in, run, copy h' out."""
        u_dev.copy_(u_host, non_blocking=True)
        self.forward(u_dev, e, b, update_bias, stream)
        out_host.copy_(self.out, non_blocking=True)
        return out_host

    def forward_host_pipelined(self, u_hosts, e, b, out_hosts, u_devs, update_bias=True):
        """End to end over a sequence of batches in pinned host memory, with the
        copies overlapped with the kernels: batch i+1's input goes to the
        device, and batch i-1's h' to the host, on a copy stream while batch i
        runs on the current stream. u_devs holds two device input buffers. On
        return everything is enqueued; out_hosts[i] holds batch i's h' once the
        current stream is synchronised."""
        comp = torch.cuda.current_stream(self.device)
        if getattr(self, "_copy_stream", None) is None:
            self._copy_stream = torch.cuda.Stream(self.device)
        copy = self._copy_stream
        n = len(u_hosts)
        h2d_done = [torch.cuda.Event(), torch.cuda.Event()]   # input buffer k filled
        read_done = [torch.cuda.Event(), torch.cuda.Event()]  # input buffer k no longer read
        out_ready, d2h_done = torch.cuda.Event(), torch.cuda.Event()
        copy.wait_stream(comp)            # inputs and buffers as the caller left them
        with torch.cuda.stream(copy):
            u_devs[0].copy_(u_hosts[0], non_blocking=True)
            h2d_done[0].record(copy)
        for i in range(n):
            k = i % 2
            if i + 1 < n:
                with torch.cuda.stream(copy):
                    if i >= 1:            # batch i-1 used the buffer batch i+1 fills
                        copy.wait_event(read_done[(i + 1) % 2])
                    u_devs[(i + 1) % 2].copy_(u_hosts[i + 1], non_blocking=True)
                    h2d_done[(i + 1) % 2].record(copy)
            comp.wait_event(h2d_done[k])
            self.route(u_devs[k], e, b)
            self.quant(u_devs[k])
            self.permute()
            self.experts()
            if i >= 1:                    # batch i-1's h' has left self.out
                comp.wait_event(d2h_done)
            self.combine(u_devs[k])
            read_done[k].record(comp)
            out_ready.record(comp)
            if update_bias:
                self.bias_update(b)
            with torch.cuda.stream(copy):
                copy.wait_event(out_ready)
                out_hosts[i].copy_(self.out, non_blocking=True)
                d2h_done.record(copy)
        comp.wait_event(d2h_done)
        for t in u_devs:
            t.record_stream(copy)
        return out_hosts
