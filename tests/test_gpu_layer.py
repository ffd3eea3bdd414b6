"""End-to-end parity of the whole layer (MoELayerFP8 over the C ABI) with
the CPU oracle on the five workloads, and on batches of 1 and 129 tokens.

tiny, mid and decode are compared on every token. prefill and skew run at
full size in the same launch configuration as the benchmark; the oracle
routes all tokens (selection, counts, bias update) and computes the expert
outputs for 256 tokens: the first, the last, the 16 with the largest
|u| (the outlier-heavy ones) and a seeded draw of the rest. Weights are drawn
on the device by the seeded generator; the oracle receives the same FP32
weights copied to the host and quantises them itself (its codes and scales
must equal the GPU's).
"""
import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np
import pytest
import torch

import workloads
from oracle import moe as O
from tests.parity import accumulation_bound, assert_bf16_rounding, assert_close, down_bound, f64, near_tie_rows
from tests.test_gpu_kernels import _check_routing

pytestmark = pytest.mark.gpu

SAMPLE = 256
N_LARGEST = 16

# The oracle's quantised weights of the last seed used, by slot: decode and
# the T = 1 / T = 129 batches of the same layer share them.
_QCACHE = {"key": None, "w": {}}


def _threads():
    return max(2, min(32, os.cpu_count() or 8))


def _build(cfg, weights_on="cuda", gather=None, fuse_quant=False):
    from fine_grained_fp8_sigmoid_b200 import MoELayerFP8
    layer = MoELayerFP8(cfg.T, cfg.d, cfg.N_r, cfg.K_r, cfg.I, gather=gather, fuse_quant=fuse_quant)
    for slot in range(cfg.N_r + 1):
        w = workloads.expert_weights(cfg, slot, device=weights_on)
        layer.load_expert(slot, *[x.cuda() for x in w])
    return layer


def _oracle_weights(cfg, slots, weights_on, ex):
    """The oracle's own quantisation of the experts in `slots` (from the same
    FP32 weights the layer received), a chunk of slots at a time."""
    key = (cfg.seed, cfg.d, cfg.I, cfg.N_r, weights_on)
    if _QCACHE["key"] != key:
        _QCACHE["key"], _QCACHE["w"] = key, {}
    cache = _QCACHE["w"]
    todo = [s_ for s_ in slots if s_ not in cache]
    quant = lambda h: O.quantise_expert(*[a.astype(np.float64) for a in h])
    step = _threads()
    for i in range(0, len(todo), step):
        chunk = todo[i:i + step]
        host = [[x.cpu().numpy() for x in workloads.expert_weights(cfg, s_, device=weights_on)]
                for s_ in chunk]
        cache.update(zip(chunk, ex.map(quant, host)))
        del host
    return {s_: cache[s_] for s_ in slots}


def _sample(cfg, u, n=SAMPLE):
    """Token sample: all tokens if there are at most n; else the first, the
    last, the N_LARGEST tokens with the largest max |u|, and a seeded draw."""
    T = cfg.T
    if T <= n:
        return np.arange(T)
    big = np.argsort(-np.abs(u).max(axis=1), kind="stable")[:N_LARGEST]
    fixed = np.unique(np.concatenate([[0, T - 1], big]))
    rest = np.setdiff1d(np.arange(T), fixed)
    rng = np.random.default_rng(cfg.seed + 17)
    extra = rng.choice(rest, size=n - len(fixed), replace=False)
    return np.sort(np.concatenate([fixed, extra]))


def _run(cfg, weights_on, all_tokens=False):
    dev_inputs = cfg.T * cfg.d > 8_000_000
    gen_dev = "cuda" if dev_inputs else "cpu"
    u = workloads.activations(cfg, device=gen_dev)
    e = workloads.centroids(cfg, device=gen_dev)
    b = workloads.bias(cfg, device=gen_dev)
    layer = _build(cfg, weights_on)
    ud, ed, bd = u.cuda(), e.cuda(), b.cuda().clone()
    out = layer.forward(ud, ed, bd, update_bias=True)
    torch.cuda.synchronize()
    from fine_grained_fp8_sigmoid_b200 import binding as B
    assert B.moe_get_error() == 0

    un, en, bn = u.cpu().double().numpy(), e.cpu().double().numpy(), b.cpu().double().numpy()
    sample = np.arange(cfg.T) if all_tokens else _sample(cfg, un)
    gpu_idx = layer.topk_idx.cpu().numpy().astype(np.int64)
    s64 = O.router_scores(un, en)
    diff = _check_routing(gpu_idx, s64, bn, cfg.K_r)
    assert len(diff) <= max(2, cfg.T // 200), len(diff)

    # permutation and bias update given the GPU's selection: bit-exact
    rc, ro, rst, rinv = O.permute(gpu_idx, cfg.N_r)
    assert np.array_equal(layer.counts.cpu().numpy(), rc)
    assert np.array_equal(layer.offsets.cpu().numpy(), ro)
    assert np.array_equal(layer.sorted_token.cpu().numpy(), rst)
    assert np.array_equal(layer.inv.cpu().numpy(), rinv)
    rb, ratio = O.bias_update(bn, rc, cfg.T, cfg.K_r)
    assert np.array_equal(bd.cpu().double().numpy(), rb)

    # expert outputs and h' on the sample, under the GPU's selection; the
    # oracle quantises the same FP32 weights itself (threads: numpy releases
    # the GIL), and its codes and scales must equal the GPU's
    slots = sorted(set(gpu_idx[sample].reshape(-1).tolist()) | {cfg.N_r})
    with ThreadPoolExecutor(max_workers=_threads()) as ex:
        quant = _oracle_weights(cfg, slots, weights_on, ex)
        for s_, q in quant.items():
            for key, t in [("gate_q", layer.w_gate), ("up_q", layer.w_up), ("down_q", layer.w_down)]:
                assert np.array_equal(t[s_].cpu().numpy(), q[key]), (s_, key)
            for key, t in [("gate_s", layer.s_gate), ("up_s", layer.s_up), ("down_s", layer.s_down)]:
                assert np.array_equal(t[s_].cpu().double().numpy(), q[key]), (s_, key)
        ref = O.moe_forward(un, en, bn, cfg.K_r, quant.__getitem__, tokens=sample, select=gpu_idx,
                            map_fn=ex.map)
    assert np.array_equal(layer.xq[torch.as_tensor(sample).cuda()].cpu().numpy(), ref["xq"])

    # the intermediate H of the sampled rows under the near-tie rule; rows
    # with an accepted near-tie code are re-evaluated on the kernel's codes
    P, S, K = cfg.T * cfg.K_r, len(sample), cfg.K_r
    inv = layer.inv.cpu().numpy()
    hq_all, hs_all = layer.intermediate()
    rows_r = inv[sample].reshape(-1)                      # routed rows (j, k) in H
    rows_s = P + sample                                   # shared rows in H
    take = lambda t, r: t[torch.as_tensor(r).cuda()].cpu().numpy()
    hq_g = np.concatenate([take(hq_all, rows_r), take(hq_all, rows_s)])
    hs_g = np.concatenate([take(hs_all, rows_r), take(hs_all, rows_s)]).astype(np.float64)
    rp, sp = ref["routed_parts"], ref["shared_parts"]
    I = cfg.I
    flat = lambda key, w: np.concatenate([rp[key].reshape(S * K, w), sp[key]])
    a32, hq_o, hs_o = flat("a32", I), flat("hq", I), flat("hs", I // 128)
    G, U = flat("G", I), flat("U", I)
    slot_of = np.concatenate([gpu_idx[sample].reshape(-1), np.full(S, cfg.N_r)])
    tok_of = np.concatenate([np.repeat(np.arange(S), K), np.arange(S)])   # row -> sample index
    da = np.zeros_like(a32)
    for s_ in np.unique(slot_of):
        rr = np.nonzero(slot_of == s_)[0]
        da[rr] = accumulation_bound(ref["xq"][tok_of[rr]], ref["xs"][tok_of[rr]], quant[int(s_)], G[rr], U[rr])
    flip, dist = near_tie_rows(hq_g, hs_g, a32, da, hq_o, hs_o, f"{cfg.name} intermediate")
    y_r = ref["y_routed"].reshape(S * K, cfg.d).copy()
    y_s = ref["y_shared"].copy()
    for s_ in np.unique(slot_of[flip]):
        rr = flip[slot_of[flip] == s_]
        y = O.expert_down(hq_g[rr], hs_g[rr], quant[int(s_)])
        routed = rr < S * K
        y_r[rr[routed]] = y[routed]
        y_s[rr[~routed] - S * K] = y[~routed]
    print(f"[parity] {cfg.name} T={cfg.T}: {flip.size} of {hq_g.shape[0]} intermediate rows hold a "
          f"near-tie code (max distance to the boundary {dist:.3g} of the bound)")

    # bf16 expert outputs: each the rounding of the kernel's FP32 sum, which
    # lies within the accumulation bound of the oracle's value (near a bf16
    # midpoint either neighbour is valid); h' is then checked against the
    # oracle's combine of those outputs
    yb_s = f64(layer.y_shared)[sample]
    yp = f64(layer.y_perm)
    yb_r = np.concatenate([yp[inv[t]] for t in sample])
    assert_close(yb_s, y_s, "shared expert")
    for j, t in enumerate(sample):
        assert_close(yb_r[j * K:(j + 1) * K], y_r[j * K:(j + 1) * K], f"routed rows of token {t}")
    yb = np.concatenate([yb_r, yb_s])
    y64 = np.concatenate([y_r, y_s])
    n_flip = 0
    for s_ in np.unique(slot_of):
        rr = np.nonzero(slot_of == s_)[0]
        n_flip += assert_bf16_rounding(yb[rr], y64[rr], down_bound(hq_g[rr], hs_g[rr], quant[int(s_)]),
                                       f"{cfg.name} expert {int(s_)} outputs")
    print(f"[parity] {cfg.name} T={cfg.T}: {n_flip} of {yb.size} bf16 expert outputs on the other side "
          f"of a rounding midpoint (within the accumulation bound)")
    out_ref = O.combine(un[sample], yb_r, yb_s, np.arange(S * K).reshape(S, K), ref["gates"][sample])
    assert_close(f64(out)[sample], out_ref, "h'")
    return layer


def test_layer_tiny_all_tokens(lib):
    cfg = workloads.CONFIGS["tiny"]
    _run(cfg, weights_on="cpu", all_tokens=True)


def test_layer_tiny_ragged_tokens(lib):
    cfg = workloads.CONFIGS["tiny"].with_tokens(37)
    _run(cfg, weights_on="cpu", all_tokens=True)


def test_layer_mid_all_tokens(lib):
    cfg = workloads.CONFIGS["mid"]
    _run(cfg, weights_on="cuda", all_tokens=True)


@pytest.mark.parametrize("T", [1, 129])
def test_layer_mid_small_batches(lib, T):
    # T = 1: one row per group and a one-row shared expert; T = 129: a
    # ragged second row tile of the shared expert
    _run(workloads.CONFIGS["mid"].with_tokens(T), weights_on="cuda", all_tokens=True)


# decode and its 1- and 129-token batches run back to back (same weights)
@pytest.mark.parametrize("name,T", [("decode", None), ("decode", 1), ("decode", 129),
                                    ("prefill", None), ("skew", None)])
def test_layer_full_size(lib, name, T):
    cfg = workloads.CONFIGS[name]
    if T is not None:
        cfg = cfg.with_tokens(T)
    _run(cfg, weights_on="cuda")


@pytest.mark.parametrize("name", ["tiny", "mid"])
def test_layer_gather_fused_equals_materialised(lib, name):
    """The layer with the row gather fused into the GEMM and with xq_perm
    materialised by moe_permute give the same h', bit for bit."""
    cfg = workloads.CONFIGS[name]
    u = workloads.activations(cfg, device="cuda")
    e = workloads.centroids(cfg, device="cuda")
    b = workloads.bias(cfg, device="cuda")
    outs = []
    for gather in (True, False):
        layer = _build(cfg, "cuda", gather=gather)
        bb = b.clone()
        outs.append((layer.forward(u, e, bb).clone(), layer.y_perm.clone(), bb))
        torch.cuda.synchronize()
    for a_, b_ in zip(*outs):
        assert torch.equal(a_, b_)


@pytest.mark.parametrize("name", ["tiny", "mid"])
def test_layer_fused_quantisation_equals_separate(lib, name):
    """The layer with the activation quantisation fused into the router and
    with moe_quant_1x128 apart give the same xq, xs and h', bit for bit."""
    cfg = workloads.CONFIGS[name]
    u = workloads.activations(cfg, device="cuda")
    e = workloads.centroids(cfg, device="cuda")
    b = workloads.bias(cfg, device="cuda")
    outs = []
    for fuse in (True, False):
        layer = _build(cfg, "cuda", fuse_quant=fuse)
        bb = b.clone()
        out = layer.forward(u, e, bb).clone()
        torch.cuda.synchronize()
        outs.append((out, layer.xq.clone(), layer.xs.clone(), bb))
        assert layer.launches_per_step() == (9 if fuse else 10) - (1 if layer.gather else 0)
    for a_, b_ in zip(*outs):
        assert torch.equal(a_, b_)


def test_layer_pipelined_host_path_matches_plain():
    """forward_host_pipelined (copies on a second stream, two input buffers)
    gives, batch for batch and bit for bit, what forward_host gives, bias
    updates included."""
    cfg = workloads.CONFIGS["tiny"]
    layer = _build(cfg, "cuda")
    u = workloads.activations(cfg, device="cuda")
    e = workloads.centroids(cfg, device="cuda")
    b = workloads.bias(cfg, device="cuda")
    u_hosts = [u.cpu().pin_memory(), torch.roll(u, 1, 0).cpu().pin_memory(), (u * 0.5).cpu().pin_memory()]
    outs = [torch.empty(cfg.T, cfg.d, dtype=torch.bfloat16).pin_memory() for _ in u_hosts]
    refs = [torch.empty(cfg.T, cfg.d, dtype=torch.bfloat16).pin_memory() for _ in u_hosts]
    b_pipe, b_plain = b.clone(), b.clone()
    layer.forward_host_pipelined(u_hosts, e, b_pipe, outs, [torch.empty_like(u), torch.empty_like(u)])
    torch.cuda.synchronize()
    u_dev = torch.empty_like(u)
    for src, ref in zip(u_hosts, refs):
        layer.forward_host(src, e, b_plain, ref, u_dev)
    torch.cuda.synchronize()
    for i, (o, r) in enumerate(zip(outs, refs)):
        assert torch.equal(o, r), f"batch {i}"
    assert torch.equal(b_pipe, b_plain)
