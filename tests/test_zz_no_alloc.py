"""moe_permute_noalloc, the permutation entry point for callers that cannot
allocate device memory (for example an engine plugin whose execute step may
not allocate and reserved no workspace, or a serving loop held to a fixed
memory budget). It takes no workspace: its scratch is a static device array
inside the library. This file is collected last so that a failure here,
under `-x`, comes after every other test has run.

Checked through the C ABI against moe_permute (given a workspace from the
caller): bit-exact, on consecutive calls with different sizes, since every
call reuses the same static array.
"""
import ctypes

import pytest
import torch

import workloads

pytestmark = pytest.mark.gpu


def _outputs(T, N, K, d, dev):
    return dict(counts=torch.empty(N, dtype=torch.int32, device=dev),
                offsets=torch.empty(N + 1, dtype=torch.int32, device=dev),
                sorted_token=torch.empty(T * K, dtype=torch.int32, device=dev),
                inv=torch.empty(T, K, dtype=torch.int32, device=dev),
                xq_perm=torch.empty(T * K, d, dtype=torch.uint8, device=dev),
                xs_perm=torch.empty(T * K, d // 128, dtype=torch.float32, device=dev))


@pytest.mark.parametrize("calls", [[(5000, 256, 8, "uniform"), (3000, 64, 6, "one_hot_expert"),
                                    (5000, 256, 8, "uniform")]])
def test_permute_noalloc_matches_permute(lib, calls):
    from fine_grained_fp8_sigmoid_b200 import binding as B
    dev = "cuda"
    d = 256
    for T, N, K, pattern in calls:
        idx = workloads.topk_indices(T, N, K, seed=T + N, pattern=pattern).to(dev)
        g = torch.Generator().manual_seed(T)
        xq = torch.randint(0, 256, (T, d), generator=g, dtype=torch.uint8).to(dev)
        xs = torch.rand(T, d // 128, generator=g).to(dev)
        ref = _outputs(T, N, K, d, dev)
        ws = torch.empty(B.moe_permute_workspace(T, N), dtype=torch.uint8, device=dev)
        B.moe_permute(idx, N, ref["counts"], ref["offsets"], ref["sorted_token"], ref["inv"], ws,
                      xq, xs, ref["xq_perm"], ref["xs_perm"])
        got = _outputs(T, N, K, d, dev)
        B.moe_permute_noalloc(idx, N, got["counts"], got["offsets"], got["sorted_token"], got["inv"],
                              xq, xs, got["xq_perm"], got["xs_perm"])
        torch.cuda.synchronize()
        for key in ref:
            assert torch.equal(got[key], ref[key]), key


def test_permute_noalloc_rejects_sizes_beyond_its_buffer(lib):
    from fine_grained_fp8_sigmoid_b200 import _lib
    # 2 * ceil(T/256) * N_r int32 > 1 MiB
    st = lib.moe_permute_noalloc(None, 1 << 20, 8, 1024, None, None, 0, None, None, None, None,
                                 None, None, ctypes.c_void_p(0))
    assert st == _lib.MOE_ERR_UNSUPPORTED
    assert b"static buffer" in lib.moe_last_error_detail()
