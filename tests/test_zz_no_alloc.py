"""The allocation-free permutation (moe_permute_noalloc) against moe_permute.

moe_permute_noalloc serves callers that cannot allocate device memory for a
workspace (an engine that owns all device memory, a serving loop where
cudaMalloc's device-wide synchronisation is not allowed, a plugin that only
sees its tensors).  It keeps its scratch in a static array inside the library,
shared by every call, so this file checks that two calls in a row (a large one,
then a smaller one that must not see the first call's leftovers) give exactly
what the workspace version gives.  Index work, so the comparison is bit-exact.
This module is collected last on purpose and needs nothing from other tests.
"""
import ctypes

import numpy as np
import pytest
import torch

from sigmoid_routed_mixture_b200 import moe

pytestmark = pytest.mark.gpu


def topk_ids(T, E, K, seed):
    g = torch.Generator(device="cuda")
    g.manual_seed(seed)
    scores = torch.rand((T, E), generator=g, device="cuda")
    return torch.argsort(scores, dim=1)[:, :K].to(torch.int32).contiguous()


def call_noalloc(cfg, idx, counts, offsets, sorted_):
    """Straight through the C ABI."""
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    p = lambda t: ctypes.c_void_p(t.data_ptr())  # noqa: E731
    return moe.lib().moe_permute_noalloc(ctypes.byref(cfg.c()), p(idx), p(counts), p(offsets),
                                         p(sorted_), stream)


@pytest.mark.parametrize("has_shared", [True, False])
def test_noalloc_matches_workspace_permute_on_two_calls(has_shared):
    # both calls above 16384 assignments, so both take the chunked path whose
    # per-chunk counts live in the static array; the second has fewer chunks and
    # another expert count, so leftovers of the first would show; the third is
    # the one-CTA path for small batches
    for T, E, K, seed in [(32768, 256, 8, 11), (3000, 64, 8, 12), (1000, 64, 4, 14)]:
        cfg = moe.Config(T=T, H=256, I=128, E=E, K=K, has_shared=has_shared)
        idx = topk_ids(T, E, K, seed)
        ref = moe.permute(cfg, idx, moe.workspace(cfg))
        out = (torch.full((E + 1,), -7, dtype=torch.int32, device="cuda"),
               torch.full((E + 2,), -7, dtype=torch.int32, device="cuda"),
               torch.full((cfg.rows,), -7, dtype=torch.int32, device="cuda"))
        assert call_noalloc(cfg, idx, *out) == 0
        torch.cuda.synchronize()
        for a, b in zip(ref, out):
            assert torch.equal(a, b)
        assert int(out[1][0]) == 0


@pytest.mark.parametrize("T,E,K", [(300, 16, 4), (3000, 64, 8)])  # one-CTA path, chunked path
def test_noalloc_limits_and_bad_ids(T, E, K):
    L = moe.lib()
    big = moe.Config(T=262144 // 8 + 1, H=256, I=128, E=256, K=8)
    assert L.moe_permute_noalloc(ctypes.byref(big.c()), None, None, None, None, None) == 2
    cfg = moe.Config(T=T, H=256, I=128, E=E, K=K)
    idx = topk_ids(T, E, K, 13)
    idx[5, 1] = 999  # out of range: skipped and flagged in offsets[0]
    counts, offsets, sorted_ = moe.permute_noalloc(cfg, idx)
    torch.cuda.synchronize()
    assert int(offsets[0]) == -1
    idx[5, 1] = next(v for v in range(E) if v not in idx[5].tolist())
    counts, offsets, sorted_ = moe.permute_noalloc(cfg, idx)  # the next call starts clean
    ref = moe.permute(cfg, idx, moe.workspace(cfg))
    torch.cuda.synchronize()
    assert torch.equal(counts, ref[0]) and torch.equal(offsets, ref[1]) and torch.equal(sorted_, ref[2])
    assert np.all(np.diff(offsets.cpu().numpy()) >= 0)
