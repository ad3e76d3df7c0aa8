"""moe_permute_static: the permutation for callers that cannot allocate.

Some callers of this library cannot allocate device memory at the moment they
run the permutation -- an engine plugin whose device memory is all planned
ahead, or a latency-critical loop that cannot take cudaMalloc's implicit
synchronisation.  moe_permute_static gives them the same results as
moe_permute with the scratch taken from a fixed array inside the library.

These tests call it through the C ABI and compare every output with
moe_permute's (integer outputs bit for bit; x_perm and w_perm are copies, so
bit for bit too) on two calls in a row of different shapes, so a second call
that picked up the first call's leftovers would be caught.  This file is
collected last on purpose: the array is shared by every call in the process.
"""
import ctypes

import numpy as np
import pytest
import torch

import top_routing_grouped_softmax_b200 as moe

pytestmark = pytest.mark.gpu


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _inputs(T, d, E, k, seed):
    rng = np.random.default_rng(seed)
    ids = np.stack([rng.permutation(E)[:k] for _ in range(T)]).astype(np.int32)
    w = rng.random((T, k)).astype(np.float32)
    x = torch.randn(T, d, generator=torch.Generator().manual_seed(seed)).to(torch.bfloat16)
    return x.cuda(), torch.from_numpy(ids).cuda(), torch.from_numpy(w).cuda()


def _static(x, ids, w, E):
    T, k = ids.shape
    d = x.shape[1]
    M = T * k
    dev = ids.device
    out = {
        "counts": torch.full((E,), -7, dtype=torch.int32, device=dev),
        "offsets": torch.full((E + 1,), -7, dtype=torch.int32, device=dev),
        "perm": torch.full((M,), -7, dtype=torch.int32, device=dev),
        "inv": torch.full((M,), -7, dtype=torch.int32, device=dev),
        "w_perm": torch.full((M,), -7.0, dtype=torch.float32, device=dev),
        "x_perm": torch.zeros(M, d, dtype=torch.bfloat16, device=dev),
    }
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    rc = moe.lib().moe_permute_static(_p(x), _p(ids), _p(w), T, d, E, k, _p(out["counts"]), _p(out["offsets"]),
                                      _p(out["perm"]), _p(out["inv"]), _p(out["x_perm"]), _p(out["w_perm"]),
                                      stream)
    assert rc == moe.MOE_OK, moe.strerror(rc)
    return out


def _same(a, b):
    for key in ("counts", "offsets", "perm", "inv", "w_perm"):
        assert torch.equal(a[key], b[key]), key
    assert torch.equal(a["x_perm"].view(torch.int16), b["x_perm"].view(torch.int16)), "x_perm"


def test_static_permute_matches_workspace_permute_twice():
    # first call: many chunks, 128 experts; second call: fewer tokens, fewer
    # experts -- leftovers of the first call in the shared array must not leak
    for T, d, E, k, seed in [(9000, 128, 128, 8, 1), (3000, 64, 64, 6, 2)]:
        x, ids, w = _inputs(T, d, E, k, seed)
        got = _static(x, ids, w, E)
        ref = moe.permute(x, ids, w, E)
        torch.cuda.synchronize()
        assert moe.get_status() == moe.MOE_OK
        _same(got, ref)


def test_static_permute_rejects_sizes_beyond_its_array():
    E, k = 512, 1
    T = 64 * 513                      # E * ceil(T / 64) = 262656 > 262144
    ids = torch.zeros(T, k, dtype=torch.int32, device="cuda")
    w = torch.zeros(T, k, dtype=torch.float32, device="cuda")
    buf = torch.zeros(T * k + E + 1, dtype=torch.int32, device="cuda")
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    rc = moe.lib().moe_permute_static(None, _p(ids), _p(w), T, 64, E, k, _p(buf), _p(buf), _p(buf), _p(buf),
                                      None, _p(w), stream)
    assert rc == moe.MOE_ERR_STATIC_SCRATCH_TOO_SMALL
    assert "262144" in moe.strerror(rc)
