"""Permutation kernels against the oracle's stable grouping, bit-exact."""
import numpy as np
import pytest
import torch

import top_routing_grouped_softmax_b200 as moe
from oracle.oracle import default_oracle
from tests import gpu_cases as gc

pytestmark = pytest.mark.gpu


def _check_permute(x_dev, ids_np, w_np, E):
    T, k = ids_np.shape
    ids = torch.from_numpy(ids_np).cuda()
    w = torch.from_numpy(w_np).cuda()
    out = moe.permute(x_dev, ids, w, E)
    torch.cuda.synchronize()
    assert moe.get_status() == moe.MOE_OK
    ref = default_oracle().permute(ids_np, E)
    assert np.array_equal(out["counts"].cpu().numpy(), ref.counts)
    assert np.array_equal(out["offsets"].cpu().numpy(), ref.offsets)
    assert np.array_equal(out["perm"].cpu().numpy(), ref.perm)
    assert np.array_equal(out["inv"].cpu().numpy(), ref.inv)
    assert np.array_equal(out["w_perm"].cpu().numpy(), w_np.ravel()[ref.perm])
    if x_dev is not None:
        xp = out["x_perm"].view(torch.int16).cpu().numpy()
        xs = x_dev.view(torch.int16).cpu().numpy()
        assert np.array_equal(xp, xs[ref.perm // k])
    return out


@pytest.mark.parametrize("T,d,E,k", [(1000, 256, 16, 4), (4097, 64, 8, 2), (1, 128, 8, 8), (9000, 64, 512, 32),
                                     (12345, 128, 64, 6)])
def test_permute_random_ids(T, d, E, k):
    rng = np.random.default_rng(T + E)
    ids = np.stack([rng.permutation(E)[:k] for _ in range(T)]).astype(np.int32)
    w = rng.random((T, k)).astype(np.float32)
    x = torch.randn(T, d, generator=torch.Generator().manual_seed(3)).to(torch.bfloat16).cuda()
    _check_permute(x, ids, w, E)


def test_permute_skewed_and_empty_groups():
    """One expert takes every token, most experts stay empty."""
    T, E, k = 5000, 64, 4
    rng = np.random.default_rng(1)
    ids = np.empty((T, k), np.int32)
    ids[:, 0] = 17
    for t in range(T):
        ids[t, 1:] = rng.choice([e for e in (3, 5, 40, 63) if e != 17], size=k - 1, replace=False)
    w = rng.random((T, k)).astype(np.float32)
    x = torch.randn(T, 64).to(torch.bfloat16).cuda()
    out = _check_permute(x, ids, w, E)
    counts = out["counts"].cpu().numpy()
    assert counts[17] == T and (counts == 0).sum() == E - 5


def test_permute_from_routing_full_size():
    cfg = gc.FULL[1]  # the Qwen3-shaped layer
    d = gc.on_device(gc.inputs(cfg))
    ids, w = moe.route(d["x"], d["w_router"], cfg.k)
    _check_permute(d["x"], ids.cpu().numpy(), w.cpu().numpy(), cfg.E)


def test_permute_without_gather():
    T, E, k = 300, 8, 2
    rng = np.random.default_rng(2)
    ids = np.stack([rng.permutation(E)[:k] for _ in range(T)]).astype(np.int32)
    w = rng.random((T, k)).astype(np.float32)
    out = moe.permute(None, torch.from_numpy(ids).cuda(), torch.from_numpy(w).cuda(), E, gather=False)
    torch.cuda.synchronize()
    ref = default_oracle().permute(ids, E)
    assert np.array_equal(out["perm"].cpu().numpy(), ref.perm)


def test_permute_out_of_range_ids_reported():
    """An id outside [0, E) is reported through the status word, not a fault."""
    T, E, k = 64, 8, 2
    ids = np.tile(np.array([[0, 1]], np.int32), (T, 1))
    ids[5, 1] = 99
    ids[9, 0] = -3
    w = np.ones((T, k), np.float32)
    x = torch.zeros(T, 64, dtype=torch.bfloat16, device="cuda")
    moe.permute(x, torch.from_numpy(ids).cuda(), torch.from_numpy(w).cuda(), E)
    assert moe.get_status() == moe.MOE_ERR_DEVICE_BOUNDS
    assert moe.get_status() == moe.MOE_OK  # cleared by the read
