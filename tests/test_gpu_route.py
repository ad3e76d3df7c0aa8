"""Router kernel (GEMM + fp32 softmax + top-k) against the oracle, on the GPU.

Expert ids bit-exact (near ties excepted, see tests/parity.py), weights to
5e-5 relative and within their a-priori fp32 bound (tests/parity.py)."""
import numpy as np
import pytest
import torch

import top_routing_grouped_softmax_b200 as moe
from tests import gpu_cases as gc
from tests.parity import W_REL, route_check

pytestmark = pytest.mark.gpu

SMALL = [
    gc.small_cfg(1000, 256, 16, 4, 320, sigma=0.1),       # ragged T, several tiles
    gc.small_cfg(129, 128, 8, 2, 64, sigma=0.1),          # one full tile + 1 token
    gc.small_cfg(1, 64, 8, 1, 64, sigma=0.1),             # single token, minimal d
    gc.small_cfg(300, 192, 264, 8, 64, sigma=0.1),        # E not a multiple of 64: two MMAs per k-step
    gc.small_cfg(257, 128, 512, 32, 64, sigma=0.1),       # maximum E and k
    gc.small_cfg(200, 64, 8, 8, 64, sigma=0.1),           # k = E
    gc.small_cfg(640, 256, 64, 6, 64, sigma=0.1, skew=True),  # per-expert bias
]


def _route(cfg):
    d = gc.on_device(gc.inputs(cfg))
    ids, w = moe.route(d["x"], d["w_router"], cfg.k, bias=d["bias"])
    torch.cuda.synchronize()
    assert moe.get_status() == moe.MOE_OK
    return ids.cpu().numpy(), w.cpu().numpy()


@pytest.mark.parametrize("cfg", SMALL, ids=lambda c: c.name)
def test_route_small(cfg):
    ids, w = _route(cfg)
    r = gc.oracle_route(cfg)
    route_check(ids, w, r.probs, r.ids, cfg.k, logit_err=gc.logit_error(cfg))


@pytest.mark.parametrize("cfg", gc.FULL, ids=lambda c: c.name)
def test_route_full_size(cfg):
    ids, w = _route(cfg)
    r = gc.oracle_route(cfg)
    excluded, stats = route_check(ids, w, r.probs, r.ids, cfg.k, logit_err=gc.logit_error(cfg))
    print(cfg.name, stats)
    assert stats["excluded_near_tie"] < max(1, cfg.T // 100)


def test_route_exact_ties_lowest_index():
    """Identical router columns: every probability is 1/E and ids are 0..k-1."""
    cfg = gc.small_cfg(300, 128, 16, 4, 64)
    inp = gc.inputs(cfg)
    d = gc.on_device(inp)
    wr = d["w_router"].clone()
    wr[:] = wr[:, :1]
    ids, w = moe.route(d["x"], wr, 4)
    torch.cuda.synchronize()
    assert np.all(ids.cpu().numpy() == np.arange(4)[None, :])
    assert torch.all(w == 1.0 / 16).item()


def test_route_rejects_bad_shapes():
    x = torch.zeros(4, 64, dtype=torch.bfloat16, device="cuda")
    wr = torch.zeros(64, 12, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(moe.MoEError) as e:
        moe.route(x, wr, 2)
    assert e.value.status == moe.MOE_ERR_UNSUPPORTED_SHAPE
    wr = torch.zeros(64, 8, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(moe.MoEError) as e:
        moe.route(x, wr, 9)
    assert e.value.status == moe.MOE_ERR_UNSUPPORTED_SHAPE


RENORM = [SMALL[0], SMALL[4], SMALL[5], SMALL[6]]   # group top-k, whole-warp top-k (k = 32), k = E, bias


@pytest.mark.parametrize("cfg", RENORM, ids=lambda c: c.name)
def test_route_renormalized(cfg):
    """MOE_FLAG_RENORMALIZE: the same ids; each weight is the oracle's
    probability divided by the sum over the token's selected experts."""
    d = gc.on_device(gc.inputs(cfg))
    ids_t, w_t = moe.route(d["x"], d["w_router"], cfg.k, bias=d["bias"], renormalize=True)
    ids_p, _ = moe.route(d["x"], d["w_router"], cfg.k, bias=d["bias"])
    torch.cuda.synchronize()
    assert moe.get_status() == moe.MOE_OK
    assert torch.equal(ids_t, ids_p)
    ids, w = ids_t.cpu().numpy(), w_t.cpu().numpy().astype(np.float64)
    r = gc.oracle_route(cfg)
    p_sel = np.take_along_axis(r.probs, ids.astype(np.int64), axis=1)
    want = p_sel / p_sel.sum(axis=1, keepdims=True)
    worst = float(np.max(np.abs(w - want) / want))
    assert worst <= W_REL, f"renormalised weight relative error {worst:.3e}"
    np.testing.assert_allclose(w.sum(axis=1), 1.0, rtol=0, atol=k_sum_tol(cfg.k))


def k_sum_tol(k):
    """fp32 sum of k weights that each carry relative error <= W_REL."""
    return k * W_REL
