"""The a-priori routing-weight bound (tests/parity.py: logit_error_bound,
weight_bound) against fp32 renderings of the router on the CPU: it must hold
for every slot whatever the fp32 summation order, and it must not be vacuous
(a bound that forgot the length of the dot product fails).  CPU only."""
import numpy as np
import pytest

from tests.parity import logit_error_bound, weight_bound, widen
from top_routing_grouped_softmax_b200.synth import MoEConfig, make_inputs


def _case(T=256, d=2048, E=128, k=8, skew=True):
    cfg = MoEConfig("bound", T=T, d=d, E=E, k=k, f=64, sigma=0.02, seed=11, skew=skew)
    inp = make_inputs(cfg)
    x = widen(inp.bits("x")).reshape(T, d)
    w = widen(inp.bits("W_router")).reshape(d, E)
    b = inp.bias_np().astype(np.float64) if inp.bias is not None else np.zeros(E)
    return cfg, x, w, b


def _softmax64(l):
    z = np.exp(l - l.max(axis=1, keepdims=True))
    return z / z.sum(axis=1, keepdims=True)


def _softmax32(l32):
    l32 = l32.astype(np.float32)
    z = np.exp(l32 - l32.max(axis=1, keepdims=True)).astype(np.float32)
    return (z / z.sum(axis=1, keepdims=True, dtype=np.float32)).astype(np.float32)


def _logits32_sequential(x, w, b):
    """fp32 dot products summed strictly left to right (the longest chain of
    roundings any order has), then the bias."""
    x32, w32 = x.astype(np.float32), w.astype(np.float32)
    acc = np.zeros((x.shape[0], w.shape[1]), np.float32)
    for i in range(x.shape[1]):
        acc = (acc + np.outer(x32[:, i], w32[i, :]).astype(np.float32)).astype(np.float32)
    return (acc + b.astype(np.float32)).astype(np.float32)


def _logits32_blas(x, w, b):
    return (x.astype(np.float32) @ w.astype(np.float32) + b.astype(np.float32)).astype(np.float32)


def _rel_err_over_bound(x, w, b, d, k, logits32, d_in_bound=None):
    l64 = x @ w + b
    p = _softmax64(l64)
    ids = np.argsort(-p, axis=1, kind="stable")[:, :k]
    p32 = _softmax32(logits32).astype(np.float64)
    w_gpu = np.take_along_axis(p32, ids, axis=1)
    p_sel = np.take_along_axis(p, ids, axis=1)
    scale = np.abs(x) @ np.abs(w) + np.abs(b)[None, :]
    bound = weight_bound(logit_error_bound(scale, d if d_in_bound is None else d_in_bound), p, ids)
    return np.abs(w_gpu - p_sel) / p_sel / bound


@pytest.mark.parametrize("order", ["sequential", "blas"])
def test_bound_holds_for_fp32_routers(order):
    cfg, x, w, b = _case()
    l32 = _logits32_sequential(x, w, b) if order == "sequential" else _logits32_blas(x, w, b)
    use = _rel_err_over_bound(x, w, b, cfg.d, cfg.k, l32)
    assert use.max() <= 1.0


def _adversarial(T=16, d=2048, E=16):
    """Every token: x = (1, 2^-13, ..., 2^-13); expert e's column: (1 + e/16,
    2^-12, ..., 2^-12) for even e, (1 + e/16, 0, ..., 0) for odd e (all bf16
    values).  The even experts' 2047 products of 2^-25 each fall below half
    an ulp of the running fp32 sum (between 1 and 2), so a left-to-right fp32
    sum drops all of them: logit error 2047 * 2^-25, near the worst case,
    and different for even and odd experts, so the softmax does not cancel
    it."""
    x = np.full((T, d), 2.0 ** -13)
    x[:, 0] = 1.0
    w = np.zeros((d, E))
    w[0, :] = 1.0 + np.arange(E) / 16.0
    w[1:, 0::2] = 2.0 ** -12
    return x, w, np.zeros(E)


def test_bound_holds_on_a_near_worst_case_sum():
    x, w, b = _adversarial()
    l32 = _logits32_sequential(x, w, b)
    assert np.all(l32[:, 0] == np.float32(1.0))   # every small product was lost
    use = _rel_err_over_bound(x, w, b, x.shape[1], 4, l32)
    assert use.max() <= 1.0
    assert use.max() > 0.02   # the logit part of the bound is what holds it


def test_bound_that_forgets_the_dot_product_length_fails():
    """A slip that takes one rounding per logit instead of d + 1 is caught on
    the near-worst-case sum."""
    x, w, b = _adversarial()
    use = _rel_err_over_bound(x, w, b, x.shape[1], 4, _logits32_sequential(x, w, b), d_in_bound=-1)
    assert use.max() > 1.0


def test_bound_exact_logits_leave_only_softmax_rounding():
    """Integer-valued inputs make every fp32 logit exact: the error is the
    fp32 softmax's alone, and the bound's logit part vanishes with a zero
    scale."""
    T, d, E, k = 64, 32, 16, 4
    rng = np.random.default_rng(3)
    x = rng.integers(-3, 4, size=(T, d)).astype(np.float64)
    w = rng.integers(-2, 3, size=(d, E)).astype(np.float64) / 8.0
    b = np.zeros(E)
    l32 = _logits32_blas(x, w, b)
    assert np.array_equal(l32.astype(np.float64), x @ w)
    p = _softmax64(x @ w)
    ids = np.argsort(-p, axis=1, kind="stable")[:, :k]
    bound = weight_bound(np.zeros((T, E)), p, ids)
    p32 = np.take_along_axis(_softmax32(l32).astype(np.float64), ids, axis=1)
    p_sel = np.take_along_axis(p, ids, axis=1)
    assert (np.abs(p32 - p_sel) / p_sel <= bound).all()
    assert bound.max() < 1e-5
