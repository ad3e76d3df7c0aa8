"""The block's backward on the GPU (moe_backward) against the fp64 oracle.

Small shapes compare every element of every gradient with oracle_backward.
At the Qwen3-shaped layer's full size the oracle computes sampled dx rows
one token at a time and one expert's weight gradients, and properties that
hold at any size are checked on everything: exact doubling with 2 * dout,
bit-identical repeats, zero gradients for experts no token selects.

Tolerance.  The GPU rounds each GEMM operand to bf16 once (dout, g and u
after the recompute, dg, du, w h, dlogit): three roundings of 2^-9 relative
lie on the longest path (dout, g/u, dg), so an element of an operand is off
by up to about 0.6 % of its own size and typically by a third of that, and
the fp32 sums add little.  A gradient element sums such products, so its
error scales with the size of the terms it sums, not with the RMS of the
whole tensor: weight gradients are outer products of two heavy-tailed
factors (x and dg, h and dout), whose largest elements sit many RMS out.
The criteria are therefore norms of the whole tensor plus a bound against
its largest element:
    ||gpu - oracle||_F <= 1e-2 * ||oracle||_F
    sum |gpu - oracle| <= 1e-2 * sum |oracle|
    max |gpu - oracle| <= 2e-2 * max |oracle|
per gradient tensor -- a few times the expected 0.2-0.4 %.
"""
import numpy as np
import pytest
import torch

import top_routing_grouped_softmax_b200 as moe
from oracle.oracle import default_oracle, topk_gap
from tests import gpu_cases as gc
from tests.parity import TIE_EPS
from top_routing_grouped_softmax_b200.synth import CONFIGS, make_dout

pytestmark = pytest.mark.gpu

BWD_FROB = 1e-2
BWD_MEAN_REL = 1e-2
BWD_MAX_OF_MAX = 2e-2
NAMES = ("dx", "dw_router", "dbias", "dw_gate", "dw_up", "dw_down")


def grad_check(gpu, ref, what):
    """The backward's criteria; returns (frobenius, mean, max-of-max) relative errors."""
    gpu = np.asarray(gpu, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert gpu.shape == ref.shape, (what, gpu.shape, ref.shape)
    assert np.all(np.isfinite(gpu)), f"{what}: non-finite values"
    diff = np.abs(gpu - ref)
    nref = float(np.sqrt(np.sum(ref * ref)))
    frob = float(np.sqrt(np.sum(diff * diff)) / nref) if nref > 0 else float(diff.max())
    denom = float(np.abs(ref).sum())
    mean_rel = float(diff.sum() / denom) if denom > 0 else float(diff.sum())
    mref = float(np.abs(ref).max())
    mx = float(diff.max() / mref) if mref > 0 else float(diff.max())
    assert frob <= BWD_FROB, f"{what}: ||gpu-oracle||_F = {frob:.3e} * ||oracle||_F > {BWD_FROB}"
    assert mean_rel <= BWD_MEAN_REL, f"{what}: mean relative error {mean_rel:.3e} > {BWD_MEAN_REL}"
    assert mx <= BWD_MAX_OF_MAX, f"{what}: max|gpu-oracle| = {mx:.3e} * max|oracle| > {BWD_MAX_OF_MAX}"
    return frob, mean_rel, mx


def _run(cfg, renorm=False, scale=1.0):
    inp = gc.inputs(cfg)
    d = gc.on_device(inp)
    dout = (make_dout(cfg.T, cfg.d, cfg.seed) * scale).cuda()
    g = moe.backward(d["x"], d["w_router"], d["w_gate"], d["w_up"], d["w_down"], cfg.k, dout, bias=d["bias"],
                     renormalize=renorm)
    torch.cuda.synchronize()
    status = moe.get_status()
    assert status == moe.MOE_OK, moe.strerror(status)
    return {n: (None if v is None else v.cpu().numpy()) for n, v in g.items()}


SMALL = [
    (gc.small_cfg(200, 128, 8, 2, 128, sigma=0.1), False),
    (gc.small_cfg(300, 256, 16, 4, 320, sigma=0.1, skew=True), False),   # partial N tile over f, bias
    (gc.small_cfg(129, 192, 64, 6, 192, sigma=0.1), False),              # many small groups
    (gc.small_cfg(160, 320, 8, 8, 64, sigma=0.1), False),                # k = E, d not a multiple of 256
    (gc.small_cfg(250, 128, 16, 4, 256, seed=8, sigma=0.1, skew=True), True),    # renormalised weights
    (gc.small_cfg(1, 64, 8, 1, 64, sigma=0.1), False),                   # one token
]


@pytest.mark.parametrize("cfg,renorm", SMALL, ids=[c.name + ("_renorm" if r else "") for c, r in SMALL])
def test_backward_small_every_element(cfg, renorm):
    inp = gc.inputs(cfg)
    r = default_oracle().route(inp.bits("x"), inp.bits("W_router"), inp.bias_np(), cfg.k)
    assert not (topk_gap(r.probs, cfg.k) < TIE_EPS).any(), "near-tie routing in a small case: pick another seed"
    got = _run(cfg, renorm)
    dout = make_dout(cfg.T, cfg.d, cfg.seed).numpy().astype(np.float64)
    ref = default_oracle().backward(inp.bits("x"), inp.bits("W_router"), inp.bias_np(), inp.bits("W_gate"),
                                    inp.bits("W_up"), inp.bits("W_down"), cfg.k, dout, renormalize=renorm)
    stats = {n: grad_check(got[n], getattr(ref, n), n) for n in NAMES}
    print(cfg.name, {n: "/".join(f"{v:.2e}" for v in st) for n, st in stats.items()})
    # experts no token selects: exactly zero
    unused = np.setdiff1d(np.arange(cfg.E), r.ids.ravel())
    for e in unused:
        assert not got["dw_gate"][e].any() and not got["dw_up"][e].any() and not got["dw_down"][e].any(), e


def test_backward_empty_batch():
    cfg = gc.small_cfg(64, 128, 8, 2, 64, sigma=0.1)
    d = gc.on_device(gc.inputs(cfg))
    x0 = d["x"][:0]
    dout = torch.zeros(0, cfg.d, dtype=torch.float32, device="cuda")
    g = moe.backward(x0, d["w_router"], d["w_gate"], d["w_up"], d["w_down"], cfg.k, dout)
    torch.cuda.synchronize()
    assert moe.get_status() == moe.MOE_OK
    for n in ("dw_router", "dbias", "dw_gate", "dw_up", "dw_down"):
        assert not g[n].any().item(), n


@pytest.fixture(scope="module")
def qwen_grads():
    cfg = CONFIGS["qwen"]
    return cfg, _run(cfg)


@pytest.fixture(scope="module")
def fine_grads():
    cfg = CONFIGS["fine"]
    return cfg, _run(cfg)


@pytest.fixture(params=["qwen", "fine"])
def full_grads(request):
    """The Qwen3-shaped layer and the fine-grained one (E = 256, f = 256: a
    short K for the dh and weight-gradient GEMMs, 256 experts in the router
    gradient's split)."""
    return request.getfixturevalue(f"{request.param}_grads")


def test_backward_full_size_sampled_rows(full_grads):
    cfg, got = full_grads
    inp = gc.inputs(cfg)
    r = gc.oracle_route(cfg)
    excluded = topk_gap(r.probs, cfg.k) < TIE_EPS
    rows = [int(t) for t in gc.sample_for(cfg, 24) if not excluded[t]]
    dout = make_dout(cfg.T, cfg.d, cfg.seed).numpy().astype(np.float64)
    from concurrent.futures import ThreadPoolExecutor
    o = default_oracle()
    args = (inp.bits("x"), inp.bits("W_router"), inp.bias_np(), inp.bits("W_gate"), inp.bits("W_up"),
            inp.bits("W_down"), cfg.k, dout)
    chunks = [c for c in np.array_split(np.array(rows, dtype=np.int64), 16) if c.size]
    with ThreadPoolExecutor(max_workers=len(chunks)) as pool:
        parts = list(pool.map(lambda c: o.backward_rows(*args, c), chunks))
    ref = np.concatenate(parts, axis=0)
    print("dx rows", grad_check(got["dx"][rows], ref, "dx (sampled rows)"))


def test_backward_full_size_one_expert(full_grads):
    cfg, got = full_grads
    inp = gc.inputs(cfg)
    r = gc.oracle_route(cfg)
    counts = np.bincount(r.ids.ravel(), minlength=cfg.E)
    # an expert whose token set cannot change under a near tie: no excluded
    # token has it among its k selected experts
    excluded = topk_gap(r.probs, cfg.k) < TIE_EPS
    touched = set(r.ids[excluded].ravel().tolist())
    order = [int(e) for e in np.argsort(counts) if counts[e] > 0 and int(e) not in touched]
    e = order[0]
    dout = make_dout(cfg.T, cfg.d, cfg.seed).numpy().astype(np.float64)
    gg, gu, gd = default_oracle().backward_expert(inp.bits("x"), inp.bits("W_router"), inp.bias_np(),
                                                  inp.bits("W_gate"), inp.bits("W_up"), inp.bits("W_down"), cfg.k,
                                                  dout, e)
    print("expert", e, counts[e], grad_check(got["dw_gate"][e], gg, "dW_gate[e]"),
          grad_check(got["dw_up"][e], gu, "dW_up[e]"), grad_check(got["dw_down"][e], gd, "dW_down[e]"))


def test_backward_full_size_properties(qwen_grads):
    cfg, got = qwen_grads
    # bit-identical when repeated (no atomics anywhere)
    again = _run(cfg)
    for n in NAMES:
        assert np.array_equal(got[n], again[n]), f"{n} differs between two identical calls"
    # linear in dout, exactly: doubling dout doubles every rounding step
    twice = _run(cfg, scale=2.0)
    for n in NAMES:
        assert np.array_equal(twice[n], 2.0 * got[n]), f"{n} is not exactly doubled by 2 * dout"
    # the softmax Jacobian's rows sum to zero, so the bias gradient (summed
    # in fp32 from the unrounded dlogit) sums to zero up to fp32 rounding
    db = got["dbias"].astype(np.float64)
    assert abs(db.sum()) <= 2.0 ** -8 * np.abs(db).sum() + 1e-6


def _run_dtype(cfg, grad_dtype):
    inp = gc.inputs(cfg)
    d = gc.on_device(inp)
    dout = make_dout(cfg.T, cfg.d, cfg.seed).cuda()
    g = moe.backward(d["x"], d["w_router"], d["w_gate"], d["w_up"], d["w_down"], cfg.k, dout, bias=d["bias"],
                     grad_dtype=grad_dtype)
    torch.cuda.synchronize()
    assert moe.get_status() == moe.MOE_OK
    return g


@pytest.mark.parametrize("cfg", [SMALL[0][0], SMALL[1][0], CONFIGS["qwen"]], ids=lambda c: c.name)
def test_backward_bf16_weight_gradients_are_rounded_fp32(cfg):
    """MOE_FLAG_GRAD_BF16: each weight gradient is the fp32 one rounded to
    bf16 once, bit for bit; dx and dbias are unchanged; the bf16 gradients
    are within the backward's criteria of the oracle on a small shape."""
    g32 = _run_dtype(cfg, torch.float32)
    g16 = _run_dtype(cfg, torch.bfloat16)
    for n in ("dw_router", "dw_gate", "dw_up", "dw_down"):
        assert g16[n].dtype == torch.bfloat16
        assert torch.equal(g16[n], g32[n].to(torch.bfloat16)), n
    for n in ("dx", "dbias"):
        assert torch.equal(g16[n], g32[n]), n
    if cfg.T <= 1000:
        inp = gc.inputs(cfg)
        dout = make_dout(cfg.T, cfg.d, cfg.seed).numpy().astype(np.float64)
        ref = default_oracle().backward(inp.bits("x"), inp.bits("W_router"), inp.bias_np(), inp.bits("W_gate"),
                                        inp.bits("W_up"), inp.bits("W_down"), cfg.k, dout)
        for n in ("dw_router", "dw_gate", "dw_up", "dw_down"):
            grad_check(g16[n].float().cpu().numpy(), getattr(ref, n), f"{n} (bf16)")
