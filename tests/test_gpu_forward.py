"""The fused moe_forward against the oracle, on the GPU: small cases on every
token, the five workloads at full size on sampled tokens (the launch
configuration the benchmark times), and the equalities the path must keep."""
import numpy as np
import pytest
import torch

import top_routing_grouped_softmax_b200 as moe
from tests import gpu_cases as gc
from tests.parity import route_check, value_check

pytestmark = pytest.mark.gpu

SMALL = [
    gc.small_cfg(1000, 256, 16, 4, 320),
    gc.small_cfg(513, 192, 8, 2, 256, skew=True),
    gc.small_cfg(130, 64, 8, 8, 64),
    gc.small_cfg(2000, 128, 264, 8, 128),
]


VARIANTS = {"x_perm": 0, "fused_gather": moe.MOE_FLAG_FUSED_GATHER}


def _forward(cfg, d, flags=0):
    ids = torch.empty(cfg.T, cfg.k, dtype=torch.int32, device="cuda")
    w = torch.empty(cfg.T, cfg.k, dtype=torch.float32, device="cuda")
    out = moe.forward(d["x"], d["w_router"], d["w_gate"], d["w_up"], d["w_down"], cfg.k, bias=d["bias"],
                      topk_ids=ids, topk_w=w, flags=flags)
    torch.cuda.synchronize()
    assert moe.get_status() == moe.MOE_OK
    return out, ids, w


def _check(cfg, out, ids, w, rows, ref_out):
    r = gc.oracle_route(cfg)
    excluded, stats = route_check(ids.cpu().numpy(), w.cpu().numpy(), r.probs, r.ids, cfg.k,
                                  logit_err=gc.logit_error(cfg))
    keep = ~excluded[rows]
    got = out.double().cpu().numpy()[rows]
    return value_check(got[keep], ref_out[keep], f"out[{cfg.name}]"), stats


@pytest.mark.parametrize("variant", list(VARIANTS))
@pytest.mark.parametrize("cfg", SMALL, ids=lambda c: c.name)
def test_forward_small_all_tokens(cfg, variant):
    d = gc.on_device(gc.inputs(cfg))
    out, ids, w = _forward(cfg, d, VARIANTS[variant])
    rows, ref = gc.oracle_rows(cfg, cfg.T)
    _check(cfg, out, ids, w, rows, ref)


def test_forward_full_size_fused_gather_matches_default():
    """The fused-gather variant on the Qwen3-shaped layer: bit-identical to the default."""
    cfg = gc.FULL[1]
    d = gc.on_device(gc.inputs(cfg))
    a, _, _ = _forward(cfg, d, 0)
    b, _, _ = _forward(cfg, d, moe.MOE_FLAG_FUSED_GATHER)
    assert torch.equal(a, b)


@pytest.mark.parametrize("cfg", gc.FULL, ids=lambda c: c.name)
def test_forward_full_size_sampled(cfg):
    d = gc.on_device(gc.inputs(cfg))
    out, ids, w = _forward(cfg, d)
    rows, ref = gc.oracle_rows(cfg, gc.SAMPLES[cfg.name])
    (mx, mean), stats = _check(cfg, out, ids, w, rows, ref)
    print(cfg.name, "sampled", len(rows), "max/rms", mx, "mean_rel", mean, stats)


@pytest.mark.parametrize("variant", list(VARIANTS))
def test_forward_equals_stages_bitwise(variant):
    cfg = gc.small_cfg(1000, 256, 16, 4, 320, skew=True)
    d = gc.on_device(gc.inputs(cfg))
    out, ids, w = _forward(cfg, d, VARIANTS[variant])
    ids2, w2 = moe.route(d["x"], d["w_router"], cfg.k, bias=d["bias"])
    pm = moe.permute(d["x"], ids2, w2, cfg.E)
    h, y = moe.expert_ffn(pm["x_perm"], pm["w_perm"], pm["offsets"], d["w_gate"], d["w_up"], d["w_down"])
    out2 = moe.combine(y, pm["inv"], cfg.T, cfg.k)
    torch.cuda.synchronize()
    assert torch.equal(ids, ids2) and torch.equal(w, w2)
    assert torch.equal(out, out2)


def test_forward_deterministic_and_block_api():
    cfg = gc.small_cfg(900, 128, 32, 4, 128)
    d = gc.on_device(gc.inputs(cfg))
    blk = moe.MoEBlock(d["w_router"], d["w_gate"], d["w_up"], d["w_down"], cfg.k)
    a = blk(d["x"]).clone()
    b = blk(d["x"]).clone()
    c, _, _ = _forward(cfg, d)
    torch.cuda.synchronize()
    assert torch.equal(a, b)
    assert torch.equal(a, c)


def test_forward_single_expert_is_dense_swiglu():
    """All tokens forced onto expert 0 with k = 1 through a dominant bias: the
    block is one dense SwiGLU MLP scaled by p_0 (checked against the oracle)."""
    cfg = gc.small_cfg(256, 128, 8, 1, 128)
    inp = gc.inputs(cfg)
    d = gc.on_device(inp)
    bias = torch.full((8,), -30.0, device="cuda")
    bias[0] = 30.0
    d["bias"] = bias
    out, ids, w = _forward(cfg, d)
    assert torch.all(ids == 0).item()
    from oracle.oracle import default_oracle
    r, ex = default_oracle().forward(inp.bits("x"), inp.bits("W_router"), bias.cpu().numpy(), inp.bits("W_gate"),
                                     inp.bits("W_up"), inp.bits("W_down"), 1)
    value_check(out.double().cpu().numpy(), ex.out, "dense")


def test_forward_empty_batch():
    cfg = gc.small_cfg(8, 64, 8, 2, 64)
    d = gc.on_device(gc.inputs(cfg))
    x0 = d["x"][:0]
    out = moe.forward(x0, d["w_router"], d["w_gate"], d["w_up"], d["w_down"], 2)
    torch.cuda.synchronize()
    assert out.shape == (0, 64)
    assert moe.get_status() == moe.MOE_OK


def test_forward_profiled_events():
    cfg = gc.small_cfg(512, 128, 8, 2, 128)
    d = gc.on_device(gc.inputs(cfg))
    evs = [torch.cuda.Event(enable_timing=True) for _ in range(6)]
    out = moe.forward(d["x"], d["w_router"], d["w_gate"], d["w_up"], d["w_down"], 2, events=evs)
    torch.cuda.synchronize()
    times = [evs[i].elapsed_time(evs[i + 1]) for i in range(5)]
    assert all(t >= 0 for t in times)
    ref, _, _ = _forward(cfg, d)
    assert torch.equal(out, ref)


@pytest.mark.parametrize("cfg", [SMALL[0], SMALL[1], gc.small_cfg(257, 128, 64, 16, 128)], ids=lambda c: c.name)
def test_forward_renormalized(cfg):
    """MOE_FLAG_RENORMALIZE end to end, every token, against the oracle with
    renormalised weights (k = 16 runs the whole-warp top-k)."""
    d = gc.on_device(gc.inputs(cfg))
    out, ids, w = _forward(cfg, d, moe.MOE_FLAG_RENORMALIZE)
    inp = gc.inputs(cfg)
    o = gc.default_oracle()
    r = o.route(inp.bits("x"), inp.bits("W_router"), inp.bias_np(), cfg.k, renormalize=True)
    excluded, inner = gc.near_tie_masks(cfg)
    g = ids.cpu().numpy()
    exact = ~excluded & ~inner
    assert np.array_equal(g[exact], r.ids[exact])
    assert np.array_equal(np.sort(g[inner], axis=1), np.sort(r.ids[inner], axis=1))
    rows = np.arange(cfg.T, dtype=np.int64)
    ex = o.expert_rows(inp.bits("x"), inp.bits("W_gate"), inp.bits("W_up"), inp.bits("W_down"), r.ids, r.weights,
                       rows)
    keep = ~excluded
    value_check(out.double().cpu().numpy()[keep], ex.out[keep], f"out[{cfg.name}, renormalised]")
    np.testing.assert_allclose(w.cpu().numpy().sum(axis=1), 1.0, rtol=0, atol=cfg.k * 5e-5)


def test_forward_cuda_graph_replay_equals_eager():
    """moe_forward captured in a CUDA graph (its launches carry the
    programmatic-dependent-launch attribute) replays bit-identically to the
    eager call, also after the input changes in place."""
    cfg = SMALL[0]
    d = gc.on_device(gc.inputs(cfg))
    blk = moe.MoEBlock(d["w_router"], d["w_gate"], d["w_up"], d["w_down"], cfg.k, bias=d["bias"])
    x = d["x"].clone()
    out = torch.empty(cfg.T, cfg.d, dtype=torch.float32, device="cuda")
    blk(x, out=out)                                   # eager: sets up the device and the workspace
    torch.cuda.synchronize()
    ref = out.clone()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        blk(x, out=out)
    out.zero_()
    g.replay()
    torch.cuda.synchronize()
    assert moe.get_status() == moe.MOE_OK
    assert torch.equal(out, ref)
    x2 = torch.flip(d["x"], dims=[0]).contiguous()
    x.copy_(x2)
    g.replay()
    eager = blk(x2)
    torch.cuda.synchronize()
    assert torch.equal(out, eager)


@pytest.mark.parametrize("cfg", SMALL, ids=lambda c: c.name)
def test_forward_f16_out_small_all_tokens(cfg):
    """MOE_FLAG_OUT_F16: the fp32 output rounded to fp16 bit for bit, and every
    token within the out criteria of the oracle."""
    d = gc.on_device(gc.inputs(cfg))
    out32, _, _ = _forward(cfg, d)
    out16, ids, w = _forward(cfg, d, moe.MOE_FLAG_OUT_F16)
    assert out16.dtype == torch.float16 and out16.shape == out32.shape
    assert torch.equal(out16, out32.half())
    rows, ref = gc.oracle_rows(cfg, cfg.T)
    _check(cfg, out16, ids, w, rows, ref)


def test_forward_f16_out_full_size_is_rounded_fp32():
    """The Qwen3-shaped layer in the launch configuration the benchmark's
    fp16-output leg times: out16 == fp16(out32), sampled tokens against the
    oracle."""
    cfg = gc.FULL[1]
    d = gc.on_device(gc.inputs(cfg))
    out32, _, _ = _forward(cfg, d)
    out16, ids, w = _forward(cfg, d, moe.MOE_FLAG_OUT_F16)
    assert torch.equal(out16, out32.half())
    rows, ref = gc.oracle_rows(cfg, gc.SAMPLES[cfg.name])
    _check(cfg, out16, ids, w, rows, ref)


def test_forward_f16_out_range_is_reported():
    """Eight identical experts, all selected (k = E) with equal weights 1/8
    (a zero router): out is the expert's output o and each y row is o / 8.
    W_down scaled by a power of two so that max|o| lands in [65520, 131040):
    the fp32 call is clean (y stays in range), the fp16 call stores inf and
    reports MOE_ERR_DEVICE_RANGE, and the context stays usable."""
    import math
    cfg = gc.small_cfg(256, 128, 8, 8, 128)
    d = gc.on_device(gc.inputs(cfg))
    wr = torch.zeros_like(d["w_router"])
    wg = d["w_gate"][:1].expand_as(d["w_gate"]).contiguous()
    wu = d["w_up"][:1].expand_as(d["w_up"]).contiguous()
    wd = d["w_down"][:1].expand_as(d["w_down"]).contiguous()
    o = moe.forward(d["x"], wr, wg, wu, wd, 8)
    torch.cuda.synchronize()
    assert moe.get_status() == moe.MOE_OK
    n = math.ceil(math.log2(65520.0 / o.abs().max().item()))
    wd2 = (wd.float() * 2.0 ** n).to(torch.bfloat16)
    o2 = moe.forward(d["x"], wr, wg, wu, wd2, 8)
    torch.cuda.synchronize()
    assert moe.get_status() == moe.MOE_OK
    assert 65520.0 <= o2.abs().max().item() < 131040.0
    o16 = moe.forward(d["x"], wr, wg, wu, wd2, 8, flags=moe.MOE_FLAG_OUT_F16)
    torch.cuda.synchronize()
    assert moe.get_status() == moe.MOE_ERR_DEVICE_RANGE
    assert torch.isinf(o16).any().item()
    assert torch.equal(o16, o2.half())
    o16 = moe.forward(d["x"], wr, wg, wu, wd, 8, flags=moe.MOE_FLAG_OUT_F16)
    torch.cuda.synchronize()
    assert moe.get_status() == moe.MOE_OK
    assert torch.equal(o16, o.half())


@pytest.mark.parametrize("flags", [moe.MOE_FLAG_RENORMALIZE, moe.MOE_FLAG_FUSED_GATHER,
                                   moe.MOE_FLAG_RENORMALIZE | moe.MOE_FLAG_FUSED_GATHER],
                         ids=["renorm", "fused_gather", "both"])
def test_forward_f16_out_with_other_flags(flags):
    """The fp16 output composes with the other flags: fp16 of the fp32 output
    computed with the same flags, bit for bit."""
    cfg = gc.small_cfg(1000, 256, 16, 4, 320, skew=True)
    d = gc.on_device(gc.inputs(cfg))
    out32, ids32, w32 = _forward(cfg, d, flags)
    out16, ids16, w16 = _forward(cfg, d, flags | moe.MOE_FLAG_OUT_F16)
    assert torch.equal(ids16, ids32) and torch.equal(w16, w32)
    assert torch.equal(out16, out32.half())
