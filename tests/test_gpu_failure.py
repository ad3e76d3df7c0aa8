"""Failure detection on the GPU without a fault: a bounded wait that nothing
satisfies gives up, reports MOE_ERR_DEVICE_TIMEOUT, and the context stays
usable."""
import pytest
import torch

import top_routing_grouped_softmax_b200 as moe
from tests import gpu_cases as gc

pytestmark = pytest.mark.gpu


def test_bounded_wait_times_out_and_context_survives():
    assert moe.get_status() == moe.MOE_OK
    moe.selftest_wait_timeout(20_000_000)   # 20 ms
    assert moe.get_status() == moe.MOE_ERR_DEVICE_TIMEOUT
    assert moe.get_status() == moe.MOE_OK
    cfg = gc.small_cfg(256, 128, 8, 2, 128)
    d = gc.on_device(gc.inputs(cfg))
    out = moe.forward(d["x"], d["w_router"], d["w_gate"], d["w_up"], d["w_down"], 2)
    torch.cuda.synchronize()
    assert moe.get_status() == moe.MOE_OK
    assert torch.isfinite(out.float()).all().item()


def test_wait_limit_setting_roundtrip():
    moe.set_wait_limit_ns(500_000_000)
    moe.set_wait_limit_ns(0)   # back to the default
    cfg = gc.small_cfg(128, 64, 8, 2, 64)
    d = gc.on_device(gc.inputs(cfg))
    moe.forward(d["x"], d["w_router"], d["w_gate"], d["w_up"], d["w_down"], 2)
    assert moe.get_status() == moe.MOE_OK


def test_y_outside_fp16_range_is_reported():
    """y is stored as fp16.  A block whose contributions exceed the fp16 range
    (here W_down scaled by 2^30, so |y| reaches about 1e6) stores inf and
    reports MOE_ERR_DEVICE_RANGE;
    the context stays usable and an in-range call is clean again."""
    cfg = gc.small_cfg(256, 128, 8, 2, 128)
    d = gc.on_device(gc.inputs(cfg))
    assert moe.get_status() == moe.MOE_OK
    big = (d["w_down"].float() * 2.0 ** 30).to(torch.bfloat16)
    out = moe.forward(d["x"], d["w_router"], d["w_gate"], d["w_up"], big, 2)
    torch.cuda.synchronize()
    assert moe.get_status() == moe.MOE_ERR_DEVICE_RANGE
    assert not torch.isfinite(out).all().item()
    out = moe.forward(d["x"], d["w_router"], d["w_gate"], d["w_up"], d["w_down"], 2)
    torch.cuda.synchronize()
    assert moe.get_status() == moe.MOE_OK
    assert torch.isfinite(out).all().item()


def test_tiny_wait_limit_is_raised_to_one_millisecond():
    """A limit below 1 ms is raised to 1 ms: with a 1 ns limit taken as is,
    nearly every pipeline wait would give up; raised, a small forward and
    backward finish cleanly (their waits last microseconds)."""
    cfg = gc.small_cfg(256, 128, 8, 2, 128)
    d = gc.on_device(gc.inputs(cfg))
    assert moe.get_status() == moe.MOE_OK
    moe.set_wait_limit_ns(1)
    try:
        out = moe.forward(d["x"], d["w_router"], d["w_gate"], d["w_up"], d["w_down"], 2)
        dout = torch.ones(cfg.T, cfg.d, dtype=torch.float32, device="cuda")
        moe.backward(d["x"], d["w_router"], d["w_gate"], d["w_up"], d["w_down"], 2, dout)
        torch.cuda.synchronize()
        assert moe.get_status() == moe.MOE_OK
        assert torch.isfinite(out).all().item()
    finally:
        moe.set_wait_limit_ns(0)
