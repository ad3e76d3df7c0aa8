"""Grouped expert GEMMs (gate/up + SwiGLU, down + routing weight) and the
combine, against the oracle, on the GPU.

The oracle is handed the GPU's own routing (ids, and its fp32 weights widened
exactly) so that these stages are checked in isolation from routing."""
import numpy as np
import pytest
import torch

import top_routing_grouped_softmax_b200 as moe
from oracle.oracle import default_oracle
from tests import gpu_cases as gc
from tests.parity import bf16_rounded_check, bf16_tensor_to_f64, bound_check, value_check, widen

pytestmark = pytest.mark.gpu

CASES = [
    gc.small_cfg(1000, 256, 16, 4, 320),    # ragged T; f = 320: partial last gate/up tile
    gc.small_cfg(700, 320, 8, 2, 128),      # d = 320: partial last down tile
    gc.small_cfg(64, 64, 8, 8, 64),         # k = E, minimal d and f
    gc.small_cfg(3000, 128, 64, 6, 192, skew=True),  # skewed groups, many empty
    gc.small_cfg(1, 128, 8, 2, 128),        # a single token
]


def _stages(cfg, rows=None):
    inp = gc.inputs(cfg)
    d = gc.on_device(inp)
    ids, w = moe.route(d["x"], d["w_router"], cfg.k, bias=d["bias"])
    pm = moe.permute(d["x"], ids, w, cfg.E)
    h, y = moe.expert_ffn(pm["x_perm"], pm["w_perm"], pm["offsets"], d["w_gate"], d["w_up"], d["w_down"])
    out = moe.combine(y, pm["inv"], cfg.T, cfg.k)
    torch.cuda.synchronize()
    assert moe.get_status() == moe.MOE_OK
    return inp, d, ids, w, pm, h, y, out


@pytest.mark.parametrize("cfg", CASES, ids=lambda c: c.name)
def test_ffn_and_combine_small(cfg):
    inp, d, ids, w, pm, h, y, out = _stages(cfg)
    ids_np = ids.cpu().numpy()
    w_np = w.cpu().numpy().astype(np.float64)
    rows = np.arange(cfg.T)
    ex = default_oracle().expert_rows(inp.bits("x"), inp.bits("W_gate"), inp.bits("W_up"), inp.bits("W_down"),
                                      ids_np, w_np, rows, want_y=True, want_h=True)
    inv = pm["inv"].cpu().numpy().reshape(cfg.T, cfg.k)
    h_gpu = bf16_tensor_to_f64(h)[inv]      # [T, k, f]
    y_gpu = y.double().cpu().numpy()[inv]   # [T, k, d]
    value_check(out.double().cpu().numpy(), ex.out, "out")
    # y = w * o with o = h . W_down.  h is rounded to bf16 once (it is the
    # second GEMM's operand), so each element of o may differ from the fp64
    # value by at most (2^-8 + f * 2^-23) * sum_n |h_n| |W_down[n, c]|.
    wv = w_np[:, :, None]
    Wd = np.abs(widen(inp.bits("W_down")))
    bound = np.empty_like(ex.y)
    for e in range(cfg.E):
        sel = ids_np == e
        if sel.any():
            bound[sel] = np.abs(ex.h[sel]) @ Wd[e]
    bound *= 2.0 ** -8 + cfg.f * 2.0 ** -23
    bound_check(y_gpu / wv, ex.y / wv, bound, "o = y / w")
    bf16_rounded_check(h_gpu, ex.h, "h")


def test_combine_exact_fp32_sum():
    """The combine widens the fp16 rows to fp32 and sums them in slot order:
    an fp32 numpy sum of the same widened rows in the same order matches bit
    for bit."""
    cfg = gc.small_cfg(777, 192, 16, 4, 64)
    inp, d, ids, w, pm, h, y, out = _stages(cfg)
    yf = y.cpu().numpy().astype(np.float32)   # fp16 -> fp32 is exact
    inv = pm["inv"].cpu().numpy().reshape(cfg.T, cfg.k)
    acc = np.zeros((cfg.T, cfg.d), np.float32)
    for j in range(cfg.k):
        acc = acc + yf[inv[:, j]]
    assert np.array_equal(out.cpu().numpy(), acc)


def test_ffn_rejects_corrupt_offsets():
    """Non-monotone group offsets are reported, and nothing is written."""
    cfg = gc.small_cfg(256, 128, 8, 2, 128)
    inp, d, ids, w, pm, h, y, out = _stages(cfg)
    bad = pm["offsets"].clone()
    bad[3] = bad[5] + 7
    y2 = torch.full_like(y, 0)
    moe.expert_ffn(pm["x_perm"], pm["w_perm"], bad, d["w_gate"], d["w_up"], d["w_down"], y=y2)
    assert moe.get_status() == moe.MOE_ERR_DEVICE_BOUNDS
    assert torch.count_nonzero(y2).item() == 0
    bad = pm["offsets"].clone()
    bad[-1] = bad[-1] - 1  # offsets[E] != M
    moe.expert_ffn(pm["x_perm"], pm["w_perm"], bad, d["w_gate"], d["w_up"], d["w_down"], y=y2)
    assert moe.get_status() == moe.MOE_ERR_DEVICE_BOUNDS
