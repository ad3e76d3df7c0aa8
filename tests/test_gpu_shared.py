"""Shared experts (every token, weight one) on the GPU against the oracle:
small cases on every token, the Qwen3-shaped layer with one shared expert on
sampled tokens, and the stage-by-stage calls against the fused call."""
import numpy as np
import pytest
import torch

import top_routing_grouped_softmax_b200 as moe
from tests import gpu_cases as gc
from tests.parity import route_check, value_check
from top_routing_grouped_softmax_b200.synth import CONFIGS, bf16_bits, make_shared_weights

pytestmark = pytest.mark.gpu

CASES = [
    (gc.small_cfg(1000, 256, 16, 4, 320), 1, 320),
    (gc.small_cfg(513, 192, 8, 2, 256, skew=True), 2, 128),
    (gc.small_cfg(130, 64, 8, 8, 64), 3, 192),        # f_shared not a multiple of 128: partial N tiles
]


def _shared(cfg, n_s, f_s):
    sw = make_shared_weights(cfg, n_s, f_s)
    dev = {k: v.cuda() for k, v in sw.items()}
    bits = tuple(bf16_bits(sw[n]) for n in ("W_gate_s", "W_up_s", "W_down_s"))
    return dev, bits


def _run(cfg, d, sdev):
    ids = torch.empty(cfg.T, cfg.k, dtype=torch.int32, device="cuda")
    w = torch.empty(cfg.T, cfg.k, dtype=torch.float32, device="cuda")
    out = moe.forward_shared(d["x"], d["w_router"], d["w_gate"], d["w_up"], d["w_down"], sdev["W_gate_s"],
                             sdev["W_up_s"], sdev["W_down_s"], cfg.k, bias=d["bias"], topk_ids=ids, topk_w=w)
    torch.cuda.synchronize()
    assert moe.get_status() == moe.MOE_OK
    return out, ids, w


def _check(cfg, out, ids, w, bits, rows):
    inp = gc.inputs(cfg)
    r = gc.oracle_route(cfg)
    excluded, _ = route_check(ids.cpu().numpy(), w.cpu().numpy(), r.probs, r.ids, cfg.k,
                              logit_err=gc.logit_error(cfg))
    _, ex = gc.default_oracle().forward(inp.bits("x"), inp.bits("W_router"), inp.bias_np(), inp.bits("W_gate"),
                                        inp.bits("W_up"), inp.bits("W_down"), cfg.k, rows=rows, shared=bits)
    keep = ~excluded[rows]
    value_check(out.double().cpu().numpy()[rows][keep], ex.out[keep], f"out[{cfg.name}, shared]")


@pytest.mark.parametrize("cfg,n_s,f_s", CASES, ids=[f"{c.name}_ns{n}_fs{f}" for c, n, f in CASES])
def test_forward_shared_small_all_tokens(cfg, n_s, f_s):
    d = gc.on_device(gc.inputs(cfg))
    sdev, bits = _shared(cfg, n_s, f_s)
    out, ids, w = _run(cfg, d, sdev)
    _check(cfg, out, ids, w, bits, np.arange(cfg.T, dtype=np.int64))


def test_forward_shared_qwen_sampled():
    """The Qwen3-shaped layer with one shared expert of the routed size."""
    cfg = CONFIGS["qwen"]
    d = gc.on_device(gc.inputs(cfg))
    sdev, bits = _shared(cfg, 1, cfg.f)
    out, ids, w = _run(cfg, d, sdev)
    rows = gc.sample_for(cfg, 96)
    _check(cfg, out, ids, w, bits, rows)


def test_shared_stages_equal_fused_bitwise():
    """route -> permute -> expert_ffn -> shared_ffn -> combine_shared gives the
    fused call's output bit for bit."""
    cfg, n_s, f_s = CASES[1]
    d = gc.on_device(gc.inputs(cfg))
    sdev, _ = _shared(cfg, n_s, f_s)
    out, _, _ = _run(cfg, d, sdev)
    ids, w = moe.route(d["x"], d["w_router"], cfg.k, bias=d["bias"])
    pm = moe.permute(d["x"], ids, w, cfg.E)
    _, y = moe.expert_ffn(pm["x_perm"], pm["w_perm"], pm["offsets"], d["w_gate"], d["w_up"], d["w_down"])
    _, y_s = moe.shared_ffn(d["x"], sdev["W_gate_s"], sdev["W_up_s"], sdev["W_down_s"])
    out2 = moe.combine_shared(y, pm["inv"], y_s, cfg.T, cfg.k)
    torch.cuda.synchronize()
    assert moe.get_status() == moe.MOE_OK
    assert torch.equal(out, out2)
