"""Token rounding on the GPU against the oracle.

The GPU decides the rounding on its fp32 probabilities, the oracle on fp64;
an expert whose selection boundary is a near tie may therefore move a
different token.  The checks: every rounded count is a multiple of the tile;
the GPU's rounded routing obeys the order-statistic rule on the oracle's
probabilities up to a 1e-6 relative tolerance; it differs from the oracle's
on at most a few tokens; and on every token whose expert set agrees, the
output matches the oracle's within the block's output tolerance."""
import numpy as np
import pytest
import torch

import top_routing_grouped_softmax_b200 as moe
from tests import gpu_cases as gc
from tests.parity import value_check
from top_routing_grouped_softmax_b200.synth import CONFIGS

pytestmark = pytest.mark.gpu

EPS = 1e-6

CASES = [
    (gc.small_cfg(1000, 256, 16, 4, 320), 64),
    (gc.small_cfg(1000, 256, 16, 4, 320), 256),
    (gc.small_cfg(513, 192, 8, 2, 256, skew=True), 128),
    (gc.small_cfg(300, 128, 64, 6, 128), 32),
]


def _run(cfg, tile):
    d = gc.on_device(gc.inputs(cfg))
    rows = torch.empty(cfg.T, cfg.E, dtype=torch.int32, device="cuda")
    out, counts, rows = moe.forward_rounded(d["x"], d["w_router"], d["w_gate"], d["w_up"], d["w_down"], cfg.k,
                                            tile=tile, bias=d["bias"], rows=rows)
    torch.cuda.synchronize()
    assert moe.get_status() == moe.MOE_OK
    return out.double().cpu().numpy(), counts.cpu().numpy(), rows.cpu().numpy()


def _rule_holds(probs, mask0, mask, tile):
    """The rounding rule on the oracle's probabilities, with a relative
    tolerance at the selection boundary."""
    T, E = probs.shape
    for e in range(E):
        m0, m1 = mask0[:, e], mask[:, e]
        c, r = int(m0.sum()), int(m0.sum()) % tile
        added, dropped = np.nonzero(m1 & ~m0)[0], np.nonzero(m0 & ~m1)[0]
        assert added.size == 0 or dropped.size == 0
        if r == 0:
            assert added.size == 0 and dropped.size == 0
        elif added.size:
            assert 2 * r > tile and added.size == tile - r
            rest = probs[~m0 & ~m1, e]
            if rest.size:
                assert probs[added, e].min() >= rest.max() * (1 - EPS), e
        else:
            assert dropped.size == r and (2 * r <= tile or T - c < tile - r)
            if m1.any():  # an expert with fewer than half a tile of tokens keeps none
                assert probs[dropped, e].max() <= probs[m1, e].min() * (1 + EPS), e


@pytest.mark.parametrize("cfg,tile", CASES, ids=[f"{c.name}_tile{t}" for c, t in CASES])
def test_rounded_small_all_tokens(cfg, tile):
    out, counts, rows = _run(cfg, tile)
    mask = rows >= 0
    assert np.all(counts % tile == 0)
    assert np.array_equal(counts, mask.sum(axis=0))
    r = gc.oracle_route(cfg)
    d = gc.on_device(gc.inputs(cfg))
    ids_gpu, _ = moe.route(d["x"], d["w_router"], cfg.k, bias=d["bias"])   # the routing the GPU rounded
    mask0 = np.zeros((cfg.T, cfg.E), bool)
    np.put_along_axis(mask0, ids_gpu.cpu().numpy().astype(np.int64), True, axis=1)
    _rule_holds(r.probs, mask0, mask, tile)
    o = gc.default_oracle()
    mask_o, counts_o = o.round_tokens(r.probs, r.ids, tile)
    same = np.all(mask == mask_o, axis=1)
    assert (~same).sum() <= max(2, cfg.T // 200), f"{(~same).sum()} tokens routed differently"
    inp = gc.inputs(cfg)
    rows_all = np.arange(cfg.T, dtype=np.int64)
    ref = o.masked_rows(inp.bits("x"), inp.bits("W_gate"), inp.bits("W_up"), inp.bits("W_down"), mask_o, r.probs,
                        rows_all)
    value_check(out[same], ref[same], f"out[{cfg.name}, rounded to {tile}]")


def test_rounded_tile_one_is_the_block():
    """Tile 1 rounds nothing: the routing is the top-k routing and the output
    is the block's (summed in expert order instead of slot order)."""
    cfg = CASES[0][0]
    out, counts, rows = _run(cfg, 1)
    r = gc.oracle_route(cfg)
    mask0 = np.zeros((cfg.T, cfg.E), bool)
    np.put_along_axis(mask0, r.ids.astype(np.int64), True, axis=1)
    excluded, _ = gc.near_tie_masks(cfg)
    assert np.array_equal((rows >= 0)[~excluded], mask0[~excluded])
    rows_all, ref = gc.oracle_rows(cfg, cfg.T)
    value_check(out[rows_all][~excluded[rows_all]], ref[~excluded[rows_all]], "out[tile 1]")


def test_rounded_qwen_full_size():
    """The Qwen3-shaped layer rounded to the 256-row GEMM tile: every count a
    multiple of 256; sampled tokens against the oracle."""
    cfg = CONFIGS["qwen"]
    out, counts, rows = _run(cfg, 256)
    assert np.all(counts % 256 == 0)
    r = gc.oracle_route(cfg)
    o = gc.default_oracle()
    mask_o, counts_o = o.round_tokens(r.probs, r.ids, 256)
    mask = rows >= 0
    same = np.all(mask == mask_o, axis=1)
    assert (~same).sum() <= cfg.T // 200
    sample = gc.sample_for(cfg, 96)
    sample = sample[same[sample]]
    inp = gc.inputs(cfg)
    ref = o.masked_rows(inp.bits("x"), inp.bits("W_gate"), inp.bits("W_up"), inp.bits("W_down"), mask_o, r.probs,
                        sample)
    value_check(out[sample], ref, "out[qwen, rounded to 256]")
