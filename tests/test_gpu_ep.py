"""The expert-parallel forward's CUDA stages on one GPU (a one-rank NCCL
group): the dispatch, regroup, local grouped GEMMs, return and combine give
the single-GPU forward's output bit for bit, and the row gather reports
out-of-range indices instead of faulting."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist

import top_routing_grouped_softmax_b200 as moe
from tests import gpu_cases as gc
from top_routing_grouped_softmax_b200.ep import ExpertParallelMoE

pytestmark = pytest.mark.gpu


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


@pytest.fixture(scope="module")
def one_rank_group():
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(_free_port()))
    torch.cuda.set_device(0)
    dist.init_process_group("nccl", rank=0, world_size=1, device_id=torch.device("cuda", 0))
    yield
    dist.destroy_process_group()


@pytest.mark.parametrize("cfg", [gc.small_cfg(600, 256, 16, 4, 320, sigma=0.1, skew=True),
                                 gc.small_cfg(1000, 512, 64, 8, 256, sigma=0.05)], ids=lambda c: c.name)
def test_ep_one_rank_equals_forward(one_rank_group, cfg):
    d = gc.on_device(gc.inputs(cfg))
    blk = ExpertParallelMoE(d["w_router"], d["w_gate"], d["w_up"], d["w_down"], cfg.k, bias=d["bias"])
    out_ep = blk.forward(d["x"])
    out = moe.forward(d["x"], d["w_router"], d["w_gate"], d["w_up"], d["w_down"], cfg.k, bias=d["bias"])
    torch.cuda.synchronize()
    assert moe.get_status() == moe.MOE_OK
    assert torch.equal(out_ep, out)


def test_gather_rows_wide_and_narrow():
    src = torch.arange(40 * 16, dtype=torch.float32, device="cuda").view(40, 16)
    idx = torch.tensor([3, 0, 39, 7], dtype=torch.int32, device="cuda")
    assert torch.equal(moe.gather_rows(src, idx), src[idx.long()])
    w = torch.arange(40, dtype=torch.float32, device="cuda")
    assert torch.equal(moe.gather_rows(w, idx), w[idx.long()])
    bad = torch.tensor([1, 40], dtype=torch.int32, device="cuda")
    got = moe.gather_rows(src, bad)
    torch.cuda.synchronize()
    assert moe.get_status() == moe.MOE_ERR_DEVICE_BOUNDS
    assert torch.equal(got[0], src[1]) and not got[1].any().item()
