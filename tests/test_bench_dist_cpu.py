"""The benchmark's multi-process host logic on CPU ranks (gloo, world size 2):
per-rank replica seeds, and the whole-job rate taken over the slowest rank."""
import os

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    r, local, w = bench.dist_env()
    assert (r, local, w) == (rank, rank, world)
    seed = bench.replica_seed(1, r)
    seeds = [None] * world
    dist.all_gather_object(seeds, seed)
    # each rank "takes" a different time; the job rate uses the slowest
    t = torch.tensor([0.5 + rank], dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    rate = bench.whole_job_rate(1000, w, [t.item()])
    dist.barrier()
    dist.destroy_process_group()
    q.put((rank, seeds, t.item(), rate))


@pytest.mark.timeout(120)
def test_two_rank_replicas_gloo():
    world, port = 2, 29517
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=90) for _ in range(world))
    for p in procs:
        p.join(timeout=30)
        assert p.exitcode == 0
    for rank, seeds, tmax, rate in res:
        assert seeds == [1, 1001]            # distinct replicas
        assert tmax == 1.5                   # max over ranks
        assert rate == pytest.approx(2000 / 1.5)


def test_single_process_env_defaults(monkeypatch):
    for k in ("WORLD_SIZE", "RANK", "LOCAL_RANK"):
        monkeypatch.delenv(k, raising=False)
    assert bench.dist_env() == (0, 0, 1)
    assert bench.whole_job_rate(10, 1, [2.0]) == 5.0


def test_algorithmic_counts():
    from top_routing_grouped_softmax_b200.synth import CONFIGS
    a = bench.algorithmic(CONFIGS["qwen"])
    assert a["flops"] == 2 * 8192 * (2048 * 128 + 3 * 8 * 2048 * 768)
    assert a["gateup_flops"] + a["down_flops"] + 2 * 8192 * 2048 * 128 == a["flops"]


def test_peaks_source(monkeypatch, tmp_path):
    """The roofline denominators come from the peaks file when it exists and
    are labelled as the fallback figures when it does not."""
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    p = bench.load_peaks()
    assert p["source"] == "fallback"
    assert p["bf16_tflops"] == bench.FALLBACK_PEAKS["bf16_tflops"]
    (tmp_path / "MEASURED_PEAKS.json").write_text('{"hbm_gbs": 6554.6, "bf16_tflops": 1657.0}')
    p = bench.load_peaks()
    assert p == {"hbm_gbs": 6554.6, "bf16_tflops": 1657.0, "bf16_tflops_sustained": 1657.0, "source": "measured"}
