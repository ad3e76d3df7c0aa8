"""Expert parallelism's host logic on CPU ranks (gloo, world size 2): the
count exchange, the split sizes, the regroup / ungroup permutations and the
reassembly give each rank's tokens the rows a single-process forward gives.

The library's kernels need a GPU, so the stages here are CPU stand-ins (the
fp64 oracle's routing and grouping, numpy expert MLPs); the orchestration in
top_routing_grouped_softmax_b200.ep is the product code under test."""
import os

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from top_routing_grouped_softmax_b200.ep import ExpertParallelMoE, owner_block, plan_dispatch


def _widen(t):
    """bf16 torch tensor -> float64 numpy, exactly."""
    return t.to(torch.float64).numpy()


class CpuStages:
    """Test stand-ins for the kernels: fp64 routing / grouping from the oracle
    and numpy SwiGLU experts; y rows stay fp64."""

    y_dtype = torch.float64

    def __init__(self, oracle, E_total):
        self.o = oracle
        self.E_total = E_total

    def route(self, x, w_router, k, bias):
        from top_routing_grouped_softmax_b200.synth import bf16_bits
        r = self.o.route(bf16_bits(x), bf16_bits(w_router), None if bias is None else bias.numpy(), k)
        return torch.from_numpy(r.ids), torch.from_numpy(r.weights)

    def permute(self, x, ids, w, E):
        pr = self.o.permute(ids.numpy(), E)
        k = ids.shape[1]
        tok = torch.from_numpy(pr.perm.astype(np.int64) // k)
        return {"counts": torch.from_numpy(pr.counts), "offsets": torch.from_numpy(pr.offsets),
                "inv": torch.from_numpy(pr.inv), "x_perm": x[tok].contiguous(),
                "w_perm": w.reshape(-1)[torch.from_numpy(pr.perm.astype(np.int64))].contiguous()}

    def gather_rows(self, src, idx):
        return src[idx.to(torch.int64)].contiguous()

    def expert_ffn(self, x_rows, w_rows, offsets, w_gate, w_up, w_down):
        X = _widen(x_rows)
        Wg, Wu, Wd = _widen(w_gate), _widen(w_up), _widen(w_down)
        off = offsets.numpy()
        y = np.zeros((X.shape[0], Wd.shape[2]))
        for e in range(Wg.shape[0]):
            a, b = int(off[e]), int(off[e + 1])
            if b > a:
                g = X[a:b] @ Wg[e]
                u = X[a:b] @ Wu[e]
                y[a:b] = (g / (1.0 + np.exp(-g)) * u) @ Wd[e]
        return torch.from_numpy(y * w_rows.numpy().astype(np.float64)[:, None])

    def combine(self, y, inv, T, k):
        Y = y.numpy()
        idx = inv.numpy().astype(np.int64).reshape(T, k)
        out = np.zeros((T, Y.shape[1]))
        for j in range(k):
            out += Y[idx[:, j]]
        return torch.from_numpy(out)


def _inputs():
    from top_routing_grouped_softmax_b200.synth import MoEConfig, make_inputs
    cfg = MoEConfig("ep", T=96, d=64, E=8, k=2, f=48, sigma=0.2, seed=21, skew=True)
    return cfg, make_inputs(cfg)


def _token_ranges(T, world, uneven):
    """Each rank's token slice: equal shares, uneven ones (rank r gets r + 1
    parts) so that ranks send and receive different row counts, or
    ("empty") every token on rank 0 and none on the others."""
    if uneven == "empty":
        return [(0, T)] + [(T, T)] * (world - 1)
    w = [r + 1 for r in range(world)] if uneven else [1] * world
    cuts = [0]
    for r in range(world):
        cuts.append(cuts[-1] + T * w[r] // sum(w) if r < world - 1 else T)
    return [(cuts[r], cuts[r + 1]) for r in range(world)]


def _cold_bias(cfg):
    """A router bias that no expert of the upper half survives: their owner
    ranks receive no rows at all."""
    b = torch.zeros(cfg.E, dtype=torch.float32)
    b[cfg.E // 2:] = -1.0e4
    return b


def _worker(rank, world, port, q, uneven=False, cold=False):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    from oracle.oracle import default_oracle
    cfg, inp = _inputs()
    if cold:
        inp.bias = _cold_bias(cfg)
    e0, e1 = owner_block(cfg.E, world, rank)
    t0, t1 = _token_ranges(cfg.T, world, uneven)[rank]
    x = inp.x[t0:t1].contiguous()
    blk = ExpertParallelMoE(inp.W_router, inp.W_gate[e0:e1].contiguous(), inp.W_up[e0:e1].contiguous(),
                            inp.W_down[e0:e1].contiguous(), cfg.k, bias=inp.bias,
                            stages=CpuStages(default_oracle(), cfg.E))
    out = blk.forward(x).numpy()
    plan = blk.last_plan
    dist.barrier()
    dist.destroy_process_group()
    q.put((rank, out, plan.recv_counts, plan.offsets))


def _run_ranks(world, port, uneven, cold=False):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q, uneven, cold)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted((q.get(timeout=150) for _ in range(world)), key=lambda r: r[0])
    for p in procs:
        p.join(timeout=30)
        assert p.exitcode == 0
    return res


def _single_process_reference(cold=False):
    from oracle.oracle import default_oracle
    cfg, inp = _inputs()
    if cold:
        inp.bias = _cold_bias(cfg)
    st = CpuStages(default_oracle(), cfg.E)
    ids, w = st.route(inp.x, inp.W_router, cfg.k, inp.bias)
    pm = st.permute(inp.x, ids, w, cfg.E)
    y = st.expert_ffn(pm["x_perm"], pm["w_perm"], pm["offsets"], inp.W_gate, inp.W_up, inp.W_down)
    return cfg, ids.numpy(), st.combine(y, pm["inv"], cfg.T, cfg.k).numpy()


@pytest.mark.timeout(240)
def test_four_ranks_uneven_tokens_match_single_process():
    """Four ranks (two experts each) with uneven token shares: different
    send and receive counts on every rank; the outputs still equal the
    single-process forward, rank by rank."""
    world = 4
    res = _run_ranks(world, 29541, uneven=True)
    cfg, ids, ref = _single_process_reference()
    counts = np.bincount(ids.ravel(), minlength=cfg.E)
    for (rank, out, recv_counts, offsets), (t0, t1) in zip(res, _token_ranges(cfg.T, world, True)):
        np.testing.assert_allclose(out, ref[t0:t1], rtol=1e-12, atol=1e-14)
        e0, e1 = owner_block(cfg.E, world, rank)
        assert recv_counts.shape == (world, e1 - e0)
        assert recv_counts.sum(axis=0).tolist() == counts[e0:e1].tolist()


@pytest.mark.timeout(240)
def test_rank_without_tokens():
    """A rank with no tokens of its own still serves its experts: it sends
    nothing, receives rank 0's rows for its experts, and returns an empty
    output; rank 0's output equals the single-process forward."""
    world = 2
    res = _run_ranks(world, 29547, uneven="empty")
    cfg, ids, ref = _single_process_reference()
    counts = np.bincount(ids.ravel(), minlength=cfg.E)
    (r0, out0, rc0, _), (r1, out1, rc1, off1) = res
    np.testing.assert_allclose(out0, ref, rtol=1e-12, atol=1e-14)
    assert out1.shape == (0, cfg.d)
    e0, e1 = owner_block(cfg.E, world, 1)
    assert rc1[1].sum() == 0 and rc1[0].tolist() == counts[e0:e1].tolist()
    assert off1[-1] == counts[e0:e1].sum()


@pytest.mark.timeout(240)
def test_rank_whose_experts_get_no_rows():
    """No token picks the experts of rank 1: it receives nothing, computes
    nothing, and the return exchange still delivers every rank's rows."""
    world = 2
    res = _run_ranks(world, 29551, uneven=False, cold=True)
    cfg, ids, ref = _single_process_reference(cold=True)
    assert ids.max() < cfg.E // 2
    for (rank, out, recv_counts, offsets), (t0, t1) in zip(res, _token_ranges(cfg.T, world, False)):
        np.testing.assert_allclose(out, ref[t0:t1], rtol=1e-12, atol=1e-14)
        if rank == 1:
            assert recv_counts.sum() == 0 and offsets[-1] == 0


@pytest.mark.timeout(180)
def test_two_rank_expert_parallel_matches_single_process():
    world, port = 2, 29533
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted((q.get(timeout=150) for _ in range(world)), key=lambda r: r[0])
    for p in procs:
        p.join(timeout=30)
        assert p.exitcode == 0
    # the single-process forward with the same stand-ins, all experts local
    from oracle.oracle import default_oracle
    cfg, inp = _inputs()
    st = CpuStages(default_oracle(), cfg.E)
    ids, w = st.route(inp.x, inp.W_router, cfg.k, inp.bias)
    pm = st.permute(inp.x, ids, w, cfg.E)
    y = st.expert_ffn(pm["x_perm"], pm["w_perm"], pm["offsets"], inp.W_gate, inp.W_up, inp.W_down)
    ref = st.combine(y, pm["inv"], cfg.T, cfg.k).numpy()
    T_r = cfg.T // world
    counts = np.bincount(ids.numpy().ravel(), minlength=cfg.E)
    for rank, out, recv_counts, offsets in res:
        np.testing.assert_allclose(out, ref[rank * T_r:(rank + 1) * T_r], rtol=1e-12, atol=1e-14)
        e0, e1 = owner_block(cfg.E, world, rank)
        # every row of this rank's experts arrived, from both sources
        assert recv_counts.sum(axis=0).tolist() == counts[e0:e1].tolist()
        assert offsets[-1] == counts[e0:e1].sum()


def test_plan_dispatch_permutations():
    c = np.array([[2, 0, 3], [1, 4, 0]])      # 2 sources x 3 local experts
    p = plan_dispatch(c)
    # received, source-major: s0e0 (rows 0-1), s0e2 (2-4), s1e0 (5), s1e1 (6-9)
    # grouped, expert-major: e0 = s0 rows 0-1 then s1 row 5; e1 = 6-9; e2 = 2-4
    assert p.regroup.tolist() == [0, 1, 5, 6, 7, 8, 9, 2, 3, 4]
    assert p.offsets.tolist() == [0, 3, 7, 10]
    assert np.array_equal(p.regroup[p.ungroup], np.arange(10))
    assert np.array_equal(p.ungroup[p.regroup], np.arange(10))
    empty = plan_dispatch(np.zeros((3, 2), dtype=np.int64))
    assert empty.regroup.size == 0 and empty.offsets.tolist() == [0, 0, 0]


def test_owner_blocks_cover_the_experts():
    assert [owner_block(128, 8, r) for r in (0, 7)] == [(0, 16), (112, 128)]
    with pytest.raises(ValueError):
        owner_block(12, 8, 0)
