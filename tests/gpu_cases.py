"""Shared helpers for the GPU parity tests: seeded inputs on the device and
cached oracle results (the oracle is slow, so each configuration's routing
and sampled expert rows are computed once per session)."""
from __future__ import annotations

import functools

import numpy as np
import torch

from oracle.oracle import default_oracle
from top_routing_grouped_softmax_b200.synth import CONFIGS, MoEConfig, make_inputs, sample_tokens


def small_cfg(T, d, E, k, f, seed=7, skew=False, sigma=0.02):
    return MoEConfig(f"T{T}_d{d}_E{E}_k{k}_f{f}", T=T, d=d, E=E, k=k, f=f, sigma=sigma, seed=seed, skew=skew)


@functools.lru_cache(maxsize=4)
def inputs(cfg: MoEConfig):
    return make_inputs(cfg)


def on_device(inp):
    dev = torch.device("cuda")
    return {
        "x": inp.x.to(dev), "w_router": inp.W_router.to(dev), "w_gate": inp.W_gate.to(dev),
        "w_up": inp.W_up.to(dev), "w_down": inp.W_down.to(dev),
        "bias": None if inp.bias is None else inp.bias.to(dev),
    }


@functools.lru_cache(maxsize=4)
def logit_error(cfg: MoEConfig):
    """logit_error_bound of a configuration's inputs: from
    sum_i |x[t, i]| |W_router[i, e]| + |b_e| in fp64 ([T, E])."""
    from tests.parity import logit_error_bound, widen
    inp = inputs(cfg)
    ax = np.abs(widen(inp.bits("x")).reshape(cfg.T, cfg.d))
    aw = np.abs(widen(inp.bits("W_router")).reshape(cfg.d, cfg.E))
    scale = ax @ aw
    b = inp.bias_np()
    if b is not None:
        scale += np.abs(b.astype(np.float64))[None, :]
    return logit_error_bound(scale, cfg.d)


@functools.lru_cache(maxsize=8)
def oracle_route(cfg: MoEConfig):
    inp = inputs(cfg)
    return default_oracle().route(inp.bits("x"), inp.bits("W_router"), inp.bias_np(), cfg.k)


def sample_for(cfg: MoEConfig, n: int):
    """Sampled tokens, always including one token of the largest and of the
    smallest non-empty expert group, and, for every non-empty expert, the
    last token routed to it.  Groups list their tokens in ascending order, so
    that token's grouped row is the group's last row: it lies in the group's
    last (usually partial) 256-row GEMM tile, where the epilogue masks the
    rows past the group's end."""
    r = oracle_route(cfg)
    counts = np.bincount(r.ids.ravel(), minlength=cfg.E)
    big = int(np.argmax(counts))
    nz = np.nonzero(counts)[0]
    small = int(nz[np.argmin(counts[nz])])
    t_big = int(np.nonzero((r.ids == big).any(axis=1))[0][0])
    t_small = int(np.nonzero((r.ids == small).any(axis=1))[0][0])
    last = [int(np.nonzero((r.ids == e).any(axis=1))[0][-1]) for e in nz]
    return sample_tokens(cfg.T, n, cfg.seed, must_include=(t_big, t_small, 0, cfg.T - 1, *last))


def expert_rows_parallel(inp, ids, weights, rows, workers: int = 0):
    """The oracle's expert rows for ``rows``, evaluated in chunks on host
    threads.  The oracle is single-threaded C called through ctypes (which
    releases the GIL) and keeps no global state, so chunks run side by side;
    each row is computed exactly as in one call, so the result is identical."""
    import os
    from concurrent.futures import ThreadPoolExecutor
    o = default_oracle()
    args = (inp.bits("x"), inp.bits("W_gate"), inp.bits("W_up"), inp.bits("W_down"))
    workers = workers or max(1, min(16, (os.cpu_count() or 1)))
    chunks = [c for c in np.array_split(np.asarray(rows, dtype=np.int64), workers) if c.size]
    if len(chunks) <= 1:
        return o.expert_rows(*args, ids, weights, rows).out
    with ThreadPoolExecutor(max_workers=len(chunks)) as pool:
        parts = list(pool.map(lambda c: o.expert_rows(*args, ids, weights, c).out, chunks))
    return np.concatenate(parts, axis=0)


@functools.lru_cache(maxsize=8)
def oracle_rows(cfg: MoEConfig, n: int):
    inp = inputs(cfg)
    r = oracle_route(cfg)
    rows = sample_for(cfg, n)
    return rows, expert_rows_parallel(inp, r.ids, r.weights, rows)


SAMPLES = {"tiny": 256, "qwen": 384, "fine": 384, "coarse": 160, "skew": 256}
FULL = [CONFIGS[n] for n in ("tiny", "qwen", "fine", "coarse", "skew")]


def near_tie_masks(cfg: MoEConfig):
    """(excluded, inner) token masks of the oracle routing: a k-th / (k+1)-th
    probability gap below the tie threshold (left out), and a near tie
    inside the selected set (ids compared as a set)."""
    from oracle.oracle import inner_gap, topk_gap
    from tests.parity import TIE_EPS
    probs = oracle_route(cfg).probs
    excluded = topk_gap(probs, cfg.k) < TIE_EPS
    inner = (inner_gap(probs, cfg.k) < TIE_EPS) & ~excluded
    return excluded, inner
