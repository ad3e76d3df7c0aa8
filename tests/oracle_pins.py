"""Checks that pin the fp64 oracle to computations other than itself.

Each ``check_*`` function takes an ``Oracle`` handle and raises
AssertionError on a mismatch.  test_oracle_pins.py runs them on the real
oracle; test_oracle_mutants.py runs them on copies of the oracle with a
planted mistake and requires that at least one check fails for every mutant.

The independent computations used here:
  * a dense brute force: every expert evaluated for every token with numpy
    matmuls, masked by a one-hot of the top-k chosen by numpy's lexsort over
    scipy's softmax, weighted and summed -- a different algorithm from the
    oracle's sparse per-token loop;
  * library routines for single steps: numpy matmul, scipy.special.softmax,
    scipy.special.expit (for silu(z) = z * expit(z)), numpy's stable argsort;
  * special cases with closed forms: E = 1, k = 1 is a dense SwiGLU MLP;
    k = E with identical experts is that MLP times sum(p) = 1; exact ties;
  * invariants: counts sum to T*k, the permutation is a bijection, etc.;
  * for the backward: torch autograd through an fp64 torch rendering of the
    forward (a library differentiator, independent of the oracle's
    hand-derived chain rule), central finite differences of a numpy forward
    that is itself checked against the oracle's forward, and the softmax
    gradient's zero sum over experts.
"""
from __future__ import annotations

import numpy as np
import scipy.special as sps
import torch

from top_routing_grouped_softmax_b200.synth import bf16_bits, make_inputs


def widen(bits: np.ndarray) -> np.ndarray:
    """bf16 bit patterns -> float64, exactly."""
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def _rand_case(T, d, E, k, f, seed, bias=False, sigma=0.05):
    from top_routing_grouped_softmax_b200.synth import MoEConfig
    cfg = MoEConfig("pin", T=T, d=d, E=E, k=k, f=f, sigma=sigma, seed=seed, skew=bias)
    return make_inputs(cfg)


def _args(inp):
    return (inp.bits("x"), inp.bits("W_router"), inp.bias_np(), inp.bits("W_gate"),
            inp.bits("W_up"), inp.bits("W_down"))


def dense_reference(x, wr, bias, wg, wu, wd, k):
    """Brute force: evaluate all E experts densely, mask with one-hot top-k."""
    X, Wr = widen(x), widen(wr)
    Wg, Wu, Wd = widen(wg), widen(wu), widen(wd)
    T = X.shape[0]
    E = Wr.shape[1]
    logits = X @ Wr
    if bias is not None:
        logits = logits + bias.astype(np.float64)[None, :]
    p = sps.softmax(logits, axis=1)
    idx = np.broadcast_to(np.arange(E), (T, E))
    order = np.lexsort((idx, -p), axis=1)       # primary -p, then index
    top = order[:, :k]
    mask = np.zeros((T, E))
    np.put_along_axis(mask, top, 1.0, axis=1)
    out = np.zeros((T, X.shape[1]))
    for e in range(E):
        G = X @ Wg[e]
        U = X @ Wu[e]
        H = G * sps.expit(G) * U
        out += (mask[:, e] * p[:, e])[:, None] * (H @ Wd[e])
    return out, p, top, logits


def _rel(a, b):
    scale = max(np.sqrt(np.mean(b * b)), 1e-300)
    return float(np.max(np.abs(a - b)) / scale)


# ---------------------------------------------------------------------------
def check_brute_force(o):
    for (T, d, E, k, f, seed, bias) in [(48, 64, 8, 2, 32, 11, False), (33, 32, 5, 3, 48, 12, True),
                                        (64, 96, 8, 1, 64, 13, False), (17, 64, 4, 4, 16, 14, True)]:
        inp = _rand_case(T, d, E, k, f, seed, bias=bias)
        r, ex = o.forward(*_args(inp), k)
        ref, p, top, _ = dense_reference(*_args(inp), k)
        assert _rel(ex.out, ref) < 1e-10, ("brute force", T, d, E, k, f)
        assert np.array_equal(r.ids, top), "top-k ids differ from lexsort"


def check_softmax_library(o):
    inp = _rand_case(40, 64, 16, 4, 16, 21, bias=True, sigma=0.3)
    r = o.route(inp.bits("x"), inp.bits("W_router"), inp.bias_np(), 4, want_logits=True)
    logits = widen(inp.bits("x")) @ widen(inp.bits("W_router")) + inp.bias_np().astype(np.float64)
    assert np.allclose(r.logits, logits, rtol=1e-12, atol=1e-12), "logits != x @ Wr + b"
    assert np.allclose(r.probs, sps.softmax(logits, axis=1), rtol=1e-12, atol=1e-15), "softmax"
    assert np.allclose(r.probs.sum(axis=1), 1.0, atol=1e-14)


def check_topk_library_sort(o):
    inp = _rand_case(64, 64, 32, 6, 16, 22, sigma=0.2)
    r = o.route(inp.bits("x"), inp.bits("W_router"), None, 6)
    p = r.probs
    T, E = p.shape
    order = np.lexsort((np.broadcast_to(np.arange(E), (T, E)), -p), axis=1)[:, :6]
    assert np.array_equal(r.ids, order), "top-k ids"
    assert np.array_equal(r.weights, np.take_along_axis(p, r.ids.astype(np.int64), 1)), \
        "weights are not the softmax entries at the selected ids (renormalised?)"
    assert np.all(np.diff(r.weights, axis=1) <= 0), "slots not in descending probability"
    for t in range(T):
        assert len(set(r.ids[t].tolist())) == 6, "duplicate expert in one token"


def check_topk_of_logits(o):
    """Softmax is monotone: top-k of the logits picks the same experts."""
    inp = _rand_case(64, 64, 16, 3, 16, 23, bias=True, sigma=0.2)
    r = o.route(inp.bits("x"), inp.bits("W_router"), inp.bias_np(), 3, want_logits=True)
    T, E = r.logits.shape
    order = np.lexsort((np.broadcast_to(np.arange(E), (T, E)), -r.logits), axis=1)[:, :3]
    assert np.array_equal(np.sort(r.ids, 1), np.sort(order, 1)), "topk(logits) != topk(p)"


def check_exact_ties(o):
    """All router columns identical: p = 1/E exactly, ids are 0..k-1."""
    inp = _rand_case(16, 32, 8, 3, 16, 24)
    wr = inp.bits("W_router").copy()
    wr[:, :] = wr[:, :1]
    r = o.route(inp.bits("x"), wr, None, 3)
    assert np.all(r.ids == np.arange(3)[None, :]), "tie-break is not lowest index first"
    assert np.all(r.weights == 0.125), "equal logits must give p = 1/E"
    # a two-way tie at the top: columns 5 and 2 equal and largest
    wr = np.zeros((32, 8), np.uint16)
    one = np.uint16(0x3F80)       # bf16 1.0
    half = np.uint16(0x3F00)      # bf16 0.5
    wr[0, 5] = one
    wr[0, 2] = one
    wr[0, 7] = half
    xb = np.zeros((4, 32), np.uint16)
    xb[:, 0] = one
    r = o.route(xb, wr, None, 3)
    assert np.all(r.ids == np.array([2, 5, 7])[None, :]), r.ids


def check_dense_special_case(o):
    """E = 1, k = 1: p = 1 exactly and the block is one dense SwiGLU MLP."""
    inp = _rand_case(24, 64, 1, 1, 96, 25)
    r, ex = o.forward(*_args(inp), 1)
    assert np.all(r.ids == 0) and np.all(r.weights == 1.0)
    X = widen(inp.bits("x"))
    G = X @ widen(inp.bits("W_gate"))[0]
    U = X @ widen(inp.bits("W_up"))[0]
    ref = (G * sps.expit(G) * U) @ widen(inp.bits("W_down"))[0]
    assert _rel(ex.out, ref) < 1e-12, "E=1,k=1 != dense SwiGLU"


def check_all_experts_identical(o):
    """k = E with every expert identical: out = MLP(x) * sum_e p_e = MLP(x)."""
    inp = _rand_case(20, 32, 4, 4, 48, 26)
    wg, wu, wd = inp.bits("W_gate").copy(), inp.bits("W_up").copy(), inp.bits("W_down").copy()
    wg[:] = wg[0]
    wu[:] = wu[0]
    wd[:] = wd[0]
    r, ex = o.forward(inp.bits("x"), inp.bits("W_router"), None, wg, wu, wd, 4)
    X = widen(inp.bits("x"))
    G = X @ widen(wg[0])
    U = X @ widen(wu[0])
    ref = (G * sps.expit(G) * U) @ widen(wd[0])
    assert _rel(ex.out, ref) < 1e-12, "k=E identical experts != MLP(x)"


def check_zero_expert(o):
    """An expert with W_down = 0 contributes nothing; unselected experts are inert."""
    inp = _rand_case(40, 64, 8, 2, 32, 27)
    x, wr, _, wg, wu, wd = _args(inp)
    r, ex = o.forward(x, wr, None, wg, wu, wd, 2)
    wd0 = wd.copy()
    wd0[3] = 0
    r0, ex0 = o.forward(x, wr, None, wg, wu, wd0, 2)
    ref, p, top, _ = dense_reference(x, wr, None, wg, wu, wd, 2)
    # remove expert 3's term from the brute force
    X = widen(x)
    G = X @ widen(wg[3])
    U = X @ widen(wu[3])
    term = ((top == 3).any(axis=1) * p[:, 3])[:, None] * ((G * sps.expit(G) * U) @ widen(wd[3]))
    assert _rel(ex0.out, ref - term) < 1e-10, "zeroed expert still contributes"
    # change the weights of an expert that no token selects: bit-identical out
    # a strongly negative bias keeps expert 6 out of every token's top-k
    bias = np.zeros(8, np.float32)
    bias[6] = -1.0e4
    r, ex = o.forward(x, wr, bias, wg, wu, wd, 2)
    assert 6 not in set(r.ids.ravel().tolist())
    e = 6
    wg2, wu2, wd2 = wg.copy(), wu.copy(), wd.copy()
    wg2[e] = wg2[(e + 1) % 8]
    wu2[e] = 0
    wd2[e] = wd2[(e + 2) % 8]
    _, ex2 = o.forward(x, wr, bias, wg2, wu2, wd2, 2)
    assert np.array_equal(ex2.out, ex.out), "unselected expert changed the output"


def check_scale_down(o):
    """Doubling W_down (exact in bf16) doubles the output exactly."""
    inp = _rand_case(16, 64, 8, 2, 32, 28)
    x, wr, _, wg, wu, wd = _args(inp)
    _, ex = o.forward(x, wr, None, wg, wu, wd, 2)
    wd2 = bf16_bits(torch.from_numpy(widen(wd).astype(np.float32) * 2).to(torch.bfloat16))
    _, ex2 = o.forward(x, wr, None, wg, wu, wd2, 2)
    assert np.array_equal(ex2.out, 2.0 * ex.out), "2*W_down did not double out"


def check_permute_library(o):
    """Grouping equals numpy's stable argsort of the flat expert ids."""
    rng = np.random.default_rng(5)
    for (T, E, k) in [(100, 8, 2), (257, 16, 4), (1, 4, 4), (64, 32, 1)]:
        ids = np.stack([rng.permutation(E)[:k] for _ in range(T)]).astype(np.int32)
        pr = o.permute(ids, E)
        flat = ids.ravel()
        assert np.array_equal(pr.counts, np.bincount(flat, minlength=E))
        assert pr.offsets[0] == 0 and pr.offsets[-1] == T * k
        assert np.all(np.diff(pr.offsets) >= 0)
        assert np.array_equal(pr.perm, np.argsort(flat, kind="stable")), "not a stable grouping"
        assert np.array_equal(np.sort(pr.perm), np.arange(T * k)), "perm not a bijection"
        assert np.array_equal(pr.inv[pr.perm], np.arange(T * k)), "inv o perm != id"
        for e in range(E):
            seg = pr.perm[pr.offsets[e]:pr.offsets[e + 1]]
            assert np.all(flat[seg] == e)


def check_expert_rows_outputs(o):
    """y and h side outputs agree with the dense pieces for each slot."""
    inp = _rand_case(12, 32, 4, 2, 40, 30)
    x, wr, _, wg, wu, wd = _args(inp)
    r = o.route(x, wr, None, 2)
    rows = np.array([0, 5, 11])
    ex = o.expert_rows(x, wg, wu, wd, r.ids, r.weights, rows, want_y=True, want_h=True)
    X = widen(x)
    for i, t in enumerate(rows):
        for j in range(2):
            e = r.ids[t, j]
            g = X[t] @ widen(wg[e])
            u = X[t] @ widen(wu[e])
            h = g * sps.expit(g) * u
            assert np.allclose(ex.h[i, j], h, rtol=1e-12, atol=1e-14)
            assert np.allclose(ex.y[i, j], r.weights[t, j] * (h @ widen(wd[e])), rtol=1e-12, atol=1e-15)
        assert np.allclose(ex.out[i], ex.y[i].sum(axis=0), rtol=1e-13, atol=1e-15)


def check_renormalize(o):
    """Renormalised routing weights equal a softmax over the k selected
    logits only (scipy, from the numpy logits) -- a different formula for
    the same quantity; they sum to one; with k = E they are the plain
    probabilities; the selected ids do not change."""
    inp = _rand_case(48, 64, 16, 4, 32, seed=31, bias=True)
    x, wr, b = inp.bits("x"), inp.bits("W_router"), inp.bias_np()
    plain = o.route(x, wr, b, 4)
    r = o.route(x, wr, b, 4, renormalize=True)
    assert np.array_equal(r.ids, plain.ids)
    logits = widen(x) @ widen(wr) + b.astype(np.float64)[None, :]
    sel = np.take_along_axis(logits, r.ids.astype(np.int64), axis=1)
    np.testing.assert_allclose(r.weights, sps.softmax(sel, axis=1), rtol=1e-12, atol=0)
    np.testing.assert_allclose(r.weights.sum(axis=1), 1.0, rtol=0, atol=1e-14)
    full = o.route(x, wr, b, 16, renormalize=True)
    np.testing.assert_allclose(full.weights, o.route(x, wr, b, 16).weights, rtol=1e-14, atol=0)


def check_shared_experts(o):
    """Shared experts: the oracle's output equals the dense brute force plus
    every shared SwiGLU evaluated densely with numpy matmuls (weight one);
    zero shared down-projections leave the output bit-identical."""
    from top_routing_grouped_softmax_b200.synth import MoEConfig, make_shared_weights
    inp = _rand_case(40, 64, 8, 2, 32, seed=41, bias=True)
    sw = make_shared_weights(MoEConfig("pin", T=40, d=64, E=8, k=2, f=32, sigma=0.05, seed=41), 2, 48)
    shared = tuple(bf16_bits(sw[n]) for n in ("W_gate_s", "W_up_s", "W_down_s"))
    x = inp.bits("x")
    _, ex = o.forward(*_args(inp), 2, shared=shared)
    ref, _, _, _ = dense_reference(*_args(inp), 2)
    X = widen(x)
    for s_idx in range(2):
        G = X @ widen(shared[0][s_idx])
        U = X @ widen(shared[1][s_idx])
        ref = ref + (G * sps.expit(G) * U) @ widen(shared[2][s_idx])
    assert _rel(ex.out, ref) < 1e-12, _rel(ex.out, ref)
    zero = (shared[0], shared[1], np.zeros_like(shared[2]))
    _, ex0 = o.forward(*_args(inp), 2, shared=zero)
    _, plain = o.forward(*_args(inp), 2)
    assert np.array_equal(ex0.out, plain.out)


def _rounding_ok(probs, mask0, mask, tile):
    """Order-statistic characterisation of token rounding, expert by expert:
    the count becomes a multiple of the tile; a dropped token ranks below
    every kept one by (p, then the smaller index kept); an added token ranks
    above every unrouted one left out (p, then the smaller index added)."""
    T, E = probs.shape
    for e in range(E):
        m0, m1 = mask0[:, e], mask[:, e]
        c, r = int(m0.sum()), int(m0.sum()) % tile
        n = int(m1.sum())
        added, dropped = np.nonzero(m1 & ~m0)[0], np.nonzero(m0 & ~m1)[0]
        assert added.size == 0 or dropped.size == 0, f"expert {e} both gains and loses tokens"
        if r == 0:
            assert n == c
            continue
        if added.size:
            assert 2 * r > tile and n == c + tile - r, (e, c, n)
            rest = np.nonzero(~m0 & ~m1)[0]
            for a in added:
                assert np.all((probs[a, e] > probs[rest, e]) | ((probs[a, e] == probs[rest, e]) & (a < rest)))
        else:
            assert (2 * r <= tile or T - c < tile - r) and n == c - r, (e, c, n)
            kept = np.nonzero(m1)[0]
            for dd in dropped:
                assert np.all((probs[dd, e] < probs[kept, e]) | ((probs[dd, e] == probs[kept, e]) & (dd > kept)))


def check_token_rounding(o):
    """Token rounding: tile 1 changes nothing; on random routing every
    expert's count becomes a tile multiple by the order-statistic rule; the
    masked block output equals a dense numpy evaluation with the rounded
    mask; exact ties drop the larger and add the smaller token index."""
    inp = _rand_case(300, 64, 8, 2, 32, seed=53, bias=True)
    x, wr, b = inp.bits("x"), inp.bits("W_router"), inp.bias_np()
    r = o.route(x, wr, b, 2)
    mask0 = np.zeros((300, 8), bool)
    np.put_along_axis(mask0, r.ids.astype(np.int64), True, axis=1)
    same, c1 = o.round_tokens(r.probs, r.ids, 1)
    assert np.array_equal(same, mask0) and np.array_equal(c1, mask0.sum(0))
    for tile in (16, 48):
        mask, counts = o.round_tokens(r.probs, r.ids, tile)
        assert np.array_equal(counts, mask.sum(0))
        _rounding_ok(r.probs, mask0, mask, tile)
    mask, _ = o.round_tokens(r.probs, r.ids, 16)
    rows = np.arange(300, dtype=np.int64)
    got = o.masked_rows(x, inp.bits("W_gate"), inp.bits("W_up"), inp.bits("W_down"), mask, r.probs, rows)
    X = widen(x)
    ref = np.zeros_like(got)
    for e in range(8):
        G = X @ widen(inp.bits("W_gate")[e])
        U = X @ widen(inp.bits("W_up")[e])
        ref += (mask[:, e] * r.probs[:, e])[:, None] * ((G * sps.expit(G) * U) @ widen(inp.bits("W_down")[e]))
    assert _rel(got, ref) < 1e-12, _rel(got, ref)
    # exact ties: tokens 0..19 prefer expert 0, tokens 20..39 expert 1, all
    # with the same probability pair
    T = 40
    v = widen(inp.bits("x")[0, :64])
    xs = np.vstack([np.tile(v, (20, 1)), np.tile(-v, (20, 1))])
    wcol = widen(inp.bits("W_router")[:, 0])
    wr2 = np.stack([wcol, -wcol], axis=1)
    xb, wb = bf16_bits(torch.from_numpy(xs).to(torch.bfloat16)), bf16_bits(torch.from_numpy(wr2).to(torch.bfloat16))
    rt = o.route(xb, wb, None, 1)
    assert set(rt.ids[:20, 0]) == {0} and set(rt.ids[20:, 0]) == {1}
    m16, _ = o.round_tokens(rt.probs, rt.ids, 16)      # 20 each, r = 4: drop the 4 largest indices
    assert np.array_equal(np.nonzero(m16[:, 0])[0], np.arange(16))
    assert np.array_equal(np.nonzero(m16[:, 1])[0], np.arange(20, 36))
    m24, _ = o.round_tokens(rt.probs, rt.ids, 24)      # r = 20 > 12: add the 4 smallest unrouted indices
    assert np.array_equal(np.nonzero(m24[:, 0])[0], np.arange(24))
    assert np.array_equal(np.nonzero(m24[:, 1])[0], np.concatenate([np.arange(4), np.arange(20, 40)]))


# --------------------------------------------------------------- backward
def _torch_block_grads(x, wr, bias, wg, wu, wd, k, dout, renormalize):
    """Gradients of sum(dout * out) by torch autograd (fp64) through a dense
    torch rendering of the block; the top-k choice is numpy's lexsort over
    scipy's softmax (no gradient flows through a selection)."""
    _, _, top, _ = dense_reference(x, wr, bias, wg, wu, wd, k)
    X = torch.tensor(widen(x), requires_grad=True)
    Wr = torch.tensor(widen(wr), requires_grad=True)
    E = Wr.shape[1]
    b = torch.tensor(np.zeros(E) if bias is None else bias.astype(np.float64), requires_grad=True)
    Wg = torch.tensor(widen(wg), requires_grad=True)
    Wu = torch.tensor(widen(wu), requires_grad=True)
    Wd = torch.tensor(widen(wd), requires_grad=True)
    ids = torch.tensor(top.astype(np.int64))
    p = torch.softmax(X @ Wr + b, dim=1)
    w = torch.gather(p, 1, ids)
    if renormalize:
        w = w / w.sum(dim=1, keepdim=True)
    out = torch.zeros_like(X)
    for j in range(k):
        e = ids[:, j]
        G = torch.einsum("td,tdf->tf", X, Wg[e])
        U = torch.einsum("td,tdf->tf", X, Wu[e])
        H = torch.nn.functional.silu(G) * U
        out = out + w[:, j:j + 1] * torch.einsum("tf,tfd->td", H, Wd[e])
    (out * torch.tensor(dout)).sum().backward()
    return {"dx": X.grad.numpy(), "dw_router": Wr.grad.numpy(), "dbias": b.grad.numpy(),
            "dw_gate": Wg.grad.numpy(), "dw_up": Wu.grad.numpy(), "dw_down": Wd.grad.numpy()}


_BWD_CASES = [(24, 32, 6, 2, 16, 21, False, False), (17, 16, 8, 3, 24, 22, True, False),
              (20, 32, 5, 5, 8, 23, False, True), (9, 16, 1, 1, 16, 24, False, False),
              (16, 24, 8, 4, 16, 25, True, True)]


def _dout(T, d, seed):
    return np.random.default_rng(seed).standard_normal((T, d))


def check_backward_autograd(o):
    for (T, d, E, k, f, seed, bias, renorm) in _BWD_CASES:
        inp = _rand_case(T, d, E, k, f, seed, bias=bias, sigma=0.2)
        dout = _dout(T, d, seed)
        g = o.backward(*_args(inp), k, dout, renormalize=renorm)
        ref = _torch_block_grads(*_args(inp), k, dout, renorm)
        for name, want in ref.items():
            got = getattr(g, name)
            assert got.shape == want.shape, (name, got.shape, want.shape)
            assert _rel(got, want) < 1e-10 or np.abs(want).max() < 1e-300, ("autograd", name, T, d, E, k, f, renorm)


def _np_block(X, Wr, b, Wg, Wu, Wd, ids, renormalize):
    """Plain fp64 numpy forward with a fixed expert choice (for finite differences)."""
    p = sps.softmax(X @ Wr + b[None, :], axis=1)
    w = np.take_along_axis(p, ids, axis=1)
    if renormalize:
        w = w / w.sum(axis=1, keepdims=True)
    out = np.zeros_like(X)
    for t in range(X.shape[0]):
        for j in range(ids.shape[1]):
            e = ids[t, j]
            G = X[t] @ Wg[e]
            H = G * sps.expit(G) * (X[t] @ Wu[e])
            out[t] += w[t, j] * (H @ Wd[e])
    return out


def check_backward_finite_differences(o):
    for (T, d, E, k, f, seed, bias, renorm) in _BWD_CASES[:3]:
        inp = _rand_case(T, d, E, k, f, seed, bias=bias, sigma=0.2)
        args = _args(inp)
        dout = _dout(T, d, seed)
        r, ex = o.forward(*args, k, renormalize=renorm)
        base = [widen(args[0]), widen(args[1]),
                np.zeros(E) if args[2] is None else args[2].astype(np.float64),
                widen(args[3]), widen(args[4]), widen(args[5])]
        ids = r.ids.astype(np.int64)
        # the numpy forward is the oracle's forward at the bf16 point
        assert _rel(_np_block(*base, ids, renorm), ex.out) < 1e-12, ("numpy forward", T, E, k)
        g = o.backward(*args, k, dout, renormalize=renorm)
        grads = [g.dx, g.dw_router, g.dbias, g.dw_gate, g.dw_up, g.dw_down]
        rng = np.random.default_rng(seed + 1)
        for pos in range(6):
            v = rng.standard_normal(base[pos].shape)
            eps = 1e-6 * max(1.0, float(np.abs(base[pos]).max()))

            def loss(sign):
                pts = list(base)
                pts[pos] = base[pos] + sign * eps * v
                return float(np.sum(_np_block(*pts, ids, renorm) * dout))

            fd = (loss(1.0) - loss(-1.0)) / (2 * eps)
            an = float(np.sum(grads[pos] * v))
            assert abs(fd - an) <= 1e-6 * max(1.0, abs(an)), ("finite differences", pos, fd, an)


def check_backward_invariants(o):
    # the softmax gradient sums to zero over experts, so do dbias and each row of dW_router
    inp = _rand_case(24, 32, 8, 3, 16, 31, bias=True, sigma=0.2)
    dout = _dout(24, 32, 31)
    g = o.backward(*_args(inp), 3, dout)
    assert abs(g.dbias.sum()) <= 1e-12 * np.abs(g.dbias).sum()
    assert np.all(np.abs(g.dw_router.sum(axis=1)) <= 1e-12 * np.abs(g.dw_router).sum(axis=1) + 1e-300)
    # experts no token selects get exactly zero weight gradients
    r, _ = o.forward(*_args(inp), 3)
    unused = np.setdiff1d(np.arange(8), r.ids.ravel())
    for e in unused:
        assert not g.dw_gate[e].any() and not g.dw_up[e].any() and not g.dw_down[e].any()
    # linear in dout: doubling it doubles every gradient exactly
    g2 = o.backward(*_args(inp), 3, 2.0 * dout)
    for name in ("dx", "dw_router", "dbias", "dw_gate", "dw_up", "dw_down"):
        assert np.array_equal(getattr(g2, name), 2.0 * getattr(g, name)), name


def check_backward_restricted(o):
    """The per-token dx and per-expert weight gradients (for sampled checks
    at full size) equal the corresponding entries of the whole backward."""
    for (T, d, E, k, f, seed, bias, ren) in [(24, 32, 8, 3, 16, 31, True, False), (30, 64, 8, 2, 32, 5, False, True)]:
        inp = _rand_case(T, d, E, k, f, seed, bias=bias, sigma=0.2)
        dout = _dout(T, d, seed)
        g = o.backward(*_args(inp), k, dout, renormalize=ren)
        rows = np.array([0, T // 2, T - 1])
        assert np.array_equal(o.backward_rows(*_args(inp), k, dout, rows, renormalize=ren), g.dx[rows]), "dx rows"
        for e in range(E):
            gg, gu, gd = o.backward_expert(*_args(inp), k, dout, e, renormalize=ren)
            assert np.array_equal(gg, g.dw_gate[e]) and np.array_equal(gu, g.dw_up[e]), ("expert", e)
            assert np.array_equal(gd, g.dw_down[e]), ("expert down", e)


ALL_CHECKS = [
    check_brute_force, check_softmax_library, check_topk_library_sort, check_topk_of_logits,
    check_exact_ties, check_dense_special_case, check_all_experts_identical, check_zero_expert,
    check_scale_down, check_permute_library, check_expert_rows_outputs,
    check_renormalize, check_shared_experts, check_token_rounding, check_backward_autograd,
    check_backward_finite_differences, check_backward_invariants, check_backward_restricted,
]
