"""Parity criteria between the CUDA path and the fp64 oracle.

Tolerances (floating point; inputs bf16, fp32 accumulation, fp32 outputs):
  * outputs y and out:          max|gpu - oracle| <= 2e-2 * RMS(oracle)
                                sum|gpu - oracle| / sum|oracle| <= 5e-3
  * h, the bf16 operand of the second GEMM: within one bf16 rounding of the
    oracle value, |gpu - oracle| <= 2^-8 * |oracle| + 1e-3 * RMS(oracle)
    (the second term covers the fp32 accumulation of g and u)
  * o = h . W_down (y before the routing weight): each element within the
    worst-case effect of that one rounding of h plus fp32 accumulation,
    |gpu - oracle| <= (2^-8 + f * 2^-23) * sum_n |h_n| |W_down[n, c]|
  * routing weights:            |w_gpu - w_oracle| <= W_REL * w_oracle, and,
                                where the caller passes the logits' magnitudes,
                                within the a-priori bound of weight_bound
Integer results (expert ids, counts, offsets, perm, inv) must be bit-exact,
except for tokens whose k-th and (k+1)-th oracle probabilities differ by less
than 1e-6: the fp32 logits of the GPU may order such a pair differently, so
those tokens are counted and left out of the id check.  A near tie between
two selected slots (inside the top k) may swap their order without changing
the set; such tokens are compared as sets.
"""
from __future__ import annotations

import numpy as np

from oracle.oracle import inner_gap, topk_gap

TIE_EPS = 1e-6
MAX_ABS_REL_RMS = 2e-2
MEAN_REL = 5e-3
# Routing weights come from fp32 logits.  p_j = exp(l_j - m) / s, so the
# relative error of p_j is the absolute error of (l_j - m) plus that of log s.
# An fp32 GEMM of these inputs (cuBLAS, no TF32) misses the fp64 logits by up
# to 7e-6 on the five workloads (logits reach |l| ~ 12 with the Zipf bias),
# and the router's worst weight error measured there is 1.3e-5; 5e-5 bounds
# two such logit errors plus the normaliser's with margin.
W_REL = 5e-5


def logit_error_bound(abs_scale: np.ndarray, d: int) -> np.ndarray:
    """A-priori bound on |l_gpu - l| per (token, expert) for fp32 logits.

    abs_scale[t, e] = sum_i |x[t, i]| |W_router[i, e]| + |b_e| (fp64).  The
    products of two bf16 values are exact in fp32; the d - 1 additions of the
    dot product, the sum of the split-K partials and the bias add are at
    most d + 1 roundings, in any order.  With unit roundoff u the classical
    bound is gamma_n * abs_scale, gamma_n = n u / (1 - n u).  u = 2^-23, not
    2^-24: neither the order nor the rounding mode inside the tensor-core
    accumulation is specified, and 2^-23 also covers truncation.
    """
    u = 2.0 ** -23
    n = d + 2
    return (n * u / (1.0 - n * u)) * abs_scale


def weight_bound(logit_err: np.ndarray, probs: np.ndarray, ids: np.ndarray) -> np.ndarray:
    """A-priori bound on |w_gpu - p| / p for each selected slot [T, k].

    With logit errors |delta_j| <= b_j, exp(l_e + delta_e - m) / sum_j
    exp(l_j + delta_j - m) differs from p_e by a factor within
    exp(+-(b_e + max_j b_j)).  The fp32 softmax adds: the rounding of l - m
    and of (l - m) log2(e) before the exponential (relative error of the
    term up to |l - m| 2^-23, with |l_e - m| = log(p_max / p_e), and, for the
    sum, the p-weighted mean H of |l_j - m|), the approximate exponential
    (2^-21 for the numerator and for the sum's terms), and the E-term sum plus
    the division ((E + 1) 2^-24).  The first-order terms are added and the
    total is scaled by 1.25 to cover the neglected second-order products.
    """
    T, E = probs.shape
    ids = ids.astype(np.int64)
    b_e = np.take_along_axis(logit_err, ids, axis=1)
    b_max = logit_err.max(axis=1, keepdims=True)
    p_max = probs.max(axis=1, keepdims=True)
    p_e = np.take_along_axis(probs, ids, axis=1)
    with np.errstate(divide="ignore", invalid="ignore"):
        r_e = np.log(p_max / p_e)
        terms = np.where(probs > 0, probs * np.log(p_max / np.where(probs > 0, probs, 1.0)), 0.0)
    H = terms.sum(axis=1, keepdims=True)
    fp = (r_e + H) * 2.0 ** -23 + 2 * 2.0 ** -21 + (E + 1) * 2.0 ** -24
    return 1.25 * (np.expm1(b_e + b_max) + fp)


def widen(bits: np.ndarray) -> np.ndarray:
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def bf16_tensor_to_f64(t) -> np.ndarray:
    import torch
    return widen(t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16))


def route_check(ids_gpu: np.ndarray, w_gpu: np.ndarray, probs: np.ndarray, oracle_ids: np.ndarray, k: int,
                logit_err: np.ndarray | None = None):
    """Check GPU routing against the oracle's fp64 probabilities.

    logit_err (optional, [T, E]): logit_error_bound of the inputs; the
    weights must then also lie within weight_bound.
    Returns (excluded token mask, stats).  Raises AssertionError on mismatch.
    """
    T = probs.shape[0]
    excluded = topk_gap(probs, k) < TIE_EPS
    inner = (inner_gap(probs, k) < TIE_EPS) & ~excluded
    ok = ~excluded
    exact = ok & ~inner
    bad = np.nonzero(exact & np.any(ids_gpu != oracle_ids, axis=1))[0]
    assert bad.size == 0, f"{bad.size} tokens with different expert ids, first {bad[:5]}: " \
                          f"gpu {ids_gpu[bad[:3]]} oracle {oracle_ids[bad[:3]]}"
    if inner.any():
        a = np.sort(ids_gpu[inner], axis=1)
        b = np.sort(oracle_ids[inner], axis=1)
        assert np.array_equal(a, b), "near-tie tokens select different expert sets"
    # every token: ids distinct and in range
    assert ids_gpu.min() >= 0 and ids_gpu.max() < probs.shape[1]
    srt = np.sort(ids_gpu, axis=1)
    assert np.all(srt[:, 1:] != srt[:, :-1]) if k > 1 else True, "duplicate expert for a token"
    # weights: the oracle probability of the expert the GPU chose
    p_sel = np.take_along_axis(probs, ids_gpu.astype(np.int64), axis=1)
    err = np.abs(w_gpu.astype(np.float64) - p_sel)
    worst = float(np.max(err[ok] / p_sel[ok])) if ok.any() else 0.0
    assert worst <= W_REL, f"routing weight relative error {worst:.3e} > {W_REL}"
    bound_use = None
    if logit_err is not None:
        bound = weight_bound(logit_err, probs, ids_gpu)
        ratio = err / (p_sel * bound)
        bound_use = float(ratio[ok].max()) if ok.any() else 0.0
        assert bound_use <= 1.0, f"routing weight beyond its a-priori bound (x{bound_use:.3f})"
    assert np.all(np.diff(w_gpu, axis=1) <= 0), "slots not in descending probability order"
    stats = {"tokens": int(T), "excluded_near_tie": int(excluded.sum()), "inner_near_tie": int(inner.sum()),
             "w_max_rel_err": worst, "w_bound_use": bound_use}
    return excluded, stats


def bf16_rounded_check(gpu: np.ndarray, ref: np.ndarray, what: str):
    """A bf16-rounded intermediate: each value within one rounding of the oracle."""
    gpu = gpu.astype(np.float64)
    ref = ref.astype(np.float64)
    assert np.all(np.isfinite(gpu)), f"{what}: non-finite values"
    rms = float(np.sqrt(np.mean(ref * ref)))
    excess = np.abs(gpu - ref) - (2.0 ** -8 * np.abs(ref) + 1e-3 * rms)
    worst = float(excess.max())
    assert worst <= 0, f"{what}: {int((excess > 0).sum())} values beyond one bf16 rounding (worst by {worst:.3e})"
    return worst


def bound_check(gpu: np.ndarray, ref: np.ndarray, bound: np.ndarray, what: str):
    """Elementwise |gpu - ref| <= bound; returns the largest |gpu - ref| / bound."""
    gpu = gpu.astype(np.float64)
    assert np.all(np.isfinite(gpu)), f"{what}: non-finite values"
    ratio = np.abs(gpu - ref) / np.maximum(bound, 1e-300)
    worst = float(ratio.max())
    assert worst <= 1.0, f"{what}: {int((ratio > 1).sum())} values beyond the bound (worst x{worst:.3f})"
    return worst


def value_check(gpu: np.ndarray, ref: np.ndarray, what: str):
    """The floating-point output criterion; returns (max_abs/rms, mean_rel)."""
    gpu = gpu.astype(np.float64)
    ref = ref.astype(np.float64)
    assert np.all(np.isfinite(gpu)), f"{what}: non-finite values"
    rms = float(np.sqrt(np.mean(ref * ref)))
    diff = np.abs(gpu - ref)
    max_rel_rms = float(diff.max() / rms) if rms > 0 else float(diff.max())
    denom = float(np.abs(ref).sum())
    mean_rel = float(diff.sum() / denom) if denom > 0 else float(diff.sum())
    assert max_rel_rms <= MAX_ABS_REL_RMS, f"{what}: max|gpu-oracle| = {max_rel_rms:.3e} * RMS > {MAX_ABS_REL_RMS}"
    assert mean_rel <= MEAN_REL, f"{what}: mean relative error {mean_rel:.3e} > {MEAN_REL}"
    return max_rel_rms, mean_rel
