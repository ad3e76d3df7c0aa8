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
  * routing weights:            |w_gpu - w_oracle| <= W_REL * w_oracle
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


def widen(bits: np.ndarray) -> np.ndarray:
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def bf16_tensor_to_f64(t) -> np.ndarray:
    import torch
    return widen(t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16))


def route_check(ids_gpu: np.ndarray, w_gpu: np.ndarray, probs: np.ndarray, oracle_ids: np.ndarray, k: int):
    """Check GPU routing against the oracle's fp64 probabilities.

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
    assert np.all(np.diff(w_gpu, axis=1) <= 0), "slots not in descending probability order"
    stats = {"tokens": int(T), "excluded_near_tie": int(excluded.sum()), "inner_near_tie": int(inner.sum()),
             "w_max_rel_err": worst}
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
