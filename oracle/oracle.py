"""Python wrapper of the fp64 C oracle (``moe_oracle.c``).

TEST INFRASTRUCTURE ONLY: the tests, the smoke check and the benchmark's
CPU-baseline leg may import this module; the product path never does.

The C source is compiled with plain ``gcc -O2`` (no fast-math, so every sum
keeps its written order) into ``liboracle.so`` beside it, on first use or
when the source changed.  Inputs are numpy arrays: bf16 tensors as uint16 bit
patterns, the bias as float32.
"""
from __future__ import annotations

import ctypes
import hashlib
import os
import subprocess
from dataclasses import dataclass

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "moe_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_STAMP = _LIB + ".srchash"


def _source_hash(src: str) -> str:
    with open(src, "rb") as fh:
        return hashlib.sha256(fh.read()).hexdigest()


def compile_oracle(src: str = _SRC, out: str = _LIB, extra_flags=(), force: bool = False) -> str:
    """Compile an oracle source file to a shared library; returns its path."""
    stamp = out + ".srchash"
    h = _source_hash(src) + " " + " ".join(extra_flags)
    if not force and os.path.exists(out) and os.path.exists(stamp):
        with open(stamp) as fh:
            if fh.read() == h:
                return out
    cmd = ["gcc", "-O2", "-std=c99", "-fPIC", "-shared", "-o", out, src, "-lm", *extra_flags]
    subprocess.run(cmd, check=True)
    with open(stamp, "w") as fh:
        fh.write(h)
    return out


_P = ctypes.c_void_p
_I64 = ctypes.c_int64


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


class Oracle:
    """Handle on one compiled oracle library (the real one, or a test mutant)."""

    def __init__(self, lib_path: str | None = None):
        self.path = lib_path or compile_oracle()
        lib = ctypes.CDLL(self.path)
        lib.oracle_route.argtypes = [_P, _P, _P, _I64, _I64, _I64, _I64, _P, _P, _P, _P]
        lib.oracle_permute.argtypes = [_P, _I64, _I64, _I64, _P, _P, _P, _P]
        lib.oracle_expert_rows.argtypes = [_P, _P, _P, _P, _I64, _I64, _I64, _I64, _I64,
                                           _P, _P, _I64, _P, _P, _P, _P]
        lib.oracle_renormalize.argtypes = [_P, _I64, _I64]
        lib.oracle_shared_rows.argtypes = [_P, _P, _P, _P, _I64, _I64, _I64, _I64, _I64, _P, _P]
        lib.oracle_shared_rows.restype = ctypes.c_int
        lib.oracle_round_tokens.argtypes = [_P, _P, _I64, _I64, _I64, _I64, _P, _P]
        lib.oracle_round_tokens.restype = ctypes.c_int
        lib.oracle_masked_rows.argtypes = [_P, _P, _P, _P, _I64, _I64, _I64, _I64, _P, _P, _I64, _P, _P]
        lib.oracle_masked_rows.restype = ctypes.c_int
        lib.oracle_backward.argtypes = [_P, _P, _P, _P, _P, _P, _I64, _I64, _I64, _I64, _I64, ctypes.c_int,
                                        _P, _P, _P, _P, _P, _P, _P]
        lib.oracle_backward.restype = ctypes.c_int
        lib.oracle_backward_rows.argtypes = [_P, _P, _P, _P, _P, _P, _I64, _I64, _I64, _I64, _I64, ctypes.c_int,
                                             _P, _I64, _P, _P]
        lib.oracle_backward_rows.restype = ctypes.c_int
        lib.oracle_backward_expert.argtypes = [_P, _P, _P, _P, _P, _P, _I64, _I64, _I64, _I64, _I64,
                                               ctypes.c_int, _P, _I64, _P, _P, _P]
        lib.oracle_backward_expert.restype = ctypes.c_int
        for fn in (lib.oracle_route, lib.oracle_permute, lib.oracle_expert_rows, lib.oracle_renormalize):
            fn.restype = ctypes.c_int
        self.lib = lib

    # -- stage 1 + 2 ------------------------------------------------------
    def route(self, x, w_router, bias, k, want_logits=False, want_probs=True, renormalize=False):
        x = np.ascontiguousarray(x, dtype=np.uint16)
        w_router = np.ascontiguousarray(w_router, dtype=np.uint16)
        T, d = x.shape
        d2, E = w_router.shape
        assert d == d2
        b = None if bias is None else np.ascontiguousarray(bias, dtype=np.float32)
        logits = np.empty((T, E), np.float64) if want_logits else None
        probs = np.empty((T, E), np.float64) if want_probs else None
        ids = np.empty((T, k), np.int32)
        w = np.empty((T, k), np.float64)
        rc = self.lib.oracle_route(_ptr(x), _ptr(w_router), _ptr(b), T, d, E, k,
                                   _ptr(logits), _ptr(probs), _ptr(ids), _ptr(w))
        if rc != 0:
            raise ValueError(f"oracle_route failed ({rc})")
        if renormalize:
            rc = self.lib.oracle_renormalize(_ptr(w), T, k)
            if rc != 0:
                raise ValueError(f"oracle_renormalize failed ({rc})")
        return RouteResult(ids=ids, weights=w, probs=probs, logits=logits)

    # -- grouping -----------------------------------------------------------
    def permute(self, ids, E):
        ids = np.ascontiguousarray(ids, dtype=np.int32)
        T, k = ids.shape
        counts = np.empty(E, np.int32)
        offsets = np.empty(E + 1, np.int32)
        perm = np.empty(T * k, np.int32)
        inv = np.empty(T * k, np.int32)
        rc = self.lib.oracle_permute(_ptr(ids), T, E, k, _ptr(counts), _ptr(offsets),
                                     _ptr(perm), _ptr(inv))
        if rc != 0:
            raise ValueError(f"oracle_permute failed ({rc})")
        return PermuteResult(counts, offsets, perm, inv)

    # -- stage 3 + 4 ----------------------------------------------------------
    def expert_rows(self, x, w_gate, w_up, w_down, ids, weights, rows,
                    want_y=False, want_h=False):
        x = np.ascontiguousarray(x, dtype=np.uint16)
        w_gate = np.ascontiguousarray(w_gate, dtype=np.uint16)
        w_up = np.ascontiguousarray(w_up, dtype=np.uint16)
        w_down = np.ascontiguousarray(w_down, dtype=np.uint16)
        ids = np.ascontiguousarray(ids, dtype=np.int32)
        weights = np.ascontiguousarray(weights, dtype=np.float64)
        rows = np.ascontiguousarray(rows, dtype=np.int64)
        T, d = x.shape
        E, _, f = w_gate.shape
        k = ids.shape[1]
        n = rows.shape[0]
        out = np.empty((n, d), np.float64)
        y = np.empty((n, k, d), np.float64) if want_y else None
        h = np.empty((n, k, f), np.float64) if want_h else None
        rc = self.lib.oracle_expert_rows(_ptr(x), _ptr(w_gate), _ptr(w_up), _ptr(w_down),
                                         T, d, E, k, f, _ptr(ids), _ptr(weights), n,
                                         _ptr(rows), _ptr(out), _ptr(y), _ptr(h))
        if rc != 0:
            raise ValueError(f"oracle_expert_rows failed ({rc})")
        return ExpertResult(out=out, y=y, h=h)

    # -- shared experts -------------------------------------------------------
    def shared_rows(self, x, w_gate_s, w_up_s, w_down_s, rows, out):
        """out + sum over shared experts s of SwiGLU_s(x[rows]) (a new array)."""
        x = np.ascontiguousarray(x, dtype=np.uint16)
        w_gate_s = np.ascontiguousarray(w_gate_s, dtype=np.uint16)
        w_up_s = np.ascontiguousarray(w_up_s, dtype=np.uint16)
        w_down_s = np.ascontiguousarray(w_down_s, dtype=np.uint16)
        rows = np.ascontiguousarray(rows, dtype=np.int64)
        res = np.array(out, dtype=np.float64, copy=True, order="C")
        T, d = x.shape
        n_s, _, f_s = w_gate_s.shape
        rc = self.lib.oracle_shared_rows(_ptr(x), _ptr(w_gate_s), _ptr(w_up_s), _ptr(w_down_s), T, d, n_s, f_s,
                                         rows.shape[0], _ptr(rows), _ptr(res))
        if rc != 0:
            raise ValueError(f"oracle_shared_rows failed ({rc})")
        return res

    # -- token rounding -------------------------------------------------------
    def round_tokens(self, probs, ids, tile):
        """Token rounding of the top-k routing to multiples of ``tile`` rows per
        expert; returns (mask [T, E] bool, counts [E] int32)."""
        probs = np.ascontiguousarray(probs, dtype=np.float64)
        ids = np.ascontiguousarray(ids, dtype=np.int32)
        T, E = probs.shape
        k = ids.shape[1]
        mask = np.empty((T, E), np.uint8)
        counts = np.empty(E, np.int32)
        rc = self.lib.oracle_round_tokens(_ptr(probs), _ptr(ids), T, E, k, tile, _ptr(mask), _ptr(counts))
        if rc != 0:
            raise ValueError(f"oracle_round_tokens failed ({rc})")
        return mask.astype(bool), counts

    def masked_rows(self, x, w_gate, w_up, w_down, mask, probs, rows):
        """out[r] = sum over experts e (ascending) with mask[t, e] of probs[t, e] * expert_e(x[t])."""
        x = np.ascontiguousarray(x, dtype=np.uint16)
        w_gate = np.ascontiguousarray(w_gate, dtype=np.uint16)
        w_up = np.ascontiguousarray(w_up, dtype=np.uint16)
        w_down = np.ascontiguousarray(w_down, dtype=np.uint16)
        m = np.ascontiguousarray(mask, dtype=np.uint8)
        probs = np.ascontiguousarray(probs, dtype=np.float64)
        rows = np.ascontiguousarray(rows, dtype=np.int64)
        T, d = x.shape
        E, _, f = w_gate.shape
        out = np.empty((rows.shape[0], d), np.float64)
        rc = self.lib.oracle_masked_rows(_ptr(x), _ptr(w_gate), _ptr(w_up), _ptr(w_down), T, d, E, f, _ptr(m),
                                         _ptr(probs), rows.shape[0], _ptr(rows), _ptr(out))
        if rc != 0:
            raise ValueError(f"oracle_masked_rows failed ({rc})")
        return out

    # -- whole block ----------------------------------------------------------
    def forward(self, x, w_router, bias, w_gate, w_up, w_down, k, rows=None,
                want_y=False, want_h=False, renormalize=False, shared=None):
        """Route every token; evaluate the expert MLPs for ``rows`` (all if
        None).  ``shared``: optional (W_gate_s, W_up_s, W_down_s) bit arrays of
        shared experts, added to ``out`` with weight one."""
        r = self.route(x, w_router, bias, k, renormalize=renormalize)
        if rows is None:
            rows = np.arange(x.shape[0], dtype=np.int64)
        ex = self.expert_rows(x, w_gate, w_up, w_down, r.ids, r.weights, rows,
                              want_y=want_y, want_h=want_h)
        if shared is not None:
            ex = ExpertResult(out=self.shared_rows(x, *shared, rows, ex.out), y=ex.y, h=ex.h)
        return r, ex

    # -- backward ---------------------------------------------------------------
    def backward(self, x, w_router, bias, w_gate, w_up, w_down, k, dout, renormalize=False):
        """Gradient of sum(dout * out) with respect to x, W_router, the bias
        and the expert weights (fp64; the routing choice passes no gradient)."""
        x = np.ascontiguousarray(x, dtype=np.uint16)
        w_router = np.ascontiguousarray(w_router, dtype=np.uint16)
        w_gate = np.ascontiguousarray(w_gate, dtype=np.uint16)
        w_up = np.ascontiguousarray(w_up, dtype=np.uint16)
        w_down = np.ascontiguousarray(w_down, dtype=np.uint16)
        dout = np.ascontiguousarray(dout, dtype=np.float64)
        T, d = x.shape
        E = w_router.shape[1]
        f = w_gate.shape[2]
        assert w_gate.shape == (E, d, f) and w_up.shape == (E, d, f) and w_down.shape == (E, f, d)
        assert dout.shape == (T, d)
        b = None if bias is None else np.ascontiguousarray(bias, dtype=np.float32)
        g = BackwardResult(dx=np.empty((T, d)), dw_router=np.empty((d, E)), dbias=np.empty(E),
                           dw_gate=np.empty((E, d, f)), dw_up=np.empty((E, d, f)), dw_down=np.empty((E, f, d)))
        rc = self.lib.oracle_backward(_ptr(x), _ptr(w_router), _ptr(b), _ptr(w_gate), _ptr(w_up), _ptr(w_down),
                                      T, d, E, k, f, 1 if renormalize else 0, _ptr(dout), _ptr(g.dx),
                                      _ptr(g.dw_router), _ptr(g.dbias), _ptr(g.dw_gate), _ptr(g.dw_up),
                                      _ptr(g.dw_down))
        if rc != 0:
            raise ValueError(f"oracle_backward failed ({rc})")
        return g


    def _bwd_args(self, x, w_router, bias, w_gate, w_up, w_down, dout):
        x = np.ascontiguousarray(x, dtype=np.uint16)
        w_router = np.ascontiguousarray(w_router, dtype=np.uint16)
        w_gate = np.ascontiguousarray(w_gate, dtype=np.uint16)
        w_up = np.ascontiguousarray(w_up, dtype=np.uint16)
        w_down = np.ascontiguousarray(w_down, dtype=np.uint16)
        dout = np.ascontiguousarray(dout, dtype=np.float64)
        b = None if bias is None else np.ascontiguousarray(bias, dtype=np.float32)
        return x, w_router, b, w_gate, w_up, w_down, dout

    def backward_rows(self, x, w_router, bias, w_gate, w_up, w_down, k, dout, rows, renormalize=False):
        """dx of the chosen tokens only ([len(rows), d] fp64), equal to the
        corresponding rows of backward()'s dx."""
        x, w_router, b, w_gate, w_up, w_down, dout = self._bwd_args(x, w_router, bias, w_gate, w_up, w_down, dout)
        rows = np.ascontiguousarray(rows, dtype=np.int64)
        T, d = x.shape
        E = w_router.shape[1]
        f = w_gate.shape[2]
        out = np.empty((rows.shape[0], d), np.float64)
        rc = self.lib.oracle_backward_rows(_ptr(x), _ptr(w_router), _ptr(b), _ptr(w_gate), _ptr(w_up), _ptr(w_down),
                                           T, d, E, k, f, 1 if renormalize else 0, _ptr(dout), rows.shape[0],
                                           _ptr(rows), _ptr(out))
        if rc != 0:
            raise ValueError(f"oracle_backward_rows failed ({rc})")
        return out

    def backward_expert(self, x, w_router, bias, w_gate, w_up, w_down, k, dout, e, renormalize=False):
        """(dW_gate[e], dW_up[e], dW_down[e]) in fp64, equal to backward()'s."""
        x, w_router, b, w_gate, w_up, w_down, dout = self._bwd_args(x, w_router, bias, w_gate, w_up, w_down, dout)
        T, d = x.shape
        E = w_router.shape[1]
        f = w_gate.shape[2]
        gg, gu, gd = np.empty((d, f)), np.empty((d, f)), np.empty((f, d))
        rc = self.lib.oracle_backward_expert(_ptr(x), _ptr(w_router), _ptr(b), _ptr(w_gate), _ptr(w_up),
                                             _ptr(w_down), T, d, E, k, f, 1 if renormalize else 0, _ptr(dout), e,
                                             _ptr(gg), _ptr(gu), _ptr(gd))
        if rc != 0:
            raise ValueError(f"oracle_backward_expert failed ({rc})")
        return gg, gu, gd


@dataclass
class BackwardResult:
    dx: np.ndarray         # [T, d]
    dw_router: np.ndarray  # [d, E]
    dbias: np.ndarray      # [E]
    dw_gate: np.ndarray    # [E, d, f]
    dw_up: np.ndarray      # [E, d, f]
    dw_down: np.ndarray    # [E, f, d]


@dataclass
class RouteResult:
    ids: np.ndarray        # [T, k] int32
    weights: np.ndarray    # [T, k] float64
    probs: np.ndarray | None   # [T, E] float64
    logits: np.ndarray | None  # [T, E] float64


@dataclass
class PermuteResult:
    counts: np.ndarray     # [E]
    offsets: np.ndarray    # [E+1]
    perm: np.ndarray       # [T*k]
    inv: np.ndarray        # [T*k]


@dataclass
class ExpertResult:
    out: np.ndarray                # [n, d] float64
    y: np.ndarray | None = None    # [n, k, d]
    h: np.ndarray | None = None    # [n, k, f]


def topk_gap(probs: np.ndarray, k: int) -> np.ndarray:
    """p_(k-1) - p_(k) per token, with p_(0) >= p_(1) >= ... the probabilities
    sorted in descending order: the margin between the last selected expert
    and the best unselected one (inf when k >= E)."""
    T, E = probs.shape
    if k >= E:
        return np.full(T, np.inf)
    s = -np.sort(-probs, axis=1)
    return s[:, k - 1] - s[:, k]


def inner_gap(probs: np.ndarray, k: int) -> np.ndarray:
    """Smallest gap between consecutive probabilities inside the top k, per token.

    min over j < k-1 of p_(j) - p_(j+1), with p_(0) >= p_(1) >= ... the
    probabilities sorted in descending order (inf when k < 2): a near tie
    here may swap the order of two selected slots without changing the
    selected set.
    """
    T, E = probs.shape
    if k < 2:
        return np.full(T, np.inf)
    s = -np.sort(-probs, axis=1)[:, :k]
    return np.min(s[:, :-1] - s[:, 1:], axis=1)


_default: Oracle | None = None


def default_oracle() -> Oracle:
    global _default
    if _default is None:
        _default = Oracle()
    return _default


__all__ = ["Oracle", "compile_oracle", "default_oracle", "topk_gap", "inner_gap",
           "RouteResult", "PermuteResult", "ExpertResult"]
