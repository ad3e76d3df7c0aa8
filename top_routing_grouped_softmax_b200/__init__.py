"""B200-native sparse Mixture-of-Experts block forward (sm_100a CUDA).

A thin ctypes binding over the C ABI of ``libmoe.so`` (declared in
``include/moe.h``).  Every step of the block runs in the library's CUDA
kernels; this module only checks tensor properties, allocates outputs and
workspace through PyTorch, and passes raw device pointers and the current
CUDA stream.  There is no CPU or PyTorch fallback: if the library is missing
or the device is not a B200, the calls raise.

Functions mirror the ABI entry points:
  route, permute, expert_ffn, combine, forward, backward, the shared-expert
  and token-rounding variants, the *_workspace_size queries, get_status,
  set_wait_limit_ns.
``MoEBlock`` keeps the weights and a reusable workspace for repeated calls.
"""
from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libmoe.so")

MOE_OK = 0
MOE_ERR_INVALID_ARG = 1
MOE_ERR_UNSUPPORTED_SHAPE = 2
MOE_ERR_WORKSPACE_TOO_SMALL = 3
MOE_ERR_CUDA = 4
MOE_ERR_DEVICE_TIMEOUT = 5
MOE_ERR_DEVICE_BOUNDS = 6
MOE_ERR_UNSUPPORTED_DEVICE = 7
MOE_ERR_STATIC_SCRATCH_TOO_SMALL = 8
MOE_ERR_DEVICE_RANGE = 9

# Every symbol include/moe.h declares.
ABI_SYMBOLS = (
    "moe_strerror", "moe_version", "moe_workspace_size", "moe_route_workspace_size",
    "moe_permute_workspace_size", "moe_route", "moe_permute", "moe_expert_ffn", "moe_combine", "moe_forward",
    "moe_forward_ex", "moe_get_status", "moe_set_wait_limit_ns", "moe_selftest_wait_timeout",
    "moe_permute_static", "moe_route_ex", "moe_workspace_size_shared", "moe_shared_ffn", "moe_combine_shared",
    "moe_forward_shared", "moe_workspace_size_rounded", "moe_forward_rounded",
    "moe_backward_workspace_size", "moe_backward", "moe_gather_rows",
)


class MoEError(RuntimeError):
    """A non-zero status from the C ABI."""

    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {strerror(status)} (status {status})")


_P = ctypes.c_void_p
_I64 = ctypes.c_int64
_SZ = ctypes.c_size_t
_lib = None


def lib() -> ctypes.CDLL:
    """Load libmoe.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(
                f"{LIB_PATH} is missing: build it with `python -m top_routing_grouped_softmax_b200._build` "
                "or __graft_entry__.build(); there is no fallback implementation")
        L = ctypes.CDLL(LIB_PATH)
        L.moe_strerror.restype = ctypes.c_char_p
        L.moe_strerror.argtypes = [ctypes.c_int]
        L.moe_version.restype = ctypes.c_int
        L.moe_workspace_size.restype = _SZ
        L.moe_workspace_size.argtypes = [_I64] * 5
        L.moe_route_workspace_size.restype = _SZ
        L.moe_route_workspace_size.argtypes = [_I64] * 3
        L.moe_permute_workspace_size.restype = _SZ
        L.moe_permute_workspace_size.argtypes = [_I64] * 3
        L.moe_route.argtypes = [_P, _P, _P, _I64, _I64, _I64, _I64, _P, _P, _P, _SZ, _P]
        L.moe_route_ex.argtypes = [_P, _P, _P, _I64, _I64, _I64, _I64, _P, _P, _P, _SZ, _P, ctypes.c_uint]
        L.moe_permute.argtypes = [_P, _P, _P, _I64, _I64, _I64, _I64, _P, _P, _P, _P, _P, _P, _P, _SZ, _P]
        L.moe_permute_static.argtypes = [_P, _P, _P, _I64, _I64, _I64, _I64, _P, _P, _P, _P, _P, _P, _P]
        L.moe_expert_ffn.argtypes = [_P, _P, _P, _P, _P, _P, _I64, _I64, _I64, _I64, _P, _P, _P]
        L.moe_combine.argtypes = [_P, _P, _I64, _I64, _I64, _P, _P]
        L.moe_forward.argtypes = [_P, _P, _P, _P, _P, _P, _I64, _I64, _I64, _I64, _I64, _P, _P, _P, _P, _SZ, _P]
        L.moe_forward_ex.argtypes = L.moe_forward.argtypes + [_P, ctypes.c_int, ctypes.c_uint]
        L.moe_workspace_size_shared.restype = _SZ
        L.moe_workspace_size_shared.argtypes = [_I64] * 7
        L.moe_shared_ffn.argtypes = [_P, _P, _P, _P, _I64, _I64, _I64, _I64, _P, _P, _P]
        L.moe_combine_shared.argtypes = [_P, _P, _P, _I64, _I64, _I64, _I64, _P, _P]
        L.moe_workspace_size_rounded.restype = _SZ
        L.moe_workspace_size_rounded.argtypes = [_I64] * 6
        L.moe_forward_rounded.argtypes = [_P] * 6 + [_I64] * 6 + [_P, _P, _P, _P, _SZ, _P, _P, ctypes.c_int]
        L.moe_forward_shared.argtypes = ([_P] * 9 + [_I64] * 7 + [_P, _P, _P, _P, _SZ, _P, _P, ctypes.c_int,
                                                                   ctypes.c_uint])
        L.moe_backward_workspace_size.restype = _SZ
        L.moe_backward_workspace_size.argtypes = [_I64] * 5
        L.moe_backward.argtypes = [_P] * 7 + [_I64] * 5 + [_P] * 7 + [_SZ, _P, ctypes.c_uint]
        L.moe_gather_rows.argtypes = [_P, _P, _I64, _I64, _I64, _P, _P]
        L.moe_get_status.argtypes = [_P]
        L.moe_set_wait_limit_ns.argtypes = [_I64]
        L.moe_selftest_wait_timeout.argtypes = [_I64, _P]
        for name in ("moe_route", "moe_permute", "moe_expert_ffn", "moe_combine", "moe_forward",
                     "moe_forward_ex", "moe_get_status", "moe_set_wait_limit_ns",
                     "moe_selftest_wait_timeout", "moe_permute_static", "moe_route_ex", "moe_shared_ffn",
                     "moe_combine_shared", "moe_forward_shared", "moe_forward_rounded", "moe_backward", "moe_gather_rows"):
            getattr(L, name).restype = ctypes.c_int
        _lib = L
    return _lib


def strerror(status: int) -> str:
    try:
        return lib().moe_strerror(int(status)).decode()
    except ImportError:
        return f"status {status}"


def _check(rc: int, where: str):
    if rc != MOE_OK:
        raise MoEError(rc, where)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _need(t, name, dtype, ndim=None):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if ndim is not None and t.dim() != ndim:
        raise ValueError(f"{name} must have {ndim} dims, got {t.dim()}")
    return t


# ------------------------------------------------------------------ sizes
def workspace_size(T: int, d: int, E: int, k: int, f: int) -> int:
    return int(lib().moe_workspace_size(T, d, E, k, f))


def route_workspace_size(T: int, d: int, E: int) -> int:
    return int(lib().moe_route_workspace_size(T, d, E))


def permute_workspace_size(T: int, E: int, k: int) -> int:
    return int(lib().moe_permute_workspace_size(T, E, k))


def _workspace(nbytes: int, device) -> torch.Tensor:
    return torch.empty(max(nbytes, 256), dtype=torch.uint8, device=device)


# ----------------------------------------------------------------- stages
def route(x, w_router, k, bias=None, topk_ids=None, topk_w=None, workspace=None, renormalize=False):
    """Router GEMM + fp32 softmax + top-k; returns (topk_ids int32 [T,k], topk_w fp32 [T,k]).

    ``renormalize``: divide each token's k weights by their sum
    (MOE_FLAG_RENORMALIZE); by default they are the softmax probabilities."""
    _need(x, "x", torch.bfloat16, 2)
    _need(w_router, "w_router", torch.bfloat16, 2)
    T, d = x.shape
    E = w_router.shape[1]
    if bias is not None:
        _need(bias, "bias", torch.float32, 1)
    if topk_ids is None:
        topk_ids = torch.empty(T, k, dtype=torch.int32, device=x.device)
    if topk_w is None:
        topk_w = torch.empty(T, k, dtype=torch.float32, device=x.device)
    need = route_workspace_size(T, d, E)
    if need > 0 and (workspace is None or workspace.numel() < need):
        workspace = _workspace(need, x.device)
    ws_bytes = 0 if workspace is None else workspace.numel()
    flags = MOE_FLAG_RENORMALIZE if renormalize else 0
    _check(lib().moe_route_ex(_ptr(x), _ptr(w_router), _ptr(bias), T, d, E, k, _ptr(topk_ids),
                              _ptr(topk_w), _ptr(workspace), ws_bytes, _stream(), flags), "moe_route_ex")
    return topk_ids, topk_w


def permute(x, topk_ids, topk_w, E, gather=True):
    """Stable grouping by expert; returns dict(counts, offsets, perm, inv, x_perm, w_perm)."""
    _need(topk_ids, "topk_ids", torch.int32, 2)
    _need(topk_w, "topk_w", torch.float32, 2)
    T, k = topk_ids.shape
    dev = topk_ids.device
    d = x.shape[1] if x is not None else 64
    if x is not None:
        _need(x, "x", torch.bfloat16, 2)
    M = T * k
    out = {
        "counts": torch.empty(E, dtype=torch.int32, device=dev),
        "offsets": torch.empty(E + 1, dtype=torch.int32, device=dev),
        "perm": torch.empty(M, dtype=torch.int32, device=dev),
        "inv": torch.empty(M, dtype=torch.int32, device=dev),
        "w_perm": torch.empty(M, dtype=torch.float32, device=dev),
        "x_perm": torch.empty(M, d, dtype=torch.bfloat16, device=dev) if (gather and x is not None) else None,
    }
    nbytes = permute_workspace_size(T, E, k)
    ws = _workspace(nbytes, dev)
    _check(lib().moe_permute(_ptr(x), _ptr(topk_ids), _ptr(topk_w), T, d, E, k, _ptr(out["counts"]),
                             _ptr(out["offsets"]), _ptr(out["perm"]), _ptr(out["inv"]), _ptr(out["x_perm"]),
                             _ptr(out["w_perm"]), _ptr(ws), ws.numel(), _stream()), "moe_permute")
    return out


def expert_ffn(x_perm, w_perm, offsets, w_gate, w_up, w_down, h=None, y=None):
    """Grouped gate/up + SwiGLU and grouped down + routing weight; returns (h bf16, y fp16)."""
    _need(x_perm, "x_perm", torch.bfloat16, 2)
    _need(w_perm, "w_perm", torch.float32, 1)
    _need(offsets, "offsets", torch.int32, 1)
    for n, t in (("w_gate", w_gate), ("w_up", w_up), ("w_down", w_down)):
        _need(t, n, torch.bfloat16, 3)
    M, d = x_perm.shape
    E, _, f = w_gate.shape
    if h is None:
        h = torch.empty(M, f, dtype=torch.bfloat16, device=x_perm.device)
    if y is None:
        y = torch.empty(M, d, dtype=torch.float16, device=x_perm.device)
    _need(y, "y", torch.float16, 2)
    _check(lib().moe_expert_ffn(_ptr(x_perm), _ptr(w_perm), _ptr(offsets), _ptr(w_gate), _ptr(w_up),
                                _ptr(w_down), M, d, E, f, _ptr(h), _ptr(y), _stream()), "moe_expert_ffn")
    return h, y


def shared_ffn(x, w_gate_s, w_up_s, w_down_s, h_s=None, y_s=None):
    """Shared experts on every token; returns (h_s bf16 [T, f_s] scratch, y_s fp16 [n_s, T, d])."""
    _need(x, "x", torch.bfloat16, 2)
    for n, t in (("w_gate_s", w_gate_s), ("w_up_s", w_up_s), ("w_down_s", w_down_s)):
        _need(t, n, torch.bfloat16, 3)
    T, d = x.shape
    n_s, _, f_s = w_gate_s.shape
    if h_s is None:
        h_s = torch.empty(T, f_s, dtype=torch.bfloat16, device=x.device)
    if y_s is None:
        y_s = torch.empty(n_s, T, d, dtype=torch.float16, device=x.device)
    _need(y_s, "y_s", torch.float16, 3)
    _check(lib().moe_shared_ffn(_ptr(x), _ptr(w_gate_s), _ptr(w_up_s), _ptr(w_down_s), T, d, n_s, f_s, _ptr(h_s),
                                _ptr(y_s), _stream()), "moe_shared_ffn")
    return h_s, y_s


def combine_shared(y, inv, y_s, T, k, out=None):
    """out[t] = sum_j y[inv[t*k+j]] + sum_s y_s[s, t] (fp32 sum: routed slots, then ascending s)."""
    _need(y, "y", torch.float16, 2)
    _need(inv, "inv", torch.int32, 1)
    _need(y_s, "y_s", torch.float16, 3)
    d = y.shape[1]
    if out is None:
        out = torch.empty(T, d, dtype=torch.float32, device=y.device)
    _need(out, "out", torch.float32, 2)
    _check(lib().moe_combine_shared(_ptr(y), _ptr(inv), _ptr(y_s), y_s.shape[0], T, d, k, _ptr(out), _stream()),
           "moe_combine_shared")
    return out


def forward_shared(x, w_router, w_gate, w_up, w_down, w_gate_s, w_up_s, w_down_s, k, bias=None, out=None,
                   workspace=None, topk_ids=None, topk_w=None, events=None, flags=0):
    """The MoE block plus shared experts (weight one on every token); returns out [T, d] fp32."""
    T, d, E, f = _forward_args(x, w_router, w_gate, w_up, w_down, bias)
    for n, t in (("w_gate_s", w_gate_s), ("w_up_s", w_up_s), ("w_down_s", w_down_s)):
        _need(t, n, torch.bfloat16, 3)
    n_s, _, f_s = w_gate_s.shape
    if out is None:
        out = torch.empty(T, d, dtype=torch.float32, device=x.device)
    _need(out, "out", torch.float32, 2)
    nbytes = int(lib().moe_workspace_size_shared(T, d, E, k, f, n_s, f_s))
    if nbytes == 0:
        raise MoEError(MOE_ERR_UNSUPPORTED_SHAPE, "moe_workspace_size_shared")
    if workspace is None or workspace.numel() < nbytes:
        workspace = _workspace(nbytes, x.device)
    arr, n = _event_array(events)
    _check(lib().moe_forward_shared(_ptr(x), _ptr(w_router), _ptr(bias), _ptr(w_gate), _ptr(w_up), _ptr(w_down),
                                    _ptr(w_gate_s), _ptr(w_up_s), _ptr(w_down_s), T, d, E, k, f, n_s, f_s,
                                    _ptr(out), _ptr(topk_ids), _ptr(topk_w), _ptr(workspace), workspace.numel(),
                                    _stream(), arr, n, int(flags or 0)), "moe_forward_shared")
    return out


def forward_rounded(x, w_router, w_gate, w_up, w_down, k, tile=256, bias=None, out=None, workspace=None,
                    counts=None, rows=None, events=None):
    """The block with token rounding (every expert's token count rounded to a
    multiple of ``tile``); returns (out fp32 [T, d], counts int32 [E], rows).
    ``rows`` (optional int32 [T, E] output): the grouped row of (t, e), -1
    where token t does not go to expert e."""
    T, d, E, f = _forward_args(x, w_router, w_gate, w_up, w_down, bias)
    if out is None:
        out = torch.empty(T, d, dtype=torch.float32, device=x.device)
    _need(out, "out", torch.float32, 2)
    if counts is None:
        counts = torch.empty(E, dtype=torch.int32, device=x.device)
    if rows is not None:
        _need(rows, "rows", torch.int32, 2)
    nbytes = int(lib().moe_workspace_size_rounded(T, d, E, k, f, tile))
    if nbytes == 0:
        raise MoEError(MOE_ERR_UNSUPPORTED_SHAPE, "moe_workspace_size_rounded")
    if workspace is None or workspace.numel() < nbytes:
        workspace = _workspace(nbytes, x.device)
    arr, n = _event_array(events)
    _check(lib().moe_forward_rounded(_ptr(x), _ptr(w_router), _ptr(bias), _ptr(w_gate), _ptr(w_up), _ptr(w_down),
                                     T, d, E, k, f, tile, _ptr(out), _ptr(counts), _ptr(rows), _ptr(workspace),
                                     workspace.numel(), _stream(), arr, n), "moe_forward_rounded")
    return out, counts, rows


def combine(y, inv, T, k, out=None):
    """out[t] = sum_j y[inv[t*k+j]] (fp16 rows widened to fp32, fp32 sum, fp32 result)."""
    _need(y, "y", torch.float16, 2)
    _need(inv, "inv", torch.int32, 1)
    d = y.shape[1]
    if out is None:
        out = torch.empty(T, d, dtype=torch.float32, device=y.device)
    _need(out, "out", torch.float32, 2)
    _check(lib().moe_combine(_ptr(y), _ptr(inv), T, d, k, _ptr(out), _stream()), "moe_combine")
    return out


def _forward_args(x, w_router, w_gate, w_up, w_down, bias):
    _need(x, "x", torch.bfloat16, 2)
    _need(w_router, "w_router", torch.bfloat16, 2)
    for n, t in (("w_gate", w_gate), ("w_up", w_up), ("w_down", w_down)):
        _need(t, n, torch.bfloat16, 3)
    if bias is not None:
        _need(bias, "bias", torch.float32, 1)
    T, d = x.shape
    E, _, f = w_gate.shape
    return T, d, E, f


MOE_FLAG_FUSED_GATHER = 1
MOE_FLAG_RENORMALIZE = 2
MOE_FLAG_OUT_F16 = 4
MOE_FLAG_GRAD_BF16 = 8


def forward(x, w_router, w_gate, w_up, w_down, k, bias=None, out=None, workspace=None,
            topk_ids=None, topk_w=None, events=None, flags=None):
    """The whole MoE block; returns out [T, d] fp32 (fp16 with MOE_FLAG_OUT_F16).

    ``events`` (optional): a list of >= 6 torch.cuda.Event objects (or None
    to skip a boundary) recorded at the stage boundaries (before route, after
    route, after permute, after gate/up, after down, after combine).  ``flags`` (optional):
    MOE_FLAG_FUSED_GATHER selects the variant whose gate/up GEMM gathers the
    rows of x itself (identical results); MOE_FLAG_RENORMALIZE divides each
    token's k routing weights by their sum; MOE_FLAG_OUT_F16 stores out as
    fp16 (the fp32 result rounded once).
    """
    T, d, E, f = _forward_args(x, w_router, w_gate, w_up, w_down, bias)
    out_dtype = torch.float16 if (flags or 0) & MOE_FLAG_OUT_F16 else torch.float32
    if out is None:
        out = torch.empty(T, d, dtype=out_dtype, device=x.device)
    _need(out, "out", out_dtype, 2)
    nbytes = workspace_size(T, d, E, k, f)
    if nbytes == 0:
        raise MoEError(MOE_ERR_UNSUPPORTED_SHAPE, "moe_workspace_size")
    if workspace is None:
        workspace = _workspace(nbytes, x.device)
    args = [_ptr(x), _ptr(w_router), _ptr(bias), _ptr(w_gate), _ptr(w_up), _ptr(w_down), T, d, E, k, f,
            _ptr(out), _ptr(topk_ids), _ptr(topk_w), _ptr(workspace), workspace.numel(), _stream()]
    if events is None and flags is None:
        _check(lib().moe_forward(*args), "moe_forward")
    else:
        arr, n = _event_array(events)
        _check(lib().moe_forward_ex(*args, arr, n, int(flags or 0)), "moe_forward_ex")
    return out


def gather_rows(src, idx, out=None):
    """out[i] = src[idx[i]] (whole rows) on the GPU; src is 1-D or 2-D and
    contiguous, each row a multiple of 4 bytes; idx int32 on the same device."""
    if not (src.is_cuda and src.is_contiguous() and src.dim() in (1, 2)):
        raise ValueError("src: contiguous 1-D or 2-D CUDA tensor expected")
    if src.dim() == 1:
        return gather_rows(src.view(-1, 1), idx, None if out is None else out.view(-1, 1)).view(-1)
    _need(idx, "idx", torch.int32, 1)
    n = idx.shape[0]
    if out is None:
        out = torch.empty(n, src.shape[1], dtype=src.dtype, device=src.device)
    row_bytes = src.shape[1] * src.element_size()
    _check(lib().moe_gather_rows(_ptr(src), _ptr(idx), src.shape[0], n, row_bytes, _ptr(out), _stream()),
           "moe_gather_rows")
    return out


def backward_workspace_size(T: int, d: int, E: int, k: int, f: int) -> int:
    return int(lib().moe_backward_workspace_size(T, d, E, k, f))


def backward(x, w_router, w_gate, w_up, w_down, k, dout, bias=None, workspace=None, renormalize=False,
             want_dbias=True, grad_dtype=torch.float32):
    """Gradient of sum(dout * out) of the block (moe_backward): returns a dict
    of tensors dx [T, d] fp32, dw_router [d, E], dbias [E] fp32 (None unless
    want_dbias), dw_gate / dw_up [E, d, f], dw_down [E, f, d].  The four
    weight gradients are fp32, or bf16 with grad_dtype=torch.bfloat16
    (MOE_FLAG_GRAD_BF16: the fp32 results rounded once)."""
    T, d, E, f = _forward_args(x, w_router, w_gate, w_up, w_down, bias)
    _need(dout, "dout", torch.float32, 2)
    if grad_dtype not in (torch.float32, torch.bfloat16):
        raise ValueError("grad_dtype: torch.float32 or torch.bfloat16")
    dev = x.device
    gd = grad_dtype
    g = {
        "dx": torch.empty(T, d, dtype=torch.float32, device=dev),
        "dw_router": torch.empty(d, E, dtype=gd, device=dev),
        "dbias": torch.empty(E, dtype=torch.float32, device=dev) if want_dbias else None,
        "dw_gate": torch.empty(E, d, f, dtype=gd, device=dev),
        "dw_up": torch.empty(E, d, f, dtype=gd, device=dev),
        "dw_down": torch.empty(E, f, d, dtype=gd, device=dev),
    }
    nbytes = backward_workspace_size(T, d, E, k, f)
    if nbytes == 0:
        raise MoEError(MOE_ERR_UNSUPPORTED_SHAPE, "moe_backward_workspace_size")
    if workspace is None:
        workspace = _workspace(nbytes, dev)
    flags = (MOE_FLAG_RENORMALIZE if renormalize else 0) | (MOE_FLAG_GRAD_BF16 if gd == torch.bfloat16 else 0)
    _check(lib().moe_backward(_ptr(x), _ptr(w_router), _ptr(bias), _ptr(w_gate), _ptr(w_up), _ptr(w_down),
                              _ptr(dout), T, d, E, k, f, _ptr(g["dx"]), _ptr(g["dw_router"]), _ptr(g["dbias"]),
                              _ptr(g["dw_gate"]), _ptr(g["dw_up"]), _ptr(g["dw_down"]), _ptr(workspace),
                              workspace.numel(), _stream(), flags), "moe_backward")
    return g


def _event_array(events):
    """ctypes array of cudaEvent_t handles (None entries stay NULL), and its length."""
    if events is None:
        return None, 0
    arr = (ctypes.c_void_p * len(events))()
    for i, ev in enumerate(events):
        if ev is None:
            continue
        if ev.cuda_event == 0:
            ev.record()  # the event handle is created lazily by torch
        arr[i] = ev.cuda_event
    return arr, len(events)


def get_status() -> int:
    """Synchronise the current stream; return and clear the device status word."""
    return int(lib().moe_get_status(_stream()))


def set_wait_limit_ns(limit_ns: int):
    _check(lib().moe_set_wait_limit_ns(int(limit_ns)), "moe_set_wait_limit_ns")


def selftest_wait_timeout(limit_ns: int):
    _check(lib().moe_selftest_wait_timeout(int(limit_ns), _stream()), "moe_selftest_wait_timeout")


class MoEBlock:
    """Weights of one MoE block on the GPU plus a reusable workspace."""

    def __init__(self, w_router, w_gate, w_up, w_down, k, bias=None, renormalize=False):
        self.w_router, self.w_gate, self.w_up, self.w_down = w_router, w_gate, w_up, w_down
        self.bias = bias
        self.renormalize = bool(renormalize)
        self.k = int(k)
        self.E, self.d, self.f = w_gate.shape
        self._ws = None

    def workspace(self, T: int) -> torch.Tensor:
        need = workspace_size(T, self.d, self.E, self.k, self.f)
        if self._ws is None or self._ws.numel() < need:
            self._ws = _workspace(need, self.w_gate.device)
        return self._ws

    def __call__(self, x, out=None, topk_ids=None, topk_w=None, events=None, flags=None):
        if self.renormalize:
            flags = (flags or 0) | MOE_FLAG_RENORMALIZE
        return forward(x, self.w_router, self.w_gate, self.w_up, self.w_down, self.k, bias=self.bias,
                       out=out, workspace=self.workspace(x.shape[0]), topk_ids=topk_ids, topk_w=topk_w,
                       events=events, flags=flags)


__all__ = [
    "lib", "strerror", "MoEError", "ABI_SYMBOLS", "workspace_size", "route_workspace_size",
    "permute_workspace_size", "MOE_FLAG_FUSED_GATHER", "MOE_FLAG_RENORMALIZE", "MOE_FLAG_OUT_F16", "MOE_FLAG_GRAD_BF16", "route",
    "permute", "expert_ffn", "combine", "forward", "shared_ffn", "combine_shared", "forward_shared", "forward_rounded",
    "get_status", "set_wait_limit_ns", "backward", "backward_workspace_size", "gather_rows",
    "selftest_wait_timeout", "MoEBlock",
]
