"""The C-ABI library builds, loads and exports every declared entry point;
host-side validation answers without touching a GPU (CPU only)."""
import ctypes
import os
import re
import subprocess

import pytest

import top_routing_grouped_softmax_b200 as moe

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "moe.h")


def _declared():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(moe_[a-z0-9_]+)\s*\(", text)))


def test_header_matches_binding_list():
    assert set(_declared()) == set(moe.ABI_SYMBOLS)


def test_flag_values_match_header():
    flags = dict(re.findall(r"#define\s+(MOE_FLAG_[A-Z0-9_]+)\s+(\d+)u", open(HEADER).read()))
    assert flags and {k: int(v) for k, v in flags.items()} == {k: getattr(moe, k) for k in flags}


def test_library_exports_every_declared_symbol(moe_lib):
    out = subprocess.run(["nm", "-D", "--defined-only", moe.LIB_PATH], capture_output=True, text=True,
                         check=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if " T " in line}
    missing = [s for s in _declared() if s not in exported]
    assert not missing, f"not exported: {missing}"
    for s in _declared():
        getattr(moe_lib, s)


def test_strerror_and_version(moe_lib):
    assert moe_lib.moe_version() == 203
    for code in range(10):
        assert moe.strerror(code).startswith("MOE_")


def test_workspace_sizes(moe_lib):
    ws = moe.workspace_size(8192, 2048, 128, 8, 768)
    M = 8192 * 8
    assert ws >= M * (2048 * 2 + 768 * 2)     # y (fp16) + h (bf16) at least
    assert ws % 256 == 0
    assert moe.workspace_size(8192, 2048, 12, 8, 768) == 0       # E % 8 != 0
    assert moe.workspace_size(8192, 2000, 128, 8, 768) == 0      # d % 64 != 0
    assert moe.workspace_size(8192, 2048, 128, 33, 768) == 0     # k > 32
    assert moe.workspace_size(0, 2048, 128, 8, 768) > 0
    assert moe.permute_workspace_size(8192, 128, 8) == (8192 // 64) * 128 * 4
    assert moe.route_workspace_size(8192, 2048, 128) == 0   # logits stay on chip
    assert moe.route_workspace_size(8192, 2048, 12) == 0


def test_validation_happens_before_any_device_call(moe_lib):
    L = moe_lib
    null = ctypes.c_void_p(0)
    # null pointers
    assert L.moe_route(null, null, null, 16, 64, 8, 2, null, null, null, 0, null) == moe.MOE_ERR_INVALID_ARG
    # unsupported shapes are rejected before pointers are even looked at
    assert L.moe_route(null, null, null, 16, 64, 12, 2, null, null, null, 0, null) == moe.MOE_ERR_UNSUPPORTED_SHAPE
    assert L.moe_route(null, null, null, 16, 64, 8, 9, null, null, null, 0, null) == moe.MOE_ERR_UNSUPPORTED_SHAPE
    assert L.moe_route(null, null, null, -1, 64, 8, 2, null, null, null, 0, null) == moe.MOE_ERR_INVALID_ARG
    # misaligned (odd) pointer
    odd = ctypes.c_void_p(0x1001)
    assert L.moe_route(odd, odd, null, 16, 64, 8, 2, odd, odd, odd, 1 << 20, null) == moe.MOE_ERR_INVALID_ARG
    fake = ctypes.c_void_p(0x10000)
    assert L.moe_permute(fake, fake, fake, 1000, 64, 8, 2, fake, fake, fake, fake, null, fake, fake, 16,
                         null) == moe.MOE_ERR_WORKSPACE_TOO_SMALL
    # unknown flag bits
    assert L.moe_forward_ex(fake, fake, null, fake, fake, fake, 16, 64, 8, 2, 64, fake, null, null, fake, 1 << 30,
                            null, null, 0, 8) == moe.MOE_ERR_INVALID_ARG
    # fp16 output is an option of moe_forward_ex only
    assert L.moe_forward_shared(null, null, null, null, null, null, null, null, null, 16, 64, 8, 2, 64, 1, 64, null,
                                null, null, null, 0, null, null, 0, moe.MOE_FLAG_OUT_F16) == moe.MOE_ERR_INVALID_ARG
    assert L.moe_combine(null, null, 4, 64, 2, null, null) == moe.MOE_ERR_INVALID_ARG
    assert L.moe_combine(null, null, 4, 65, 2, null, null) == moe.MOE_ERR_UNSUPPORTED_SHAPE
    # workspace too small is caught on the host
    assert L.moe_forward(fake, fake, null, fake, fake, fake, 16, 64, 8, 2, 64, fake, null, null, fake, 16,
                         null) == moe.MOE_ERR_WORKSPACE_TOO_SMALL


def test_binding_fails_loudly_without_library(monkeypatch):
    monkeypatch.setattr(moe, "_lib", None)
    monkeypatch.setattr(moe, "LIB_PATH", "/nonexistent/libmoe.so")
    with pytest.raises(ImportError):
        moe.lib()


def test_product_never_touches_the_oracle():
    pkg = os.path.join(ROOT, "top_routing_grouped_softmax_b200")
    for dirpath, _, files in os.walk(pkg):
        for fn in files:
            if fn.endswith((".py", ".cu", ".cuh", ".h")):
                text = open(os.path.join(dirpath, fn)).read()
                assert "import oracle" not in text and "from oracle" not in text, fn
                assert "moe_oracle" not in text and "liboracle" not in text, fn


def test_shared_expert_validation(moe_lib):
    """Shared-expert entry points reject bad counts and sizes on the host."""
    L = moe_lib
    null = ctypes.c_void_p(0)
    assert moe.lib().moe_workspace_size_shared(8192, 2048, 128, 8, 768, 1, 768) > \
        moe.workspace_size(8192, 2048, 128, 8, 768)
    assert L.moe_workspace_size_shared(8192, 2048, 128, 8, 768, 9, 768) == 0     # more than 8 shared experts
    assert L.moe_workspace_size_shared(8192, 2048, 128, 8, 768, 1, 700) == 0     # f_shared % 64 != 0
    fake = ctypes.c_void_p(0x10000)
    args = [fake] * 9 + [16, 64, 8, 2, 64]
    assert L.moe_forward_shared(*args, 0, 64, fake, null, null, fake, 1 << 30, null, null, 0, 0) == \
        moe.MOE_ERR_INVALID_ARG                                                    # n_shared = 0
    assert L.moe_forward_shared(*args, 9, 64, fake, null, null, fake, 1 << 30, null, null, 0, 0) == \
        moe.MOE_ERR_UNSUPPORTED_SHAPE
    assert L.moe_combine_shared(fake, fake, null, 1, 4, 64, 2, fake, null) == moe.MOE_ERR_INVALID_ARG
