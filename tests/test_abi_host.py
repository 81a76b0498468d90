"""The C-ABI library loads on a machine without a GPU and exports every
symbol include/attn.h declares; argument checks run before any device work."""

import ctypes
import os
import re

from io_aware_exact_30_b200 import attn, build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_symbols():
    text = open(os.path.join(ROOT, "include", "attn.h")).read()
    return sorted(set(re.findall(r"^\s*(?:const\s+)?[\w\s\*]*?\b(attn_\w+)\s*\(", text, re.M)))


def test_header_and_binding_agree():
    assert declared_symbols() == sorted(attn.EXPORTS)


def test_library_exports_every_declared_symbol():
    build.build()
    L = attn.lib()
    for name in declared_symbols():
        assert hasattr(L, name), name


def test_host_side_errors_without_device_work():
    L = attn.lib()
    assert L.attn_fwd(None, None, None, None, None, 1, 1, 16, 64, 0, 0.125, 0, None) == -1
    p = ctypes.c_void_p(16)
    assert L.attn_fwd(p, p, p, p, p, 1, 1, 16, 80, 0, 0.125, 0, None) == -3
    assert L.attn_fwd(p, p, p, p, p, 1, 1, 0, 64, 0, 0.125, 0, None) == -2
    assert L.attn_fwd(p, p, p, p, p, 1, 1, 16, 64, 0, 0.125, 3, None) == -5
    assert L.attn_fwd(p, p, p, p, p, 1, 1, 16, 64, 0, 0.0, 0, None) == -9
    assert L.attn_fwd(ctypes.c_void_p(17), p, p, p, p, 1, 1, 16, 64, 0, 0.125, 0, None) == -4
    assert L.attn_fwd(p, p, p, p, p, 1 << 16, 1 << 16, 16, 64, 0, 0.125, 0, None) == -2
    assert L.attn_bwd(*([None] * 10), 1, 1, 16, 64, 0, 0.125, 0, None) == -1
    # sizes: L2 and D (B*H*Np fp32 each, Np = N rounded up to 128) + dQ accumulator
    # (B*H*N*d fp32) + counters (B*H int32), each section 256-byte aligned
    assert attn.attn_bwd_workspace_bytes(1, 1, 1, 64) == 512 + 512 + 256 + 256
    assert attn.attn_bwd_workspace_bytes(4, 16, 4096, 128) == 2 * 64 * 4096 * 4 + 64 * 4096 * 128 * 4 + 256
    assert attn.attn_bwd_workspace_bytes(1, 1, 16, 96) == 0
    for s in attn.STATUS:
        assert attn.strerror(s)
