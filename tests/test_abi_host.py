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


def _entry_calls(L, p, B=1, H=1, N=16, d=64, dt=0, scale=0.125, drop=0.1):
    """One call of every compute entry point, with pointer p in every pointer slot
    (never dereferenced on the host) and the given sizes and scalars."""
    return {
        "attn_fwd": lambda: L.attn_fwd(p, p, p, p, p, B, H, N, d, 0, scale, dt, None),
        "attn_bwd": lambda: L.attn_bwd(*([p] * 10), B, H, N, d, 0, scale, dt, None),
        "attn_bwd_main": lambda: L.attn_bwd_main(*([p] * 8), B, H, N, d, 0, scale, dt, None),
        "attn_bwd_noalloc": lambda: L.attn_bwd_noalloc(*([p] * 9), B, H, N, d, 0, scale, dt, None),
        "attn_fwd_blocksparse": lambda: L.attn_fwd_blocksparse(*([p] * 6), B, H, N, d, 0, scale,
                                                               dt, None),
        "attn_bwd_blocksparse": lambda: L.attn_bwd_blocksparse(*([p] * 11), B, H, N, d, 0, scale,
                                                               dt, None),
        "attn_fwd_fp8": lambda: L.attn_fwd_fp8(*([p] * 7), B, H, N, d, 0, scale, 1, dt, None),
        "attn_fwd_dropout": lambda: L.attn_fwd_dropout(*([p] * 5), B, H, N, d, 0, scale, drop, 7,
                                                       dt, None),
        "attn_bwd_dropout": lambda: L.attn_bwd_dropout(*([p] * 10), B, H, N, d, 0, scale, drop,
                                                       7, dt, None),
        "attn_linear_fwd": lambda: L.attn_linear_fwd(*([p] * 5), B, H, N,
                                                     128 if d == 64 else d, scale, dt, None),
        "attn_sdpa_host": lambda: L.attn_sdpa_host(*([p] * 10), 1 << 30, B, H, N, d, 0, scale,
                                                   dt, 0, None),
        # no scale argument
        "attn_bwd_prep": lambda: L.attn_bwd_prep(p, p, p, p, B, H, N, d, dt, None),
        "attn_fp8_quantize": lambda: L.attn_fp8_quantize(p, p, p, p, 1, B, H, N, d, dt, None),
    }


def test_every_entry_point_checks_its_arguments_before_device_work():
    """Each compute entry returns the header's argument errors synchronously,
    before it queries or touches a device: a NULL pointer, a head dimension
    other than 64/128 (128 only for linear attention), B, H or N below 1, an
    unknown dtype, a scale that is not finite and positive, a dropout
    probability outside [0, 1)."""
    L = attn.lib()
    p = ctypes.c_void_p(256)
    no_scale = {"attn_bwd_prep", "attn_fp8_quantize"}
    for name, f in _entry_calls(L, None).items():
        assert f() == -1, name
    cases = [({"d": 80}, -3), ({"N": 0}, -2), ({"B": 0}, -2), ({"H": 0}, -2), ({"dt": 3}, -5)]
    for kw, want in cases:
        for name, f in _entry_calls(L, p, **kw).items():
            assert f() == want, (name, kw)
    for bad in (0.0, -1.0, float("nan"), float("inf")):
        for name, f in _entry_calls(L, p, scale=bad).items():
            if name not in no_scale:
                assert f() == -9, (name, bad)
    for bad in (1.0, -0.1, 1.5):
        calls = _entry_calls(L, p, drop=bad)
        assert calls["attn_fwd_dropout"]() == -9, bad
        assert calls["attn_bwd_dropout"]() == -9, bad
    assert L.attn_linear_fwd(p, p, p, p, p, 1, 1, 16, 64, 0.125, 0, None) == -3


def test_linear_and_host_entry_sizes():
    """Host-side size queries: linear attention keeps per (head, chunk of 128
    rows) a 128 x 128 fp32 K^T V and a 16-bit state (d = 128 only); the host
    entry's scratch grows with the chunk of heads and with the backward."""
    def a256(x):
        return (x + 255) // 256 * 256
    for B, H, N in ((1, 1, 128), (1, 1, 1), (2, 3, 300), (4, 16, 4096)):
        states = B * H * -(-N // 128) * 128 * 128
        assert attn.attn_linear_workspace_bytes(B, H, N, 128) == a256(4 * states) + a256(2 * states)
    assert attn.attn_linear_workspace_bytes(1, 1, 128, 64) == 0
    assert attn.attn_linear_workspace_bytes(1, 0, 128, 128) == 0
    f = attn.attn_sdpa_host_scratch_bytes
    assert f(4, 16, 4096, 128, 1, 0) > f(4, 16, 4096, 128, 0, 0) > 0
    assert f(4, 16, 4096, 128, 1, 16) > f(4, 16, 4096, 128, 1, 8) > f(4, 16, 4096, 128, 1, 1)
    assert f(4, 16, 4096, 96, 1, 0) == 0 and f(0, 16, 4096, 128, 1, 0) == 0
