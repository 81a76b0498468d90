"""fp64 CPU oracle for exact attention (forward and backward).

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and
the benchmark's CPU-baseline / reference leg may import this package.  The
CUDA product path never calls it and has no CPU fallback.

All functions take float64 arrays shaped (B, H, N, d) (or (BH, N, d)) and
return float64 results; the C routines are in ``attn_oracle.c`` (see its
header for the passages each routine follows).
"""

from __future__ import annotations

import ctypes
import os

import numpy as np

from . import build as _build

_lib = None


def lib():
    global _lib
    if _lib is None:
        path = _build.build()
        L = ctypes.CDLL(path)
        dp = ctypes.POINTER(ctypes.c_double)
        lp = ctypes.POINTER(ctypes.c_int64)
        i64, ci, cd = ctypes.c_int64, ctypes.c_int, ctypes.c_double
        L.oracle_fwd.argtypes = [dp, dp, dp, dp, dp, i64, i64, i64, ci, cd]
        L.oracle_fwd.restype = None
        L.oracle_fwd_rows.argtypes = [dp, dp, dp, i64, i64, i64, ci, cd, lp, i64, dp, dp]
        L.oracle_fwd_rows.restype = None
        L.oracle_fwd_online.argtypes = [dp, dp, dp, dp, dp, i64, i64, i64, ci, cd, i64]
        L.oracle_fwd_online.restype = None
        L.oracle_bwd_heads.argtypes = [dp, dp, dp, dp, i64, i64, i64, ci, cd, lp, i64, dp, dp, dp]
        L.oracle_bwd_heads.restype = None
        u8 = ctypes.POINTER(ctypes.c_uint8)
        L.oracle_fwd_blocksparse.argtypes = [dp, dp, dp, dp, dp, i64, i64, i64, ci, cd, u8, i64]
        L.oracle_fwd_blocksparse.restype = None
        L.oracle_bwd_blocksparse_heads.argtypes = [dp, dp, dp, dp, i64, i64, i64, ci, cd, u8, i64,
                                                   lp, i64, dp, dp, dp]
        L.oracle_bwd_blocksparse_heads.restype = None
        fp = ctypes.POINTER(ctypes.c_float)
        L.oracle_e4m3_round.argtypes = [ctypes.c_float]
        L.oracle_e4m3_round.restype = ctypes.c_float
        L.oracle_fwht32.argtypes = [fp, i64, i64]
        L.oracle_fwht32.restype = None
        L.oracle_fp8_quantize.argtypes = [dp, i64, i64, i64, ctypes.POINTER(ctypes.c_int8), ci,
                                          fp, fp]
        L.oracle_fp8_quantize.restype = None
        u32p = ctypes.POINTER(ctypes.c_uint32)
        L.oracle_philox4x32_10.argtypes = [u32p, u32p, u32p]
        L.oracle_philox4x32_10.restype = None
        L.oracle_dropout_mask.argtypes = [i64, i64, ctypes.c_uint64, ci, ctypes.POINTER(ctypes.c_uint8)]
        L.oracle_dropout_mask.restype = None
        L.oracle_fwd_dropout.argtypes = [dp, dp, dp, dp, dp, i64, i64, i64, ci, cd,
                                         ctypes.c_uint64, ci]
        L.oracle_fwd_dropout.restype = None
        L.oracle_bwd_dropout_heads.argtypes = [dp, dp, dp, dp, i64, i64, i64, ci, cd,
                                               ctypes.c_uint64, ci, lp, i64, dp, dp, dp]
        L.oracle_bwd_dropout_heads.restype = None
        L.oracle_linear_attn.argtypes = [dp, dp, dp, dp, i64, i64, i64, cd]
        L.oracle_linear_attn.restype = None
        L.oracle_linear_attn_chunked.argtypes = [dp, dp, dp, dp, i64, i64, i64, cd, i64]
        L.oracle_linear_attn_chunked.restype = None
        L.oracle_num_threads.argtypes = []
        L.oracle_num_threads.restype = ci
        L.oracle_set_num_threads.argtypes = [ci]
        L.oracle_set_num_threads.restype = None
        _lib = L
    return _lib


def _f64(a):
    return np.ascontiguousarray(a, dtype=np.float64)


def _p(a, t=ctypes.c_double):
    return a.ctypes.data_as(ctypes.POINTER(t))


def _dims(q):
    if q.ndim == 4:
        B, H, N, d = q.shape
        return B * H, N, d
    if q.ndim == 3:
        return q.shape
    raise ValueError("expected (B,H,N,d) or (BH,N,d)")


def num_threads() -> int:
    return lib().oracle_num_threads()


def set_num_threads(n: int) -> None:
    lib().oracle_set_num_threads(int(n))


def fwd(q, k, v, causal: bool, scale: float):
    """Two-pass exact forward: returns (O, LSE) shaped like q and q.shape[:-1]."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    BH, N, d = _dims(q)
    o = np.empty_like(q)
    lse = np.empty(q.shape[:-1], dtype=np.float64)
    lib().oracle_fwd(_p(q), _p(k), _p(v), _p(o), _p(lse), BH, N, d, int(bool(causal)), float(scale))
    return o, lse


def fwd_rows(q, k, v, causal: bool, scale: float, rows):
    """Forward for selected rows; ``rows`` are flat indices bh*N + i.

    Returns (O_rows (len, d), LSE_rows (len,))."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    BH, N, d = _dims(q)
    rows = np.ascontiguousarray(rows, dtype=np.int64)
    if rows.size and (rows.min() < 0 or rows.max() >= BH * N):
        raise IndexError("row index out of range")
    o = np.empty((rows.size, d), dtype=np.float64)
    lse = np.empty(rows.size, dtype=np.float64)
    lib().oracle_fwd_rows(_p(q), _p(k), _p(v), BH, N, d, int(bool(causal)), float(scale),
                          _p(rows, ctypes.c_int64), rows.size, _p(o), _p(lse))
    return o, lse


def fwd_online(q, k, v, causal: bool, scale: float, block: int):
    """The per-block online-softmax pseudo-code in fp64 (self-check only)."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    BH, N, d = _dims(q)
    o = np.empty_like(q)
    lse = np.empty(q.shape[:-1], dtype=np.float64)
    lib().oracle_fwd_online(_p(q), _p(k), _p(v), _p(o), _p(lse), BH, N, d, int(bool(causal)),
                            float(scale), int(block))
    return o, lse


def bwd_heads(q, k, v, dout, causal: bool, scale: float, heads=None):
    """Exact gradients of sum(O * dO) for the listed flat heads (bh indices).

    Returns (dQ, dK, dV), each (len(heads), N, d)."""
    q, k, v, dout = _f64(q), _f64(k), _f64(v), _f64(dout)
    BH, N, d = _dims(q)
    if heads is None:
        heads = np.arange(BH)
    heads = np.ascontiguousarray(heads, dtype=np.int64)
    if heads.size and (heads.min() < 0 or heads.max() >= BH):
        raise IndexError("head index out of range")
    shp = (heads.size, N, d)
    dq, dk, dv = np.empty(shp), np.empty(shp), np.empty(shp)
    lib().oracle_bwd_heads(_p(q), _p(k), _p(v), _p(dout), BH, N, d, int(bool(causal)),
                           float(scale), _p(heads, ctypes.c_int64), heads.size,
                           _p(dq), _p(dk), _p(dv))
    return dq, dk, dv


def bwd(q, k, v, dout, causal: bool, scale: float):
    """Exact gradients for every head, shaped like q."""
    shape = np.shape(q)
    dq, dk, dv = bwd_heads(q, k, v, dout, causal, scale)
    return dq.reshape(shape), dk.reshape(shape), dv.reshape(shape)


def _block_mask(mask, N, blk):
    mask = np.ascontiguousarray(mask, dtype=np.uint8)
    nb = (N + blk - 1) // blk
    if mask.shape != (nb, nb):
        raise ValueError(f"block mask must be ({nb}, {nb}) for N={N}, block {blk}")
    return mask


def fwd_blocksparse(q, k, v, mask, causal: bool, scale: float, block: int = 128):
    """Block-sparse forward: key j is visible to query i iff
    mask[i // block, j // block] != 0 (and j <= i when causal).  Rows with no
    visible key get O = 0 and LSE = -inf.  Returns (O, LSE)."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    BH, N, d = _dims(q)
    mask = _block_mask(mask, N, block)
    o = np.empty_like(q)
    lse = np.empty(q.shape[:-1], dtype=np.float64)
    lib().oracle_fwd_blocksparse(_p(q), _p(k), _p(v), _p(o), _p(lse), BH, N, d,
                                 int(bool(causal)), float(scale), _p(mask, ctypes.c_uint8),
                                 int(block))
    return o, lse


def bwd_blocksparse_heads(q, k, v, dout, mask, causal: bool, scale: float, heads=None,
                          block: int = 128):
    """Exact gradients of sum(O * dO) under the block mask, for the listed heads."""
    q, k, v, dout = _f64(q), _f64(k), _f64(v), _f64(dout)
    BH, N, d = _dims(q)
    mask = _block_mask(mask, N, block)
    if heads is None:
        heads = np.arange(BH)
    heads = np.ascontiguousarray(heads, dtype=np.int64)
    if heads.size and (heads.min() < 0 or heads.max() >= BH):
        raise IndexError("head index out of range")
    shp = (heads.size, N, d)
    dq, dk, dv = np.empty(shp), np.empty(shp), np.empty(shp)
    lib().oracle_bwd_blocksparse_heads(_p(q), _p(k), _p(v), _p(dout), BH, N, d,
                                       int(bool(causal)), float(scale), _p(mask, ctypes.c_uint8),
                                       int(block), _p(heads, ctypes.c_int64), heads.size,
                                       _p(dq), _p(dk), _p(dv))
    return dq, dk, dv


def bwd_blocksparse(q, k, v, dout, mask, causal: bool, scale: float, block: int = 128):
    """Block-sparse gradients for every head, shaped like q."""
    shape = np.shape(q)
    dq, dk, dv = bwd_blocksparse_heads(q, k, v, dout, mask, causal, scale, block=block)
    return dq.reshape(shape), dk.reshape(shape), dv.reshape(shape)


def e4m3_round(x: float) -> float:
    """Nearest e4m3 value of an fp32 number (ties to even, saturating at 448)."""
    return float(lib().oracle_e4m3_round(float(x)))


def fwht32(x):
    """Unnormalised Walsh-Hadamard transform of each row of x in fp32 butterflies."""
    y = np.ascontiguousarray(x, dtype=np.float32).copy()
    d = y.shape[-1]
    lib().oracle_fwht32(_p(y, ctypes.c_float), y.size // d, d)
    return y


def fp8_quantize(x, signs=None, rotate: bool = True):
    """Block-wise e4m3 quantisation of x (B, H, N, d) or (BH, N, d), after the
    randomised Hadamard rotation when `rotate`.  Returns (codes, scales): codes
    shaped like x (the e4m3 values, as float32), scales (..., ceil(N / 128))."""
    x = _f64(x)
    BH, N, d = _dims(x)
    nb = (N + 127) // 128
    codes = np.empty(x.shape, dtype=np.float32)
    scales = np.empty(x.shape[:-2] + (nb,), dtype=np.float32)
    sg = None
    if signs is not None:
        sg = np.ascontiguousarray(signs, dtype=np.int8)
        if sg.shape != (d,):
            raise ValueError("signs must have d entries")
    lib().oracle_fp8_quantize(_p(x), BH, N, d,
                              None if sg is None else _p(sg, ctypes.c_int8), int(bool(rotate)),
                              _p(codes, ctypes.c_float), _p(scales, ctypes.c_float))
    return codes, scales


def fp8_dequantize(codes, scales):
    """codes * their block's scale, in fp64 (exact)."""
    codes = np.asarray(codes, dtype=np.float64)
    N = codes.shape[-2]
    per_row = np.repeat(np.asarray(scales, dtype=np.float64), 128, axis=-1)[..., :N]
    return codes * per_row[..., None]


def fwd_fp8(q, k, v, causal: bool, scale: float, signs=None, rotate: bool = True):
    """The FP8 forward as the method computes it: Q and K rotated and quantised
    block-wise to e4m3 (fp8_quantize), the scores scale (q~ . k~) / d (the
    rotation multiplies dot products by d; 1 without it), then the exact
    two-pass attention in fp64 with the 16-bit V.  Returns (O, LSE)."""
    d = np.shape(q)[-1]
    qc, qs = fp8_quantize(q, signs, rotate)
    kc, ks = fp8_quantize(k, signs, rotate)
    return fwd(fp8_dequantize(qc, qs), fp8_dequantize(kc, ks), v, causal,
               scale / (d if rotate else 1.0))


def dropout_threshold(p: float) -> int:
    """The 8-bit keep threshold t = round(256 (1 - p)), clamped to 1 .. 256."""
    return int(min(256, max(1, round(256.0 * (1.0 - float(p))))))


def philox4x32_10(ctr, key):
    """Philox4x32-10 of four 32-bit counter words and two key words."""
    c = (ctypes.c_uint32 * 4)(*[int(x) & 0xFFFFFFFF for x in ctr])
    k = (ctypes.c_uint32 * 2)(*[int(x) & 0xFFFFFFFF for x in key])
    out = (ctypes.c_uint32 * 4)()
    lib().oracle_philox4x32_10(c, k, out)
    return [int(x) for x in out]


def dropout_mask(BH: int, N: int, seed: int, p: float):
    """Z (BH, N, N) uint8: 1 where the probability P_ij is kept."""
    z = np.empty((BH, N, N), dtype=np.uint8)
    lib().oracle_dropout_mask(BH, N, int(seed), dropout_threshold(p), _p(z, ctypes.c_uint8))
    return z


def fwd_dropout(q, k, v, causal: bool, scale: float, p: float, seed: int):
    """Forward with dropout on P (kept values scaled by 256 / t): (O, LSE)."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    BH, N, d = _dims(q)
    o = np.empty_like(q)
    lse = np.empty(q.shape[:-1], dtype=np.float64)
    lib().oracle_fwd_dropout(_p(q), _p(k), _p(v), _p(o), _p(lse), BH, N, d, int(bool(causal)),
                             float(scale), int(seed), dropout_threshold(p))
    return o, lse


def bwd_dropout_heads(q, k, v, dout, causal: bool, scale: float, p: float, seed: int,
                      heads=None):
    """Exact gradients of sum(O * dO) with the same dropout mask, listed heads."""
    q, k, v, dout = _f64(q), _f64(k), _f64(v), _f64(dout)
    BH, N, d = _dims(q)
    if heads is None:
        heads = np.arange(BH)
    heads = np.ascontiguousarray(heads, dtype=np.int64)
    shp = (heads.size, N, d)
    dq, dk, dv = np.empty(shp), np.empty(shp), np.empty(shp)
    lib().oracle_bwd_dropout_heads(_p(q), _p(k), _p(v), _p(dout), BH, N, d, int(bool(causal)),
                                   float(scale), int(seed), dropout_threshold(p),
                                   _p(heads, ctypes.c_int64), heads.size, _p(dq), _p(dk), _p(dv))
    return dq, dk, dv


def bwd_dropout(q, k, v, dout, causal: bool, scale: float, p: float, seed: int):
    shape = np.shape(q)
    dq, dk, dv = bwd_dropout_heads(q, k, v, dout, causal, scale, p, seed)
    return dq.reshape(shape), dk.reshape(shape), dv.reshape(shape)


def linear_attn(q, k, v, scale: float):
    """Causal linear attention O_i = scale sum_{j <= i} (q_i . k_j) v_j."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    BH, N, d = _dims(q)
    o = np.empty_like(q)
    lib().oracle_linear_attn(_p(q), _p(k), _p(v), _p(o), BH, N, d, float(scale))
    return o


def linear_attn_chunked(q, k, v, scale: float, chunk: int):
    """The chunked form (in-chunk product + running state), self-check only."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    BH, N, d = _dims(q)
    o = np.empty_like(q)
    lib().oracle_linear_attn_chunked(_p(q), _p(k), _p(v), _p(o), BH, N, d, float(scale), int(chunk))
    return o
