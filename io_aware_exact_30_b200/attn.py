"""Python binding of libattn.so — argument marshalling only.

Every step of the attention path runs in the library's CUDA kernels; this
module converts torch tensors to pointers and sizes, passes the current CUDA
stream, and raises on a non-zero status.  There is no CPU fallback: if the
library is missing or the device is not sm_100, calls raise.
"""

from __future__ import annotations

import ctypes
import math
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libattn.so")

ATTN_BF16, ATTN_FP16 = 0, 1
_DTYPES = {torch.bfloat16: ATTN_BF16, torch.float16: ATTN_FP16}

STATUS = {
    0: "ATTN_OK", -1: "ATTN_ERR_NULL", -2: "ATTN_ERR_SHAPE", -3: "ATTN_ERR_HEADDIM",
    -4: "ATTN_ERR_ALIGN", -5: "ATTN_ERR_DTYPE", -6: "ATTN_ERR_DEVICE", -7: "ATTN_ERR_LAUNCH",
    -8: "ATTN_ERR_TIMEOUT", -9: "ATTN_ERR_ARG", -10: "ATTN_ERR_SCRATCH",
}

# Kernel launches one attn_bwd call makes: the preprocess, then the main
# backward (d = 64), or the main backward and the dQ conversion (d = 128).
def bwd_launches(d: int) -> int:
    return 2 if d == 64 else 3

# Every symbol include/attn.h declares.
EXPORTS = ("attn_fwd", "attn_bwd", "attn_bwd_prep", "attn_bwd_main", "attn_bwd_workspace_bytes",
           "attn_bwd_noalloc", "attn_sdpa_host", "attn_sdpa_host_scratch_bytes",
           "attn_fwd_blocksparse", "attn_bwd_blocksparse", "attn_fp8_quantize", "attn_fwd_fp8",
           "attn_fwd_dropout", "attn_bwd_dropout", "attn_linear_fwd", "attn_linear_workspace_bytes",
           "attn_last_device_status", "attn_selftest_wait_timeout",
           "attn_last_cuda_error_string", "attn_strerror", "attn_version")

# Size of the built-in scratch attn_bwd_noalloc uses (bytes, per device).
NOALLOC_SCRATCH_BYTES = 32 * 1024 * 1024


class AttnError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        extra = ""
        if status in (-6, -7):
            extra = f"; CUDA: {lib().attn_last_cuda_error_string().decode()}"
        super().__init__(f"{where}: {STATUS.get(status, status)} ({strerror(status)}{extra})")


_lib = None


def lib() -> ctypes.CDLL:
    """Load libattn.so from the package directory (never from elsewhere)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is not built: run `python -m io_aware_exact_30_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        vp, ci, cf, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
        L.attn_fwd.argtypes = [vp, vp, vp, vp, vp, ci, ci, ci, ci, ci, cf, ci, vp]
        L.attn_fwd.restype = ci
        L.attn_bwd.argtypes = [vp] * 10 + [ci, ci, ci, ci, ci, cf, ci, vp]
        L.attn_bwd.restype = ci
        L.attn_bwd_prep.argtypes = [vp, vp, vp, vp, ci, ci, ci, ci, ci, vp]
        L.attn_bwd_prep.restype = ci
        L.attn_bwd_main.argtypes = [vp] * 8 + [ci, ci, ci, ci, ci, cf, ci, vp]
        L.attn_bwd_main.restype = ci
        L.attn_bwd_noalloc.argtypes = [vp] * 9 + [ci, ci, ci, ci, ci, cf, ci, vp]
        L.attn_bwd_noalloc.restype = ci
        L.attn_fwd_blocksparse.argtypes = [vp] * 6 + [ci, ci, ci, ci, ci, cf, ci, vp]
        L.attn_fwd_blocksparse.restype = ci
        L.attn_bwd_blocksparse.argtypes = [vp] * 11 + [ci, ci, ci, ci, ci, cf, ci, vp]
        L.attn_bwd_blocksparse.restype = ci
        L.attn_linear_workspace_bytes.argtypes = [ci, ci, ci, ci]
        L.attn_linear_workspace_bytes.restype = sz
        L.attn_linear_fwd.argtypes = [vp] * 5 + [ci, ci, ci, ci, cf, ci, vp]
        L.attn_linear_fwd.restype = ci
        u64 = ctypes.c_ulonglong
        L.attn_fwd_dropout.argtypes = [vp] * 5 + [ci, ci, ci, ci, ci, cf, cf, u64, ci, vp]
        L.attn_fwd_dropout.restype = ci
        L.attn_bwd_dropout.argtypes = [vp] * 10 + [ci, ci, ci, ci, ci, cf, cf, u64, ci, vp]
        L.attn_bwd_dropout.restype = ci
        L.attn_fp8_quantize.argtypes = [vp, vp, vp, vp, ci, ci, ci, ci, ci, ci, vp]
        L.attn_fp8_quantize.restype = ci
        L.attn_fwd_fp8.argtypes = [vp] * 7 + [ci, ci, ci, ci, ci, cf, ci, ci, vp]
        L.attn_fwd_fp8.restype = ci
        L.attn_sdpa_host_scratch_bytes.argtypes = [ci, ci, ci, ci, ci, ci]
        L.attn_sdpa_host_scratch_bytes.restype = sz
        L.attn_sdpa_host.argtypes = [vp] * 10 + [sz, ci, ci, ci, ci, ci, cf, ci, ci, vp]
        L.attn_sdpa_host.restype = ci
        L.attn_bwd_workspace_bytes.argtypes = [ci, ci, ci, ci]
        L.attn_bwd_workspace_bytes.restype = sz
        L.attn_last_device_status.argtypes = [vp]
        L.attn_last_device_status.restype = ci
        L.attn_selftest_wait_timeout.argtypes = [ctypes.c_uint, vp]
        L.attn_selftest_wait_timeout.restype = ci
        L.attn_strerror.argtypes = [ci]
        L.attn_strerror.restype = ctypes.c_char_p
        L.attn_last_cuda_error_string.argtypes = []
        L.attn_last_cuda_error_string.restype = ctypes.c_char_p
        L.attn_version.argtypes = []
        L.attn_version.restype = ctypes.c_char_p
        _lib = L
    return _lib


def strerror(status: int) -> str:
    return lib().attn_strerror(int(status)).decode()


def version() -> str:
    return lib().attn_version().decode()


def _stream(device, stream):
    if stream is not None:
        return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)
    return torch.cuda.current_stream(device).cuda_stream


def _check(rc: int, where: str):
    if rc != 0:
        raise AttnError(rc, where)


def _shape(q):
    if q.dim() != 4:
        raise ValueError("q must be (B, H, N, d)")
    return q.shape


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else None


def _dtype(q):
    if q.dtype not in _DTYPES:
        raise TypeError(f"dtype must be bfloat16 or float16, got {q.dtype}")
    return _DTYPES[q.dtype]


def _same(ref, *ts, names):
    for t, n in zip(ts, names):
        if t.dtype != ref.dtype or t.shape != ref.shape or not t.is_contiguous():
            raise ValueError(f"{n} must be contiguous with the shape and dtype of q")


def attn_fwd(q, k, v, o, lse, causal: bool, scale: float | None = None, stream=None) -> None:
    """O, LSE <- attention(q, k, v); all tensors caller-allocated, (B, H, N, d) / (B, H, N)."""
    B, H, N, d = _shape(q)
    _same(q, k, v, o, names=("k", "v", "o"))
    if lse.dtype != torch.float32 or tuple(lse.shape) != (B, H, N) or not lse.is_contiguous():
        raise ValueError("lse must be a contiguous float32 (B, H, N) tensor")
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    rc = lib().attn_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, H, N, d, int(bool(causal)),
                        scale, _dtype(q), ctypes.c_void_p(_stream(q.device, stream)))
    _check(rc, "attn_fwd")


def attn_bwd_workspace_bytes(B: int, H: int, N: int, d: int) -> int:
    return int(lib().attn_bwd_workspace_bytes(B, H, N, d))


def attn_bwd(q, k, v, o, lse, dout, dq, dk, dv, workspace, causal: bool,
             scale: float | None = None, stream=None) -> None:
    """dQ, dK, dV <- gradients of sum(O * dout), recomputing P from lse."""
    B, H, N, d = _shape(q)
    _same(q, k, v, o, dout, dq, dk, dv, names=("k", "v", "o", "dout", "dq", "dk", "dv"))
    if lse.dtype != torch.float32 or tuple(lse.shape) != (B, H, N) or not lse.is_contiguous():
        raise ValueError("lse must be a contiguous float32 (B, H, N) tensor")
    need = attn_bwd_workspace_bytes(B, H, N, d)
    if workspace.numel() * workspace.element_size() < need:
        raise ValueError(f"workspace needs {need} bytes")
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    rc = lib().attn_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(dout), _ptr(dq), _ptr(dk),
                        _ptr(dv), _ptr(workspace), B, H, N, d, int(bool(causal)), scale, _dtype(q),
                        ctypes.c_void_p(_stream(q.device, stream)))
    _check(rc, "attn_bwd")


def attn_bwd_prep(o, dout, lse, workspace, stream=None) -> None:
    """Stage D = rowdot(dout, o) and lse * log2(e) in the workspace; clear the dQ accumulator."""
    B, H, N, d = _shape(o)
    _same(o, dout, names=("dout",))
    if lse.dtype != torch.float32 or tuple(lse.shape) != (B, H, N) or not lse.is_contiguous():
        raise ValueError("lse must be a contiguous float32 (B, H, N) tensor")
    need = attn_bwd_workspace_bytes(B, H, N, d)
    if workspace.numel() * workspace.element_size() < need:
        raise ValueError(f"workspace needs {need} bytes")
    rc = lib().attn_bwd_prep(_ptr(o), _ptr(dout), _ptr(lse), _ptr(workspace), B, H, N, d, _dtype(o),
                             ctypes.c_void_p(_stream(o.device, stream)))
    _check(rc, "attn_bwd_prep")


def attn_bwd_main(q, k, v, dout, dq, dk, dv, workspace, causal: bool,
                  scale: float | None = None, stream=None) -> None:
    """Recompute backward on a workspace prepared by attn_bwd_prep."""
    B, H, N, d = _shape(q)
    _same(q, k, v, dout, dq, dk, dv, names=("k", "v", "dout", "dq", "dk", "dv"))
    need = attn_bwd_workspace_bytes(B, H, N, d)
    if workspace.numel() * workspace.element_size() < need:
        raise ValueError(f"workspace needs {need} bytes")
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    rc = lib().attn_bwd_main(_ptr(q), _ptr(k), _ptr(v), _ptr(dout), _ptr(dq), _ptr(dk), _ptr(dv),
                             _ptr(workspace), B, H, N, d, int(bool(causal)), scale, _dtype(q),
                             ctypes.c_void_p(_stream(q.device, stream)))
    _check(rc, "attn_bwd_main")


def attn_bwd_noalloc(q, k, v, o, lse, dout, dq, dk, dv, causal: bool,
                     scale: float | None = None, stream=None) -> None:
    """attn_bwd without a workspace argument: the library uses its own fixed
    device array (``NOALLOC_SCRATCH_BYTES`` per device) and allocates nothing.
    For callers that have their inputs and outputs but no way to obtain
    scratch memory.  Calls that overlap on the GPU share that array and race."""
    B, H, N, d = _shape(q)
    _same(q, k, v, o, dout, dq, dk, dv, names=("k", "v", "o", "dout", "dq", "dk", "dv"))
    if lse.dtype != torch.float32 or tuple(lse.shape) != (B, H, N) or not lse.is_contiguous():
        raise ValueError("lse must be a contiguous float32 (B, H, N) tensor")
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    rc = lib().attn_bwd_noalloc(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(dout), _ptr(dq),
                                _ptr(dk), _ptr(dv), B, H, N, d, int(bool(causal)), scale, _dtype(q),
                                ctypes.c_void_p(_stream(q.device, stream)))
    _check(rc, "attn_bwd_noalloc")


# Block size of attn_fwd_blocksparse / attn_bwd_blocksparse masks (rows and keys).
BLOCK = 128


def _check_mask(mask, N, device):
    nb = (N + BLOCK - 1) // BLOCK
    if (mask.dtype not in (torch.uint8, torch.bool) or tuple(mask.shape) != (nb, nb)
            or not mask.is_contiguous() or mask.device != device):
        raise ValueError(f"block mask must be a contiguous ({nb}, {nb}) uint8/bool tensor on {device}")


def attn_fwd_blocksparse(q, k, v, o, lse, block_mask, causal: bool, scale: float | None = None,
                         stream=None) -> None:
    """attn_fwd over the 128 x 128 blocks ``block_mask`` marks (one mask for all heads)."""
    B, H, N, d = _shape(q)
    _same(q, k, v, o, names=("k", "v", "o"))
    if lse.dtype != torch.float32 or tuple(lse.shape) != (B, H, N) or not lse.is_contiguous():
        raise ValueError("lse must be a contiguous float32 (B, H, N) tensor")
    _check_mask(block_mask, N, q.device)
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    rc = lib().attn_fwd_blocksparse(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(block_mask),
                                    B, H, N, d, int(bool(causal)), scale, _dtype(q),
                                    ctypes.c_void_p(_stream(q.device, stream)))
    _check(rc, "attn_fwd_blocksparse")


def attn_bwd_blocksparse(q, k, v, o, lse, dout, dq, dk, dv, workspace, block_mask, causal: bool,
                         scale: float | None = None, stream=None) -> None:
    """attn_bwd over the 128 x 128 blocks ``block_mask`` marks."""
    B, H, N, d = _shape(q)
    _same(q, k, v, o, dout, dq, dk, dv, names=("k", "v", "o", "dout", "dq", "dk", "dv"))
    if lse.dtype != torch.float32 or tuple(lse.shape) != (B, H, N) or not lse.is_contiguous():
        raise ValueError("lse must be a contiguous float32 (B, H, N) tensor")
    _check_mask(block_mask, N, q.device)
    need = attn_bwd_workspace_bytes(B, H, N, d)
    if workspace.numel() * workspace.element_size() < need:
        raise ValueError(f"workspace needs {need} bytes")
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    rc = lib().attn_bwd_blocksparse(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(dout),
                                    _ptr(dq), _ptr(dk), _ptr(dv), _ptr(workspace),
                                    _ptr(block_mask), B, H, N, d, int(bool(causal)), scale,
                                    _dtype(q), ctypes.c_void_p(_stream(q.device, stream)))
    _check(rc, "attn_bwd_blocksparse")


def attn_fp8_quantize(x, x8, scales, signs=None, rotate: bool = True, stream=None) -> None:
    """x8 <- e4m3 codes of x's rows (times ``signs``, Hadamard-rotated when
    ``rotate``), one scale per 128-row block of each head into ``scales``."""
    B, H, N, d = _shape(x)
    nb = (N + 127) // 128
    if x8.dtype != torch.uint8 or tuple(x8.shape) != (B, H, N, d) or not x8.is_contiguous():
        raise ValueError("x8 must be a contiguous uint8 (B, H, N, d) tensor")
    if scales.dtype != torch.float32 or tuple(scales.shape) != (B, H, nb) or not scales.is_contiguous():
        raise ValueError(f"scales must be a contiguous float32 (B, H, {nb}) tensor")
    if signs is not None and (signs.dtype != torch.int8 or tuple(signs.shape) != (d,)):
        raise ValueError("signs must be an int8 tensor of d entries")
    rc = lib().attn_fp8_quantize(_ptr(x), _ptr(x8), _ptr(scales), _ptr(signs), int(bool(rotate)),
                                 B, H, N, d, _dtype(x), ctypes.c_void_p(_stream(x.device, stream)))
    _check(rc, "attn_fp8_quantize")


def attn_fwd_fp8(q8, k8, q_scale, k_scale, v, o, lse, causal: bool, scale: float | None = None,
                 rotated: bool = True, stream=None) -> None:
    """Forward with e4m3 scores (codes and scales from attn_fp8_quantize)."""
    B, H, N, d = _shape(v)
    _same(v, o, names=("o",))
    for t, n in ((q8, "q8"), (k8, "k8")):
        if t.dtype != torch.uint8 or tuple(t.shape) != (B, H, N, d) or not t.is_contiguous():
            raise ValueError(f"{n} must be a contiguous uint8 (B, H, N, d) tensor")
    if lse.dtype != torch.float32 or tuple(lse.shape) != (B, H, N) or not lse.is_contiguous():
        raise ValueError("lse must be a contiguous float32 (B, H, N) tensor")
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    rc = lib().attn_fwd_fp8(_ptr(q8), _ptr(k8), _ptr(q_scale), _ptr(k_scale), _ptr(v), _ptr(o),
                            _ptr(lse), B, H, N, d, int(bool(causal)), scale, int(bool(rotated)),
                            _dtype(v), ctypes.c_void_p(_stream(v.device, stream)))
    _check(rc, "attn_fwd_fp8")


def attn_fwd_dropout(q, k, v, o, lse, causal: bool, dropout_p: float, seed: int,
                     scale: float | None = None, stream=None) -> None:
    """attn_fwd with dropout on P (Philox4x32-10 mask from ``seed``)."""
    B, H, N, d = _shape(q)
    _same(q, k, v, o, names=("k", "v", "o"))
    if lse.dtype != torch.float32 or tuple(lse.shape) != (B, H, N) or not lse.is_contiguous():
        raise ValueError("lse must be a contiguous float32 (B, H, N) tensor")
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    rc = lib().attn_fwd_dropout(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, H, N, d,
                                int(bool(causal)), scale, float(dropout_p),
                                int(seed) & 0xFFFFFFFFFFFFFFFF, _dtype(q),
                                ctypes.c_void_p(_stream(q.device, stream)))
    _check(rc, "attn_fwd_dropout")


def attn_bwd_dropout(q, k, v, o, lse, dout, dq, dk, dv, workspace, causal: bool,
                     dropout_p: float, seed: int, scale: float | None = None, stream=None) -> None:
    """attn_bwd for attn_fwd_dropout (the same dropout_p and seed)."""
    B, H, N, d = _shape(q)
    _same(q, k, v, o, dout, dq, dk, dv, names=("k", "v", "o", "dout", "dq", "dk", "dv"))
    if lse.dtype != torch.float32 or tuple(lse.shape) != (B, H, N) or not lse.is_contiguous():
        raise ValueError("lse must be a contiguous float32 (B, H, N) tensor")
    need = attn_bwd_workspace_bytes(B, H, N, d)
    if workspace.numel() * workspace.element_size() < need:
        raise ValueError(f"workspace needs {need} bytes")
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    rc = lib().attn_bwd_dropout(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(dout),
                                _ptr(dq), _ptr(dk), _ptr(dv), _ptr(workspace), B, H, N, d,
                                int(bool(causal)), scale, float(dropout_p),
                                int(seed) & 0xFFFFFFFFFFFFFFFF, _dtype(q),
                                ctypes.c_void_p(_stream(q.device, stream)))
    _check(rc, "attn_bwd_dropout")


def attn_linear_workspace_bytes(B: int, H: int, N: int, d: int) -> int:
    return int(lib().attn_linear_workspace_bytes(B, H, N, d))


def attn_linear_fwd(q, k, v, o, workspace, scale: float | None = None, stream=None) -> None:
    """Causal linear attention O_i = scale sum_{j<=i} (q_i . k_j) v_j (d = 128)."""
    B, H, N, d = _shape(q)
    _same(q, k, v, o, names=("k", "v", "o"))
    need = attn_linear_workspace_bytes(B, H, N, d)
    if need == 0 or workspace.numel() * workspace.element_size() < need:
        raise ValueError(f"workspace needs {need} bytes (d must be 128)")
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    rc = lib().attn_linear_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(workspace), B, H, N, d,
                               scale, _dtype(q), ctypes.c_void_p(_stream(q.device, stream)))
    _check(rc, "attn_linear_fwd")


def attn_sdpa_host_scratch_bytes(B: int, H: int, N: int, d: int, with_backward: bool,
                                 heads_per_chunk: int = 0) -> int:
    return int(lib().attn_sdpa_host_scratch_bytes(B, H, N, d, int(bool(with_backward)),
                                                  int(heads_per_chunk)))


def attn_sdpa_host(q, k, v, dout, o, lse, dq, dk, dv, scratch, causal: bool,
                   scale: float | None = None, heads_per_chunk: int = 0, stream=None) -> None:
    """Attention from host buffers: q, k, v, dout and the outputs are CPU
    tensors (pinned, for the copies to overlap); ``dout=None`` runs the forward
    alone (o and lse required).  ``scratch`` is a CUDA uint8 tensor of
    attn_sdpa_host_scratch_bytes() bytes."""
    B, H, N, d = _shape(q)
    host = [t for t in (q, k, v, dout, o, lse, dq, dk, dv) if t is not None]
    if any(t.device.type != "cpu" or not t.is_contiguous() for t in host):
        raise ValueError("host tensors must be contiguous CPU tensors")
    if scratch.device.type != "cuda":
        raise ValueError("scratch must be device memory")
    sc = 1.0 / math.sqrt(d) if scale is None else float(scale)
    rc = lib().attn_sdpa_host(_ptr(q), _ptr(k), _ptr(v), _ptr(dout), _ptr(o), _ptr(lse),
                              _ptr(dq), _ptr(dk), _ptr(dv), _ptr(scratch),
                              scratch.numel() * scratch.element_size(), B, H, N, d,
                              int(bool(causal)), sc, _dtype(q), int(heads_per_chunk),
                              ctypes.c_void_p(_stream(scratch.device, stream)))
    _check(rc, "attn_sdpa_host")


def attn_last_device_status(stream=None, device=None) -> int:
    st = _stream(device or torch.cuda.current_device(), stream)
    return int(lib().attn_last_device_status(ctypes.c_void_p(st)))


def attn_selftest_wait_timeout(timeout_us: int, stream=None) -> None:
    st = _stream(torch.cuda.current_device(), stream)
    _check(lib().attn_selftest_wait_timeout(int(timeout_us), ctypes.c_void_p(st)),
           "attn_selftest_wait_timeout")


# ------------------------------------------------------------ conveniences --
def forward(q, k, v, causal: bool = False, scale: float | None = None):
    """Allocates O and LSE with torch and runs attn_fwd; returns (o, lse)."""
    B, H, N, d = _shape(q)
    o = torch.empty_like(q)
    lse = torch.empty((B, H, N), dtype=torch.float32, device=q.device)
    attn_fwd(q, k, v, o, lse, causal, scale)
    return o, lse


def backward(q, k, v, o, lse, dout, causal: bool = False, scale: float | None = None,
             workspace=None):
    """Allocates dQ, dK, dV (and the workspace if not given); returns (dq, dk, dv)."""
    B, H, N, d = _shape(q)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    if workspace is None:
        workspace = torch.empty(attn_bwd_workspace_bytes(B, H, N, d), dtype=torch.uint8,
                                device=q.device)
    attn_bwd(q, k, v, o, lse, dout, dq, dk, dv, workspace, causal, scale)
    return dq, dk, dv


def forward_blocksparse(q, k, v, block_mask, causal: bool = False, scale: float | None = None):
    """Allocates O and LSE and runs attn_fwd_blocksparse; returns (o, lse)."""
    B, H, N, d = _shape(q)
    o = torch.empty_like(q)
    lse = torch.empty((B, H, N), dtype=torch.float32, device=q.device)
    attn_fwd_blocksparse(q, k, v, o, lse, block_mask, causal, scale)
    return o, lse


def backward_blocksparse(q, k, v, o, lse, dout, block_mask, causal: bool = False,
                         scale: float | None = None):
    """Allocates dQ, dK, dV and the workspace; returns (dq, dk, dv)."""
    B, H, N, d = _shape(q)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    ws = torch.empty(attn_bwd_workspace_bytes(B, H, N, d), dtype=torch.uint8, device=q.device)
    attn_bwd_blocksparse(q, k, v, o, lse, dout, dq, dk, dv, ws, block_mask, causal, scale)
    return dq, dk, dv


def forward_fp8(q, k, v, causal: bool = False, scale: float | None = None, signs=None,
                rotate: bool = True):
    """Quantises q and k (rotated unless ``rotate`` is False) and runs
    attn_fwd_fp8; returns (o, lse).  ``signs``: int8 (d,) device tensor."""
    B, H, N, d = _shape(q)
    nb = (N + 127) // 128
    q8 = torch.empty((B, H, N, d), dtype=torch.uint8, device=q.device)
    k8 = torch.empty_like(q8)
    qs = torch.empty((B, H, nb), dtype=torch.float32, device=q.device)
    ks = torch.empty_like(qs)
    attn_fp8_quantize(q, q8, qs, signs, rotate)
    attn_fp8_quantize(k, k8, ks, signs, rotate)
    o = torch.empty_like(v)
    lse = torch.empty((B, H, N), dtype=torch.float32, device=q.device)
    attn_fwd_fp8(q8, k8, qs, ks, v, o, lse, causal, scale, rotate)
    return o, lse


def forward_dropout(q, k, v, dropout_p: float, seed: int, causal: bool = False,
                    scale: float | None = None):
    """Allocates O and LSE and runs attn_fwd_dropout; returns (o, lse)."""
    B, H, N, d = _shape(q)
    o = torch.empty_like(q)
    lse = torch.empty((B, H, N), dtype=torch.float32, device=q.device)
    attn_fwd_dropout(q, k, v, o, lse, causal, dropout_p, seed, scale)
    return o, lse


def backward_dropout(q, k, v, o, lse, dout, dropout_p: float, seed: int, causal: bool = False,
                     scale: float | None = None):
    """Allocates dQ, dK, dV and the workspace; runs attn_bwd_dropout."""
    B, H, N, d = _shape(q)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    ws = torch.empty(attn_bwd_workspace_bytes(B, H, N, d), dtype=torch.uint8, device=q.device)
    attn_bwd_dropout(q, k, v, o, lse, dout, dq, dk, dv, ws, causal, dropout_p, seed, scale)
    return dq, dk, dv


def linear_forward(q, k, v, scale: float | None = None):
    """Allocates O and the workspace and runs attn_linear_fwd; returns o."""
    B, H, N, d = _shape(q)
    o = torch.empty_like(q)
    ws = torch.empty(max(1, attn_linear_workspace_bytes(B, H, N, d)), dtype=torch.uint8,
                     device=q.device)
    attn_linear_fwd(q, k, v, o, ws, scale)
    return o


# ------------------------------------------------------------ several GPUs --
# Every (batch, head) pair is independent in both passes, so one problem's heads
# split across the ranks of a process group (one GPU each) with no exchange:
# each rank runs the single-GPU calls above on a contiguous range of the
# flattened B*H heads (views of the inputs; an LSE slice that would not be
# 16-byte aligned is copied).  The one collective is an optional all-gather of the
# outputs, for callers that want the whole tensors on every rank.  (Dropout is
# not offered here: its random bytes are keyed by the head index within the
# call, so a rank's slice would draw other bytes than the whole call.)

def head_shard(BH: int, rank: int, world: int) -> tuple[int, int]:
    """(first head, number of heads) of rank `rank` among `world` for B*H = BH
    flattened heads: contiguous ranges, the first BH % world ranks one head more."""
    if world < 1 or not 0 <= rank < world or BH < 0:
        raise ValueError("need 0 <= rank < world and BH >= 0")
    base, extra = divmod(BH, world)
    return rank * base + min(rank, extra), base + (1 if rank < extra else 0)


def _heads(x, s, n):
    """Heads [s, s + n) of a (B, H, ...) tensor as a contiguous (1, n, ...) tensor:
    a view, or a copy where the view would not start on the 16-byte boundary the
    ABI requires (an fp32 LSE slice when s * N is not a multiple of 4)."""
    B, H = x.shape[0], x.shape[1]
    view = x.reshape(B * H, *x.shape[2:])[s:s + n].unsqueeze(0)
    return view if view.data_ptr() % 16 == 0 else view.clone()


def _gather_heads(parts, shape, s_n, group):
    """All-gather every rank's (1, n_r, ...) slice into one (B, H, ...) tensor;
    uneven counts are padded to the largest for the collective."""
    import torch.distributed as dist
    world = dist.get_world_size(group)
    m = max(n for _, n in s_n)
    outs = []
    for part in parts:
        pad = part.new_zeros((1, m) + tuple(part.shape[2:]))
        pad[:, :part.shape[1]] = part
        bufs = [torch.empty_like(pad) for _ in range(world)]
        dist.all_gather(bufs, pad, group=group)
        full = torch.cat([b[0, :n] for b, (_, n) in zip(bufs, s_n)], dim=0)
        outs.append(full.reshape(shape[:2] + tuple(part.shape[2:])))
    return outs


def forward_sharded(q, k, v, causal: bool = False, scale: float | None = None, group=None,
                    gather: bool = True):
    """The forward of (B, H, N, d) q, k, v (the same on every rank of `group`)
    split by heads: this rank computes its head_shard() range with attn_fwd.
    gather=True returns the whole (o, lse) on every rank (one all-gather each);
    gather=False returns this rank's (o, lse) of shape (1, n, N, d) and (1, n, N)
    and its (first head, count)."""
    import torch.distributed as dist
    B, H, N, d = _shape(q)
    world, rank = dist.get_world_size(group), dist.get_rank(group)
    s_n = [head_shard(B * H, r, world) for r in range(world)]
    s, n = s_n[rank]
    if n > 0:
        o, lse = forward(_heads(q, s, n), _heads(k, s, n), _heads(v, s, n), causal, scale)
    else:
        o = q.new_empty((1, 0, N, d))
        lse = torch.empty((1, 0, N), dtype=torch.float32, device=q.device)
    if not gather:
        return o, lse, (s, n)
    o, lse = _gather_heads([o, lse], (B, H), s_n, group)
    return o, lse


def backward_sharded(q, k, v, o, lse, dout, causal: bool = False, scale: float | None = None,
                     group=None, gather: bool = True):
    """The backward split by heads as forward_sharded: this rank runs attn_bwd on
    its head range; gather=True returns the whole (dq, dk, dv) on every rank,
    gather=False this rank's slices and its (first head, count)."""
    import torch.distributed as dist
    B, H, N, d = _shape(q)
    world, rank = dist.get_world_size(group), dist.get_rank(group)
    s_n = [head_shard(B * H, r, world) for r in range(world)]
    s, n = s_n[rank]
    if n > 0:
        grads = backward(*(_heads(x, s, n) for x in (q, k, v, o, lse, dout)), causal, scale)
    else:
        grads = tuple(x.new_empty((1, 0, N, d)) for x in (q, k, v))
    if not gather:
        return (*grads, (s, n))
    return tuple(_gather_heads(list(grads), (B, H), s_n, group))
