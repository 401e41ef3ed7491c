"""Thin ctypes binding of ``libavq_b200.so`` (the C ABI in ``include/avq.h``).

Argument marshalling only: tensors become device pointers, the current torch
stream becomes the ``stream`` argument, and every step of the path runs in
the library's CUDA kernels. There is no fallback: if the library is missing
or the tensors are not on a CUDA device, the calls raise.

Low-level names mirror the C ABI (``avq_precompute``, ``avq_attention``, ...);
``precompute`` and ``attention`` allocate outputs with torch and call them.
"""
from __future__ import annotations

import ctypes
import math
import os

import torch

from . import build as _build

AVQ_F32, AVQ_BF16 = 0, 1
AVQ_OK = 0
_STATUS = {0: "AVQ_OK", -1: "AVQ_EINVAL", -2: "AVQ_EUNSUPPORTED", -3: "AVQ_ECUDA",
           -4: "AVQ_ETIMEOUT", -5: "AVQ_EWORKSPACE", -6: "AVQ_ERANGE"}

# every symbol include/avq.h declares (checked by the tests)
EXPORTS = ("avq_precompute_workspace_bytes", "avq_precompute", "avq_attention_workspace_bytes",
           "avq_attention", "avq_device_status", "avq_status_string", "avq_version",
           "avq_kernel_launches", "avq_attention_noalloc", "avq_commitment", "avq_gilbert_order",
           "avq_gather_rows", "avq_capture_workspace_bytes", "avq_capture", "avq_precompute_deep",
           "avq_attention_deep_workspace_bytes", "avq_attention_deep", "avq_test_fail_next_wait")


class AVQError(RuntimeError):
    def __init__(self, code: int, what: str):
        self.code = code
        super().__init__(f"{what}: {_STATUS.get(code, code)} ({code})")


class AvqShape(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int32), ("H", ctypes.c_int32), ("N", ctypes.c_int32),
                ("d", ctypes.c_int32), ("M0", ctypes.c_int32), ("C", ctypes.c_int32),
                ("dtype", ctypes.c_int32)]


_LIB = None


def library_path() -> str:
    return _build.LIB


def lib() -> ctypes.CDLL:
    """Load the library (once). Raises if it has not been built."""
    global _LIB
    if _LIB is None:
        path = library_path()
        if not os.path.exists(path):
            raise ImportError(f"{path} is missing: build it with "
                              "`python -m adaptive_vector_quantized_avq_b200.build`")
        L = ctypes.CDLL(path)
        vp, sz, i32 = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int
        shp = ctypes.POINTER(AvqShape)
        L.avq_precompute_workspace_bytes.argtypes = [shp]
        L.avq_precompute_workspace_bytes.restype = sz
        L.avq_precompute.argtypes = [shp, vp, vp, vp, vp, vp, vp, vp, sz, vp]
        L.avq_precompute.restype = i32
        L.avq_attention_workspace_bytes.argtypes = [shp, i32, i32]
        L.avq_attention_workspace_bytes.restype = sz
        L.avq_attention.argtypes = [shp, vp, vp, vp, vp, i32, i32, ctypes.c_float, vp, vp, vp,
                                    sz, vp]
        L.avq_attention.restype = i32
        L.avq_device_status.argtypes = [vp, vp]
        L.avq_device_status.restype = i32
        L.avq_status_string.argtypes = [i32]
        L.avq_status_string.restype = ctypes.c_char_p
        L.avq_version.argtypes = []
        L.avq_version.restype = i32
        L.avq_attention_noalloc.argtypes = [shp, vp, vp, vp, vp, i32, i32, ctypes.c_float, vp, vp,
                                            vp, vp]
        L.avq_attention_noalloc.restype = i32
        L.avq_commitment.argtypes = [shp, vp, vp, vp, vp, vp]
        L.avq_commitment.restype = i32
        L.avq_gilbert_order.argtypes = [i32, i32, vp]
        L.avq_gilbert_order.restype = i32
        L.avq_gather_rows.argtypes = [shp, vp, vp, vp, vp]
        L.avq_gather_rows.restype = i32
        L.avq_capture_workspace_bytes.argtypes = [shp, i32, i32]
        L.avq_capture_workspace_bytes.restype = sz
        L.avq_capture.argtypes = [shp, vp, vp, vp, vp, i32, i32, ctypes.c_float, vp, vp, sz, vp]
        L.avq_capture.restype = i32
        L.avq_precompute_deep.argtypes = [shp, i32, vp, vp, vp, vp, vp, vp, vp]
        L.avq_precompute_deep.restype = i32
        L.avq_attention_deep_workspace_bytes.argtypes = [shp, i32]
        L.avq_attention_deep_workspace_bytes.restype = sz
        L.avq_attention_deep.argtypes = [shp, i32, vp, vp, vp, vp, vp, i32, ctypes.c_float, vp, vp, vp, sz,
                                         vp]
        L.avq_attention_deep.restype = i32
        L.avq_test_fail_next_wait.argtypes = []
        L.avq_test_fail_next_wait.restype = i32
        L.avq_kernel_launches.argtypes = []
        L.avq_kernel_launches.restype = ctypes.c_uint64
        _LIB = L
    return _LIB


# ------------------------------------------------------------ marshalling
def _ptr(x) -> int | None:
    if x is None:
        return None
    if isinstance(x, int):
        return x
    return x.data_ptr()


def _stream(stream) -> int | None:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def make_shape(B, H, N, d, M0, C, dtype) -> AvqShape:
    if isinstance(dtype, torch.dtype):
        dtype = {torch.float32: AVQ_F32, torch.bfloat16: AVQ_BF16}[dtype]
    return AvqShape(B, H, N, d, M0, C, dtype)


# ------------------------------------------------------- the C ABI, 1:1
def avq_version() -> int:
    return lib().avq_version()


def avq_kernel_launches() -> int:
    return int(lib().avq_kernel_launches())


def avq_status_string(code: int) -> str:
    return lib().avq_status_string(code).decode()


def avq_precompute_workspace_bytes(shape: AvqShape) -> int:
    return lib().avq_precompute_workspace_bytes(ctypes.byref(shape))


def avq_attention_workspace_bytes(shape: AvqShape, P: int, tile: int) -> int:
    return lib().avq_attention_workspace_bytes(ctypes.byref(shape), P, tile)


def avq_precompute(shape, K, V, codebook, assign, counts, vsum, workspace, workspace_bytes,
                   stream=None) -> int:
    return lib().avq_precompute(ctypes.byref(shape), _ptr(K), _ptr(V), _ptr(codebook),
                                _ptr(assign), _ptr(counts), _ptr(vsum), _ptr(workspace),
                                workspace_bytes, _stream(stream))


def avq_attention(shape, Q, codebook, counts, vsum, P, tile, scale, O, selected, workspace,
                  workspace_bytes, stream=None) -> int:
    return lib().avq_attention(ctypes.byref(shape), _ptr(Q), _ptr(codebook), _ptr(counts),
                               _ptr(vsum), P, tile, float(scale), _ptr(O), _ptr(selected),
                               _ptr(workspace), workspace_bytes, _stream(stream))


def avq_attention_noalloc(shape, Q, codebook, counts, vsum, P, tile, scale, O, selected,
                          device_status=None, stream=None) -> int:
    return lib().avq_attention_noalloc(ctypes.byref(shape), _ptr(Q), _ptr(codebook), _ptr(counts),
                                       _ptr(vsum), P, tile, float(scale), _ptr(O), _ptr(selected),
                                       _ptr(device_status), _stream(stream))


def avq_commitment(shape, K, codebook, assign, sq_err, stream=None) -> int:
    return lib().avq_commitment(ctypes.byref(shape), _ptr(K), _ptr(codebook), _ptr(assign), _ptr(sq_err),
                                _stream(stream))


def avq_gilbert_order(rows: int, cols: int, order) -> int:
    """`order`: a writable host buffer of rows*cols int32 (e.g. a numpy array)."""
    return lib().avq_gilbert_order(rows, cols, order.ctypes.data if hasattr(order, "ctypes") else order)


def avq_gather_rows(shape, src, dst, perm, stream=None) -> int:
    return lib().avq_gather_rows(ctypes.byref(shape), _ptr(src), _ptr(dst), _ptr(perm), _stream(stream))


def avq_capture_workspace_bytes(shape, P, tile) -> int:
    return lib().avq_capture_workspace_bytes(ctypes.byref(shape), P, tile)


def avq_capture(shape, Q, K, assign, selected, P, tile, scale, capture, workspace, workspace_bytes,
                stream=None) -> int:
    return lib().avq_capture(ctypes.byref(shape), _ptr(Q), _ptr(K), _ptr(assign), _ptr(selected), P, tile,
                             float(scale), _ptr(capture), _ptr(workspace), workspace_bytes, _stream(stream))


def avq_precompute_deep(shape, L, K, V, codebook, assign, counts, vsum, stream=None) -> int:
    return lib().avq_precompute_deep(ctypes.byref(shape), L, _ptr(K), _ptr(V), _ptr(codebook), _ptr(assign),
                                     _ptr(counts), _ptr(vsum), _stream(stream))


def avq_attention_deep_workspace_bytes(shape, L) -> int:
    return lib().avq_attention_deep_workspace_bytes(ctypes.byref(shape), L)


def avq_attention_deep(shape, L, P, Q, codebook, counts, vsum, tile, scale, O, selected, workspace,
                       workspace_bytes, stream=None) -> int:
    """`P`: a sequence of L-1 budgets (marshalled to a host int32 array)."""
    Pa = (ctypes.c_int32 * max(1, len(P)))(*[int(x) for x in P])
    return lib().avq_attention_deep(ctypes.byref(shape), L, ctypes.cast(Pa, ctypes.c_void_p), _ptr(Q),
                                    _ptr(codebook), _ptr(counts), _ptr(vsum), tile, float(scale), _ptr(O),
                                    _ptr(selected), _ptr(workspace), workspace_bytes, _stream(stream))


def avq_test_fail_next_wait() -> int:
    return lib().avq_test_fail_next_wait()


def avq_device_status(workspace, stream=None) -> int:
    return lib().avq_device_status(_ptr(workspace), _stream(stream))


# ------------------------------------------------ tensor-level convenience
def _check(t: torch.Tensor, name: str, dtype=None):
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")


def workspace(nbytes: int, device) -> torch.Tensor:
    """A zero-filled, 256-byte aligned workspace tensor of at least ``nbytes``."""
    return torch.zeros(max(256, (nbytes + 255) // 256 * 256), dtype=torch.uint8, device=device)


def precompute(K: torch.Tensor, V: torch.Tensor, codebook: torch.Tensor, M0: int, C: int,
               *, out=None, ws: torch.Tensor | None = None, stream=None):
    """Return (assign [B,H,N] int32, counts [B,H,Mtot] int32, vsum [B,H,Mtot,d] fp32)."""
    for t, n in ((K, "K"), (V, "V"), (codebook, "codebook")):
        _check(t, n, K.dtype)
    B, H, N, d = K.shape
    Mtot = M0 * (1 + C)
    if V.shape != K.shape or codebook.shape != (H, Mtot, d):
        raise ValueError(f"shapes: K {tuple(K.shape)}, V {tuple(V.shape)}, codebook "
                         f"{tuple(codebook.shape)} (want [{H},{Mtot},{d}])")
    shape = make_shape(B, H, N, d, M0, C, K.dtype)
    dev = K.device
    if out is None:
        out = (torch.empty((B, H, N), dtype=torch.int32, device=dev),
               torch.empty((B, H, Mtot), dtype=torch.int32, device=dev),
               torch.empty((B, H, Mtot, d), dtype=torch.float32, device=dev))
    nbytes = avq_precompute_workspace_bytes(shape)
    if ws is None:
        ws = workspace(nbytes, dev)
    rc = avq_precompute(shape, K, V, codebook, *out, ws, ws.numel(), stream)
    if rc != AVQ_OK:
        raise AVQError(rc, "avq_precompute")
    return out


def attention(Q: torch.Tensor, codebook: torch.Tensor, counts: torch.Tensor, vsum: torch.Tensor,
              M0: int, C: int, P: int, tile: int, scale: float | None = None, *, out=None,
              ws: torch.Tensor | None = None, stream=None):
    """Return (O [B,H,N,d] in Q's dtype, selected [B,H,ceil(N/tile),P] int32)."""
    _check(Q, "Q")
    _check(codebook, "codebook", Q.dtype)
    _check(counts, "counts", torch.int32)
    _check(vsum, "vsum", torch.float32)
    B, H, N, d = Q.shape
    Mtot = M0 * (1 + C)
    if codebook.shape != (H, Mtot, d) or counts.shape != (B, H, Mtot) or vsum.shape != (B, H, Mtot, d):
        raise ValueError("codebook/counts/vsum shapes do not match Q and M0, C")
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    shape = make_shape(B, H, N, d, M0, C, Q.dtype)
    ntiles = (N + tile - 1) // tile
    dev = Q.device
    if out is None:
        out = (torch.empty_like(Q),
               torch.empty((B, H, ntiles, P), dtype=torch.int32, device=dev))
    nbytes = avq_attention_workspace_bytes(shape, P, tile)
    if ws is None:
        ws = workspace(nbytes, dev)
    rc = avq_attention(shape, Q, codebook, counts, vsum, P, tile, scale, out[0],
                       out[1] if P > 0 else None, ws, ws.numel(), stream)
    if rc != AVQ_OK:
        raise AVQError(rc, "avq_attention")
    return out


def commitment(K: torch.Tensor, codebook: torch.Tensor, assign: torch.Tensor, M0: int, C: int,
               *, stream=None) -> torch.Tensor:
    """Per-(b,h) sum of ||k - codebook[h, assign]||^2 over the keys ([B,H] fp64);
    divide by N for the commitment loss."""
    _check(K, "K")
    _check(codebook, "codebook", K.dtype)
    _check(assign, "assign", torch.int32)
    B, H, N, d = K.shape
    if assign.shape != (B, H, N) or codebook.shape != (H, M0 * (1 + C), d):
        raise ValueError(f"shapes: K {tuple(K.shape)}, assign {tuple(assign.shape)}, codebook "
                         f"{tuple(codebook.shape)}")
    out = torch.empty((B, H), dtype=torch.float64, device=K.device)
    rc = avq_commitment(make_shape(B, H, N, d, M0, C, K.dtype), K, codebook, assign, out, stream)
    if rc != AVQ_OK:
        raise AVQError(rc, "avq_commitment")
    return out


def capture(Q: torch.Tensor, K: torch.Tensor, assign: torch.Tensor, selected: torch.Tensor | None,
            M0: int, C: int, P: int, tile: int, scale: float | None = None, *,
            ws: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """Top-P capture of every query ([B,H,N] fp32): the share of its exact
    softmax attention weight on keys whose parent is selected for its tile.
    Raises on a device-side timeout."""
    _check(Q, "Q")
    _check(K, "K", Q.dtype)
    _check(assign, "assign", torch.int32)
    B, H, N, d = Q.shape
    if K.shape != Q.shape or assign.shape != (B, H, N):
        raise ValueError(f"shapes: Q {tuple(Q.shape)}, K {tuple(K.shape)}, assign {tuple(assign.shape)}")
    if P > 0:
        _check(selected, "selected", torch.int32)
        if selected.shape != (B, H, (N + tile - 1) // tile, P):
            raise ValueError(f"selected has shape {tuple(selected.shape)}")
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    shape = make_shape(B, H, N, d, M0, C, Q.dtype)
    if ws is None:
        ws = workspace(avq_capture_workspace_bytes(shape, P, tile), Q.device)
    out = torch.empty((B, H, N), dtype=torch.float32, device=Q.device)
    rc = avq_capture(shape, Q, K, assign, selected if P > 0 else None, P, tile, scale, out, ws, ws.numel(),
                     stream)
    if rc != AVQ_OK:
        raise AVQError(rc, "avq_capture")
    st = avq_device_status(ws, stream)
    if st != AVQ_OK:
        raise AVQError(st, "avq_capture (device status)")
    return out


def gilbert_order(rows: int, cols: int):
    """The tokens of a rows x cols grid (token r*cols + c) in Gilbert-curve
    order, as an int32 numpy array (host)."""
    import numpy as np
    order = np.empty(rows * cols, dtype=np.int32)
    rc = avq_gilbert_order(rows, cols, order)
    if rc != AVQ_OK:
        raise AVQError(rc, "avq_gilbert_order")
    return order


def gather_rows(x: torch.Tensor, perm: torch.Tensor, *, stream=None) -> torch.Tensor:
    """y[b,h,i,:] = x[b,h,perm[i],:] for a [B,H,N,d] tensor (device kernel)."""
    _check(x, "x")
    _check(perm, "perm", torch.int32)
    B, H, N, d = x.shape
    if perm.shape != (N,):
        raise ValueError(f"perm must have shape ({N},), got {tuple(perm.shape)}")
    y = torch.empty_like(x)
    rc = avq_gather_rows(make_shape(B, H, N, d, 1, 1, x.dtype), x, y, perm, stream)
    if rc != AVQ_OK:
        raise AVQError(rc, "avq_gather_rows")
    return y


def deep_rows(M0: int, C: int, L: int) -> int:
    """Rows of a depth-L codebook: M0 (1 + C + ... + C^(L-1))."""
    return sum(M0 * C ** k for k in range(L))


def precompute_deep(K: torch.Tensor, V: torch.Tensor, codebook: torch.Tensor, M0: int, C: int, L: int,
                    *, out=None, stream=None):
    """Depth-L assignment and path statistics: (assign, counts, vsum)."""
    for t, n in ((K, "K"), (V, "V"), (codebook, "codebook")):
        _check(t, n, K.dtype)
    B, H, N, d = K.shape
    Mtot = deep_rows(M0, C, L)
    if V.shape != K.shape or codebook.shape != (H, Mtot, d):
        raise ValueError(f"shapes: K {tuple(K.shape)}, codebook {tuple(codebook.shape)} (want [{H},{Mtot},{d}])")
    shape = make_shape(B, H, N, d, M0, C, K.dtype)
    dev = K.device
    if out is None:
        out = (torch.empty((B, H, N), dtype=torch.int32, device=dev),
               torch.empty((B, H, Mtot), dtype=torch.int32, device=dev),
               torch.empty((B, H, Mtot, d), dtype=torch.float32, device=dev))
    rc = avq_precompute_deep(shape, L, K, V, codebook, *out, stream)
    if rc != AVQ_OK:
        raise AVQError(rc, "avq_precompute_deep")
    return out


def attention_deep(Q: torch.Tensor, codebook: torch.Tensor, counts: torch.Tensor, vsum: torch.Tensor,
                   M0: int, C: int, L: int, P, tile: int, scale: float | None = None, *, out=None,
                   ws: torch.Tensor | None = None, stream=None):
    """Depth-L adaptive attention: (O [B,H,N,d], selected [B,H,ntiles,sum(P)])."""
    _check(Q, "Q")
    _check(codebook, "codebook", Q.dtype)
    _check(counts, "counts", torch.int32)
    _check(vsum, "vsum", torch.float32)
    B, H, N, d = Q.shape
    P = [int(x) for x in P]
    if len(P) != L - 1:
        raise ValueError("one budget per expanded level (L - 1)")
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    shape = make_shape(B, H, N, d, M0, C, Q.dtype)
    ntiles = (N + tile - 1) // tile
    dev = Q.device
    if out is None:
        out = (torch.empty_like(Q), torch.empty((B, H, ntiles, sum(P)), dtype=torch.int32, device=dev))
    if ws is None:
        ws = workspace(avq_attention_deep_workspace_bytes(shape, L), dev)
    rc = avq_attention_deep(shape, L, P, Q, codebook, counts, vsum, tile, scale, out[0],
                            out[1] if sum(P) > 0 else None, ws, ws.numel(), stream)
    if rc != AVQ_OK:
        raise AVQError(rc, "avq_attention_deep")
    return out
