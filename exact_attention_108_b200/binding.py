"""ctypes binding over libfattn.so -- argument marshalling only.

Every step of the computation runs in the library's CUDA kernels.  There is no
fallback: if the library is missing or cannot be loaded, every call raises.
The names mirror the C ABI in include/fattn.h.
"""
from __future__ import annotations

import ctypes
import math
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libfattn.so")

FATTN_OK = 0
FATTN_ERR_INVALID_ARG = 1
FATTN_ERR_UNSUPPORTED = 2
FATTN_ERR_ALIGNMENT = 3
FATTN_ERR_CUDA = 4
FATTN_ERR_DEVICE_TIMEOUT = 5
FATTN_ERR_SCRATCH_TOO_SMALL = 6
NOALLOC_SCRATCH_BYTES = 32 << 20  # FATTN_NOALLOC_SCRATCH_BYTES

# Every symbol include/fattn.h declares (checked by the CPU test suite).
EXPORTED = ("fattn_fwd", "fattn_bwd", "fattn_bwd_workspace_size", "fattn_bwd_preprocess",
            "fattn_bwd_dkdv", "fattn_bwd_dq", "fattn_status_string", "fattn_last_cuda_error",
            "fattn_device_status", "fattn_version", "fattn_bwd_noalloc", "fattn_fwd_ex",
            "fattn_bwd_ex", "fattn_bwd_ex_workspace_size", "fattn_decode", "fattn_decode_workspace_size", "fattn_selftest_wait_timeout")


class FwdParams(ctypes.Structure):
    """fattn_fwd_params (include/fattn.h)."""
    _fields_ = [("q", ctypes.c_void_p), ("k", ctypes.c_void_p), ("v", ctypes.c_void_p),
                ("o", ctypes.c_void_p), ("lse", ctypes.c_void_p),
                ("B", ctypes.c_int), ("H", ctypes.c_int), ("H_kv", ctypes.c_int), ("N_q", ctypes.c_int),
                ("N_k", ctypes.c_int), ("d", ctypes.c_int), ("causal", ctypes.c_int),
                ("scale", ctypes.c_float), ("dropout_p", ctypes.c_float),
                ("seed", ctypes.c_ulonglong), ("offset", ctypes.c_uint)]


class DecodeParams(ctypes.Structure):
    """fattn_decode_params (include/fattn.h)."""
    _fields_ = [("q", ctypes.c_void_p), ("k", ctypes.c_void_p), ("v", ctypes.c_void_p),
                ("o", ctypes.c_void_p), ("lse", ctypes.c_void_p),
                ("B", ctypes.c_int), ("H", ctypes.c_int), ("H_kv", ctypes.c_int), ("N_q", ctypes.c_int),
                ("N_k", ctypes.c_int), ("N_k_cap", ctypes.c_int), ("d", ctypes.c_int), ("causal", ctypes.c_int),
                ("scale", ctypes.c_float), ("num_splits", ctypes.c_int), ("workspace", ctypes.c_void_p),
                ("workspace_bytes", ctypes.c_size_t)]


class BwdParams(ctypes.Structure):
    """fattn_bwd_params (include/fattn.h)."""
    _fields_ = [("q", ctypes.c_void_p), ("k", ctypes.c_void_p), ("v", ctypes.c_void_p),
                ("o", ctypes.c_void_p), ("dout", ctypes.c_void_p), ("lse", ctypes.c_void_p),
                ("dq", ctypes.c_void_p), ("dk", ctypes.c_void_p), ("dv", ctypes.c_void_p),
                ("B", ctypes.c_int), ("H", ctypes.c_int), ("H_kv", ctypes.c_int), ("N_q", ctypes.c_int),
                ("N_k", ctypes.c_int), ("d", ctypes.c_int), ("causal", ctypes.c_int),
                ("scale", ctypes.c_float), ("dropout_p", ctypes.c_float),
                ("seed", ctypes.c_ulonglong), ("offset", ctypes.c_uint),
                ("deterministic", ctypes.c_int), ("workspace", ctypes.c_void_p),
                ("workspace_bytes", ctypes.c_size_t)]

_lib = None


class FattnError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        msg = f"{where}: {status_string(status)} (status {status})"
        if status == FATTN_ERR_CUDA:
            msg += f": {last_cuda_error()}"
        super().__init__(msg)


def load():
    """Open libfattn.so (once) and declare the C signatures."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"{LIB_PATH} is missing: build it with `python -m exact_attention_108_b200.build`")
    L = ctypes.CDLL(LIB_PATH)
    vp, i, f, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
    L.fattn_fwd.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, f, vp]
    L.fattn_fwd.restype = i
    L.fattn_bwd.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, f, vp, sz, vp]
    L.fattn_bwd.restype = i
    L.fattn_bwd_noalloc.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, f, vp]
    L.fattn_bwd_noalloc.restype = i
    L.fattn_bwd_preprocess.argtypes = [vp, vp, vp, i, i, i, i, vp, sz, vp]
    L.fattn_bwd_preprocess.restype = i
    L.fattn_bwd_dkdv.argtypes = [vp, vp, vp, vp, vp, vp, i, i, i, i, i, f, vp, sz, vp]
    L.fattn_bwd_dkdv.restype = i
    L.fattn_bwd_dq.argtypes = [vp, i, i, i, i, f, vp, sz, vp]
    L.fattn_bwd_dq.restype = i
    L.fattn_bwd_workspace_size.argtypes = [i, i, i, i]
    L.fattn_bwd_workspace_size.restype = sz
    L.fattn_status_string.argtypes = [i]
    L.fattn_status_string.restype = ctypes.c_char_p
    L.fattn_last_cuda_error.argtypes = []
    L.fattn_last_cuda_error.restype = ctypes.c_char_p
    L.fattn_device_status.argtypes = [i]
    L.fattn_device_status.restype = i
    L.fattn_fwd_ex.argtypes = [ctypes.POINTER(FwdParams), vp]
    L.fattn_fwd_ex.restype = i
    L.fattn_bwd_ex.argtypes = [ctypes.POINTER(BwdParams), vp]
    L.fattn_bwd_ex.restype = i
    L.fattn_bwd_ex_workspace_size.argtypes = [ctypes.POINTER(BwdParams)]
    L.fattn_bwd_ex_workspace_size.restype = sz
    L.fattn_decode.argtypes = [ctypes.POINTER(DecodeParams), vp]
    L.fattn_decode.restype = i
    L.fattn_decode_workspace_size.argtypes = [ctypes.POINTER(DecodeParams)]
    L.fattn_decode_workspace_size.restype = sz
    L.fattn_selftest_wait_timeout.argtypes = [vp]
    L.fattn_selftest_wait_timeout.restype = i
    L.fattn_version.argtypes = []
    L.fattn_version.restype = i
    _lib = L
    return L


def status_string(status: int) -> str:
    return load().fattn_status_string(int(status)).decode()


def last_cuda_error() -> str:
    return load().fattn_last_cuda_error().decode()


def device_status(clear: bool = False) -> int:
    return int(load().fattn_device_status(1 if clear else 0))


def workspace_size(B: int, H: int, N: int, d: int) -> int:
    return int(load().fattn_bwd_workspace_size(B, H, N, d))


def _stream_handle(stream) -> int:
    s = torch.cuda.current_stream() if stream is None else stream
    return int(s.cuda_stream)


def _check(t: torch.Tensor, name: str, dtype=torch.bfloat16):
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _shape4(q: torch.Tensor):
    if q.dim() != 4:
        raise ValueError("expected [B, H, N, d] tensors")
    return tuple(int(x) for x in q.shape)


def fwd(q, k, v, causal: bool = False, scale: float | None = None, out=None, lse=None, stream=None):
    """O, LSE = attention(q, k, v); bf16 [B,H,N,d] in, bf16 O and fp32 LSE [B,H,N] out."""
    B, H, N, d = _shape4(q)
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _check(t, n)
        if tuple(t.shape) != (B, H, N, d):
            raise ValueError(f"{n} has shape {tuple(t.shape)}, expected {(B, H, N, d)}")
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, H, N), device=q.device, dtype=torch.float32)
    _check(out, "out")
    _check(lse, "lse", torch.float32)
    rc = load().fattn_fwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), lse.data_ptr(),
                          B, H, N, d, 1 if causal else 0, float(scale), _stream_handle(stream))
    if rc != FATTN_OK:
        raise FattnError(rc, "fattn_fwd")
    return out, lse


def bwd(q, k, v, o, lse, do, causal: bool = False, scale: float | None = None,
        dq=None, dk=None, dv=None, workspace=None, stream=None):
    """dQ, dK, dV of L = sum(dO * O) for the forward that produced (o, lse)."""
    B, H, N, d = _shape4(q)
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (o, "o"), (do, "do")):
        _check(t, n)
        if tuple(t.shape) != (B, H, N, d):
            raise ValueError(f"{n} has shape {tuple(t.shape)}, expected {(B, H, N, d)}")
    _check(lse, "lse", torch.float32)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    need = workspace_size(B, H, N, d)
    if workspace is None:
        workspace = torch.empty(max(need, 1), device=q.device, dtype=torch.uint8)
    rc = load().fattn_bwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), do.data_ptr(),
                          lse.data_ptr(), dq.data_ptr(), dk.data_ptr(), dv.data_ptr(),
                          B, H, N, d, 1 if causal else 0, float(scale),
                          workspace.data_ptr(), workspace.numel() * workspace.element_size(),
                          _stream_handle(stream))
    if rc != FATTN_OK:
        raise FattnError(rc, "fattn_bwd")
    return dq, dk, dv


def _nbytes(t) -> int:
    return t.numel() * t.element_size()


def bwd_preprocess(o, lse, do, workspace, stream=None):
    """Stage 1 of the backward: D, LSE*log2(e) and a zeroed dQ accumulator in `workspace`."""
    B, H, N, d = _shape4(o)
    rc = load().fattn_bwd_preprocess(o.data_ptr(), do.data_ptr(), lse.data_ptr(), B, H, N, d,
                                     workspace.data_ptr(), _nbytes(workspace), _stream_handle(stream))
    if rc != FATTN_OK:
        raise FattnError(rc, "fattn_bwd_preprocess")


def bwd_dkdv(q, k, v, do, dk, dv, workspace, causal: bool = False, scale: float | None = None, stream=None):
    """Stage 2: dK, dV, and dS K added into the workspace accumulator."""
    B, H, N, d = _shape4(q)
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    rc = load().fattn_bwd_dkdv(q.data_ptr(), k.data_ptr(), v.data_ptr(), do.data_ptr(), dk.data_ptr(),
                               dv.data_ptr(), B, H, N, d, 1 if causal else 0, float(scale),
                               workspace.data_ptr(), _nbytes(workspace), _stream_handle(stream))
    if rc != FATTN_OK:
        raise FattnError(rc, "fattn_bwd_dkdv")


def bwd_dq(dq, workspace, scale: float | None = None, stream=None):
    """Stage 3: dQ = bf16(scale * accumulator)."""
    B, H, N, d = _shape4(dq)
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    rc = load().fattn_bwd_dq(dq.data_ptr(), B, H, N, d, float(scale), workspace.data_ptr(),
                             _nbytes(workspace), _stream_handle(stream))
    if rc != FATTN_OK:
        raise FattnError(rc, "fattn_bwd_dq")


def bwd_noalloc(q, k, v, o, lse, do, causal: bool = False, scale: float | None = None,
                dq=None, dk=None, dv=None, stream=None):
    """The backward without any workspace: for callers that cannot allocate device
    memory or hand the library a buffer (see fattn_bwd_noalloc in include/fattn.h).

    Results are those of bwd(); the scratch comes from a fixed 32 MiB array the
    library keeps on each device, so larger shapes raise FattnError and calls that
    overlap on the GPU must not share a device.  (dq, dk, dv are created here when
    not given, as in bwd(); pass them to keep this wrapper allocation-free too.)
    """
    B, H, N, d = _shape4(q)
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (o, "o"), (do, "do")):
        _check(t, n)
        if tuple(t.shape) != (B, H, N, d):
            raise ValueError(f"{n} has shape {tuple(t.shape)}, expected {(B, H, N, d)}")
    _check(lse, "lse", torch.float32)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    rc = load().fattn_bwd_noalloc(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), do.data_ptr(),
                                  lse.data_ptr(), dq.data_ptr(), dk.data_ptr(), dv.data_ptr(),
                                  B, H, N, d, 1 if causal else 0, float(scale), _stream_handle(stream))
    if rc != FATTN_OK:
        raise FattnError(rc, "fattn_bwd_noalloc")
    return dq, dk, dv


def _shapes_general(q, k, v):
    if q.dim() != 4 or k.dim() != 4 or v.dim() != 4:
        raise ValueError("expected [B, H, N, d] tensors")
    B, H, N_q, d = (int(x) for x in q.shape)
    Bk, H_kv, N_k, dk_ = (int(x) for x in k.shape)
    if Bk != B or dk_ != d or tuple(v.shape) != tuple(k.shape):
        raise ValueError(f"k and v must be [B, H_kv, N_k, d] with B={B}, d={d}")
    return B, H, H_kv, N_q, N_k, d


def fwd_ex(q, k, v, causal: bool = False, scale: float | None = None, dropout_p: float = 0.0,
           seed: int = 0, offset: int = 0, out=None, lse=None, stream=None):
    """General forward (fattn_fwd_ex): q [B,H,N_q,d] against k, v [B,H_kv,N_k,d], causal mask
    aligned at the bottom right, optional dropout; returns (O, LSE)."""
    B, H, H_kv, N_q, N_k, d = _shapes_general(q, k, v)
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _check(t, n)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    out = torch.empty_like(q) if out is None else out
    lse = torch.empty((B, H, N_q), device=q.device, dtype=torch.float32) if lse is None else lse
    _check(out, "out")
    _check(lse, "lse", torch.float32)
    p = FwdParams(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), lse.data_ptr(),
                  B, H, H_kv, N_q, N_k, d, 1 if causal else 0, float(scale), float(dropout_p),
                  int(seed), int(offset))
    rc = load().fattn_fwd_ex(ctypes.byref(p), _stream_handle(stream))
    if rc != FATTN_OK:
        raise FattnError(rc, "fattn_fwd_ex")
    return out, lse


def bwd_ex(q, k, v, o, lse, do, causal: bool = False, scale: float | None = None, dropout_p: float = 0.0,
           seed: int = 0, offset: int = 0, deterministic: bool = False, dq=None, dk=None, dv=None,
           workspace=None, stream=None):
    """General backward (fattn_bwd_ex) for the forward of fwd_ex; returns (dQ, dK, dV)."""
    B, H, H_kv, N_q, N_k, d = _shapes_general(q, k, v)
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (o, "o"), (do, "do")):
        _check(t, n)
    _check(lse, "lse", torch.float32)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    p = BwdParams(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), do.data_ptr(), lse.data_ptr(),
                  dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), B, H, H_kv, N_q, N_k, d,
                  1 if causal else 0, float(scale), float(dropout_p), int(seed), int(offset),
                  1 if deterministic else 0, None, 0)
    need = int(load().fattn_bwd_ex_workspace_size(ctypes.byref(p)))
    if workspace is None:
        workspace = torch.empty(max(need, 1), device=q.device, dtype=torch.uint8)
    p.workspace = workspace.data_ptr()
    p.workspace_bytes = _nbytes(workspace)
    rc = load().fattn_bwd_ex(ctypes.byref(p), _stream_handle(stream))
    if rc != FATTN_OK:
        raise FattnError(rc, "fattn_bwd_ex")
    return dq, dk, dv


def decode(q, k_cache, v_cache, n_k: int | None = None, causal: bool = False, scale: float | None = None,
           num_splits: int = 0, out=None, lse=None, workspace=None, stream=None):
    """Decoding attention (fattn_decode): q [B,H,N_q,d] against the first n_k rows of each head
    of the caches k_cache, v_cache [B,H_kv,N_k_cap,d]; returns (O, LSE)."""
    if q.dim() != 4 or k_cache.dim() != 4 or tuple(v_cache.shape) != tuple(k_cache.shape):
        raise ValueError("expected q [B,H,N_q,d] and caches [B,H_kv,N_k_cap,d]")
    B, H, N_q, d = (int(x) for x in q.shape)
    H_kv, cap = int(k_cache.shape[1]), int(k_cache.shape[2])
    n_k = cap if n_k is None else int(n_k)
    for t, n in ((q, "q"), (k_cache, "k_cache"), (v_cache, "v_cache")):
        _check(t, n)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    out = torch.empty_like(q) if out is None else out
    lse = torch.empty((B, H, N_q), device=q.device, dtype=torch.float32) if lse is None else lse
    _check(out, "out")
    _check(lse, "lse", torch.float32)
    p = DecodeParams(q.data_ptr(), k_cache.data_ptr(), v_cache.data_ptr(), out.data_ptr(), lse.data_ptr(),
                     B, H, H_kv, N_q, n_k, cap, d, 1 if causal else 0, float(scale), int(num_splits), None, 0)
    need = int(load().fattn_decode_workspace_size(ctypes.byref(p)))
    if need > 0:
        if workspace is None:
            workspace = torch.empty(need, device=q.device, dtype=torch.uint8)
        p.workspace = workspace.data_ptr()
        p.workspace_bytes = _nbytes(workspace)
    rc = load().fattn_decode(ctypes.byref(p), _stream_handle(stream))
    if rc != FATTN_OK:
        raise FattnError(rc, "fattn_decode")
    return out, lse


def selftest_wait_timeout(stream=None):
    """Enqueue the failure-detection self-test (fattn_selftest_wait_timeout): a kernel
    whose bounded wait runs out after about a second; device_status() then reports
    FATTN_ERR_DEVICE_TIMEOUT."""
    rc = load().fattn_selftest_wait_timeout(_stream_handle(stream))
    if rc != FATTN_OK:
        raise FattnError(rc, "fattn_selftest_wait_timeout")
