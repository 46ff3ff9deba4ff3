"""ctypes binding of libattnsink.so (C ABI declared in include/attnsink.h).

Argument marshalling only: torch tensors are described as ``attn_tensor``
structs (device pointer, dtype, shape, strides) and passed to the library,
which runs every step on the GPU.  There is no CPU fallback: if the library
is missing or a call fails, an exception is raised.

The functions carry the C names.  ``stream`` defaults to torch's current CUDA
stream on the tensors' device.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libattnsink.so")

ATTN_OK = 0
ATTN_EINVAL = -1
ATTN_EUNSUPPORTED = -2
ATTN_ECUDA = -3
ATTN_ENOMEM = -4
ATTN_ETIMEOUT = -5

ATTN_DTYPE_BF16 = 1
ATTN_DTYPE_F32 = 2
ATTN_DTYPE_I32 = 3
ATTN_DTYPE_E4M3 = 4

_DTYPES = {torch.bfloat16: ATTN_DTYPE_BF16, torch.float32: ATTN_DTYPE_F32,
           torch.int32: ATTN_DTYPE_I32, torch.float8_e4m3fn: ATTN_DTYPE_E4M3}

# Every symbol include/attnsink.h declares.
EXPORTS = ("attn_sink_fwd", "attn_sink_fwd_max_logit", "attn_sink_fwd_varlen", "attn_sink_bwd", "attn_sink_fwd_cudacore", "attn_sink_decode",
           "attn_sink_decode_chunked", "attn_sink_decode_paged", "attn_sink_decode_fp8",
           "attn_sink_decode_noalloc",
           "attn_sink_get_status", "attn_sink_set_wait_limit_ns", "attn_sink_fail_workspace_allocs",
           "attn_sink_strerror", "attn_sink_last_error")


class AttnTensor(ctypes.Structure):
    _fields_ = [("data", ctypes.c_void_p), ("dtype", ctypes.c_int32), ("ndim", ctypes.c_int32),
                ("shape", ctypes.c_int64 * 4), ("stride", ctypes.c_int64 * 4)]


class AttnSinkError(RuntimeError):
    def __init__(self, code: int, where: str, detail: str):
        self.code = code
        super().__init__(f"{where}: {detail or 'error'} (code {code})")


_lib = None


def load() -> ctypes.CDLL:
    """Load libattnsink.so (built by ``python -m sliding_window_learned_b200.build``)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"libattnsink.so is not built ({LIB_PATH}); run "
                              "`python -m sliding_window_learned_b200.build`")
        lib = ctypes.CDLL(LIB_PATH)
        P = ctypes.POINTER(AttnTensor)
        V = ctypes.c_void_p
        i32, f32 = ctypes.c_int32, ctypes.c_float
        for name in ("attn_sink_fwd", "attn_sink_fwd_cudacore"):
            fn = getattr(lib, name)
            fn.argtypes = [P, P, P, P, i32, f32, P, P, V]
            fn.restype = ctypes.c_int
        lib.attn_sink_bwd.argtypes = [P, P, P, P, P, P, P, i32, f32, P, P, P, P, V]
        lib.attn_sink_bwd.restype = ctypes.c_int
        lib.attn_sink_fwd_max_logit.argtypes = [P, P, P, P, i32, f32, P, P, P, V]
        lib.attn_sink_fwd_max_logit.restype = ctypes.c_int
        lib.attn_sink_fwd_varlen.argtypes = [P, P, P, P, i32, P, i32, f32, P, P, V]
        lib.attn_sink_fwd_varlen.restype = ctypes.c_int
        lib.attn_sink_decode.argtypes = [P, P, P, P, P, i32, f32, P, V]
        lib.attn_sink_decode.restype = ctypes.c_int
        lib.attn_sink_decode_chunked.argtypes = [P, P, P, P, P, i32, f32, i32, P, V]
        lib.attn_sink_decode_chunked.restype = ctypes.c_int
        lib.attn_sink_decode_paged.argtypes = [P, P, P, P, P, P, i32, f32, P, V]
        lib.attn_sink_decode_paged.restype = ctypes.c_int
        lib.attn_sink_decode_fp8.argtypes = [P, P, P, P, P, P, P, i32, f32, P, V]
        lib.attn_sink_decode_fp8.restype = ctypes.c_int
        lib.attn_sink_decode_noalloc.argtypes = [P, P, P, P, P, i32, f32, P, V]
        lib.attn_sink_decode_noalloc.restype = ctypes.c_int
        lib.attn_sink_get_status.argtypes = [V]
        lib.attn_sink_get_status.restype = ctypes.c_int
        lib.attn_sink_set_wait_limit_ns.argtypes = [ctypes.c_uint64]
        lib.attn_sink_set_wait_limit_ns.restype = ctypes.c_int
        lib.attn_sink_fail_workspace_allocs.argtypes = [i32]
        lib.attn_sink_fail_workspace_allocs.restype = ctypes.c_int
        lib.attn_sink_strerror.argtypes = [ctypes.c_int]
        lib.attn_sink_strerror.restype = ctypes.c_char_p
        lib.attn_sink_last_error.argtypes = []
        lib.attn_sink_last_error.restype = ctypes.c_char_p
        _lib = lib
    return _lib


_DESC_CACHE: dict = {}


def describe(t: torch.Tensor | None):
    """An attn_tensor describing a torch tensor (None -> NULL).  Descriptions
    are cached by (address, dtype, shape, strides): a struct holds no more than
    those, so a cached one is exact for any tensor with the same key."""
    if t is None:
        return None
    key = (t.data_ptr(), t.dtype, tuple(t.shape), t.stride())
    d = _DESC_CACHE.get(key)
    if d is not None:
        return d
    if t.dtype not in _DTYPES:
        raise TypeError(f"unsupported dtype {t.dtype}")
    if t.dim() > 4:
        raise ValueError("at most 4 dimensions")
    if len(_DESC_CACHE) > 256:
        _DESC_CACHE.clear()
    d = AttnTensor()
    d.data = t.data_ptr() if t.numel() > 0 else None
    d.dtype = _DTYPES[t.dtype]
    d.ndim = t.dim()
    for i in range(t.dim()):
        d.shape[i] = t.shape[i]
        d.stride[i] = t.stride(i)
    _DESC_CACHE[key] = d
    return d


def _ref(d):
    return ctypes.byref(d) if d is not None else None


def _stream(stream, t: torch.Tensor):
    if stream is None:
        return torch.cuda.current_stream(t.device).cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def _check(rc: int, where: str):
    if rc != ATTN_OK:
        detail = load().attn_sink_last_error().decode()
        raise AttnSinkError(rc, where, detail)


def attn_sink_fwd(q, k, v, sinks, window: int, scale: float, out, lse=None, stream=None):
    """C ``attn_sink_fwd``: tcgen05 prefill forward into ``out`` (and ``lse``)."""
    lib = load()
    ds = [describe(x) for x in (q, k, v, sinks, out, lse)]
    rc = lib.attn_sink_fwd(_ref(ds[0]), _ref(ds[1]), _ref(ds[2]), _ref(ds[3]), int(window),
                           float(scale), _ref(ds[4]), _ref(ds[5]), _stream(stream, q))
    _check(rc, "attn_sink_fwd")


def attn_sink_bwd(q, k, v, o, lse, dout, sinks, window: int, scale: float, dq, dk, dv, dsink,
                  stream=None):
    """C ``attn_sink_bwd``: gradients of sum(dout * O) into dq, dk, dv (bf16)
    and dsink ([Hq] f32); ``o`` is the forward's output (bf16 or f32)."""
    lib = load()
    ds = [describe(x) for x in (q, k, v, o, lse, dout, sinks, dq, dk, dv, dsink)]
    rc = lib.attn_sink_bwd(_ref(ds[0]), _ref(ds[1]), _ref(ds[2]), _ref(ds[3]), _ref(ds[4]), _ref(ds[5]),
                           _ref(ds[6]), int(window), float(scale), _ref(ds[7]), _ref(ds[8]), _ref(ds[9]),
                           _ref(ds[10]), _stream(stream, q))
    _check(rc, "attn_sink_bwd")


def attn_sink_fwd_max_logit(q, k, v, sinks, window: int, scale: float, out, lse, max_logit,
                            stream=None):
    """C ``attn_sink_fwd_max_logit``: attn_sink_fwd plus the largest content
    logit of every (batch, head) into ``max_logit [B, Hq]`` (f32)."""
    lib = load()
    ds = [describe(x) for x in (q, k, v, sinks, out, lse, max_logit)]
    rc = lib.attn_sink_fwd_max_logit(_ref(ds[0]), _ref(ds[1]), _ref(ds[2]), _ref(ds[3]), int(window),
                                     float(scale), _ref(ds[4]), _ref(ds[5]), _ref(ds[6]),
                                     _stream(stream, q))
    _check(rc, "attn_sink_fwd_max_logit")


def attn_sink_fwd_varlen(q, k, v, cu_seqlens, max_seqlen: int, sinks, window: int, scale: float,
                         out, lse=None, stream=None):
    """C ``attn_sink_fwd_varlen``: forward over packed sequences (q/out
    [T,Hq,D], k/v [T,Hkv,D], cu_seqlens [B+1] int32 on the device, lse [Hq,T])."""
    lib = load()
    ds = [describe(x) for x in (q, k, v, cu_seqlens, sinks, out, lse)]
    rc = lib.attn_sink_fwd_varlen(_ref(ds[0]), _ref(ds[1]), _ref(ds[2]), _ref(ds[3]),
                                  int(max_seqlen), _ref(ds[4]), int(window), float(scale),
                                  _ref(ds[5]), _ref(ds[6]), _stream(stream, q))
    _check(rc, "attn_sink_fwd_varlen")


def attn_sink_fwd_cudacore(q, k, v, sinks, window: int, scale: float, out, lse=None, stream=None):
    """C ``attn_sink_fwd_cudacore``: the CUDA-core fp32 second implementation."""
    lib = load()
    ds = [describe(x) for x in (q, k, v, sinks, out, lse)]
    rc = lib.attn_sink_fwd_cudacore(_ref(ds[0]), _ref(ds[1]), _ref(ds[2]), _ref(ds[3]),
                                    int(window), float(scale), _ref(ds[4]), _ref(ds[5]),
                                    _stream(stream, q))
    _check(rc, "attn_sink_fwd_cudacore")


def attn_sink_decode(q, kcache, vcache, seqlens, sinks, window: int, scale: float, out,
                     stream=None):
    """C ``attn_sink_decode``: split-KV decode into ``out``."""
    lib = load()
    ds = [describe(x) for x in (q, kcache, vcache, seqlens, sinks, out)]
    rc = lib.attn_sink_decode(_ref(ds[0]), _ref(ds[1]), _ref(ds[2]), _ref(ds[3]), _ref(ds[4]),
                              int(window), float(scale), _ref(ds[5]), _stream(stream, q))
    _check(rc, "attn_sink_decode")


def attn_sink_decode_chunked(q, kcache, vcache, seqlens, sinks, window: int, scale: float,
                             chunk: int, out, stream=None):
    """C ``attn_sink_decode_chunked``: split-KV decode with ``chunk`` keys per split."""
    lib = load()
    ds = [describe(x) for x in (q, kcache, vcache, seqlens, sinks, out)]
    rc = lib.attn_sink_decode_chunked(_ref(ds[0]), _ref(ds[1]), _ref(ds[2]), _ref(ds[3]),
                                      _ref(ds[4]), int(window), float(scale), int(chunk),
                                      _ref(ds[5]), _stream(stream, q))
    _check(rc, "attn_sink_decode_chunked")


def attn_sink_decode_paged(q, kpages, vpages, block_table, seqlens, sinks, window: int,
                           scale: float, out, stream=None):
    """C ``attn_sink_decode_paged``: split-KV decode over page pools
    ``[NB, P, Hkv, D]`` addressed through ``block_table [B, MP]`` (int32)."""
    lib = load()
    ds = [describe(x) for x in (q, kpages, vpages, block_table, seqlens, sinks, out)]
    rc = lib.attn_sink_decode_paged(_ref(ds[0]), _ref(ds[1]), _ref(ds[2]), _ref(ds[3]),
                                    _ref(ds[4]), _ref(ds[5]), int(window), float(scale),
                                    _ref(ds[6]), _stream(stream, q))
    _check(rc, "attn_sink_decode_paged")


def attn_sink_decode_fp8(q, kcache, vcache, k_descale, v_descale, seqlens, sinks, window: int,
                         scale: float, out, stream=None):
    """C ``attn_sink_decode_fp8``: split-KV decode over an e4m3 cache
    (``torch.float8_e4m3fn``) with per-kv-head descales ``[Hkv]`` (f32)."""
    lib = load()
    ds = [describe(x) for x in (q, kcache, vcache, k_descale, v_descale, seqlens, sinks, out)]
    rc = lib.attn_sink_decode_fp8(_ref(ds[0]), _ref(ds[1]), _ref(ds[2]), _ref(ds[3]), _ref(ds[4]),
                                  _ref(ds[5]), _ref(ds[6]), int(window), float(scale), _ref(ds[7]),
                                  _stream(stream, q))
    _check(rc, "attn_sink_decode_fp8")


def attn_sink_decode_noalloc(q, kcache, vcache, seqlens, sinks, window: int, scale: float, out,
                             stream=None):
    """C ``attn_sink_decode_noalloc``: the split-KV decode with its workspace in
    the library's fixed 48 MiB device array, for callers that may not allocate
    device memory while decoding.  Calls that overlap on the GPU race on that
    array; make the first call on a device before any stream capture."""
    lib = load()
    ds = [describe(x) for x in (q, kcache, vcache, seqlens, sinks, out)]
    rc = lib.attn_sink_decode_noalloc(_ref(ds[0]), _ref(ds[1]), _ref(ds[2]), _ref(ds[3]),
                                      _ref(ds[4]), int(window), float(scale), _ref(ds[5]),
                                      _stream(stream, q))
    _check(rc, "attn_sink_decode_noalloc")


def attn_sink_set_wait_limit_ns(ns: int):
    """C ``attn_sink_set_wait_limit_ns`` (diagnostics): limit of every device
    wait on the current device, 0 = the default."""
    _check(load().attn_sink_set_wait_limit_ns(int(ns)), "attn_sink_set_wait_limit_ns")


def attn_sink_fail_workspace_allocs(count: int):
    """C ``attn_sink_fail_workspace_allocs`` (diagnostics): the next ``count``
    workspace allocations fail with ATTN_ENOMEM."""
    _check(load().attn_sink_fail_workspace_allocs(int(count)), "attn_sink_fail_workspace_allocs")


def attn_sink_get_status(stream=None) -> int:
    """C ``attn_sink_get_status``: sync ``stream`` and read/clear the device status."""
    lib = load()
    s = stream.cuda_stream if isinstance(stream, torch.cuda.Stream) else stream
    return int(lib.attn_sink_get_status(s))


def attn_sink_strerror(code: int) -> str:
    return load().attn_sink_strerror(int(code)).decode()


def attn_sink_last_error() -> str:
    return load().attn_sink_last_error().decode()


# ---------------------------------------------------------------- conveniences
def fwd(q, k, v, sinks, window: int, scale: float, with_lse: bool = True, stream=None):
    """Allocate outputs and run attn_sink_fwd.  Returns (out, lse or None)."""
    B, L, Hq, D = q.shape
    out = torch.empty_like(q)
    lse = torch.empty(B, Hq, L, dtype=torch.float32, device=q.device) if with_lse else None
    attn_sink_fwd(q, k, v, sinks, window, scale, out, lse, stream)
    return out, lse


def decode(q, kcache, vcache, seqlens, sinks, window: int, scale: float, chunk: int = 0,
           stream=None):
    """Allocate the output and run the split-KV decode.  Returns out [B,Hq,D]."""
    out = torch.empty_like(q)
    attn_sink_decode_chunked(q, kcache, vcache, seqlens, sinks, window, scale, chunk, out, stream)
    return out
