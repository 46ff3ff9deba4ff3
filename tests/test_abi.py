"""The C ABI without a GPU: the library loads, exports every symbol the header
declares, and rejects invalid arguments on the host before any launch."""
import ctypes
import os
import re

import pytest

from sliding_window_learned_b200 import abi

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    from sliding_window_learned_b200 import build
    build.build()
    return abi.load()


def _declared():
    text = open(os.path.join(ROOT, "include", "attnsink.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(attn_sink_\w+)\s*\(", text)))


def test_header_declares_the_binding_exports():
    assert _declared() == sorted(abi.EXPORTS)


def test_library_exports_every_declared_symbol(lib):
    for name in _declared():
        assert hasattr(lib, name), name


def test_strerror(lib):
    assert abi.attn_sink_strerror(0) == "success"
    assert "invalid" in abi.attn_sink_strerror(abi.ATTN_EINVAL)
    assert "timed out" in abi.attn_sink_strerror(abi.ATTN_ETIMEOUT)
    assert abi.attn_sink_strerror(12345) == "unknown error"


def _t(shape, dtype=abi.ATTN_DTYPE_BF16, ptr=0x10000, strides=None):
    d = abi.AttnTensor()
    d.data = ptr
    d.dtype = dtype
    d.ndim = len(shape)
    if strides is None:
        strides, acc = [], 1
        for s in reversed(shape):
            strides.insert(0, acc)
            acc *= s
    for i, (s, st) in enumerate(zip(shape, strides)):
        d.shape[i] = s
        d.stride[i] = st
    return d


def _fwd(lib, q, k, v, s, o, lse=None, window=64, scale=0.125, fn="attn_sink_fwd"):
    r = lambda x: ctypes.byref(x) if x is not None else None
    return getattr(lib, fn)(r(q), r(k), r(v), r(s), window, scale, r(o), r(lse), None)


def _good():
    return (_t([1, 256, 4, 64]), _t([1, 256, 2, 64]), _t([1, 256, 2, 64]),
            _t([4], abi.ATTN_DTYPE_F32), _t([1, 256, 4, 64]))


@pytest.mark.parametrize("case", [
    "q dtype", "q ndim", "k shape", "v shape", "out shape", "sinks len", "gqa", "window",
    "scale nan", "scale neg", "misaligned", "inner stride", "tma stride", "lse shape",
    "null data", "negative size"])
def test_fwd_rejects_invalid_arguments(lib, case):
    q, k, v, s, o = _good()
    lse = None
    window, scale = 64, 0.125
    if case == "q dtype":
        q = _t([1, 256, 4, 64], abi.ATTN_DTYPE_F32)
    elif case == "q ndim":
        q = _t([256, 4, 64])
    elif case == "k shape":
        k = _t([1, 255, 2, 64])
    elif case == "v shape":
        v = _t([1, 256, 1, 64])
    elif case == "out shape":
        o = _t([1, 256, 4, 32])
    elif case == "sinks len":
        s = _t([3], abi.ATTN_DTYPE_F32)
    elif case == "gqa":
        q, o = _t([1, 256, 3, 64]), _t([1, 256, 3, 64])
        s = _t([3], abi.ATTN_DTYPE_F32)
    elif case == "window":
        window = 0
    elif case == "scale nan":
        scale = float("nan")
    elif case == "scale neg":
        scale = -1.0
    elif case == "misaligned":
        q = _t([1, 256, 4, 64], ptr=0x10008)
    elif case == "inner stride":
        q = _t([1, 256, 4, 64], strides=[65536, 256, 64, 2])
    elif case == "tma stride":
        k = _t([1, 256, 2, 64], strides=[256 * 2 * 68, 2 * 68, 68, 1])
    elif case == "lse shape":
        lse = _t([1, 256, 4], abi.ATTN_DTYPE_F32)
    elif case == "null data":
        v = _t([1, 256, 2, 64], ptr=0)
    elif case == "negative size":
        k = _t([1, -1, 2, 64])
    rc = _fwd(lib, q, k, v, s, o, lse, window, scale)
    assert rc == abi.ATTN_EINVAL, (case, rc, abi.attn_sink_last_error())
    assert abi.attn_sink_last_error() != ""


def test_fwd_rejects_unsupported_head_dim(lib):
    q, k, v, s, o = (_t([1, 16, 2, 96]), _t([1, 16, 2, 96]), _t([1, 16, 2, 96]),
                     _t([2], abi.ATTN_DTYPE_F32), _t([1, 16, 2, 96]))
    assert _fwd(lib, q, k, v, s, o) == abi.ATTN_EUNSUPPORTED


def _dec(lib, q, kc, vc, sl, s, o, window=128, scale=0.125, chunk=0):
    r = ctypes.byref
    return lib.attn_sink_decode_chunked(r(q), r(kc), r(vc), r(sl), r(s), window, scale, chunk,
                                        r(o), None)


@pytest.mark.parametrize("case", ["seqlens dtype", "cache shape", "chunk", "gqa", "window",
                                  "head dim", "group too large"])
def test_decode_rejects_invalid_arguments(lib, case):
    q, kc, vc = _t([2, 8, 128]), _t([2, 512, 2, 128]), _t([2, 512, 2, 128])
    sl, s, o = _t([2], abi.ATTN_DTYPE_I32), _t([8], abi.ATTN_DTYPE_F32), _t([2, 8, 128])
    window, chunk = 128, 0
    expect = abi.ATTN_EINVAL
    if case == "seqlens dtype":
        sl = _t([2], abi.ATTN_DTYPE_F32)
    elif case == "cache shape":
        vc = _t([2, 511, 2, 128])
    elif case == "chunk":
        chunk = 100
    elif case == "gqa":
        kc, vc = _t([2, 512, 3, 128]), _t([2, 512, 3, 128])
    elif case == "window":
        window = -5
    elif case == "head dim":
        q, kc, vc, o = _t([2, 8, 96]), _t([2, 512, 2, 96]), _t([2, 512, 2, 96]), _t([2, 8, 96])
        expect = abi.ATTN_EUNSUPPORTED
    elif case == "group too large":
        q, o, s = _t([2, 34, 128]), _t([2, 34, 128]), _t([34], abi.ATTN_DTYPE_F32)
        expect = abi.ATTN_EUNSUPPORTED
    rc = _dec(lib, q, kc, vc, sl, s, o, window=window, chunk=chunk)
    assert rc == expect, (case, rc, abi.attn_sink_last_error())


@pytest.mark.parametrize("case", ["page not a power of two", "page too small", "table rows",
                                  "table dtype", "pool shapes differ", "gqa", "head dim"])
def test_paged_decode_rejects_invalid_arguments(lib, case):
    q, o = _t([2, 8, 128]), _t([2, 8, 128])
    kp, vp = _t([40, 64, 2, 128]), _t([40, 64, 2, 128])
    bt = _t([2, 16], abi.ATTN_DTYPE_I32)
    sl, s = _t([2], abi.ATTN_DTYPE_I32), _t([8], abi.ATTN_DTYPE_F32)
    expect = abi.ATTN_EINVAL
    if case == "page not a power of two":
        kp, vp = _t([40, 48, 2, 128]), _t([40, 48, 2, 128])
        expect = abi.ATTN_EUNSUPPORTED
    elif case == "page too small":
        kp, vp = _t([40, 8, 2, 128]), _t([40, 8, 2, 128])
        expect = abi.ATTN_EUNSUPPORTED
    elif case == "table rows":
        bt = _t([3, 16], abi.ATTN_DTYPE_I32)
    elif case == "table dtype":
        bt = _t([2, 16], abi.ATTN_DTYPE_F32)
    elif case == "pool shapes differ":
        vp = _t([41, 64, 2, 128])
    elif case == "gqa":
        kp, vp = _t([40, 64, 3, 128]), _t([40, 64, 3, 128])
    elif case == "head dim":
        q, o = _t([2, 8, 96]), _t([2, 8, 96])
        kp, vp = _t([40, 64, 2, 96]), _t([40, 64, 2, 96])
        expect = abi.ATTN_EUNSUPPORTED
    r = ctypes.byref
    rc = lib.attn_sink_decode_paged(r(q), r(kp), r(vp), r(bt), r(sl), r(s), 128, 0.125, r(o), None)
    assert rc == expect, (case, rc, abi.attn_sink_last_error())


def test_noalloc_decode_rejects_workspace_beyond_its_array(lib):
    """The no-allocation decode checks its workspace bound on the host and
    refuses, with a message naming both sizes, before any device work."""
    B, Smax, Hq, Hkv, D = 256, 131072, 32, 4, 128   # ~135 MB of workspace
    q, o = _t([B, Hq, D]), _t([B, Hq, D])
    kc = _t([B, Smax, Hkv, D])
    sl, s = _t([B], abi.ATTN_DTYPE_I32), _t([Hq], abi.ATTN_DTYPE_F32)
    r = ctypes.byref
    rc = lib.attn_sink_decode_noalloc(r(q), r(kc), r(kc), r(sl), r(s), Smax, 0.125, r(o), None)
    assert rc == abi.ATTN_EUNSUPPORTED
    assert "workspace" in abi.attn_sink_last_error()


def test_binding_fails_loudly_without_library(tmp_path, monkeypatch):
    monkeypatch.setattr(abi, "LIB_PATH", str(tmp_path / "missing.so"))
    monkeypatch.setattr(abi, "_lib", None)
    with pytest.raises(ImportError):
        abi.load()
