"""fp64 CPU oracle for sliding-window attention with a learned per-head sink.

TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check in
``__graft_entry__`` and the ``cpu_baseline`` / reference leg of ``bench.py``
may import this package.  The product library never loads it and has no CPU
fallback; the two share no code.

The arithmetic lives in ``oracle.c`` (plain C, double precision, OpenMP over
rows); this module only builds it with gcc and marshals numpy arrays.  Inputs
are passed as bf16 bit patterns (``np.uint16``) so that the oracle reads the
very bits the device reads.  Each function cites the passage it follows in
``oracle.c``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile oracle.c into liboracle.so (gcc, -O2, OpenMP).  No fast-math:
    the oracle must keep IEEE double semantics."""
    if force or not os.path.exists(_LIB_PATH) or (
        os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC)
    ):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(
            ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11",
             "-fno-fast-math", "-ffp-contract=off", _SRC, "-o", tmp, "-lm"]
        )
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB_PATH)
        P = ctypes.c_void_p
        I = ctypes.c_int
        F = ctypes.c_float
        lib.oracle_num_threads.restype = I
        lib.oracle_fwd.argtypes = [P, P, P, P, I, I, I, I, I, I, F, P, P]
        lib.oracle_fwd.restype = I
        lib.oracle_fwd_rows.argtypes = [P, P, P, P, I, I, I, I, I, I, F, I, P, P, P]
        lib.oracle_fwd_rows.restype = I
        lib.oracle_decode.argtypes = [P, P, P, P, P, I, I, I, I, I, I, F, P, P]
        lib.oracle_decode.restype = I
        lib.oracle_decode_paged.argtypes = [P, P, P, P, P, P, I, I, I, I, I, I, I, I, F, P, P]
        lib.oracle_decode_paged.restype = I
        lib.oracle_decode_fp8.argtypes = [P, P, P, P, P, P, P, I, I, I, I, I, I, F, P, P]
        lib.oracle_decode_fp8.restype = I
        lib.oracle_e4m3_to_f64.argtypes = [ctypes.c_uint8]
        lib.oracle_e4m3_to_f64.restype = ctypes.c_double
        lib.oracle_split_partial.argtypes = [P, P, P, ctypes.c_int64, I, I, I, F, P, P]
        lib.oracle_split_partial.restype = I
        lib.oracle_combine.argtypes = [I, P, P, I, F, P, P]
        lib.oracle_combine.restype = I
        _lib = lib
    return _lib


def _u16(a) -> np.ndarray:
    a = np.ascontiguousarray(a)
    if a.dtype != np.uint16:
        raise TypeError(f"expected bf16 bit patterns as uint16, got {a.dtype}")
    return a


def _f32(a) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(a, dtype=np.float32))


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def num_threads() -> int:
    """Threads the oracle's OpenMP loops use (OMP_NUM_THREADS or the cores)."""
    return int(_load().oracle_num_threads())


def fwd(q, k, v, sinks, window: int, scale: float, with_lse: bool = True):
    """Prefill forward (page 1, learned-sink softmax; see oracle.c).

    q [B,L,Hq,D], k/v [B,L,Hkv,D] as uint16 bf16 bits; sinks [Hq] float32.
    Returns (out [B,L,Hq,D] float64, lse [B,Hq,L] float64 or None)."""
    q, k, v, sinks = _u16(q), _u16(k), _u16(v), _f32(sinks)
    B, L, Hq, D = q.shape
    Hkv = k.shape[2]
    assert k.shape == (B, L, Hkv, D) and v.shape == k.shape and sinks.shape == (Hq,)
    out = np.empty((B, L, Hq, D), np.float64)
    lse = np.empty((B, Hq, L), np.float64) if with_lse else None
    rc = _load().oracle_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(sinks), B, L, Hq, Hkv,
                            D, int(window), float(scale), _ptr(out),
                            _ptr(lse) if with_lse else None)
    if rc != 0:
        raise ValueError("oracle_fwd: invalid sizes")
    return out, lse


def fwd_varlen(q, k, v, cu_seqlens, sinks, window: int, scale: float):
    """Prefill forward over packed variable-length sequences: the tokens of
    sequence b are rows cu_seqlens[b] .. cu_seqlens[b+1]-1 of q [T,Hq,D] and
    k/v [T,Hkv,D] (uint16 bf16 bits), and each sequence is attended on its own
    (positions restart at 0; no query sees another sequence's keys), exactly
    as one batch element of ``fwd`` (the varlen path of the flash-attention
    contributor guide's call walk-through, step 2).
    Returns (out [T,Hq,D] float64, lse [Hq,T] float64)."""
    q, k, v, sinks = _u16(q), _u16(k), _u16(v), _f32(sinks)
    cu = np.asarray(cu_seqlens, dtype=np.int64)
    T, Hq, D = q.shape
    Hkv = k.shape[1]
    assert k.shape == (T, Hkv, D) and v.shape == k.shape
    assert cu.ndim == 1 and cu[0] == 0 and cu[-1] == T and np.all(np.diff(cu) >= 0)
    out = np.empty((T, Hq, D), np.float64)
    lse = np.empty((Hq, T), np.float64)
    for b in range(len(cu) - 1):
        s0, s1 = int(cu[b]), int(cu[b + 1])
        if s1 == s0:
            continue
        o_b, l_b = fwd(q[None, s0:s1], k[None, s0:s1], v[None, s0:s1], sinks, window, scale)
        out[s0:s1] = o_b[0]
        lse[:, s0:s1] = l_b[0]
    return out, lse


def _torch_forward(qd, kd, vd, sinks, window: int, scale: float):
    """The forward as differentiable torch float64 operations: the window
    mask, one sink column per head joined to the softmax and dropped after it
    (page 1: the sink is a logit in the denominator with no value row).
    qd [B,L,Hq,D], kd/vd [B,L,Hkv,D], sinks [Hq]; returns (O [B,L,Hq,D],
    LSE [B,Hq,L])."""
    import torch
    B, L, Hq, D = qd.shape
    Hkv = kd.shape[2]
    kk = kd.repeat_interleave(Hq // Hkv, dim=2)
    vv = vd.repeat_interleave(Hq // Hkv, dim=2)
    # the scale is the float32 value the device receives, widened exactly
    s = float(np.float32(scale)) * torch.einsum("bihd,bjhd->bhij", qd, kk)
    i = torch.arange(L).view(L, 1)
    j = torch.arange(L).view(1, L)
    visible = (j <= i) & (j >= i - int(window) + 1)
    s = s.masked_fill(~visible, float("-inf"))
    full = torch.cat([s, sinks.view(1, Hq, 1, 1).expand(B, Hq, L, 1)], dim=-1)
    lse = torch.logsumexp(full, dim=-1)
    p = torch.exp(full - lse.unsqueeze(-1))[..., :L]
    o = torch.einsum("bhij,bjhd->bihd", p, vv)
    return o, lse


def bwd(q, k, v, sinks, dout, window: int, scale: float):
    """Gradients of the forward: for the loss sum(dout * O), the gradients
    with respect to q, k, v and the sinks, by float64 automatic
    differentiation of ``_torch_forward`` (the definition; page 4 names the
    sink gradient, issue #2969, as computed from the unrounded O).
    q [B,L,Hq,D], k/v [B,L,Hkv,D], dout [B,L,Hq,D] as uint16 bf16 bits,
    sinks [Hq] float32 (finite or -inf).
    Returns (dq, dk, dv, dsinks, O, LSE) float64 numpy arrays."""
    import torch
    q, k, v, dout = _u16(q), _u16(k), _u16(v), _u16(dout)
    qd = torch.from_numpy(_bits_to_f64(q)).requires_grad_()
    kd = torch.from_numpy(_bits_to_f64(k)).requires_grad_()
    vd = torch.from_numpy(_bits_to_f64(v)).requires_grad_()
    sd = torch.from_numpy(np.asarray(sinks, dtype=np.float32).astype(np.float64)).requires_grad_()
    do = torch.from_numpy(_bits_to_f64(dout))
    o, lse = _torch_forward(qd, kd, vd, sd, window, scale)
    (o * do).sum().backward()
    ds = sd.grad if sd.grad is not None else torch.zeros_like(sd)
    ds = torch.nan_to_num(ds, nan=0.0)          # an -inf sink has no gradient
    return (qd.grad.numpy(), kd.grad.numpy(), vd.grad.numpy(), ds.numpy(),
            o.detach().numpy(), lse.detach().numpy())


def max_logit(q, k, window: int, scale: float):
    """The largest pre-softmax logit of every (batch, query head): the maximum
    over rows i and visible keys j in [max(0, i-W+1), i] of scale * <q_i, k_j>
    (kv head h // (Hq/Hkv)), the sink excluded (the flash-attention contributor
    guide's task for issue #2986: one largest logit per batch and head).
    q [B,L,Hq,D], k [B,L,Hkv,D] as uint16 bf16 bits.  Returns [B, Hq] float64
    (-inf where L = 0).  Plain fp64, one key offset of the window at a time."""
    q, k = _u16(q), _u16(k)
    B, L, Hq, D = q.shape
    Hkv = k.shape[2]
    qd = _bits_to_f64(q)
    kd = _bits_to_f64(k)
    group = Hq // Hkv
    out = np.full((B, Hq), -np.inf)
    for h in range(Hq):
        qh = qd[:, :, h, :]                       # [B, L, D]
        kh = kd[:, :, h // group, :]
        for off in range(min(window, L)):         # key j = i - off
            if off >= L:
                break
            s = float(scale) * np.einsum("bld,bld->bl", qh[:, off:], kh[:, :L - off])
            out[:, h] = np.maximum(out[:, h], s.max(axis=1))
    return out


def _bits_to_f64(a: np.ndarray) -> np.ndarray:
    """bf16 bit patterns (uint16) to float64, exactly."""
    return (a.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def fwd_rows(q, k, v, sinks, window: int, scale: float, rows):
    """The forward for selected rows only.  rows: int array [n, 3] of
    (b, i, h).  Returns (out [n, D] float64, lse [n] float64)."""
    q, k, v, sinks = _u16(q), _u16(k), _u16(v), _f32(sinks)
    B, L, Hq, D = q.shape
    Hkv = k.shape[2]
    rows = np.ascontiguousarray(np.asarray(rows, dtype=np.int32).reshape(-1, 3))
    n = rows.shape[0]
    out = np.empty((n, D), np.float64)
    lse = np.empty((n,), np.float64)
    rc = _load().oracle_fwd_rows(_ptr(q), _ptr(k), _ptr(v), _ptr(sinks), B, L, Hq,
                                 Hkv, D, int(window), float(scale), n, _ptr(rows),
                                 _ptr(out), _ptr(lse))
    if rc != 0:
        raise ValueError("oracle_fwd_rows: invalid sizes or rows")
    return out, lse


def decode(q, kcache, vcache, seqlens, sinks, window: int, scale: float):
    """Single-token decode over a contiguous KV cache (see oracle.c).

    q [B,Hq,D]; kcache/vcache [B,Smax,Hkv,D] uint16 bf16 bits; seqlens [B]
    int32; sinks [Hq] float32.  Returns (out [B,Hq,D], lse [B,Hq]) float64."""
    q, kcache, vcache, sinks = _u16(q), _u16(kcache), _u16(vcache), _f32(sinks)
    seqlens = np.ascontiguousarray(np.asarray(seqlens, dtype=np.int32))
    B, Hq, D = q.shape
    _, Smax, Hkv, _ = kcache.shape
    assert kcache.shape == (B, Smax, Hkv, D) and vcache.shape == kcache.shape
    out = np.empty((B, Hq, D), np.float64)
    lse = np.empty((B, Hq), np.float64)
    rc = _load().oracle_decode(_ptr(q), _ptr(kcache), _ptr(vcache), _ptr(seqlens),
                               _ptr(sinks), B, Smax, Hq, Hkv, D, int(window),
                               float(scale), _ptr(out), _ptr(lse))
    if rc != 0:
        raise ValueError("oracle_decode: invalid sizes")
    return out, lse


def decode_paged(q, kpages, vpages, block_table, seqlens, sinks, window: int, scale: float):
    """Single-token decode over a paged KV cache (see oracle.c).

    q [B,Hq,D]; kpages/vpages [NB,P,Hkv,D] uint16 bf16 bits; block_table
    [B,MP] int32 (position t of sequence b is row t % P of page
    block_table[b, t // P]; entries outside [0, NB) are pages of zero rows);
    seqlens [B] int32 in [0, MP*P]; sinks [Hq] float32.
    Returns (out [B,Hq,D], lse [B,Hq]) float64."""
    q, kpages, vpages, sinks = _u16(q), _u16(kpages), _u16(vpages), _f32(sinks)
    block_table = np.ascontiguousarray(np.asarray(block_table, dtype=np.int32))
    seqlens = np.ascontiguousarray(np.asarray(seqlens, dtype=np.int32))
    B, Hq, D = q.shape
    NB, P, Hkv, _ = kpages.shape
    MP = block_table.shape[1]
    assert kpages.shape == (NB, P, Hkv, D) and vpages.shape == kpages.shape
    assert block_table.shape == (B, MP) and seqlens.shape == (B,)
    out = np.empty((B, Hq, D), np.float64)
    lse = np.empty((B, Hq), np.float64)
    rc = _load().oracle_decode_paged(_ptr(q), _ptr(kpages), _ptr(vpages), _ptr(block_table),
                                     _ptr(seqlens), _ptr(sinks), B, NB, P, MP, Hq, Hkv, D,
                                     int(window), float(scale), _ptr(out), _ptr(lse))
    if rc != 0:
        raise ValueError("oracle_decode_paged: invalid sizes")
    return out, lse


def e4m3_to_f64(code: int) -> float:
    """The oracle's FP8 e4m3 decoder (see oracle.c) for one byte."""
    return float(_load().oracle_e4m3_to_f64(int(code) & 0xFF))


def decode_fp8(q, kcache, vcache, k_descale, v_descale, seqlens, sinks, window: int,
               scale: float):
    """Single-token decode over an FP8 e4m3 KV cache (see oracle.c).

    q [B,Hq,D] uint16 bf16 bits; kcache/vcache [B,Smax,Hkv,D] uint8 e4m3
    codes; k_descale/v_descale [Hkv] float32 (key row = k_descale[hk] *
    e4m3(row), value row likewise); seqlens [B] int32; sinks [Hq] float32.
    Returns (out [B,Hq,D], lse [B,Hq]) float64."""
    q, sinks = _u16(q), _f32(sinks)
    kcache = np.ascontiguousarray(kcache, dtype=np.uint8)
    vcache = np.ascontiguousarray(vcache, dtype=np.uint8)
    k_descale, v_descale = _f32(k_descale), _f32(v_descale)
    seqlens = np.ascontiguousarray(np.asarray(seqlens, dtype=np.int32))
    B, Hq, D = q.shape
    _, Smax, Hkv, _ = kcache.shape
    assert kcache.shape == (B, Smax, Hkv, D) and vcache.shape == kcache.shape
    assert k_descale.shape == (Hkv,) and v_descale.shape == (Hkv,)
    out = np.empty((B, Hq, D), np.float64)
    lse = np.empty((B, Hq), np.float64)
    rc = _load().oracle_decode_fp8(_ptr(q), _ptr(kcache), _ptr(vcache), _ptr(k_descale),
                                   _ptr(v_descale), _ptr(seqlens), _ptr(sinks), B, Smax, Hq,
                                   Hkv, D, int(window), float(scale), _ptr(out), _ptr(lse))
    if rc != 0:
        raise ValueError("oracle_decode_fp8: invalid sizes")
    return out, lse


def split_partial(q_row, k_rows, v_rows, lo: int, hi: int, scale: float):
    """Split-KV step 1 (page 5, section 3): partial softmax of one query row
    over keys lo..hi (inclusive) of k_rows/v_rows [S, D], no sink.
    Returns (o_s [D], lse_s)."""
    q_row, k_rows, v_rows = _u16(q_row), _u16(k_rows), _u16(v_rows)
    D = q_row.shape[-1]
    o = np.empty((D,), np.float64)
    lse = np.empty((1,), np.float64)
    rc = _load().oracle_split_partial(_ptr(q_row), _ptr(k_rows), _ptr(v_rows),
                                      k_rows.shape[-1], int(lo), int(hi), D,
                                      float(scale), _ptr(o), _ptr(lse))
    if rc != 0:
        raise ValueError("oracle_split_partial: invalid range")
    return o, float(lse[0])


def combine(lse_s, o_s, sink: float):
    """Split-KV step 2 (page 5, section 3): log-sum-exp merge of the splits
    that exist, in order, with the sink once.  lse_s [n], o_s [n, D].
    Returns (out [D], lse)."""
    lse_s = np.ascontiguousarray(np.asarray(lse_s, dtype=np.float64))
    o_s = np.ascontiguousarray(np.asarray(o_s, dtype=np.float64))
    n = lse_s.shape[0]
    D = o_s.shape[-1]
    out = np.empty((D,), np.float64)
    lse = np.empty((1,), np.float64)
    rc = _load().oracle_combine(n, _ptr(lse_s), _ptr(o_s), D, float(sink),
                                _ptr(out), _ptr(lse))
    if rc != 0:
        raise ValueError("oracle_combine: invalid sizes")
    return out, float(lse[0])
