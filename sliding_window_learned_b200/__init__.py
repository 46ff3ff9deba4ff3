"""B200-native sliding-window attention with a learned per-head sink.

The compute path is the CUDA library ``libattnsink.so`` (C ABI in
``include/attnsink.h``); this package holds its sources (``csrc/``), its build
step (``build.py``), a thin ctypes binding (``abi.py``) and the seeded input
generators (``inputs.py``).  Importing the package does not load the library;
the first call does, and fails loudly if it is not built.
"""
from .abi import (AttnSinkError, attn_sink_bwd, attn_sink_decode, attn_sink_decode_chunked,
                  attn_sink_decode_fp8, attn_sink_decode_noalloc, attn_sink_decode_paged, attn_sink_fwd, attn_sink_fwd_max_logit, attn_sink_fwd_varlen,
                  attn_sink_fail_workspace_allocs, attn_sink_fwd_cudacore, attn_sink_get_status,
                  attn_sink_last_error, attn_sink_set_wait_limit_ns, attn_sink_strerror, decode, fwd)

__all__ = ["AttnSinkError", "attn_sink_bwd", "attn_sink_fwd", "attn_sink_fwd_max_logit", "attn_sink_fwd_varlen", "attn_sink_fwd_cudacore", "attn_sink_decode",
           "attn_sink_decode_chunked", "attn_sink_decode_paged", "attn_sink_decode_fp8", "attn_sink_decode_noalloc",
           "attn_sink_get_status", "attn_sink_strerror", "attn_sink_set_wait_limit_ns",
           "attn_sink_fail_workspace_allocs",
           "attn_sink_last_error", "fwd", "decode"]
