"""Runs a few launches of one operation on a chosen workload, for profiler
captures (Nsight Compute) of a single kernel on a bounded device footprint.

  python -m sliding_window_learned_b200.ncu_driver --op fwd --workload prefill --launches 3
  python -m sliding_window_learned_b200.ncu_driver --op decode --workload decode-small --launches 3
  python -m sliding_window_learned_b200.ncu_driver --op bwd --workload prefill --launches 2

(--op bwd runs one forward for O and LSE, then the backward passes; --op
decode_fp8 quantises the workload's cache to e4m3 per kv head first; --op
decode_paged copies the cache into pools of --page positions at random pool
positions, addressed through a block table.)

It prints no timings (numbers taken under a profiler are not measurements);
it exits non-zero if the device reports an error.
"""
from __future__ import annotations

import argparse
import sys

import torch

from . import abi, build, inputs

WORKLOADS = {
    "tiny": inputs.TINY,
    "prefill": inputs.PREFILL,
    "long-causal": inputs.LONG_CAUSAL,
    "stress": inputs.STRESS,
    "decode": inputs.DECODE,
    # same length distribution as the decode workload, 8 sequences (~1 GB of cache)
    "decode-small": inputs.Decode("decode-small B8 Hq32 Hkv4 D128 n~U[4096,131072]", 8, 32, 4,
                                  128, 131072, 4096, 131072, 131072),
}


def main(argv=None) -> int:
    ap = argparse.ArgumentParser()
    ap.add_argument("--op", choices=["fwd", "decode", "bwd", "decode_fp8", "decode_paged"], required=True)
    ap.add_argument("--workload", choices=sorted(WORKLOADS), required=True)
    ap.add_argument("--launches", type=int, default=3)
    ap.add_argument("--page", type=int, default=16, help="positions per page (--op decode_paged)")
    a = ap.parse_args(argv)
    build.build()
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    cfg = WORKLOADS[a.workload]
    if a.op in ("fwd", "bwd"):
        if not isinstance(cfg, inputs.Prefill):
            raise SystemExit(f"{a.op} needs a prefill workload")
        x = inputs.make_prefill(cfg, seed=0, device=dev)
        out = torch.empty_like(x["q"])
        lse = torch.empty(cfg.B, cfg.Hq, cfg.L, dtype=torch.float32, device=dev)
        if a.op == "fwd":
            for _ in range(a.launches):
                abi.attn_sink_fwd(x["q"], x["k"], x["v"], x["sinks"], cfg.W, cfg.scale, out, lse)
        else:
            abi.attn_sink_fwd(x["q"], x["k"], x["v"], x["sinks"], cfg.W, cfg.scale, out, lse)
            g = torch.Generator(device=dev).manual_seed(1)
            dout = torch.randn(x["q"].shape, device=dev, generator=g).to(torch.bfloat16)
            dq, dk, dv = torch.empty_like(x["q"]), torch.empty_like(x["k"]), torch.empty_like(x["v"])
            dsink = torch.empty(cfg.Hq, dtype=torch.float32, device=dev)
            for _ in range(a.launches):
                abi.attn_sink_bwd(x["q"], x["k"], x["v"], out, lse, dout, x["sinks"], cfg.W, cfg.scale,
                                  dq, dk, dv, dsink)
    else:
        if not isinstance(cfg, inputs.Decode):
            raise SystemExit("decode needs a decode workload")
        y = inputs.make_decode(cfg, seed=0, device=dev)
        out = torch.empty_like(y["q"])
        if a.op == "decode_fp8":
            kd = torch.empty(cfg.Hkv, device=dev)
            vd = torch.empty(cfg.Hkv, device=dev)
            k8 = torch.empty(y["kcache"].shape, dtype=torch.float8_e4m3fn, device=dev)
            v8 = torch.empty_like(k8)
            for hk in range(cfg.Hkv):
                for src, dst, d in ((y["kcache"], k8, kd), (y["vcache"], v8, vd)):
                    xs = src[:, :, hk].float()
                    d[hk] = torch.nan_to_num(xs, nan=0.0).abs().amax() / 448.0
                    dst[:, :, hk] = (xs / d[hk]).to(torch.float8_e4m3fn)
            for _ in range(a.launches):
                abi.attn_sink_decode_fp8(y["q"], k8, v8, kd, vd, y["seqlens"], y["sinks"], cfg.W, cfg.scale, out)
        elif a.op == "decode_paged":
            P = a.page
            n_pages = cfg.B * (cfg.Smax // P)
            perm = torch.randperm(n_pages, generator=torch.Generator(device=dev).manual_seed(0), device=dev)
            kpool = torch.empty((n_pages, P, cfg.Hkv, cfg.D), dtype=torch.bfloat16, device=dev)
            kpool[perm] = y["kcache"].reshape(n_pages, P, cfg.Hkv, cfg.D)
            vpool = torch.empty_like(kpool)
            vpool[perm] = y["vcache"].reshape(n_pages, P, cfg.Hkv, cfg.D)
            table = perm.reshape(cfg.B, cfg.Smax // P).to(torch.int32)
            del y["kcache"], y["vcache"]
            for _ in range(a.launches):
                abi.attn_sink_decode_paged(y["q"], kpool, vpool, table, y["seqlens"], y["sinks"], cfg.W,
                                           cfg.scale, out)
        else:
            for _ in range(a.launches):
                abi.attn_sink_decode(y["q"], y["kcache"], y["vcache"], y["seqlens"], y["sinks"],
                                     cfg.W, cfg.scale, out)
    torch.cuda.synchronize()
    rc = abi.attn_sink_get_status()
    print("ok" if rc == 0 else f"device status {rc}")
    return 0 if rc == 0 else 1


if __name__ == "__main__":
    sys.exit(main())
