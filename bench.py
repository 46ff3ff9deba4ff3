"""Benchmark of the hot path: prefill forward + split-KV decode.

One step = one attn_sink_fwd over the prefill workload (B2 Hq32 Hkv4 L4096
D128 W513) followed by one attn_sink_decode over the decode workload (B64
Hq32 Hkv4 D128, lengths ~ U[4096, 131072]), both on synthetic seeded inputs
already resident in HBM.  Between steps a 256 MB buffer is written to flush
L2 (the prefill inputs are smaller than L2; the decode cache is ~17 GB).

`value` is useful prefill TFLOP/s (window-visible pairs only), summed over
ranks, from CUDA events around each prefill launch; the decode figure (HBM
GB/s of algorithmic bytes) is reported beside it, and after the timed steps
the same decode over a paged copy of its cache (256-position pages at random
pool positions, attn_sink_decode_paged) is timed as `decode_paged`, the decode
over the cache quantised to e4m3 (attn_sink_decode_fp8) as `decode_fp8`, the
bf16 and e4m3 caches side by side on two more decode shapes (16 query heads per
kv head; head dim 256) as `decode_shapes`, the forward over a seeded mix of 24 packed sequences (attn_sink_fwd_varlen) as
`fwd_varlen`, and the backward pass on the prefill workload (attn_sink_bwd) as
`bwd`.  `workloads` times attn_sink_fwd on each prefill workload on its own
(tiny, prefill, long causal, sink stress), each with its own clock record.
`--impl reference` times
the fp64 CPU oracle on a bounded sample of the same prefill workload.

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
       python bench.py --profile OP --workload NAME [--launches N]   (profiler driver)
(N > 1: launch under torchrun; each rank runs its own copy of the workloads.)
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from sliding_window_learned_b200 import inputs  # noqa: E402

METRIC = "attn fwd TFLOP/s (useful) & % bf16 tensor peak; decode HBM GB/s & % of peak"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
NOMINAL_HBM_GBS = 8000.0


def useful_fwd_flops(cfg) -> float:
    """4*D per visible (query, key) pair: QK^T and PV, window-visible pairs only."""
    L, W = cfg.L, cfg.W
    i = np.arange(L, dtype=np.int64)
    pairs = int(np.minimum(i + 1, W).sum())
    return 4.0 * cfg.D * cfg.B * cfg.Hq * pairs


def decode_bytes(cfg, seqlens) -> float:
    """K and V rows of the visible keys of every (sequence, kv head), plus q and out."""
    n = np.asarray(seqlens, dtype=np.int64)
    vis = n - np.maximum(0, n - cfg.W)
    kv = int(vis.sum()) * cfg.Hkv * cfg.D * 2 * 2
    return float(kv + 2 * cfg.B * cfg.Hq * cfg.D * 2)


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def profiled_traffic(kernel: str, sources: list[str]):
    """DRAM bytes per launch from the committed ncu summary, if it was taken on
    the current source of the kernel; otherwise None."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f).get(kernel)
    if not d:
        return None
    h = hashlib.sha256()
    for s in sources:
        with open(os.path.join(ROOT, s), "rb") as f:
            h.update(f.read())
    if h.hexdigest() != d.get("src_sha256"):
        return None
    return d.get("dram_bytes_per_launch")


class ClockSampler:
    """SM clock, power and clock-event reasons sampled during a timed region.

    NVML is polled from a background thread about once a millisecond (the
    device is found by the PCI bus id torch reports, so CUDA_VISIBLE_DEVICES
    does not matter); without NVML, nvidia-smi is sampled every 50 ms.  Only
    readings are taken: no clock, power or other setting is changed."""

    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown"}
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.idx = device_index
        self.proc = None
        self.thread = None
        self.nv = None
        self.handle = None
        self.samples = []
        try:
            import pynvml
            import torch
            pynvml.nvmlInit()
            pr = torch.cuda.get_device_properties(device_index)
            bus = f"{pr.pci_domain_id:08x}:{pr.pci_bus_id:02x}:{pr.pci_device_id:02x}.0"
            self.handle = pynvml.nvmlDeviceGetHandleByPciBusId(bus.encode())
            self.nv = pynvml
        except Exception:  # noqa: BLE001 - any NVML problem: fall back to nvidia-smi
            self.nv = None

    def _poll(self):
        nv, h = self.nv, self.handle
        while not self._stop:
            try:
                sm = nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)
                pw = nv.nvmlDeviceGetPowerUsage(h) / 1000.0
                rs = nv.nvmlDeviceGetCurrentClocksEventReasons(h)
                self.samples.append((float(sm), pw, int(rs)))
            except Exception:  # noqa: BLE001
                pass
            time.sleep(0.001)

    def start(self):
        self.samples = []
        if self.nv is not None:
            import threading
            self._stop = False
            self.thread = threading.Thread(target=self._poll, daemon=True)
            self.thread.start()
            return
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-i", str(self.idx), "-lms", "50"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (OSError, ValueError):
            self.proc = None

    def stop(self):
        if self.thread is not None:
            self._stop = True
            self.thread.join()
            self.thread = None
            if not self.samples:
                return None
            mx = float(self.nv.nvmlDeviceGetMaxClockInfo(self.handle, self.nv.NVML_CLOCK_SM))
            reasons = sorted({nm for _, _, r in self.samples for bit, nm in self.REASONS.items() if r & bit})
            sm = [x for x, _, _ in self.samples]
            return {"sm_mhz": statistics.median(sm), "sm_min_mhz": min(sm), "sm_max_mhz": mx,
                    "power_w_max": round(max(p for _, p, _ in self.samples), 1),
                    "samples": len(sm), "reasons": reasons, "source": "nvml, ~1 ms"}
        if self.proc is None:
            return None
        time.sleep(0.25)
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.strip().splitlines():
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 8:
                continue
            try:
                sm.append(float(parts[0]))
                mx = float(parts[1])
            except ValueError:
                continue
            for nm, val in zip(names, parts[4:8]):
                if val.lower() == "active":
                    reasons.add(nm)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "samples": len(sm),
                "reasons": sorted(reasons), "source": "nvidia-smi, 50 ms"}


def page_cache(y, cfg, page, seed, dev):
    """The decode workload's cache copied into pools of `page` positions at
    random pool positions; returns (kpool, vpool, block_table)."""
    import torch
    n_pages = cfg.B * (cfg.Smax // page)
    perm = torch.randperm(n_pages, generator=torch.Generator(device=dev).manual_seed(seed), device=dev)
    kpool = torch.empty((n_pages, page, cfg.Hkv, cfg.D), dtype=torch.bfloat16, device=dev)
    kpool[perm] = y["kcache"].reshape(n_pages, page, cfg.Hkv, cfg.D)
    vpool = torch.empty_like(kpool)
    vpool[perm] = y["vcache"].reshape(n_pages, page, cfg.Hkv, cfg.D)
    return kpool, vpool, perm.reshape(cfg.B, cfg.Smax // page).to(torch.int32)


def quantise_e4m3(y, cfg, dev):
    """The decode workload's cache quantised to e4m3 with one descale per kv
    head (max |x| / 448); returns (k8, v8, k_descale, v_descale)."""
    import torch
    kd = torch.empty(cfg.Hkv, device=dev)
    vd = torch.empty(cfg.Hkv, device=dev)
    k8 = torch.empty(y["kcache"].shape, dtype=torch.float8_e4m3fn, device=dev)
    v8 = torch.empty_like(k8)
    for hk in range(cfg.Hkv):
        for src, dst, d in ((y["kcache"], k8, kd), (y["vcache"], v8, vd)):
            xs = src[:, :, hk].float()
            d[hk] = torch.nan_to_num(xs, nan=0.0).abs().amax() / 448.0
            dst[:, :, hk] = (xs / d[hk]).to(torch.float8_e4m3fn)
            del xs
    return k8, v8, kd, vd


def forward_leg_report(cfg, launches, seconds, clk, nsets, world, peak, peak_src):
    """One prefill workload timed on its own: useful TFLOP/s over all ranks,
    time per launch, fraction of the measured bf16 peak, and its clocks."""
    flops = useful_fwd_flops(cfg)
    per = seconds / launches
    return {"workload": cfg.name, "value": round(aggregate_rate(launches * flops, world, seconds) / 1e12, 3),
            "unit": "TFLOP/s", "launches": launches, "ms_per_call": round(per * 1e3, 5),
            "flops_per_launch": flops,
            "frac": round(flops / per / 1e12 / peak, 4), "peak": peak, "peak_source": f"{peak_src} bf16 (burst)",
            "l2": ("flushed before each launch (per-launch events)" if cfg.L <= 1024 else
                   f"back-to-back launches over {nsets} input set(s), each launch's q, k, v, O "
                   "(plus the other set's) larger than L2"),
            "clocks": clk}


# --------------------------------------------------------------- our arm
def max_over_ranks(values, world, device):
    """Element-wise maximum of per-rank timings over all ranks (every rank
    calls it, in the same order); a no-op for one rank."""
    if world <= 1:
        return list(values)
    import torch
    import torch.distributed as dist
    t = torch.tensor(list(values), dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def aggregate_rate(work_per_rank, world, seconds):
    """Whole-job rate: every rank does the same work (weak scaling), timed as
    the slowest rank's time."""
    return world * work_per_rank / seconds


def run_ours(args, rank, world, local_rank):
    import torch
    import torch.distributed as dist

    import sliding_window_learned_b200 as swl
    from sliding_window_learned_b200 import build as swl_build

    if rank == 0:
        swl_build.build()
    if world > 1:
        dist.barrier()
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream(dev)

    # ---- workloads (per rank; weak scaling) ----
    pcfg, dcfg = inputs.PREFILL, inputs.DECODE
    x = inputs.make_prefill(pcfg, seed=rank)
    q, k, v = x["q"].to(dev), x["k"].to(dev), x["v"].to(dev)
    sinks = x["sinks"].to(dev)
    out = torch.empty_like(q)
    lse = torch.empty(pcfg.B, pcfg.Hq, pcfg.L, dtype=torch.float32, device=dev)
    y = inputs.make_decode(dcfg, seed=rank, device=dev)
    dout = torch.empty_like(y["q"])
    flush = torch.empty(256 * 1024 * 1024 // 4, dtype=torch.float32, device=dev)
    fwd_flops = useful_fwd_flops(pcfg)
    dbytes = decode_bytes(dcfg, y["seqlens"].cpu().numpy())

    def fwd():
        swl.attn_sink_fwd(q, k, v, sinks, pcfg.W, pcfg.scale, out, lse, stream)

    def dec():
        swl.attn_sink_decode(y["q"], y["kcache"], y["vcache"], y["seqlens"], y["sinks"], dcfg.W,
                             dcfg.scale, dout, stream)

    for _ in range(max(3, args.warmup)):
        flush.fill_(1.0)
        fwd()
        dec()
    torch.cuda.synchronize()
    if swl.attn_sink_get_status() != 0:
        raise RuntimeError("device status error during warm-up")

    K = args.steps
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(K)]
    ev_all = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
    clocks = ClockSampler(local_rank)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    clocks.start()
    ev_all[0].record(stream)
    for s in range(K):
        flush.fill_(1.0)
        ev[s][0].record(stream)
        fwd()
        ev[s][1].record(stream)
        ev[s][2].record(stream)
        dec()
        ev[s][3].record(stream)
    ev_all[1].record(stream)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    clk = clocks.stop()
    if swl.attn_sink_get_status() != 0:
        raise RuntimeError("device status error in the timed region")
    t_fwd = sum(e[0].elapsed_time(e[1]) for e in ev) / 1e3       # s, K launches
    t_dec = sum(e[2].elapsed_time(e[3]) for e in ev) / 1e3
    t_all = ev_all[0].elapsed_time(ev_all[1]) / 1e3

    # ---- end to end through the public API: pinned host -> device -> host ----
    hq, hk, hv = x["q"].pin_memory(), x["k"].pin_memory(), x["v"].pin_memory()
    hs = x["sinks"].pin_memory()
    ho, hl = torch.empty_like(hq).pin_memory(), torch.empty(lse.shape, dtype=torch.float32).pin_memory()
    h2d = sum(t.numel() * t.element_size() for t in (hq, hk, hv, hs))
    d2h = ho.numel() * ho.element_size() + hl.numel() * hl.element_size()
    Ke = max(3, min(K, 20))

    def e2e_step():
        q.copy_(hq, non_blocking=True)
        k.copy_(hk, non_blocking=True)
        v.copy_(hv, non_blocking=True)
        sinks.copy_(hs, non_blocking=True)
        fwd()
        ho.copy_(out, non_blocking=True)
        hl.copy_(lse, non_blocking=True)

    e2e_step()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(Ke):
        e2e_step()
    e1.record(stream)
    torch.cuda.synchronize()
    t_e2e_serial = e0.elapsed_time(e1) / 1e3
    ho_serial = ho.clone()

    # The same calls as a pipeline, as a serving loop would run them: step
    # i+1's inputs are copied in on one stream (one copy engine) while step i
    # computes on the launching stream and step i-1's O, LSE are copied out
    # on another (the other engine), with two sets of device buffers.  Every
    # step still copies its inputs in and its outputs out inside the timed
    # region.
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    sets = [dict(q=torch.empty_like(q), k=torch.empty_like(k), v=torch.empty_like(v),
                 s=torch.empty_like(sinks), o=torch.empty_like(out), l=torch.empty_like(lse))
            for _ in range(2)]
    ev_in = [torch.cuda.Event() for _ in range(2)]     # set j's inputs landed
    ev_fwd = [torch.cuda.Event() for _ in range(2)]    # the forward on set j finished
    ev_out = [torch.cuda.Event() for _ in range(2)]    # set j's outputs copied out

    def e2e_pipelined(n):
        for i in range(n):
            j = i & 1
            b = sets[j]
            if i >= 2:
                s_in.wait_event(ev_fwd[j])             # set j's inputs no longer read
            with torch.cuda.stream(s_in):
                b["q"].copy_(hq, non_blocking=True)
                b["k"].copy_(hk, non_blocking=True)
                b["v"].copy_(hv, non_blocking=True)
                b["s"].copy_(hs, non_blocking=True)
            ev_in[j].record(s_in)
            stream.wait_event(ev_in[j])
            if i >= 2:
                stream.wait_event(ev_out[j])           # set j's outputs already copied out
            swl.attn_sink_fwd(b["q"], b["k"], b["v"], b["s"], pcfg.W, pcfg.scale, b["o"], b["l"], stream)
            ev_fwd[j].record(stream)
            s_out.wait_event(ev_fwd[j])
            with torch.cuda.stream(s_out):
                ho.copy_(b["o"], non_blocking=True)
                hl.copy_(b["l"], non_blocking=True)
            ev_out[j].record(s_out)

    e2e_pipelined(2)
    torch.cuda.synchronize()
    e0.record(stream)
    s_in.wait_event(e0)
    e2e_pipelined(Ke)
    stream.wait_event(ev_out[(Ke - 1) & 1])
    e1.record(stream)
    torch.cuda.synchronize()
    t_e2e = e0.elapsed_time(e1) / 1e3
    if not torch.equal(ho, ho_serial):
        raise RuntimeError("pipelined end-to-end output differs from the serial one")
    del sets

    # ---- the same decode over a paged cache (256-position pages at random
    # pool positions, addressed through a block table) ----
    page = 256
    kpool, vpool, table = page_cache(y, dcfg, page, rank, dev)

    def dec_paged():
        swl.attn_sink_decode_paged(y["q"], kpool, vpool, table, y["seqlens"], y["sinks"], dcfg.W,
                                   dcfg.scale, dout, stream)

    Kp = max(3, min(K, 50))
    for _ in range(3):
        dec_paged()
    torch.cuda.synchronize()
    e0.record(stream)
    for _ in range(Kp):
        dec_paged()
    e1.record(stream)
    torch.cuda.synchronize()
    if swl.attn_sink_get_status() != 0:
        raise RuntimeError("device status error in the paged decode")
    t_paged = e0.elapsed_time(e1) / 1e3
    del kpool, vpool, table

    # ---- the same decode over its cache quantised to FP8 e4m3 per kv head ----
    k8, v8, kdesc, vdesc = quantise_e4m3(y, dcfg, dev)

    def dec_fp8():
        swl.attn_sink_decode_fp8(y["q"], k8, v8, kdesc, vdesc, y["seqlens"], y["sinks"], dcfg.W,
                                 dcfg.scale, dout, stream)

    for _ in range(3):
        dec_fp8()
    torch.cuda.synchronize()
    e0.record(stream)
    for _ in range(Kp):
        dec_fp8()
    e1.record(stream)
    torch.cuda.synchronize()
    if swl.attn_sink_get_status() != 0:
        raise RuntimeError("device status error in the FP8 decode")
    t_fp8 = e0.elapsed_time(e1) / 1e3
    dbytes8 = (dbytes - 2 * dcfg.B * dcfg.Hq * dcfg.D * 2) // 2 + 2 * dcfg.B * dcfg.Hq * dcfg.D * 2
    del k8, v8

    # ---- two more decode shapes, bf16 and FP8 caches side by side ----
    shape_times = []
    shape_bytes = []
    for si, scfg in enumerate((inputs.DECODE_G16, inputs.DECODE_D256)):
        ys = inputs.make_decode(scfg, seed=2000 + 10 * si + rank, device=dev)
        sout = torch.empty_like(ys["q"])
        s8 = quantise_e4m3(ys, scfg, dev)
        sl = ys["seqlens"].cpu().numpy().astype(np.int64)
        qo_bytes = 2 * scfg.B * scfg.Hq * scfg.D * 2
        b16 = int(sl.sum()) * scfg.Hkv * scfg.D * 2 * 2 + qo_bytes
        shape_bytes.append((scfg.name, b16, (b16 - qo_bytes) // 2 + qo_bytes))
        calls = (lambda: swl.attn_sink_decode(ys["q"], ys["kcache"], ys["vcache"], ys["seqlens"], ys["sinks"],
                                              scfg.W, scfg.scale, sout, stream),
                 lambda: swl.attn_sink_decode_fp8(ys["q"], s8[0], s8[1], s8[2], s8[3], ys["seqlens"], ys["sinks"],
                                                  scfg.W, scfg.scale, sout, stream))
        for call in calls:
            for _ in range(3):
                call()
            torch.cuda.synchronize()
            e0.record(stream)
            for _ in range(Kp):
                call()
            e1.record(stream)
            torch.cuda.synchronize()
            if swl.attn_sink_get_status() != 0:
                raise RuntimeError(f"device status error in the {scfg.name} decode")
            shape_times.append(e0.elapsed_time(e1) / 1e3)
        del ys, sout, s8
        torch.cuda.empty_cache()
    shape_times = max_over_ranks(shape_times, world, dev)

    # ---- the forward over packed variable-length sequences: a seeded mix of
    # 24 sequences of U[1, 4096] tokens at the prefill workload's heads ----
    vl_rng = np.random.default_rng(1000 + rank)
    vl_lens = [int(n) for n in vl_rng.integers(1, 4097, size=24)]
    vl_T = sum(vl_lens)
    vl_gen = torch.Generator(device=dev).manual_seed(rank)
    vq = torch.randn(vl_T, pcfg.Hq, pcfg.D, device=dev, generator=vl_gen).bfloat16()
    vk = torch.randn(vl_T, pcfg.Hkv, pcfg.D, device=dev, generator=vl_gen).bfloat16()
    vv = torch.randn(vl_T, pcfg.Hkv, pcfg.D, device=dev, generator=vl_gen).bfloat16()
    vcu = torch.tensor(np.concatenate([[0], np.cumsum(vl_lens)]), dtype=torch.int32, device=dev)
    vout = torch.empty_like(vq)
    vlse = torch.empty(pcfg.Hq, vl_T, dtype=torch.float32, device=dev)
    vl_flops = sum(4.0 * pcfg.D * pcfg.Hq * float(np.minimum(np.arange(n) + 1, pcfg.W).sum())
                   for n in vl_lens)

    def fwd_varlen():
        swl.attn_sink_fwd_varlen(vq, vk, vv, vcu, max(vl_lens), sinks, pcfg.W, pcfg.scale, vout, vlse,
                                 stream)

    Kv = max(3, min(K, 50))
    for _ in range(3):
        fwd_varlen()
    torch.cuda.synchronize()
    t_varlen = 0.0
    for _ in range(Kv):
        flush.fill_(1.0)
        e0.record(stream)
        fwd_varlen()
        e1.record(stream)
        torch.cuda.synchronize()
        t_varlen += e0.elapsed_time(e1) / 1e3
    if swl.attn_sink_get_status() != 0:
        raise RuntimeError("device status error in the packed forward")
    del vq, vk, vv, vout, vlse

    # ---- the backward pass on the prefill workload: O and LSE from the
    # forward above, a seeded N(0, 1) upstream gradient ----
    bw_gen = torch.Generator(device=dev).manual_seed(2000 + rank)
    bdo = torch.randn(q.shape, device=dev, generator=bw_gen).bfloat16()
    bdq, bdk, bdv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    bds = torch.empty(pcfg.Hq, dtype=torch.float32, device=dev)
    fwd()

    def bwd():
        swl.attn_sink_bwd(q, k, v, out, lse, bdo, sinks, pcfg.W, pcfg.scale, bdq, bdk, bdv, bds, stream)

    Kb = max(3, min(K, 30))
    for _ in range(3):
        bwd()
    torch.cuda.synchronize()
    t_bwd = 0.0
    for _ in range(Kb):
        flush.fill_(1.0)
        e0.record(stream)
        bwd()
        e1.record(stream)
        torch.cuda.synchronize()
        t_bwd += e0.elapsed_time(e1) / 1e3
    if swl.attn_sink_get_status() != 0:
        raise RuntimeError("device status error in the backward pass")
    del bdo, bdq, bdk, bdv

    # ---- every prefill workload on its own: back-to-back launches with
    # their own clock record.  Two input sets alternate when one set (q, k, v,
    # O) is smaller than twice L2, so that a launch never finds its inputs left
    # in L2 by the previous launch; the tiny workload (launch-bound) is timed
    # per launch with L2 flushed before each. ----
    def forward_leg(cfg, launches, seed):
        one = (cfg.B * cfg.L * (2 * cfg.Hq + 2 * cfg.Hkv) * cfg.D * 2)
        nsets = 1 if one >= 256 * 1024 * 1024 else 2
        sets = []
        for si in range(nsets):
            xs = inputs.make_prefill(cfg, seed=seed + si)
            sets.append((xs["q"].to(dev), xs["k"].to(dev), xs["v"].to(dev), xs["sinks"].to(dev),
                         torch.empty(xs["q"].shape, dtype=torch.bfloat16, device=dev),
                         torch.empty(cfg.B, cfg.Hq, cfg.L, dtype=torch.float32, device=dev)))
            del xs

        def call(i):
            a = sets[i % nsets]
            swl.attn_sink_fwd(a[0], a[1], a[2], a[3], cfg.W, cfg.scale, a[4], a[5], stream)

        for i in range(5):
            call(i)
        torch.cuda.synchronize()
        per_launch = cfg.L <= 1024
        sampler = ClockSampler(local_rank)
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        sampler.start()
        if per_launch:
            tl = 0.0
            evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                   for _ in range(launches)]
            for i in range(launches):
                flush.fill_(1.0)
                evs[i][0].record(stream)
                call(i)
                evs[i][1].record(stream)
            torch.cuda.synchronize()
            tl = sum(a.elapsed_time(b) for a, b in evs) / 1e3
        else:
            e0.record(stream)
            for i in range(launches):
                call(i)
            e1.record(stream)
            torch.cuda.synchronize()
            tl = e0.elapsed_time(e1) / 1e3
        clk_leg = sampler.stop()
        if swl.attn_sink_get_status() != 0:
            raise RuntimeError(f"device status error in the {cfg.name} leg")
        del sets
        return tl, clk_leg, nsets

    leg_specs = [("tiny", inputs.TINY, 200), ("prefill", inputs.PREFILL, 1000),
                 ("long_causal", inputs.LONG_CAUSAL, 100), ("stress", inputs.STRESS, 1000)]
    leg_raw = {}
    for nm, cfg_l, n_l in leg_specs:
        leg_raw[nm] = (cfg_l, n_l) + forward_leg(cfg_l, n_l, 3000 + 10 * rank)
    leg_times = max_over_ranks([leg_raw[nm][2] for nm, _, _ in leg_specs], world, dev)

    # ---- max over ranks ----
    t_fwd, t_dec, t_all, t_e2e, t_e2e_serial, t_paged, t_varlen, t_fp8, t_bwd = max_over_ranks(
        [t_fwd, t_dec, t_all, t_e2e, t_e2e_serial, t_paged, t_varlen, t_fp8, t_bwd], world, dev)

    if rank != 0:
        return
    peaks, peak_src = load_peaks()
    bf16_peak = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    hbm_peak = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
    fwd_tflops = aggregate_rate(K * fwd_flops, world, t_fwd) / 1e12
    per_launch_fwd = t_fwd / K
    per_launch_dec = t_dec / K
    achieved_fwd = fwd_flops / per_launch_fwd / 1e12
    achieved_dec = dbytes / per_launch_dec / 1e9
    dec_gbs = aggregate_rate(K * dbytes, world, t_dec) / 1e9
    line = {
        "metric": METRIC,
        "value": round(fwd_tflops, 3),
        "unit": "TFLOP/s",
        "n_gpus": world,
        "steps": K,
        "warmup": max(3, args.warmup),
        "ms_per_step": round((t_fwd + t_dec) / K * 1e3, 4),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic (seeded; torch generator, seed = rank)",
        "config": {"workload": inputs.PREFILL.name, "decode_workload": inputs.DECODE.name,
                   "parallelism": f"replicas{world}", "l2": "flushed between steps (256 MB write)"},
        "roofline": {"kernel": "fwd_tc_kernel<128,64,1>", "bound": "tensor",
                     "achieved": round(achieved_fwd, 2), "peak": bf16_peak, "unit": "TFLOP/s",
                     "frac": round(achieved_fwd / bf16_peak, 4),
                     "peak_source": f"{peak_src} bf16 (burst)",
                     "traffic": profiled_traffic("fwd_tc", ["sliding_window_learned_b200/csrc/fwd_tc.cu",
                                                            "sliding_window_learned_b200/csrc/ptx.cuh"]),
                     "flops_per_launch": fwd_flops, "ms_per_launch": round(per_launch_fwd * 1e3, 5)},
        "decode": {"value": round(dec_gbs, 2), "unit": "GB/s", "ms_per_call": round(per_launch_dec * 1e3, 4),
                   "bytes_per_call": dbytes,
                   "roofline": {"kernel": "plan + split + combine", "bound": "hbm",
                                "achieved": round(achieved_dec, 2), "peak": hbm_peak, "unit": "GB/s",
                                "frac": round(achieved_dec / hbm_peak, 4),
                                "peak_source": f"{peak_src} copy bandwidth (read + write)",
                                "frac_of_nominal": round(achieved_dec / NOMINAL_HBM_GBS, 4),
                                "note": "the decode only reads; the copy benchmark's read+write "
                                        "figure can be exceeded, so frac_of_nominal (8 TB/s) is "
                                        "given beside it",
                                "traffic": profiled_traffic("decode_split", [
                                    "sliding_window_learned_b200/csrc/decode.cu",
                                    "sliding_window_learned_b200/csrc/ptx.cuh"])}},
        "decode_paged": {"value": round(aggregate_rate(Kp * dbytes, world, t_paged) / 1e9, 2), "unit": "GB/s",
                         "page": page, "ms_per_call": round(t_paged / Kp * 1e3, 4),
                         "frac": round(dbytes / (t_paged / Kp) / 1e9 / hbm_peak, 4),
                         "what": "attn_sink_decode_paged on the decode workload, cache in 256-position "
                                 "pages at random pool positions"},
        "decode_fp8": {"value": round(aggregate_rate(Kp * dbytes8, world, t_fp8) / 1e9, 2), "unit": "GB/s",
                       "ms_per_call": round(t_fp8 / Kp * 1e3, 4),
                       "frac": round(dbytes8 / (t_fp8 / Kp) / 1e9 / hbm_peak, 4),
                       "traffic": profiled_traffic("decode_split_fp8", [
                           "sliding_window_learned_b200/csrc/decode.cu",
                           "sliding_window_learned_b200/csrc/ptx.cuh"]),
                       "what": "attn_sink_decode_fp8 on the decode workload, cache quantised to e4m3 per "
                               "kv head (bytes counted at one per element)"},
        "decode_shapes": {nm: {
            "bf16": {"value": round(aggregate_rate(Kp * b16, world, shape_times[2 * i]) / 1e9, 2), "unit": "GB/s",
                     "ms_per_call": round(shape_times[2 * i] / Kp * 1e3, 4),
                     "frac": round(b16 / (shape_times[2 * i] / Kp) / 1e9 / hbm_peak, 4)},
            "fp8": {"value": round(aggregate_rate(Kp * b8, world, shape_times[2 * i + 1]) / 1e9, 2), "unit": "GB/s",
                    "ms_per_call": round(shape_times[2 * i + 1] / Kp * 1e3, 4),
                    "frac": round(b8 / (shape_times[2 * i + 1] / Kp) / 1e9 / hbm_peak, 4)},
            "fp8_rate_over_bf16": round((b8 / shape_times[2 * i + 1]) / (b16 / shape_times[2 * i]), 4)}
            for i, (nm, b16, b8) in enumerate(shape_bytes)},
        "fwd_varlen": {"value": round(aggregate_rate(Kv * vl_flops, world, t_varlen) / 1e12, 3), "unit": "TFLOP/s",
                       "ms_per_call": round(t_varlen / Kv * 1e3, 5),
                       "frac": round(vl_flops / (t_varlen / Kv) / 1e12 / bf16_peak, 4),
                       "what": "attn_sink_fwd_varlen on 24 packed sequences of U[1, 4096] tokens "
                               f"(T = {vl_T}), Hq32 Hkv4 D128 W513, L2 flushed before each call"},
        "bwd": {"value": round(aggregate_rate(Kb * 2.5 * fwd_flops, world, t_bwd) / 1e12, 3), "unit": "TFLOP/s",
                "ms_per_call": round(t_bwd / Kb * 1e3, 5),
                "frac": round(2.5 * fwd_flops / (t_bwd / Kb) / 1e12 / bf16_peak, 4),
                "traffic_main_pass": profiled_traffic("bwd_tc", ["sliding_window_learned_b200/csrc/bwd_tc.cu",
                                                                 "sliding_window_learned_b200/csrc/bwd.cu",
                                                                 "sliding_window_learned_b200/csrc/ptx.cuh"]),
                "what": "attn_sink_bwd (dq, dk, dv, dsink) on the prefill workload, O and LSE from "
                        "attn_sink_fwd; useful FLOPs = 10 D per visible pair (2.5x the forward's), "
                        "L2 flushed before each call"},
        "e2e": {"value": round(aggregate_rate(Ke * fwd_flops, world, t_e2e) / 1e12, 4), "unit": "TFLOP/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "serial_value": round(aggregate_rate(Ke * fwd_flops, world, t_e2e_serial) / 1e12, 4),
                "what": "attn_sink_fwd with pinned host inputs copied in and O, LSE copied out each "
                        "step; the copies of neighbouring steps overlap the forward (input copies, "
                        "forward and output copies on three streams, two sets of device buffers); "
                        "serial_value: one step at a time on one stream"},
        "workloads": {nm: forward_leg_report(leg_raw[nm][0], leg_raw[nm][1], tl_, leg_raw[nm][3],
                                            leg_raw[nm][4], world, bf16_peak, peak_src)
                      for (nm, _, _), tl_ in zip(leg_specs, leg_times)},
        "gpu_launches": K * 4,
        "clocks": clk,
        "timed_region_ms": round(t_all * 1e3, 3),
    }
    if world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(budget_s=args.cpu_seconds)
        line["decode"]["cpu_baseline"] = cpu_baseline_decode(y, dcfg)
        line["bwd"]["cpu_baseline"] = cpu_baseline_bwd(x, pcfg)
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------- oracle timing
_PREFILL_HOST = {}


def _oracle_sample(n_rows, seed=0):
    cfg = inputs.PREFILL
    if "x" not in _PREFILL_HOST:
        _PREFILL_HOST["x"] = inputs.make_prefill(cfg, seed=0)
    x = _PREFILL_HOST["x"]
    rng = np.random.default_rng(seed)
    rows = np.stack([rng.integers(cfg.B, size=n_rows), rng.integers(cfg.L, size=n_rows),
                     rng.integers(cfg.Hq, size=n_rows)], 1).astype(np.int32)
    vis = np.minimum(rows[:, 1].astype(np.int64) + 1, cfg.W)
    flops = 4.0 * cfg.D * float(vis.sum())
    import oracle
    if "bits" not in _PREFILL_HOST:
        _PREFILL_HOST["bits"] = (inputs.bits(x["q"]), inputs.bits(x["k"]), inputs.bits(x["v"]))
    qb, kb, vb = _PREFILL_HOST["bits"]
    sk = x["sinks"].numpy()

    def run():
        oracle.fwd_rows(qb, kb, vb, sk, cfg.W, cfg.scale, rows)

    return run, flops


def cpu_baseline(budget_s: float = 10.0):
    """The fp64 oracle, as it stands, on a bounded random sample of rows of the
    prefill workload; useful TFLOP/s of the sampled rows."""
    import oracle
    oracle.build()
    run, flops = _oracle_sample(256)
    t0 = time.perf_counter()
    run()
    dt = time.perf_counter() - t0
    n_rows = int(max(256, min(4000000, 256 * budget_s / max(dt, 1e-6))))
    run, flops = _oracle_sample(n_rows, seed=1)
    t0 = time.perf_counter()
    run()
    dt = time.perf_counter() - t0
    return {"value": round(flops / dt / 1e12, 6), "unit": "TFLOP/s", "cores": oracle.num_threads(),
            "kind": "oracle",
            "sample": f"{n_rows} random (b, i, h) rows of {inputs.PREFILL.name}, fp64, {dt:.1f} s"}


def cpu_baseline_decode(y, cfg, n_seq=2):
    """The oracle's decode, as it stands, on a bounded sample of the decode
    workload (n_seq of its sequences, every head); GB/s of their algorithmic
    bytes."""
    import oracle
    oracle.build()
    sl = y["seqlens"].cpu().numpy()
    pick = np.sort(np.random.default_rng(7).choice(cfg.B, size=n_seq, replace=False))
    nmax = int(sl[pick].max())
    q = inputs.bits(y["q"][pick].cpu())
    kb = inputs.bits(y["kcache"][pick, :nmax].cpu())
    vb = inputs.bits(y["vcache"][pick, :nmax].cpu())
    nbytes = float(sl[pick].sum()) * cfg.Hkv * cfg.D * 2 * 2 + 2 * n_seq * cfg.Hq * cfg.D * 2
    t0 = time.perf_counter()
    oracle.decode(q, kb, vb, sl[pick].astype(np.int32), y["sinks"].cpu().numpy(), cfg.W, cfg.scale)
    dt = time.perf_counter() - t0
    return {"value": round(nbytes / dt / 1e9, 4), "unit": "GB/s", "cores": oracle.num_threads(), "kind": "oracle",
            "sample": f"{n_seq} sequences (n = {', '.join(str(int(n)) for n in sl[pick])}) of {cfg.name}, "
                      f"every head, fp64, {dt:.1f} s"}


def cpu_baseline_bwd(x, cfg, L=2048):
    """The oracle's backward, as it stands, on a bounded slice of the prefill
    workload: the first L positions of batch 0 and the query heads of kv head
    0; useful TFLOP/s of the slice (2.5x its forward FLOPs)."""
    import torch

    import oracle
    G = cfg.Hq // cfg.Hkv
    q, k, v = (x["q"][:1, :L, :G].cpu(), x["k"][:1, :L, :1].cpu(), x["v"][:1, :L, :1].cpu())
    g = torch.Generator().manual_seed(3)
    do = torch.randn(q.shape, generator=g).to(torch.bfloat16)
    flops = 2.5 * 4.0 * cfg.D * G * float(np.minimum(np.arange(L) + 1, cfg.W).sum())
    t0 = time.perf_counter()
    oracle.bwd(inputs.bits(q), inputs.bits(k), inputs.bits(v), x["sinks"][:G].cpu().numpy(), inputs.bits(do),
               cfg.W, cfg.scale)
    dt = time.perf_counter() - t0
    return {"value": round(flops / dt / 1e12, 6), "unit": "TFLOP/s", "cores": torch.get_num_threads(),
            "kind": "oracle",
            "sample": f"positions 0..{L - 1} of batch 0, query heads 0..{G - 1} (kv head 0) of {cfg.name}, "
                      f"fp64 autograd, {dt:.1f} s"}


def run_reference(args, rank, world):
    if rank != 0:
        return
    import oracle
    oracle.build()
    run, flops = _oracle_sample(256)
    t0 = time.perf_counter()
    run()
    dt = time.perf_counter() - t0
    # each step a bounded sample: the whole run stays within ~2 minutes
    budget_per_step = min(20.0, 120.0 / max(1, args.steps + args.warmup))
    n_rows = int(max(64, min(100000, 256 * budget_per_step / max(dt, 1e-6))))
    steps = []
    for s in range(args.warmup + args.steps):
        run, flops = _oracle_sample(n_rows, seed=100 + s)
        t0 = time.perf_counter()
        run()
        if s >= args.warmup:
            steps.append((flops, time.perf_counter() - t0))
    fl = sum(f for f, _ in steps)
    tt = sum(t for _, t in steps)
    value = fl / tt / 1e12
    sample = f"{n_rows} random (b, i, h) rows of {inputs.PREFILL.name} per step, fp64"
    line = {
        "impl": "reference", "metric": METRIC, "value": round(value, 6), "unit": "TFLOP/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(tt / max(1, len(steps)) * 1e3, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded; torch generator, seed 0)",
        "config": {"workload": inputs.PREFILL.name, "parallelism": "cpu"},
        "cpu_baseline": {"kind": "oracle", "cores": oracle.num_threads(), "sample": sample,
                         "value": round(value, 6), "unit": "TFLOP/s"},
        "e2e": {"value": round(value, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ------------------------------------------------------- profiler driver
def _profile_workloads():
    return {
        "tiny": inputs.TINY,
        "prefill": inputs.PREFILL,
        "long-causal": inputs.LONG_CAUSAL,
        "stress": inputs.STRESS,
        "decode": inputs.DECODE,
        # same length distribution as the decode workload, 8 sequences (~1 GB of cache)
        "decode-small": inputs.Decode("decode-small B8 Hq32 Hkv4 D128 n~U[4096,131072]", 8, 32, 4,
                                      128, 131072, 4096, 131072, 131072),
        # the two extra decode shapes at 8 and 4 sequences (~1 GB of cache each)
        "decode-g16-small": inputs.Decode("decode-g16-small B8 Hq64 Hkv4 D128 n~U[4096,131072]", 8, 64, 4,
                                          128, 131072, 4096, 131072, 131072),
        "decode-d256-small": inputs.Decode("decode-d256-small B4 Hq32 Hkv4 D256 n~U[4096,131072]", 4, 32, 4,
                                           256, 131072, 4096, 131072, 131072),
    }


def run_profile(args) -> int:
    """A few launches of one operation on one workload, for Nsight Compute
    captures of a single kernel on a bounded device footprint.  It prints no
    timings (numbers taken under a profiler are not measurements) and exits
    non-zero if the device reports an error.

    --profile bwd runs one forward for O and LSE, then the backward passes;
    --profile decode_fp8 quantises the workload's cache to e4m3 per kv head
    first; --profile decode_paged copies the cache into pools of --page
    positions at random pool positions, addressed through a block table."""
    import torch

    from sliding_window_learned_b200 import abi, build
    build.build()
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    cfg = _profile_workloads()[args.workload]
    op, n = args.profile, args.launches
    if op in ("fwd", "bwd"):
        if not isinstance(cfg, inputs.Prefill):
            raise SystemExit(f"{op} needs a prefill workload")
        x = inputs.make_prefill(cfg, seed=0, device=dev)
        out = torch.empty_like(x["q"])
        lse = torch.empty(cfg.B, cfg.Hq, cfg.L, dtype=torch.float32, device=dev)
        if op == "fwd":
            for _ in range(n):
                abi.attn_sink_fwd(x["q"], x["k"], x["v"], x["sinks"], cfg.W, cfg.scale, out, lse)
        else:
            abi.attn_sink_fwd(x["q"], x["k"], x["v"], x["sinks"], cfg.W, cfg.scale, out, lse)
            g = torch.Generator(device=dev).manual_seed(1)
            dout = torch.randn(x["q"].shape, device=dev, generator=g).to(torch.bfloat16)
            dq, dk, dv = torch.empty_like(x["q"]), torch.empty_like(x["k"]), torch.empty_like(x["v"])
            dsink = torch.empty(cfg.Hq, dtype=torch.float32, device=dev)
            for _ in range(n):
                abi.attn_sink_bwd(x["q"], x["k"], x["v"], out, lse, dout, x["sinks"], cfg.W, cfg.scale,
                                  dq, dk, dv, dsink)
    else:
        if not isinstance(cfg, inputs.Decode):
            raise SystemExit("decode needs a decode workload")
        y = inputs.make_decode(cfg, seed=0, device=dev)
        out = torch.empty_like(y["q"])
        if op == "decode_fp8":
            k8, v8, kd, vd = quantise_e4m3(y, cfg, dev)
            for _ in range(n):
                abi.attn_sink_decode_fp8(y["q"], k8, v8, kd, vd, y["seqlens"], y["sinks"], cfg.W, cfg.scale, out)
        elif op == "decode_paged":
            kpool, vpool, table = page_cache(y, cfg, args.page, 0, dev)
            del y["kcache"], y["vcache"]
            for _ in range(n):
                abi.attn_sink_decode_paged(y["q"], kpool, vpool, table, y["seqlens"], y["sinks"], cfg.W,
                                           cfg.scale, out)
        else:
            for _ in range(n):
                abi.attn_sink_decode(y["q"], y["kcache"], y["vcache"], y["seqlens"], y["sinks"],
                                     cfg.W, cfg.scale, out)
    torch.cuda.synchronize()
    rc = abi.attn_sink_get_status()
    print("ok" if rc == 0 else f"device status {rc}")
    return 0 if rc == 0 else 1


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=400)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--profile", choices=["fwd", "decode", "bwd", "decode_fp8", "decode_paged"],
                    help="profiler driver: run --launches of one operation on --workload, no timing")
    ap.add_argument("--workload", choices=sorted(_profile_workloads()), default="prefill")
    ap.add_argument("--launches", type=int, default=3)
    ap.add_argument("--page", type=int, default=16, help="positions per page (--profile decode_paged)")
    args = ap.parse_args()
    if args.profile:
        sys.exit(run_profile(args))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, rank, world)
        return
    if world > 1:
        import datetime

        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local_rank))
    try:
        run_ours(args, rank, world, local_rank)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
