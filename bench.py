#!/usr/bin/env python
"""Benchmark: one paged decode step (slot-mapped append + paged decode attention).

A step is the whole hot path over one synthetic batch: the append of each
sequence's new key/value and the paged decode attention over contexts that
include it, in one launch of paged_attn_decode_append (a persistent decode
kernel that also merges the contexts it splits between CTAs); --two-launch
runs kv_cache_append + paged_attn_decode instead. The default workload is the
Llama-3-8B-shaped GQA batch (256 sequences, 32 q / 8 kv heads, head_dim 128,
block_size 16, context lengths U[128, 4096], pool 1.2x the needed blocks,
shuffled) -- 2.25 GB of K/V read per step, far larger than L2; L2 is also
flushed (memset of 2x its size) between timed steps, outside the step's events.

Prints one JSON line (rank 0). `value` is KV GB/s: the algorithmic bytes of
the step, sum over sequences of context_len * num_kv_heads * head_dim * 2
(K and V) * 2 (bf16), divided by the device time of the step.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
Under torchrun each rank runs its own independent batch (weak scaling, no
data-path collective); the timing is the max over ranks.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import statistics
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads  # noqa: E402

METRIC = "paged decode KV GB/s & % of B200 HBM peak; seq·tokens/s per decode step"
PREFILL_METRIC = "multi-query paged attention TFLOP/s (chunked prefill)"

# Multi-query (chunked prefill) workloads: chunk lengths and a context draw per sequence.
PREFILL_WORKLOADS = {
    "prefill_llama_chunks": dict(
        description="Llama-3-8B GQA heads: 16 seqs x 512-token chunks at the end of contexts 512 + U[0, 3584], "
                    "32/8 heads, D128, bs16",
        chunks=[512] * 16, ctx=lambda rng: [512 + int(x) for x in rng.integers(0, 3585, 16)],
        heads=(32, 8), head_dim=128, block_size=16),
}
FALLBACK_HBM_GBS = 6650.0
PROFILES = os.path.join(ROOT, "profiles")


# ----------------------------------------------------------------------------- helpers

def parse_args(argv=None):
    p = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=200)
    p.add_argument("--warmup", type=int, default=10)
    p.add_argument("--impl", choices=["ours", "reference"], default="ours")
    p.add_argument("--workload", default="llama3_8b", choices=list(workloads.CONFIGS) + list(PREFILL_WORKLOADS))
    p.add_argument("--kv-dtype", default="bf16", choices=["bf16", "fp8"],
                   help="decode workloads: bf16 pools, or e4m3 codes with per-head scales")
    p.add_argument("--num-ctas", type=int, default=0)
    p.add_argument("--num-stages", type=int, default=0)
    p.add_argument("--ctas-per-sm", type=int, default=0)
    p.add_argument("--math", type=int, default=0)
    p.add_argument("--l2-prefetch", type=int, default=0)
    p.add_argument("--piece-cost", type=int, default=0)
    p.add_argument("--head-pack", type=int, default=0)
    p.add_argument("--tile-tokens", type=int, default=0)
    p.add_argument("--prefix-tiles", type=int, default=0)
    p.add_argument("--prefix-groups", choices=["on", "off"], default="off",
                   help="on: pass the runs of sequences that share leading blocks (found on the host tables, "
                        "as an engine's block manager knows them) so that shared blocks are read once per group")
    p.add_argument("--two-launch", action="store_true",
                   help="run the step as kv_cache_append + paged_attn_decode instead of the one-launch call")
    p.add_argument("--seqs", type=int, default=0,
                   help="build the workload with only its first N context lengths (small cases for ncu)")
    p.add_argument("--no-e2e", action="store_true")
    p.add_argument("--flush", choices=["auto", "always", "never"], default="auto",
                   help="L2 flush (memset of 2x L2) between timed steps: auto = only when the step's K/V "
                        "is under 4x L2 (larger inputs leave nothing in L2 for the next step)")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--prefill-kernel", type=int, default=0, choices=[0, 1, 2],
                   help="multi-query kernel: 0 default (tcgen05 where it applies), 1 mma.sync, 2 tcgen05")
    return p.parse_args(argv)


def rank_seed(base_seed: int, rank: int) -> int:
    """Each rank decodes its own batch; rank 0 uses the workload's canonical seed."""
    return base_seed + 7919 * rank


def aggregate(sum_values, max_values):
    """Sum `sum_values` and max `max_values` over ranks (identity without a process group)."""
    import torch.distributed as dist
    s = torch.tensor(sum_values, dtype=torch.float64)
    m = torch.tensor(max_values, dtype=torch.float64)
    if dist.is_available() and dist.is_initialized():
        dev = torch.device("cuda", torch.cuda.current_device()) if dist.get_backend() == "nccl" else torch.device("cpu")
        s, m = s.to(dev), m.to(dev)
        dist.all_reduce(s, op=dist.ReduceOp.SUM)
        dist.all_reduce(m, op=dist.ReduceOp.MAX)
    return s.cpu().tolist(), m.cpu().tolist()


def job_totals(kv_bytes, seqs, ctx_tokens, steps, total_ms):
    """Whole-job figures over all ranks: each rank processed its own batch
    `steps` times in `total_ms` of device time; the job takes as long as its
    slowest rank (weak scaling: per-rank work is fixed as ranks are added)."""
    (sum_kv, sum_seq, sum_tok), (max_ms,) = aggregate(
        [kv_bytes * steps, seqs * steps, ctx_tokens * steps], [total_ms])
    seconds = max_ms / 1e3
    return {"value": sum_kv / seconds / 1e9, "seq_per_s": sum_seq / seconds,
            "ctx_tokens_per_s": sum_tok / seconds, "max_ms": max_ms}


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    return FALLBACK_HBM_GBS, "fallback"


def decode_sources_sha():
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "paged_kv_cache_377_b200", "csrc")
    for name in ("decode.cu", "decode_common.cuh", "device_utils.cuh"):
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def prefill_sources_sha():
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "paged_kv_cache_377_b200", "csrc")
    for name in ("prefill_tc.cu", "device_utils.cuh"):
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def profiled_prefill_traffic(workload: str):
    """DRAM bytes per tcgen05 prefill launch from a committed ncu capture, if it was
    taken on the current kernel sources (else None)."""
    path = os.path.join(PROFILES, "prefill_traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        e = json.load(f).get(workload)
    if not e or e.get("prefill_sources_sha") != prefill_sources_sha():
        return None
    return e.get("dram_bytes_per_launch")


def profiled_traffic(workload: str):
    """DRAM bytes per decode launch from a committed ncu capture, if it was taken
    on the current decode sources (else None)."""
    path = os.path.join(PROFILES, "decode_traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        d = json.load(f)
    e = d.get(workload)
    if not e or e.get("decode_sources_sha") != decode_sources_sha():
        return None
    return e.get("dram_bytes_per_launch")


class ClockSampler:
    """Polls SM clock, power and clock-event reasons through NVML while running."""

    NAMES = {
        0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap", 0x8: "hw_slowdown",
        0x10: "sync_boost", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
        0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting",
    }

    def __init__(self, device_index: int, period_s: float = 0.01):
        self.samples = []
        self.max_mhz = None
        self.error = None
        self._stop = threading.Event()
        self._thread = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nvml = pynvml
            self._h = self._handle(pynvml, device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
        except Exception as e:  # no NVML: report the clocks as unknown
            self.error = repr(e)
            self._nvml = None
        self.period = period_s

    @staticmethod
    def _handle(pynvml, device_index):
        props = torch.cuda.get_device_properties(device_index)
        try:
            bus = f"{props.pci_domain_id:08x}:{props.pci_bus_id:02x}:{props.pci_device_id:02x}.0"
            return pynvml.nvmlDeviceGetHandleByPciBusId(bus)
        except Exception:
            return pynvml.nvmlDeviceGetHandleByUUID(("GPU-" + str(props.uuid)).encode())

    def _run(self):
        nv = self._nvml
        while not self._stop.is_set():
            try:
                mhz = nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM)
                rs = nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
                pw = nv.nvmlDeviceGetPowerUsage(self._h) / 1000.0
                self.samples.append((time.time(), mhz, rs, pw))
            except Exception as e:
                self.error = repr(e)
            self._stop.wait(self.period)

    def __enter__(self):
        if self._nvml is not None:
            self._thread = threading.Thread(target=self._run, daemon=True)
            self._thread.start()
        return self

    def __exit__(self, *exc):
        self._stop.set()
        if self._thread is not None:
            self._thread.join()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0,
                    "note": self.error or "no samples"}
        reasons = set()
        for _, _, rs, _ in self.samples:
            for bit, name in self.NAMES.items():
                if rs & bit:
                    reasons.add(name)
        return {
            "sm_mhz": statistics.median(s[1] for s in self.samples),
            "sm_max_mhz": self.max_mhz,
            "reasons": sorted(reasons),
            "samples": len(self.samples),
            "power_w_max": max(s[3] for s in self.samples),
            "source": "NVML, polled every 10 ms during the timed region",
        }


# ----------------------------------------------------------------------------- our arm

class Step:
    """Device buffers of one decode step and the library call(s) that make it:
    paged_attn_decode_append (append + attention in one launch) by default, or
    kv_cache_append followed by paged_attn_decode with --two-launch."""

    def __init__(self, batch, args, device):
        self.fused = not args.two_launch
        import paged_kv_cache_377_b200 as pkv
        self.pkv = pkv
        b = batch
        self.b = b
        self.kc = b.k_cache.to(device)
        self.vc = b.v_cache.to(device)
        self.q = b.q.to(device)
        self.k_new = b.k_new.to(device)
        self.v_new = b.v_new.to(device)
        self.bt = b.block_tables.to(device)
        self.cl = b.context_lens.to(device)
        self.slots = b.slot_mapping.to(device)
        self.out = torch.empty_like(self.q)
        self.status = torch.zeros(1, dtype=torch.int32, device=device)
        self.opts = dict(num_ctas=args.num_ctas, num_stages=args.num_stages,
                         ctas_per_sm=args.ctas_per_sm, math=args.math, l2_prefetch=args.l2_prefetch,
                         piece_cost=args.piece_cost, head_pack=args.head_pack, tile_tokens=args.tile_tokens,
                         prefix_tiles=args.prefix_tiles)
        self.groups = None
        if getattr(args, "prefix_groups", "off") == "on" and b.kv_dtype == "bf16":
            g = pkv.find_prefix_groups(b.block_tables, b.context_lens, b.block_size)
            if len(g):
                self.groups = g
                self.opts["prefix_groups"] = g
        self.ws = pkv.allocate_workspace(b.num_seqs, b.num_q_heads, b.head_dim, device=device)
        self.fp8 = b.kv_dtype == "fp8"
        if self.fp8:
            self.ks = b.k_scale.to(device)
            self.vs = b.v_scale.to(device)

    def append(self, stream=None):
        if self.fp8:
            self.pkv.kv_cache_append_fp8(self.k_new, self.v_new, self.kc, self.vc, self.slots, self.ks, self.vs,
                                         self.status, stream=stream)
            return
        self.pkv.kv_cache_append(self.k_new, self.v_new, self.kc, self.vc, self.slots, self.status, stream=stream)

    def decode(self, stream=None):
        if self.fp8:
            self.pkv.paged_attn_decode_fp8(self.out, self.q, self.kc, self.vc, self.ks, self.vs, self.bt, self.cl,
                                           self.b.scale, self.ws, stream=stream, **self.opts)
            return
        self.pkv.paged_attn_decode(self.out, self.q, self.kc, self.vc, self.bt, self.cl, self.b.scale, self.ws,
                                   stream=stream, **self.opts)

    def fused_step(self, stream=None):
        if self.fp8:
            self.pkv.paged_attn_decode_append_fp8(self.out, self.q, self.k_new, self.v_new, self.slots, self.kc,
                                                  self.vc, self.ks, self.vs, self.bt, self.cl, self.b.scale, self.ws,
                                                  stream=stream, **self.opts)
            return
        self.pkv.paged_attn_decode_append(self.out, self.q, self.k_new, self.v_new, self.slots, self.kc, self.vc,
                                          self.bt, self.cl, self.b.scale, self.ws, stream=stream, **self.opts)

    def run(self, stream=None, mid_event=None):
        """One decode step; in two-launch mode `mid_event` is recorded between the calls."""
        if self.fused:
            self.fused_step(stream)
            return
        self.append(stream)
        if mid_event is not None:
            mid_event.record(stream if stream is not None else torch.cuda.current_stream())
        self.decode(stream)

    def decode_launches(self):
        """Decode kernels per call: one per 2048 sequences."""
        return -(-self.b.num_seqs // 2048)

    def launches(self):
        """Kernels of this library launched per step."""
        return self.decode_launches() + (0 if self.fused else 1)

    def status_word(self):
        return self.pkv.read_status(self.status) | self.pkv.read_status(self.ws)


def run_ours(args, rank, world, local_rank):
    import torch.distributed as dist
    device = torch.device("cuda", local_rank)
    torch.cuda.set_device(device)
    cfg = workloads.CONFIGS[args.workload]
    lens = None
    if args.seqs:  # the workload's recipe cut to its first N lengths (pool sized for those)
        lens = cfg.lengths(np.random.default_rng(rank_seed(cfg.seed, rank)))[:args.seqs].tolist()
    batch = workloads.make_batch(args.workload, seed=rank_seed(cfg.seed, rank), device=device, poison=False,
                                 lens_override=lens, kv_dtype=args.kv_dtype)
    step = Step(batch, args, device)
    args.groups_desc = (None if step.groups is None else
                        {"begin": step.groups.begin.tolist(), "end": step.groups.end.tolist(),
                         "blocks": step.groups.blocks.tolist()})
    kv = workloads.kv_bytes(batch)
    ctx_tokens = int(batch.context_lens.sum())
    S = batch.num_seqs
    l2 = torch.cuda.get_device_properties(device).L2_cache_size
    flush = torch.empty(2 * l2, dtype=torch.uint8, device=device)
    stream = torch.cuda.current_stream(device)
    # Inputs far larger than L2 need no flush (a memset flush also leaves L2 full of
    # dirty lines whose write-back the next step pays for: ~4 % on the Llama batch).
    do_flush = args.flush == "always" or (args.flush == "auto" and workloads.unique_kv_bytes(batch) < 4 * l2)
    args.l2_policy = ("L2 flushed (memset 2x L2) between timed steps" if do_flush else
                      f"no flush: inputs larger than L2 ({workloads.unique_kv_bytes(batch) / l2:.0f}x L2 of "
                      f"K/V read per step)")

    def barrier():
        if world > 1:
            dist.barrier()

    for _ in range(args.warmup):
        step.run()
    torch.cuda.synchronize()

    K = args.steps
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(K)]
    sampler = ClockSampler(local_rank)
    barrier()
    torch.cuda.synchronize()
    with sampler:
        for i in range(K):
            if do_flush:
                flush.zero_()                  # L2 flush, outside the step's events
            ev[i][0].record(stream)
            step.run(mid_event=ev[i][1])
            ev[i][2].record(stream)
        torch.cuda.synchronize()
    barrier()
    step_ms = [e[0].elapsed_time(e[2]) for e in ev]
    # the decode kernel's time: the whole step when the append is fused into it
    decode_ms = step_ms if step.fused else [e[1].elapsed_time(e[2]) for e in ev]
    append_ms = None if step.fused else [e[0].elapsed_time(e[1]) for e in ev]
    total_ms = sum(step_ms)
    status = step.status_word()
    if status:
        raise RuntimeError(f"device status {status} after the timed steps")

    job = job_totals(kv, S, ctx_tokens, K, total_ms)
    value, max_ms = job["value"], job["max_ms"]
    hbm, hbm_kind = measured_peaks()
    mean_decode_ms = statistics.fmean(decode_ms)
    # The roofline counts each distinct pool slot the step reads once (the DRAM
    # floor): the same as the logical bytes unless sequences share blocks, whose
    # repeated reads can come from L2.
    unique = workloads.unique_kv_bytes(batch)
    achieved = unique / (mean_decode_ms / 1e3) / 1e9

    e2e = None
    if not args.no_e2e:
        e2e = run_e2e(step, args, flush, stream, kv, world)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(batch, kv, S, ctx_tokens)

    traffic = profiled_traffic(args.workload + ("_fp8" if args.kv_dtype == "fp8" else ""))
    result = {
        "metric": METRIC,
        "value": round(value, 2),
        "unit": "GB/s",
        "n_gpus": world,
        "steps": K,
        "warmup": args.warmup,
        "ms_per_step": round(max_ms / K, 5),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": ("bf16 products, f32 accumulate" if args.kv_dtype == "bf16" else
                  "f16 products of e4m3 KV, f32 accumulate"),
        "data": "synthetic",
        "config": config_block(args, batch, world),
        "pct_of_hbm_peak": round(100.0 * value / (hbm * world), 2),
        "seq_per_s": round(job["seq_per_s"], 1),
        "ctx_tokens_per_s": round(job["ctx_tokens_per_s"], 1),
        "append_us_mean": None if append_ms is None else round(1e3 * statistics.fmean(append_ms), 3),
        "decode_us_mean": round(1e3 * mean_decode_ms, 3),
        "decode_us_median": round(1e3 * statistics.median(decode_ms), 3),
        "roofline": {
            "kernel": ("paged_decode_kernel (the step's one launch: append fused)" if step.fused else
                       "paged_decode_kernel (one launch per paged_attn_decode call)"),
            "bound": "hbm",
            "achieved": round(achieved, 2),
            "peak": hbm,
            "peak_kind": f"{hbm_kind} hbm_gbs (copy)",
            "unit": "GB/s",
            "frac": round(achieved / hbm, 4),
            "algorithmic_bytes_per_launch": unique,
            "bytes_basis": ("K/V bytes of the distinct pool slots the step reads" if unique == kv else
                            "K/V bytes of the distinct pool slots the step reads (shared blocks once; "
                            f"{kv} logical bytes through the tables)"),
            "traffic": traffic,
        },
        "clocks": sampler.summary(),
        "gpu_launches": K * step.launches(),
        "e2e": e2e,
        "cpu_baseline": cpu,
    }
    return result


def run_e2e(step, args, flush, stream, kv, world):
    """The same step through the public API with HOST inputs: every step copies its
    inputs (q, new k/v, tables, lengths, slots) from pinned memory and reads `out`
    back; the KV pool stays resident on the device (it is the cache).

    As a serving loop would, the inputs sit packed in one pinned buffer and go
    over in one copy per step; the copies run on their own streams and overlap
    the neighbouring steps' kernels: step i's inputs go to one of two device
    buffer sets while step i - 1 computes, and its output is read back while
    step i + 1 computes. The one-launch step is launched through
    ``DecodeAppendCall`` / ``DecodeAppendFp8Call`` (its buffers checked once, as
    a serving loop's static buffers are). The timed region runs from the first input copy to the last
    read-back. No L2 flush: the pool (far larger than L2) is read once per step."""
    names = ("q", "k_new", "v_new", "bt", "cl", "slots")
    srcs = {n: getattr(step, n) for n in names}
    offs, off = {}, 0
    for n in names:  # each input at a 256-byte boundary of the packed buffers
        offs[n] = off
        off += (srcs[n].numel() * srcs[n].element_size() + 255) // 256 * 256
    packed_host = torch.empty(off, dtype=torch.uint8, pin_memory=True)

    def views(buf):
        return {n: buf[offs[n]:offs[n] + srcs[n].numel() * srcs[n].element_size()].view(srcs[n].dtype)
                .view(srcs[n].shape) for n in names}

    for n, v in views(packed_host).items():
        v.copy_(srcs[n].cpu())
    packed_dev = [torch.empty(off, dtype=torch.uint8, device=step.q.device) for _ in range(2)]
    bufs = [views(d) for d in packed_dev]
    outs = [torch.empty_like(step.out) for _ in range(2)]
    out_host = [torch.empty(step.out.shape, dtype=step.out.dtype, pin_memory=True) for _ in range(2)]
    h2d = sum(t.numel() * t.element_size() for t in srcs.values())
    d2h = out_host[0].numel() * out_host[0].element_size()
    K = args.steps
    h2d_stream, d2h_stream = torch.cuda.Stream(), torch.cuda.Stream()
    prepared = None
    if step.fused and step.fp8:
        prepared = [step.pkv.DecodeAppendFp8Call(outs[b], bufs[b]["q"], bufs[b]["k_new"], bufs[b]["v_new"],
                                                 bufs[b]["slots"], step.kc, step.vc, step.ks, step.vs, bufs[b]["bt"],
                                                 bufs[b]["cl"], step.b.scale, step.ws, stream=stream, **step.opts)
                    for b in range(2)]
    elif step.fused:
        prepared = [step.pkv.DecodeAppendCall(outs[b], bufs[b]["q"], bufs[b]["k_new"], bufs[b]["v_new"],
                                              bufs[b]["slots"], step.kc, step.vc, bufs[b]["bt"], bufs[b]["cl"],
                                              step.b.scale, step.ws, stream=stream, **step.opts) for b in range(2)]

    def run(n_steps, timed):
        copied = [torch.cuda.Event() for _ in range(n_steps)]
        computed = [torch.cuda.Event() for _ in range(n_steps)]
        read = [torch.cuda.Event() for _ in range(n_steps)]
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        t0.record(h2d_stream)
        for i in range(n_steps):
            b = i % 2
            with torch.cuda.stream(h2d_stream):
                if i >= 2:
                    h2d_stream.wait_event(computed[i - 2])  # buffer set b is free again
                packed_dev[b].copy_(packed_host, non_blocking=True)
                copied[i].record(h2d_stream)
            stream.wait_event(copied[i])
            if i >= 2:
                stream.wait_event(read[i - 2])  # out[b] has been read back
            if prepared is not None:
                prepared[b]()
            else:
                for n in names:
                    setattr(step, n, bufs[b][n])
                step.out = outs[b]
                step.run()
            computed[i].record(stream)
            with torch.cuda.stream(d2h_stream):
                d2h_stream.wait_event(computed[i])
                out_host[b].copy_(outs[b], non_blocking=True)
                read[i].record(d2h_stream)
        d2h_stream.wait_stream(h2d_stream)
        t1.record(d2h_stream)
        torch.cuda.synchronize()
        return t0.elapsed_time(t1)

    run(max(args.warmup, 3), False)
    total_ms = run(K, True)
    (sum_kv,), (max_ms,) = aggregate([kv * K], [total_ms])
    return {"value": round(sum_kv / (max_ms / 1e3) / 1e9, 2), "unit": "GB/s", "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h, "ms_per_step": round(max_ms / K, 5),
            "how": "inputs packed in one pinned buffer, one H2D copy per step; H2D / D2H on their own streams, "
                   "overlapping the neighbouring steps; no L2 flush (pool > L2)"}


def config_block(args, batch, world):
    cfg = workloads.CONFIGS[args.workload]
    c = {
        "workload": args.workload,
        "description": cfg.description,
        "num_seqs": batch.num_seqs,
        "num_q_heads": batch.num_q_heads,
        "num_kv_heads": batch.num_kv_heads,
        "head_dim": batch.head_dim,
        "block_size": batch.block_size,
        "pool_blocks": batch.num_blocks,
        "context_tokens": int(batch.context_lens.sum()),
        "kv_bytes_per_step": workloads.kv_bytes(batch),
        "unique_kv_bytes_per_step": workloads.unique_kv_bytes(batch),
        "kv_dtype": batch.kv_dtype,
        "l2": getattr(args, "l2_policy", "L2 flushed (memset 2x L2) between timed steps"),
        "prefix_groups": getattr(args, "groups_desc", None),
        "parallelism": "replicas: one independent batch per GPU" if world > 1 else "single GPU",
        "step": ("kv_cache_append + paged_attn_decode (two launches)" if args.two_launch else
                 "paged_attn_decode_append (append + attention, one launch)"),
    }
    if args.seqs:
        c["seqs_kept"] = args.seqs
    for k in ("num_ctas", "num_stages", "ctas_per_sm", "math", "l2_prefetch", "piece_cost", "head_pack", "tile_tokens",
              "prefix_tiles"):
        if getattr(args, k):
            c[k] = getattr(args, k)
    return c


# ----------------------------------------------------------------------------- CPU oracle

def cpu_baseline(batch, kv, S, ctx_tokens, min_seconds=10.0, max_runs=5):
    """The fp64 oracle as it stands (append + decode), timed on the host cores on
    the same batch: runs of the whole step until ~10 s of CPU work are done."""
    import oracle
    host = batch.to("cpu")
    times = []
    t_all = time.perf_counter()
    while len(times) < max_runs and (time.perf_counter() - t_all) < min_seconds:
        t0 = time.perf_counter()
        oracle.decode_step(host)
        times.append(time.perf_counter() - t0)
    t = statistics.median(times)
    # one thread, decode only, on the first sequences of the batch (about 2 s)
    per_seq = t * host.context_lens.double() / max(1, ctx_tokens) * (os.cpu_count() or 1)
    n1 = int(max(1, min(S, int((per_seq.cumsum(0) < 2.0).sum()) or 1)))
    pairs = np.arange(n1 * host.num_q_heads, dtype=np.int64)
    t0 = time.perf_counter()
    if host.kv_dtype == "fp8":
        oracle.paged_decode_fp8(host.q, host.k_cache, host.v_cache, host.k_scale, host.v_scale,
                                host.block_tables.numpy(), host.context_lens.numpy(), host.num_kv_heads,
                                host.block_size, host.scale, pairs=pairs, num_threads=1)
    else:
        oracle.paged_decode(host.q, host.k_cache, host.v_cache, host.block_tables.numpy(), host.context_lens.numpy(),
                            host.num_kv_heads, host.block_size, host.scale, pairs=pairs, num_threads=1)
    t1 = time.perf_counter() - t0
    kv1 = int(host.context_lens[:n1].sum()) * host.num_kv_heads * host.head_dim * 2 * workloads.kv_element_bytes(host)
    return {
        "value": round(kv / t / 1e9, 3),
        "unit": "GB/s",
        "cores": os.cpu_count(),
        "kind": "oracle",
        "sample": f"whole batch ({S} seqs, {ctx_tokens} context tokens), append + decode, "
                  f"median of {len(times)} runs; {statistics.median(times):.2f} s per step",
        "seq_per_s": round(S / t, 2),
        "single_thread": {"value": round(kv1 / t1 / 1e9, 4), "unit": "GB/s", "cores": 1,
                          "sample": f"decode of the first {n1} sequences (all heads), {t1:.2f} s"},
    }


def run_reference_prefill(args):
    """The oracle's multi-query attention on a bounded sample of the workload."""
    b = make_prefill_batch(args.workload, 0, "cpu")
    sb = prefill_sample(b)
    rate, sec = oracle_prefill_rate(sb, seconds_min=10.0)
    return {
        "metric": PREFILL_METRIC, "value": round(rate, 6), "unit": "TFLOP/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(1e3 * sec, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": args.workload, "description": PREFILL_WORKLOADS[args.workload]["description"]},
        "impl": "reference",
        "cpu_baseline": {"value": round(rate, 6), "unit": "TFLOP/s", "cores": os.cpu_count(), "kind": "oracle",
                         "sample": f"the last 16 queries of the first 2 sequences, median run {sec:.2f} s"},
        "e2e": {"value": round(rate, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def run_reference(args):
    """The oracle as it stands, on bounded samples of the workload: step i decodes
    a slice of the batch's sequences (append + decode), sized so the whole run
    stays within a few minutes."""
    import oracle
    cfg = workloads.CONFIGS[args.workload]
    batch = workloads.make_batch(args.workload, device="cpu", poison=False)
    S = batch.num_seqs
    order = np.random.default_rng(0).permutation(S)

    def sub(idx):
        idx = np.sort(idx)
        return workloads.DecodeBatch(**{
            **batch.__dict__, "num_seqs": len(idx),
            "context_lens": batch.context_lens[idx], "block_tables": batch.block_tables[idx],
            "slot_mapping": batch.slot_mapping[idx], "q": batch.q[idx],
            "k_new": batch.k_new[idx], "v_new": batch.v_new[idx]})

    # size the slice from one probe step: aim at ~150 s for warmup + steps
    probe = sub(order[:8])
    t0 = time.perf_counter()
    oracle.decode_step(probe)
    t_probe = time.perf_counter() - t0
    budget = 150.0 / max(1, args.steps + args.warmup)
    n = int(max(1, min(S, 8 * budget / max(t_probe, 1e-3))))
    slices = [sub(order[(i * n) % S:(i * n) % S + n]) for i in range(args.steps + args.warmup)]
    for sl in slices[:args.warmup]:
        oracle.decode_step(sl)
    kv_total = 0
    seqs = 0
    t0 = time.perf_counter()
    for sl in slices[args.warmup:]:
        oracle.decode_step(sl)
        kv_total += workloads.kv_bytes(sl)
        seqs += sl.num_seqs
    seconds = time.perf_counter() - t0
    value = kv_total / seconds / 1e9
    sample = (f"{n} of {S} sequences per step (all heads), append + decode; "
              f"{args.steps} timed steps, {args.warmup} warm-up")
    return {
        "metric": METRIC,
        "value": round(value, 4),
        "unit": "GB/s",
        "n_gpus": args.gpus,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(1e3 * seconds / max(1, args.steps), 3),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f64",
        "data": "synthetic",
        "config": config_block(args, batch, 1),
        "impl": "reference",
        "seq_per_s": round(seqs / seconds, 3),
        "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": os.cpu_count(), "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


# ----------------------------------------------------------------------------- multi-query (prefill)

def make_prefill_batch(name, rank, device):
    w = PREFILL_WORKLOADS[name]
    seed = rank_seed(11, rank)
    ctx = w["ctx"](np.random.default_rng(seed))
    Hq, Hkv = w["heads"]
    return workloads.make_prefill(seed, w["chunks"], ctx, Hq, Hkv, w["head_dim"], w["block_size"], device=device,
                                  poison=False)


def prefill_sample(b, n_seqs=2, n_queries=16):
    """The last n_queries queries of the first n_seqs sequences, as a smaller prefill batch."""
    qs = b.query_start.numpy()
    rows, chunks = [], []
    for s in range(n_seqs):
        n = min(n_queries, int(qs[s + 1] - qs[s]))
        rows += list(range(int(qs[s + 1]) - n, int(qs[s + 1])))
        chunks.append(n)
    sub_qs = np.concatenate([[0], np.cumsum(chunks)]).astype(np.int32)
    return workloads.PrefillBatch(**{**b.__dict__, "num_seqs": n_seqs, "q": b.q[rows].cpu(),
                                     "context_lens": b.context_lens[:n_seqs], "block_tables": b.block_tables[:n_seqs],
                                     "query_start": torch.from_numpy(sub_qs), "k_cache": b.k_cache.cpu(),
                                     "v_cache": b.v_cache.cpu()})


def oracle_prefill_rate(b, seconds_min=3.0):
    import oracle
    runs, t_all = [], time.perf_counter()
    while len(runs) < 5 and time.perf_counter() - t_all < seconds_min:
        t0 = time.perf_counter()
        oracle.paged_prefill(b.q, b.k_cache, b.v_cache, b.block_tables.numpy(), b.context_lens.numpy(),
                             b.query_start.numpy(), b.num_kv_heads, b.block_size, b.scale)
        runs.append(time.perf_counter() - t0)
    return workloads.prefill_flops(b) / statistics.median(runs) / 1e12, statistics.median(runs)


def run_prefill(args, rank, world, local_rank):
    import paged_kv_cache_377_b200 as pkv
    device = torch.device("cuda", local_rank)
    torch.cuda.set_device(device)
    b = make_prefill_batch(args.workload, rank, device)
    flops = workloads.prefill_flops(b)
    T = b.q.shape[0]
    bt, cl, qs = b.block_tables.to(device), b.context_lens.to(device), b.query_start.to(device)
    mq = int((b.query_start[1:] - b.query_start[:-1]).max())
    out = torch.empty_like(b.q)
    status = torch.zeros(1, dtype=torch.int32, device=device)
    stream = torch.cuda.current_stream(device)
    l2 = torch.cuda.get_device_properties(device).L2_cache_size
    flush = torch.empty(2 * l2, dtype=torch.uint8, device=device)

    def step(q=b.q):
        pkv.paged_attn_prefill(out, q, b.k_cache, b.v_cache, bt, cl, qs, mq, b.scale, status,
                               kernel=args.prefill_kernel)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    K = args.steps
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
    sampler = ClockSampler(local_rank)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    torch.cuda.synchronize()
    with sampler:
        for i in range(K):
            flush.zero_()
            ev[i][0].record(stream)
            step()
            ev[i][1].record(stream)
        torch.cuda.synchronize()
    ms = [x.elapsed_time(y) for x, y in ev]
    if pkv.read_status(status):
        raise RuntimeError("device status set after the timed steps")
    (sum_flops,), (max_ms,) = aggregate([flops * K], [sum(ms)])
    value = sum_flops / (max_ms / 1e3) / 1e12
    mean_ms = statistics.fmean(ms)
    peak = measured_tflops()

    e2e = None if args.no_e2e else run_prefill_e2e(args, b, flops, out, status, stream, world)
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        sb = prefill_sample(b)
        rate, sec = oracle_prefill_rate(sb)
        cpu = {"value": round(rate, 6), "unit": "TFLOP/s", "cores": os.cpu_count(), "kind": "oracle",
               "sample": f"the last 16 queries of the first 2 sequences ({sb.q.shape[0]} query tokens), "
                         f"median run {sec:.2f} s"}
    w = PREFILL_WORKLOADS[args.workload]
    return {
        "metric": PREFILL_METRIC,
        "value": round(value, 2),
        "unit": "TFLOP/s",
        "n_gpus": world,
        "steps": K,
        "warmup": args.warmup,
        "ms_per_step": round(max_ms / K, 5),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16 products, f32 accumulate",
        "data": "synthetic",
        "config": {"workload": args.workload, "description": w["description"], "num_seqs": b.num_seqs,
                   "query_tokens": T, "context_tokens": int(b.context_lens.sum()), "flops_per_step": flops,
                   "l2": "L2 flushed (memset 2x L2) between timed steps",
                   "parallelism": "replicas: one independent batch per GPU" if world > 1 else "single GPU"},
        "roofline": {"kernel": ("paged_prefill_kernel (mma.sync" if args.prefill_kernel == 1 else
                               "paged_prefill_tc_kernel (tcgen05") + "; one launch per step)", "bound": "tensor",
                     "achieved": round(flops / (mean_ms / 1e3) / 1e12, 2), "peak": peak[0],
                     "peak_kind": f"{peak[1]} bf16_tflops (cuBLAS burst)", "unit": "TFLOP/s",
                     "frac": round(flops / (mean_ms / 1e3) / 1e12 / peak[0], 4),
                     "algorithmic_flops_per_launch": flops,
                     "traffic": profiled_prefill_traffic(args.workload) if args.prefill_kernel != 1 else None,
                     "traffic_unit": "DRAM bytes per launch (ncu)"},
        "clocks": sampler.summary(),
        "gpu_launches": K,
        "e2e": e2e,
        "cpu_baseline": cpu,
    }


def run_prefill_e2e(args, b, flops, out, status, stream, world):
    """The prefill step through the public API with HOST inputs: every step copies
    q, the block tables, context lengths and query starts from pinned memory and
    reads `out` back; the K/V pool stays resident (it is the cache). As in the
    decode e2e, the copies run on their own streams with two buffer sets, so step
    i's input copy and step i - 1's read-back overlap the neighbouring kernels;
    the timed region runs from the first input copy to the last read-back."""
    import paged_kv_cache_377_b200 as pkv
    mq = int((b.query_start[1:] - b.query_start[:-1]).max())
    src = {"q": b.q, "bt": b.block_tables, "cl": b.context_lens, "qs": b.query_start}
    host = {n: t.cpu().pin_memory() for n, t in src.items()}
    bufs = [{n: torch.empty(t.shape, dtype=t.dtype, device=out.device) for n, t in src.items()} for _ in range(2)]
    outs = [torch.empty_like(out) for _ in range(2)]
    out_host = [torch.empty(out.shape, dtype=out.dtype, pin_memory=True) for _ in range(2)]
    h2d = sum(t.numel() * t.element_size() for t in host.values())
    d2h = out_host[0].numel() * out_host[0].element_size()
    h2d_stream, d2h_stream = torch.cuda.Stream(), torch.cuda.Stream()

    def run(n_steps):
        copied = [torch.cuda.Event() for _ in range(n_steps)]
        computed = [torch.cuda.Event() for _ in range(n_steps)]
        read = [torch.cuda.Event() for _ in range(n_steps)]
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        t0.record(h2d_stream)
        for i in range(n_steps):
            k = i % 2
            with torch.cuda.stream(h2d_stream):
                if i >= 2:
                    h2d_stream.wait_event(computed[i - 2])  # buffer set k is free again
                for n in src:
                    bufs[k][n].copy_(host[n], non_blocking=True)
                copied[i].record(h2d_stream)
            stream.wait_event(copied[i])
            if i >= 2:
                stream.wait_event(read[i - 2])  # outs[k] has been read back
            x = bufs[k]
            pkv.paged_attn_prefill(outs[k], x["q"], b.k_cache, b.v_cache, x["bt"], x["cl"], x["qs"], mq, b.scale,
                                   status, kernel=args.prefill_kernel, stream=stream)
            computed[i].record(stream)
            with torch.cuda.stream(d2h_stream):
                d2h_stream.wait_event(computed[i])
                out_host[k].copy_(outs[k], non_blocking=True)
                read[i].record(d2h_stream)
        d2h_stream.wait_stream(h2d_stream)
        t1.record(d2h_stream)
        torch.cuda.synchronize()
        return t0.elapsed_time(t1)

    run(max(args.warmup, 3))
    K = args.steps
    total_ms = run(K)
    if pkv.read_status(status):
        raise RuntimeError("device status set in the end-to-end steps")
    (sf,), (mx,) = aggregate([flops * K], [total_ms])
    return {"value": round(sf / (mx / 1e3) / 1e12, 2), "unit": "TFLOP/s", "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h, "ms_per_step": round(mx / K, 4),
            "how": "H2D / D2H on their own streams, overlapping the neighbouring steps; no L2 flush"}


def measured_tflops():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            return float(json.load(f)["bf16_tflops"]), "measured"
    return 1590.0, "fallback"


# ----------------------------------------------------------------------------- main

def main(argv=None):
    args = parse_args(argv)
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        if rank != 0:
            return 0
        if args.workload in PREFILL_WORKLOADS:
            print(json.dumps(run_reference_prefill(args)), flush=True)
        else:
            print(json.dumps(run_reference(args)), flush=True)
        return 0
    if world > 1:
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    try:
        if args.workload in PREFILL_WORKLOADS:
            result = run_prefill(args, rank, world, local_rank)
        else:
            result = run_ours(args, rank, world, local_rank)
        if rank == 0:
            print(json.dumps(result), flush=True)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
