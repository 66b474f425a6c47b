#!/usr/bin/env python
"""Benchmark of the paged-KV attention hot path on B200.

One step = one decode step of the Llama-3-8B-shaped batch (B=128, 32 q / 8 kv
heads, head_dim 128, every context 4096, block_size 16): the cache write of one
new K/V row per sequence, then decode attention over all pages (split-KV
partials + log-sum-exp merge when the planner splits).  Metric: algorithmic
bytes of the step / step time in GB/s (the K/V read is 99.9 % of them), plus
the decode kernel's roofline fraction of the measured HBM copy bandwidth.

Other workloads (Llama-3.2-1B-shaped decode, ragged long-context decode,
chunked causal prefill in TFLOP/s) are reported under "extras" after the timed
region; they are not part of the step.

    python bench.py [--gpus N --steps K --warmup W] [--impl reference]

Multi-GPU (torchrun): every rank runs its own replica of the step on its own
GPU (the decode batch shards by sequence with no exchange); value = all
ranks' bytes / the slowest rank's time.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "decode attn KV-read GB/s (% of HBM peak); prefill TFLOP/s (% of bf16 peak)"
WORKLOAD = "llama3_8b_decode"


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="pagedkv", choices=["pagedkv", "reference"])
    ap.add_argument("--no-extras", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=10.0, help="budget of the oracle CPU baseline")
    ap.add_argument("--profile", default=None,
                    choices=["decode", "decode_full", "decode_d64", "decode_gqa8", "decode_ragged", "decode_int8",
                             "decode_int8_full", "split", "prefill", "write"],
                    help="run a few launches of one kernel on a small case (for ncu) and exit")
    return ap.parse_args()


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained", d["bf16_tflops"]),
                "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


def source_hash(*names):
    h = hashlib.sha256()
    for n in names:
        h.update(open(os.path.join(ROOT, "paged_kv_cache_477_b200", "csrc", n), "rb").read())
    return h.hexdigest()[:16]


def profiled_traffic(kernel_key: str, src_hash: str):
    """DRAM bytes per launch from a committed ncu summary, if the kernel source
    is unchanged since it was taken (else None)."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    d = json.load(open(p)).get(kernel_key)
    if not d or d.get("source_hash") != src_hash:
        return None
    return d.get("dram_bytes_per_launch")


# --------------------------------------------------------------------------- #
# clocks during the timed region                                               #
# --------------------------------------------------------------------------- #
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.idx = gpu_index
        self.proc = None
        self.path = None

    def __enter__(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.idx), f"--query-gpu={self.FIELDS}", "--format=csv,noheader",
                 "-lms", "200", "-f", self.path], stdout=subprocess.DEVNULL, stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *a):
        if self.proc is not None:
            time.sleep(0.25)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self):
        if not self.path or not os.path.exists(self.path):
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"]}
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1].split()[0]))
                smax.append(float(parts[2].split()[0]))
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        os.unlink(self.path)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(smax), "reasons": sorted(reasons),
                "samples": len(sm)}


# --------------------------------------------------------------------------- #
# algorithmic bytes / flops                                                    #
# --------------------------------------------------------------------------- #
def decode_bytes(case) -> int:
    kv = case.kv_bytes_read()
    qo = 2 * case.B * case.Hq * case.D * 2
    bt = sum(-(-L // case.bs) for L in case.lens) * 4 + case.B * 4
    return kv + qo + bt


def write_bytes(case) -> int:
    if case.new_key is None:
        return 0
    T = case.new_key.shape[0]
    return 2 * (2 * T * case.Hkv * case.D * 2) + T * 8


def prefill_flops(case) -> int:
    """4 * D per (query, visible key) per q head: QK^T and PV, 2 flop per MAC."""
    f = 0
    qsl = case.query_start_loc.cpu().tolist()
    for b in range(case.B):
        Q, L = qsl[b + 1] - qsl[b], case.lens[b]
        vis = sum(L - Q + i + 1 for i in range(Q))
        f += 4 * case.D * vis * case.Hq
    return f


# --------------------------------------------------------------------------- #
# multi-rank aggregation                                                       #
# --------------------------------------------------------------------------- #
def max_over_ranks(values, dist=None):
    """Element-wise maximum over all ranks: every device-timed figure is the
    slowest rank's.  Ranks call this in the same order (a collective)."""
    if dist is None:
        return list(values)
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor(list(values), dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def whole_job_rate(bytes_per_rank_step: int, world: int, ms_per_step: float) -> float:
    """GB/s of the whole job: every rank runs its own replica of the step, so
    the job moves world x the bytes in the slowest rank's step time."""
    return world * bytes_per_rank_step / (ms_per_step * 1e-3) / 1e9


# --------------------------------------------------------------------------- #
# the oracle on host cores                                                     #
# --------------------------------------------------------------------------- #
class OracleSample:
    """A bounded sample of the bench workload for the fp64 oracle: the first n
    of its sequences, n chosen so one oracle pass takes about `seconds`."""

    def __init__(self, seconds: float):
        import oracle
        from paged_kv_cache_477_b200 import workloads as wl
        self.orc = oracle.get()
        self.spec = wl.WORKLOADS[WORKLOAD]
        self.args, _ = self._case(1)
        t1 = self.run()
        self.n = int(max(1, min(self.spec["B"], seconds / max(t1, 1e-3))))
        self.args, self.nbytes = self._case(self.n)

    def _case(self, nseq):
        """Host arrays of the sample: (write args or None, attention args), bytes."""
        from paged_kv_cache_477_b200 import workloads as wl
        from paged_kv_cache_477_b200.workloads import bf16_bits
        sp = self.spec
        c = wl.make_case(B=nseq, Hq=sp["Hq"], Hkv=sp["Hkv"], D=sp["D"], bs=sp["bs"], lens=[sp["lens"][0]] * nseq,
                         seed=sp["seed"], device="cpu", write_tokens=sp.get("write_tokens", 0))
        k, v = bf16_bits(c.k_cache).copy(), bf16_bits(c.v_cache).copy()
        write = None
        if c.new_key is not None:
            write = (bf16_bits(c.new_key), bf16_bits(c.new_value), k, v, c.slot_mapping.numpy())
        attn = (bf16_bits(c.q), k, v, c.block_tables.numpy(), c.context_lens.numpy(), c.scale)
        return (write, attn), decode_bytes(c) + (write_bytes(c) if write is not None else 0)

    def run(self) -> float:
        """One step of the bench on the host: the cache write, then decode."""
        write, attn = self.args
        t0 = time.perf_counter()
        if write is not None:
            self.orc.kv_cache_write(*write)
        self.orc.paged_attention(*attn)
        return time.perf_counter() - t0

    def describe(self, reps: int, secs: float) -> str:
        sp = self.spec
        return (f"fp64 C oracle decode of {self.n} of the {sp['B']} sequences (ctx {sp['lens'][0]}, "
                f"{sp['Hq']} q / {sp['Hkv']} kv heads, D={sp['D']}) x {reps}, OpenMP on "
                f"{self.orc.num_threads()} threads, {secs:.1f} s")


def oracle_by_config():
    """The oracle on each workload the pages' configs name, on all host threads
    and (configs 1-3) on one: one pass each (best of 3 for the tiny case), wall
    clock.  Decode in GB/s of algorithmic bytes (cache write included where the
    workload has one), prefill in GFLOP/s; the tiny case also in microseconds."""
    import oracle
    from paged_kv_cache_477_b200 import workloads as wl
    from paged_kv_cache_477_b200.workloads import bf16_bits
    orc = oracle.get()
    cores = orc.num_threads()
    res = {"threads": cores}

    def decode_args(c):
        k, v = bf16_bits(c.k_cache).copy(), bf16_bits(c.v_cache).copy()
        write = None
        if c.new_key is not None:
            write = (bf16_bits(c.new_key), bf16_bits(c.new_value), k, v, c.slot_mapping.numpy())
        return write, (bf16_bits(c.q), k, v, c.block_tables.numpy(), c.context_lens.numpy(), c.scale)

    def run_decode(write, attn):
        t0 = time.perf_counter()
        if write is not None:
            orc.kv_cache_write(*write)
        orc.paged_attention(*attn)
        return time.perf_counter() - t0

    for cfg, name, one_core in (("1", "tiny_decode", True), ("2", "llama32_1b_decode", True),
                                ("3", WORKLOAD, True), ("4", "ragged_long_decode", False)):
        c = wl.workload(name, device="cpu")
        write, attn = decode_args(c)
        nb = decode_bytes(c) + write_bytes(c)
        entry = {}
        for label, threads in (("all_cores", cores), ("one_core", 1)):
            if label == "one_core" and not one_core:
                continue
            orc.set_num_threads(threads)
            reps = 3 if name == "tiny_decode" else 1
            t = min(run_decode(write, attn) for _ in range(reps))
            entry[label] = {"GB/s": round(nb / t / 1e9, 4), "s": round(t, 4)}
            if name == "tiny_decode":
                entry[label]["us"] = round(t * 1e6, 1)
        orc.set_num_threads(cores)
        res[f"config{cfg}_{name}"] = entry
        del c, write, attn
    c = wl.workload("chunked_prefill", device="cpu")
    k, v = bf16_bits(c.k_cache).copy(), bf16_bits(c.v_cache).copy()
    t0 = time.perf_counter()
    orc.kv_cache_write(bf16_bits(c.new_key), bf16_bits(c.new_value), k, v, c.slot_mapping.numpy())
    orc.paged_attention_prefill(bf16_bits(c.q), c.query_start_loc.numpy(), k, v, c.block_tables.numpy(),
                                c.context_lens.numpy(), c.scale)
    t = time.perf_counter() - t0
    res["config5_chunked_prefill"] = {"all_cores": {"GFLOP/s": round(prefill_flops(c) / t / 1e9, 3), "s": round(t, 2)}}
    return res


def oracle_decode_rate(seconds: float):
    """Oracle decode rate on the host cores, repeated passes over a bounded
    sample for about `seconds`.  Returns (GB/s, cores, sample description)."""
    smp = OracleSample(min(seconds, 5.0))
    t, reps = smp.run(), 1
    while t < seconds:
        t, reps = t + smp.run(), reps + 1
    return smp.nbytes * reps / t / 1e9, smp.orc.num_threads(), smp.describe(reps, t)


# --------------------------------------------------------------------------- #
# reference arm: the oracle, as it stands, on host cores                       #
# --------------------------------------------------------------------------- #
def run_reference(args, rank, world):
    """One step = one oracle pass over a bounded sample of the workload."""
    if rank != 0:
        return
    per_step = max(0.5, min(5.0, 120.0 / max(1, args.steps + args.warmup)))
    smp = OracleSample(per_step)
    for _ in range(args.warmup):
        smp.run()
    ts = [smp.run() for _ in range(args.steps)]
    secs = sum(ts)
    value = smp.nbytes * args.steps / secs / 1e9
    line = {
        "impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": "GB/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(secs / args.steps * 1e3, 3), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": f"{WORKLOAD} (bounded sample per step)", "parallelism": "host cores"},
        "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": smp.orc.num_threads(),
                         "kind": "oracle", "sample": smp.describe(args.steps, secs)},
        "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# --------------------------------------------------------------------------- #
# extras (after the timed region)                                              #
# --------------------------------------------------------------------------- #
def l2_flush_buffer():
    return torch.empty(256 << 20, dtype=torch.uint8, device="cuda")


def queue_ahead(ms: float = 5.0):
    """Keep the device busy for about `ms` so the host can queue the calls
    that follow; events around them then see device time only, not the
    host's launch overhead."""
    torch.cuda._sleep(int(ms * 2.0e6))  # ~2 GHz SM clock: cycles per ms


def time_calls(fn, iters, flush=None):
    """Per-call device times (ms): CUDA events on the current stream around
    each call, with every call queued before the first one runs."""
    st = torch.cuda.current_stream()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(iters)]
    queue_ahead()
    for e0, e1 in ev:
        if flush is not None:
            flush.zero_()
        e0.record(st)
        fn()
        e1.record(st)
    torch.cuda.synchronize()
    return [e0.elapsed_time(e1) for e0, e1 in ev]


def timed_us(fn, iters=50, flush=None):
    time_calls(fn, 3, flush)
    return statistics.median(time_calls(fn, iters, flush)) * 1e3


def extras(peaks, decode_gbs):
    import paged_kv_cache_477_b200 as pkv
    from paged_kv_cache_477_b200 import workloads as wl
    res = {}
    # read-only HBM stream (what decode does: reads K/V, writes ~nothing), 4 GiB
    buf = torch.empty(4 << 30, dtype=torch.uint8, device="cuda")
    sink = torch.empty(torch.cuda.get_device_properties(0).multi_processor_count * 2, dtype=torch.int32,
                       device="cuda")  # two CTAs per SM, 96 KB of chunks in flight each
    by_chunk = {}
    for chunk in (32768, 16384, 8192, 4096):
        us = timed_us(lambda: pkv.hbm_read_probe(buf, sink, chunk), 10)
        by_chunk[chunk] = buf.numel() / (us * 1e-6) / 1e9
    probe = max(by_chunk.values())
    res["hbm_read_probe"] = {"GB/s": round(probe, 1), "bytes": buf.numel(),
                             "GB/s_by_copy_bytes": {str(k): round(v, 1) for k, v in by_chunk.items()},
                             "in_flight": "96 KB per CTA, 2 CTAs per SM",
                             "headline_decode_frac_of_probe": round(decode_gbs / probe, 4),
                             "headline_decode_frac_of_8tbs_nominal": round(decode_gbs / 8000.0, 4)}
    del buf, sink
    torch.cuda.empty_cache()
    # the tiny parity case, warm (latency only)
    c = wl.workload("tiny_decode", device="cuda")
    us = timed_us(lambda: pkv.paged_attention(c.q, c.k_cache, c.v_cache, c.block_tables, c.context_lens,
                                              c.scale))
    res["tiny_decode"] = {"us": round(us, 2), "l2": "warm (70 KB of K/V)"}
    # cache writes of the headline step (128 new rows), plain and with RoPE on K
    c = wl.workload(WORKLOAD, device="cuda")
    T = c.new_key.shape[0]
    pos = c.context_lens.to(torch.int64) - 1
    for name, fn, nb in (
            ("kv_cache_write_128", lambda: pkv.kv_cache_write(c.new_key, c.new_value, c.k_cache, c.v_cache,
                                                              c.slot_mapping), write_bytes(c)),
            ("kv_cache_write_rope_128", lambda: pkv.kv_cache_write_rope(c.new_key, c.new_value, c.k_cache,
                                                                        c.v_cache, c.slot_mapping, pos, 500000.0),
             write_bytes(c) + 8 * T)):
        us = timed_us(fn)
        res[name] = {"us": round(us, 2), "GB/s": round(nb / (us * 1e-6) / 1e9, 1), "tokens": T, "bytes": nb,
                     "l2": "new rows warm in L2; rows scattered into a 2 GiB pool"}
    del c
    torch.cuda.empty_cache()
    for name, hint in (("llama32_1b_decode", 4096), ("ragged_long_decode", 32768), ("gqa8_decode", 4096)):
        c = wl.workload(name, device="cuda")
        out = torch.empty_like(c.q)
        ws = torch.empty(max(1, pkv.workspace_size(c.B, c.Hq, c.Hkv, c.D, c.MB, 16, hint)),
                         dtype=torch.uint8, device="cuda")
        fn = lambda: pkv.paged_attention(c.q, c.k_cache, c.v_cache, c.block_tables, c.context_lens, c.scale,
                                         out=out, max_context_len=hint, workspace=ws)
        time_calls(fn, 3)
        ts = time_calls(fn, 20)
        ms = statistics.median(ts)
        gbs = decode_bytes(c) / (ms * 1e-3) / 1e9
        res[name] = {"GB/s": round(gbs, 1), "us": round(ms * 1e3, 2), "frac_hbm": round(gbs / peaks["hbm_gbs"], 4),
                     "launches": pkv.last_launch_count(), "bytes": decode_bytes(c),
                     "l2": "inputs larger than L2"}
        del c, out, ws
        torch.cuda.empty_cache()
    # sliding window of 1024 keys over the Llama-3-8B-shaped batch (ctx 4096)
    c = wl.workload(WORKLOAD, device="cuda")
    out = torch.empty_like(c.q)
    W = 1024
    ws = torch.empty(max(1, pkv.window_workspace_size(c.B, c.Hq, c.Hkv, c.D, c.MB, 16, W)), dtype=torch.uint8,
                     device="cuda")
    fn = lambda: pkv.paged_attention_window(c.q, c.k_cache, c.v_cache, c.block_tables, c.context_lens, c.scale,
                                            W, out=out, workspace=ws)
    time_calls(fn, 3)
    ms = statistics.median(time_calls(fn, 20))
    wbytes = sum(min(L, W) for L in c.lens) * c.Hkv * c.D * 2 * 2 + 2 * c.B * c.Hq * c.D * 2 + \
        sum(-(-min(L, W) // 16) for L in c.lens) * 4 + c.B * 4
    gbs = wbytes / (ms * 1e-3) / 1e9
    res["llama3_8b_decode_window1024"] = {"GB/s": round(gbs, 1), "us": round(ms * 1e3, 2),
                                          "frac_hbm": round(gbs / peaks["hbm_gbs"], 4),
                                          "launches": pkv.last_launch_count(), "bytes": wbytes,
                                          "l2": "window pages of 128 x 8 heads: 512 MiB, larger than L2"}
    del c, out, ws
    torch.cuda.empty_cache()
    # INT8 cache (one fp32 scale per row): same shape as the headline step
    c = wl.workload("llama3_8b_decode_int8", device="cuda")
    pkv.kv_cache_write_int8(c.new_key, c.new_value, c.k_cache, c.v_cache, c.k_scale, c.v_scale, c.slot_mapping)
    out = torch.empty_like(c.q)
    ws = torch.empty(max(1, pkv.workspace_size(c.B, c.Hq, c.Hkv, c.D, c.MB, 16, 4096)), dtype=torch.uint8,
                     device="cuda")
    fn = lambda: pkv.paged_attention_int8(c.q, c.k_cache, c.v_cache, c.k_scale, c.v_scale, c.block_tables,
                                          c.context_lens, c.scale, out=out, max_context_len=4096, workspace=ws)
    time_calls(fn, 3)
    ms = statistics.median(time_calls(fn, 20))
    gbs = decode_bytes(c) / (ms * 1e-3) / 1e9
    res["llama3_8b_decode_int8"] = {"GB/s": round(gbs, 1), "us": round(ms * 1e3, 2),
                                    "frac_hbm": round(gbs / peaks["hbm_gbs"], 4), "launches": pkv.last_launch_count(),
                                    "bytes": decode_bytes(c), "kv_bytes_vs_bf16": 0.5 + 2.0 / c.D,
                                    "traffic": profiled_traffic("decode_attn_i8", source_hash(
                                        "decode_attn_i8.cuh", "decode_attn.cuh", "tcgen05.cuh", "pkv_common.cuh")),
                                    "l2": "inputs larger than L2"}
    # the same batch under a 1024-key sliding window
    W = 1024
    wsw = torch.empty(max(1, pkv.window_workspace_size(c.B, c.Hq, c.Hkv, c.D, c.MB, 16, W)), dtype=torch.uint8,
                      device="cuda")
    fnw = lambda: pkv.paged_attention_int8_window(c.q, c.k_cache, c.v_cache, c.k_scale, c.v_scale, c.block_tables,
                                                  c.context_lens, c.scale, W, out=out, workspace=wsw)
    us = timed_us(fnw, 20)
    wb = sum(min(L, W) for L in c.lens) * c.Hkv * (c.D + 4) * 2 + 2 * c.B * c.Hq * c.D * 2 + \
        sum(-(-min(L, W) // 16) for L in c.lens) * 4 + c.B * 4
    res["llama3_8b_decode_int8_window1024"] = {"GB/s": round(wb / (us * 1e-6) / 1e9, 1), "us": round(us, 2),
                                               "frac_hbm": round(wb / (us * 1e-6) / 1e9 / peaks["hbm_gbs"], 4),
                                               "launches": pkv.last_launch_count(), "bytes": wb,
                                               "l2": "window codes of 128 x 8 heads: 268 MiB, larger than L2"}
    del wsw
    T = c.new_key.shape[0]
    nb = 2 * T * c.Hkv * c.D * 2 + 2 * T * c.Hkv * (c.D + 4) + 8 * T
    us = timed_us(lambda: pkv.kv_cache_write_int8(c.new_key, c.new_value, c.k_cache, c.v_cache, c.k_scale,
                                                  c.v_scale, c.slot_mapping))
    res["kv_cache_write_int8_128"] = {"us": round(us, 2), "GB/s": round(nb / (us * 1e-6) / 1e9, 1), "tokens": T,
                                      "bytes": nb, "l2": "new rows warm in L2; rows scattered into the int8 pool"}
    del c, out, ws
    torch.cuda.empty_cache()
    # INT8 cache at the Llama-3.2-1B shape (D=64)
    c = wl.workload("llama32_1b_decode", device="cuda", kv_dtype="int8")
    out = torch.empty_like(c.q)
    ws = torch.empty(max(1, pkv.workspace_size(c.B, c.Hq, c.Hkv, c.D, c.MB, 16, 4096)), dtype=torch.uint8,
                     device="cuda")
    us = timed_us(lambda: pkv.paged_attention_int8(c.q, c.k_cache, c.v_cache, c.k_scale, c.v_scale, c.block_tables,
                                                   c.context_lens, c.scale, out=out, max_context_len=4096,
                                                   workspace=ws), 20)
    res["llama32_1b_decode_int8"] = {"GB/s": round(decode_bytes(c) / (us * 1e-6) / 1e9, 1), "us": round(us, 2),
                                     "frac_hbm": round(decode_bytes(c) / (us * 1e-6) / 1e9 / peaks["hbm_gbs"], 4),
                                     "launches": pkv.last_launch_count(), "bytes": decode_bytes(c),
                                     "l2": "inputs larger than L2"}
    del c, out, ws
    torch.cuda.empty_cache()
    # INT8 cache over the ragged long-context batch (split-KV through the int8 kernel)
    c = wl.workload("ragged_long_decode", device="cuda", kv_dtype="int8")
    out = torch.empty_like(c.q)
    ws = torch.empty(max(1, pkv.workspace_size(c.B, c.Hq, c.Hkv, c.D, c.MB, 16, 32768)), dtype=torch.uint8,
                     device="cuda")
    us = timed_us(lambda: pkv.paged_attention_int8(c.q, c.k_cache, c.v_cache, c.k_scale, c.v_scale, c.block_tables,
                                                   c.context_lens, c.scale, out=out, max_context_len=32768,
                                                   workspace=ws), 20)
    res["ragged_long_decode_int8"] = {"GB/s": round(decode_bytes(c) / (us * 1e-6) / 1e9, 1), "us": round(us, 2),
                                      "frac_hbm": round(decode_bytes(c) / (us * 1e-6) / 1e9 / peaks["hbm_gbs"], 4),
                                      "launches": pkv.last_launch_count(), "bytes": decode_bytes(c),
                                      "l2": "inputs larger than L2"}
    del c, out, ws
    torch.cuda.empty_cache()
    c = wl.workload("chunked_prefill", device="cuda")
    # the prefill's pre-step: the chunk's 2048 rows into the cache
    wfn = lambda: pkv.kv_cache_write(c.new_key, c.new_value, c.k_cache, c.v_cache, c.slot_mapping)
    us = timed_us(wfn)
    res["kv_cache_write_2048"] = {"us": round(us, 2), "GB/s": round(write_bytes(c) / (us * 1e-6) / 1e9, 1),
                                  "tokens": c.new_key.shape[0], "bytes": write_bytes(c),
                                  "l2": "new rows warm in L2"}
    out = torch.empty_like(c.q)
    fn = lambda: pkv.paged_attention_prefill(c.q, c.query_start_loc, c.k_cache, c.v_cache, c.block_tables,
                                             c.context_lens, c.scale, c.max_q_len, out=out)
    try:
        flush = l2_flush_buffer()
        time_calls(fn, 3, flush)
        ts = time_calls(fn, 20, flush)
        ms = statistics.median(ts)
        tf = prefill_flops(c) / (ms * 1e-3) / 1e12
        res["chunked_prefill"] = {"TFLOP/s": round(tf, 1), "us": round(ms * 1e3, 2),
                                  "frac_bf16_burst": round(tf / peaks["bf16_tflops"], 4),
                                  "frac_bf16_nominal_2250": round(tf / 2250.0, 4),
                                  "flops": prefill_flops(c), "l2": "flushed (256 MiB write) before each call"}
        us = timed_us(fn, 20)
        res["chunked_prefill_warm"] = {"TFLOP/s": round(prefill_flops(c) / (us * 1e-6) / 1e12, 1),
                                       "us": round(us, 2), "l2": "warm (no flush between calls)"}
        # the same chunks at head size 64 (Llama-3.2-1B's), 32 q / 8 kv heads
        del c, out
        c = wl.workload("chunked_prefill", device="cuda", D=64)
        pkv.kv_cache_write(c.new_key, c.new_value, c.k_cache, c.v_cache, c.slot_mapping)
        out = torch.empty_like(c.q)
        fn = lambda: pkv.paged_attention_prefill(c.q, c.query_start_loc, c.k_cache, c.v_cache, c.block_tables,
                                                 c.context_lens, c.scale, c.max_q_len, out=out)
        us = timed_us(fn, 20, flush)
        tf = prefill_flops(c) / (us * 1e-6) / 1e12
        res["chunked_prefill_d64"] = {"TFLOP/s": round(tf, 1), "us": round(us, 2),
                                      "frac_bf16_burst": round(tf / peaks["bf16_tflops"], 4),
                                      "flops": prefill_flops(c), "l2": "flushed (256 MiB write) before each call"}
    except pkv.PagedKVError as e:
        res["chunked_prefill"] = {"unavailable": str(e)}
    return res


# --------------------------------------------------------------------------- #
# main arm                                                                     #
# --------------------------------------------------------------------------- #
def profile_case(kind: str, launches: int = 3):
    """A few launches of one kernel on a case small enough for a full ncu
    capture (a few GB on the device at most, inputs still larger than L2)."""
    import paged_kv_cache_477_b200 as pkv
    from paged_kv_cache_477_b200 import workloads as wl
    torch.cuda.set_device(0)
    if kind == "decode_full":
        # the bench's own decode launch (Llama-3-8B-shaped, B=128): 2 GiB of K/V
        c = wl.workload(WORKLOAD, device="cuda")
        out = torch.empty_like(c.q)
        ws = torch.empty(max(1, pkv.workspace_size(c.B, c.Hq, c.Hkv, c.D, c.MB, 16, 4096)), dtype=torch.uint8,
                         device="cuda")
        for _ in range(launches):
            pkv.paged_attention(c.q, c.k_cache, c.v_cache, c.block_tables, c.context_lens, c.scale, out=out,
                                max_context_len=4096, workspace=ws)
    elif kind == "decode_gqa8":
        # eight query heads per kv head (64 q / 8 kv heads, D=128, ctx 4096): 1 GiB of K/V
        c = wl.workload("gqa8_decode", device="cuda")
        out = torch.empty_like(c.q)
        for _ in range(launches):
            pkv.paged_attention(c.q, c.k_cache, c.v_cache, c.block_tables, c.context_lens, c.scale, out=out,
                                max_context_len=4096)
    elif kind == "decode_d64":
        # the Llama-3.2-1B-shaped decode (D=64): 300 MB of K/V
        c = wl.workload("llama32_1b_decode", device="cuda")
        out = torch.empty_like(c.q)
        for _ in range(launches):
            pkv.paged_attention(c.q, c.k_cache, c.v_cache, c.block_tables, c.context_lens, c.scale, out=out,
                                max_context_len=4096)
    elif kind == "decode_ragged":
        # the ragged long-context batch (4 x 32768 + 12 shorter, split-KV + merge): 620 MB of K/V
        c = wl.workload("ragged_long_decode", device="cuda")
        out = torch.empty_like(c.q)
        ws = torch.empty(max(1, pkv.workspace_size(c.B, c.Hq, c.Hkv, c.D, c.MB, 16, 32768)), dtype=torch.uint8,
                         device="cuda")
        for _ in range(launches):
            pkv.paged_attention(c.q, c.k_cache, c.v_cache, c.block_tables, c.context_lens, c.scale, out=out,
                                max_context_len=32768, workspace=ws)
    elif kind == "decode_int8_full":
        # the bench's Llama-3-8B-shaped INT8 decode, full size: 1.1 GB of codes and scales
        c = wl.workload("llama3_8b_decode_int8", device="cuda")
        out = torch.empty_like(c.q)
        for _ in range(launches):
            pkv.paged_attention_int8(c.q, c.k_cache, c.v_cache, c.k_scale, c.v_scale, c.block_tables,
                                     c.context_lens, c.scale, out=out, max_context_len=4096)
    elif kind == "decode_int8":
        # 32 of the Llama-3-8B-shaped sequences over the INT8 cache: 264 MiB of codes and scales
        c = wl.make_case(B=32, Hq=32, Hkv=8, D=128, bs=16, lens=[4096] * 32, seed=1006, device="cuda",
                         kv_dtype="int8")
        out = torch.empty_like(c.q)
        for _ in range(launches):
            pkv.paged_attention_int8(c.q, c.k_cache, c.v_cache, c.k_scale, c.v_scale, c.block_tables,
                                     c.context_lens, c.scale, out=out, max_context_len=4096)
    elif kind in ("decode", "split", "write"):
        # 32 of the Llama-3-8B-shaped sequences: 512 MiB of K/V
        c = wl.make_case(B=32, Hq=32, Hkv=8, D=128, bs=16, lens=[4096] * 32, seed=1003, device="cuda",
                         write_tokens=1)
        out = torch.empty_like(c.q)
        for _ in range(launches):
            if kind == "write":
                pkv.kv_cache_write(c.new_key, c.new_value, c.k_cache, c.v_cache, c.slot_mapping)
            elif kind == "decode":
                pkv.paged_attention(c.q, c.k_cache, c.v_cache, c.block_tables, c.context_lens, c.scale,
                                    out=out, max_context_len=4096)
            else:
                pkv.paged_attention_split(c.q, c.k_cache, c.v_cache, c.block_tables, c.context_lens,
                                          c.scale, pages_per_split=32, out=out, max_context_len=4096)
    else:
        c = wl.workload("chunked_prefill", device="cuda")
        pkv.kv_cache_write(c.new_key, c.new_value, c.k_cache, c.v_cache, c.slot_mapping)
        out = torch.empty_like(c.q)
        for _ in range(launches):
            pkv.paged_attention_prefill(c.q, c.query_start_loc, c.k_cache, c.v_cache, c.block_tables,
                                        c.context_lens, c.scale, c.max_q_len, out=out)
    torch.cuda.synchronize()
    assert pkv.get_device_error() == 0
    print(f"profile case {kind}: ok")


def main():
    args = parse()
    if args.profile:
        profile_case(args.profile)
        return
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, rank, world)
        return
    assert args.warmup >= 3, "at least 3 warm-up steps"
    torch.cuda.set_device(local)
    dist = None
    if world > 1:
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))

    import paged_kv_cache_477_b200 as pkv
    from paged_kv_cache_477_b200 import workloads as wl

    pkv.load_library()
    peaks = measured_peaks()
    case = wl.workload(WORKLOAD, device="cuda")
    hint = max(case.lens)
    out = torch.empty_like(case.q)
    ws_bytes = pkv.workspace_size(case.B, case.Hq, case.Hkv, case.D, case.MB, case.bs, hint)
    ws = torch.empty(max(ws_bytes, 1), dtype=torch.uint8, device="cuda")
    st = torch.cuda.current_stream()

    def step():
        pkv.kv_cache_write(case.new_key, case.new_value, case.k_cache, case.v_cache, case.slot_mapping)
        n = pkv.last_launch_count()
        pkv.paged_attention(case.q, case.k_cache, case.v_cache, case.block_tables, case.context_lens,
                            case.scale, out=out, max_context_len=hint, workspace=ws)
        return n + pkv.last_launch_count()

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    assert pkv.get_device_error() == 0

    # ---- timed region: K steps, events around the attention launches ----------
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    launches = 0
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(torch.cuda.current_device()) as clk:
        queue_ahead()
        t0.record(st)
        for i in range(args.steps):
            pkv.kv_cache_write(case.new_key, case.new_value, case.k_cache, case.v_cache, case.slot_mapping)
            launches += pkv.last_launch_count()
            ev[i][0].record(st)
            pkv.paged_attention(case.q, case.k_cache, case.v_cache, case.block_tables, case.context_lens,
                                case.scale, out=out, max_context_len=hint, workspace=ws)
            launches += pkv.last_launch_count()
            ev[i][1].record(st)
        t1.record(st)
        torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    elapsed_ms = t0.elapsed_time(t1)
    attn_each = sorted(a.elapsed_time(b) for a, b in ev)
    attn_ms = statistics.mean(attn_each)
    clocks = clk.summary()
    attn_launches = pkv.last_launch_count()
    assert pkv.get_device_error() == 0

    # ---- end to end through the public API with host buffers -----------------
    # Every step copies its own inputs from pinned host memory and reads its
    # result back, double-buffered as a serving loop runs: step i+1's inputs
    # cross on a copy stream while step i computes, and step i's output
    # returns on that stream while step i+1 runs.  The events bracket both
    # streams (the copy stream starts after the first event; the last event
    # follows the last read-back).
    names = ("q", "new_key", "new_value", "slot_mapping", "block_tables", "context_lens")
    host_in = [{k: getattr(case, k).cpu().pin_memory() for k in names} for _ in range(2)]
    dev_in = [{k: torch.empty_like(getattr(case, k)) for k in names} for _ in range(2)]
    dev_out = [torch.empty_like(out) for _ in range(2)]
    host_out = [torch.empty(out.shape, dtype=out.dtype, pin_memory=True) for _ in range(2)]
    h2d = sum(t.numel() * t.element_size() for t in host_in[0].values())
    d2h = host_out[0].numel() * host_out[0].element_size()
    cs = torch.cuda.Stream()
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_done = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]

    def h2d_copy(b):
        with torch.cuda.stream(cs):
            cs.wait_event(ev_done[b])  # the step that last read these buffers has computed
            for k in names:
                dev_in[b][k].copy_(host_in[b][k], non_blocking=True)
            ev_in[b].record(cs)

    def compute(b):
        st.wait_event(ev_in[b])
        st.wait_event(ev_out[b])  # the last read-back of this output buffer is done
        pkv.kv_cache_write(dev_in[b]["new_key"], dev_in[b]["new_value"], case.k_cache, case.v_cache,
                           dev_in[b]["slot_mapping"])
        pkv.paged_attention(dev_in[b]["q"], case.k_cache, case.v_cache, dev_in[b]["block_tables"],
                            dev_in[b]["context_lens"], case.scale, out=dev_out[b], max_context_len=hint,
                            workspace=ws)
        ev_done[b].record(st)
        with torch.cuda.stream(cs):
            cs.wait_event(ev_done[b])
            host_out[b].copy_(dev_out[b], non_blocking=True)
            ev_out[b].record(cs)

    def e2e_run(n, e0=None, e1=None):
        if e0 is not None:
            e0.record(st)
            cs.wait_event(e0)
        h2d_copy(0)
        for i in range(n):
            if i + 1 < n:
                h2d_copy((i + 1) % 2)
            compute(i % 2)
        if e1 is not None:
            st.wait_event(ev_out[(n - 1) % 2])
            e1.record(st)
        torch.cuda.synchronize()

    e2e_run(3)
    if dist is not None:
        dist.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e2e_run(args.steps, e0, e1)
    e2e_ms = e0.elapsed_time(e1)
    assert pkv.get_device_error() == 0

    step_bytes = decode_bytes(case) + write_bytes(case)
    attn_bytes = decode_bytes(case)
    elapsed_ms, e2e_ms = max_over_ranks([elapsed_ms, e2e_ms], dist)

    if rank == 0:
        ms_step = elapsed_ms / args.steps
        value = whole_job_rate(step_bytes, world, ms_step)
        e2e_val = whole_job_rate(step_bytes, world, e2e_ms / args.steps)
        achieved = attn_bytes / (attn_ms * 1e-3) / 1e9
        src = source_hash("decode_attn.cuh", "pkv_common.cuh")
        line = {
            "metric": METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_step, 4),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic",
            "config": {"workload": wl.describe(WORKLOAD), "step": "kv_cache_write (128 rows) + paged_attention",
                       "bytes_per_step": step_bytes,
                       "l2": "inputs larger than L2: 2 GiB of K/V read per step, no flush needed",
                       "parallelism": f"replicas{world}" if world > 1 else "single GPU"},
            "roofline": {"bound": "hbm", "kernel": "decode_attn" + (" + lse_merge" if attn_launches == 2 else ""),
                         "achieved": round(achieved, 1), "peak": peaks["hbm_gbs"], "unit": "GB/s",
                         "frac": round(achieved / peaks["hbm_gbs"], 4), "peak_source": peaks["source"],
                         "bytes_per_launch": attn_bytes, "us_per_launch": round(attn_ms * 1e3, 2),
                         "us_per_launch_spread": {"min": round(attn_each[0] * 1e3, 2),
                                                  "median": round(statistics.median(attn_each) * 1e3, 2),
                                                  "max": round(attn_each[-1] * 1e3, 2), "n": len(attn_each)},
                         "traffic": profiled_traffic("decode_attn", src)},
            "e2e": {"value": round(e2e_val, 2), "unit": "GB/s", "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h, "how": "pinned host buffers, each step's inputs copied in "
                    "and its output read back; steps double-buffered over a copy stream"},
            "gpu_launches": launches,
            "clocks": clocks,
        }
        if not args.no_extras and world == 1:
            line["extras"] = extras(peaks, achieved)
        if world == 1:
            v, cores, desc = oracle_decode_rate(args.cpu_seconds)
            line["cpu_baseline"] = {"value": round(v, 4), "unit": "GB/s", "cores": cores, "kind": "oracle",
                                    "sample": desc}
            if "extras" in line:
                import oracle
                oracle.get().set_num_threads(1)
                v1, _, desc1 = oracle_decode_rate(min(4.0, args.cpu_seconds))
                oracle.get().set_num_threads(cores)
                line["extras"]["oracle_one_core"] = {"value": round(v1, 4), "unit": "GB/s", "sample": desc1}
                line["extras"]["oracle_by_config"] = oracle_by_config()
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
