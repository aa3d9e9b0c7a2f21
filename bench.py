#!/usr/bin/env python
"""Throughput benchmark of the grouped-query attention hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One step = one pass of the whole hot path over one batch of synthetic input:
  1. causal prefill, B=1, Hq=32, Hkv=8, T=4096, d=128 (Llama-3-8B head
     shapes), bf16 in/out, fp32 accumulation -- the headline workload;
  2. batched decode, B=64 sequences, Hq=32, Hkv=8, d=128, cache lengths
     uniform on [1024, 8192], split-KV kernel whose last split per group
     merges the splits (log-sum-exp).
Inputs are seeded synthetic tensors already resident in HBM.  L2 (126 MB) is
flushed before every timed launch by writing a 256 MB buffer and reading it
back (so no dirty lines are left for the timed kernel to write back); each
launch is timed with CUDA events on the stream it runs on.

The JSON line's ``value`` is prefill TFLOP/s (algorithmic FLOPs: 4*B*Hq*d*
unmasked pairs, all ranks) and ``decode.value`` is decode KV GB/s.  ``e2e``
repeats the prefill through the host-buffer entry point (pinned q/k/v in, o
out, the copies inside the call and the timed region).
``cpu_baseline`` times the CPU oracle on a sample of query rows of the same
workload.  With --gpus N > 1 (torchrun) every rank runs its own copy of the
workload (the path has no exchange step): weak scaling, time = max over ranks.

``--impl reference`` times the CPU oracle instead (rank 0 only), on bounded
samples of the same workload, and prints the same metric.
"""

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "GQA prefill TFLOP/s and decode KV GB/s on 1 B200 (% of roofline)"
PREFILL = dict(B=1, Hq=32, Hkv=8, T=4096, d=128, causal=True)
DECODE = dict(B=64, Hq=32, Hkv=8, d=128, Lmin=1024, Lmax=8192)
WORKLOAD = "prefill_causal_llama3_8b_t4096 + decode_b64_l1024_8192"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "traffic.txt")


def prefill_flops(c):
    pairs = c["T"] * (c["T"] + 1) // 2 if c["causal"] else c["T"] * c["T"]
    return 4 * c["B"] * c["Hq"] * c["d"] * pairs


def decode_bytes(seqlens, c):
    kv = int(seqlens.sum()) * c["Hkv"] * c["d"] * 2 * 2
    return kv + 2 * c["B"] * c["Hq"] * c["d"] * 2          # + q and o


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return p, "measured"
    except (OSError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


def kernel_source_hash(names):
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "grouped_query_attention_attn_b200", "csrc")
    for n in names:
        with open(os.path.join(csrc, n), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def recorded_traffic(kernel, src_hash):
    """DRAM bytes per launch from the committed ncu summary, if the kernel is unchanged.

    profiles/traffic.txt lines: <kernel> <source sha256[:16]> <dram read+write bytes>."""
    try:
        with open(TRAFFIC_FILE) as f:
            for line in f:
                parts = line.split()
                if len(parts) == 3 and parts[0] == kernel and parts[1] == src_hash:
                    return int(parts[2])
    except OSError:
        pass
    return None


class ClockSampler:
    """SM clock and throttle reasons sampled while a timed region runs.

    A background thread polls NVML (read-only queries) every ``period_s``, so
    even a region of a few milliseconds gets samples; without NVML it falls back
    to ``nvidia-smi -lms``.  ``stop()`` returns the median SM clock under load,
    the maximum SM clock, the sample count and every throttle reason seen."""

    REASONS = (("hw_slowdown", "nvmlClocksEventReasonHwSlowdown"),
               ("hw_thermal_slowdown", "nvmlClocksEventReasonHwThermalSlowdown"),
               ("sw_thermal_slowdown", "nvmlClocksEventReasonSwThermalSlowdown"),
               ("sw_power_cap", "nvmlClocksEventReasonSwPowerCap"))

    def __init__(self, device, period_s=0.001):
        import threading
        self.period_s = period_s
        self.samples, self.reasons, self.smax = [], set(), None
        self.stop_evt = threading.Event()
        self.thread = None
        self.handle = None
        self.proc = None
        try:
            self.uuid = "GPU-" + str(torch.cuda.get_device_properties(device).uuid)
        except Exception:
            self.uuid = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nvml = pynvml
            self.handle = pynvml.nvmlDeviceGetHandleByUUID(self.uuid.encode()) if self.uuid \
                else pynvml.nvmlDeviceGetHandleByIndex(torch.cuda.current_device())
            self.smax = float(pynvml.nvmlDeviceGetMaxClockInfo(self.handle, pynvml.NVML_CLOCK_SM))
        except Exception:
            self.handle = None

    def _poll(self):
        nv, h = self.nvml, self.handle
        masks = [(name, getattr(nv, attr, 0)) for name, attr in self.REASONS]
        while not self.stop_evt.is_set():
            try:
                self.samples.append(float(nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)))
                bits = nv.nvmlDeviceGetCurrentClocksEventReasons(h)
                for name, m in masks:
                    if m and bits & m:
                        self.reasons.add(name)
            except Exception:
                pass
            self.stop_evt.wait(self.period_s)

    def start(self):
        if self.handle is not None:
            import threading
            # the launch loop holds the GIL between launches: switch threads
            # every 0.1 ms so the poller runs during a short timed region
            self.old_switch = sys.getswitchinterval()
            sys.setswitchinterval(1e-4)
            self.thread = threading.Thread(target=self._poll, daemon=True)
            self.thread.start()
            return
        fields = ("clocks.sm,clocks.max.sm,clocks_event_reasons.hw_slowdown,"
                  "clocks_event_reasons.hw_thermal_slowdown,"
                  "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
        cmd = ["nvidia-smi", f"--query-gpu={fields}", "--format=csv,noheader,nounits", "-lms", "10"]
        if self.uuid:
            cmd += ["-i", self.uuid]
        try:
            self.proc = subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.DEVNULL,
                                         text=True)
        except OSError:
            self.proc = None

    def stop(self):
        if self.thread is not None:
            self.stop_evt.set()
            self.thread.join(timeout=5)
            sys.setswitchinterval(self.old_switch)
            src = "nvml"
        elif self.proc is not None:
            self.proc.terminate()
            out, _ = self.proc.communicate(timeout=10)
            names = [n for n, _ in self.REASONS]
            for line in out.strip().splitlines():
                parts = [x.strip() for x in line.split(",")]
                if len(parts) < 6:
                    continue
                try:
                    self.samples.append(float(parts[0]))
                    self.smax = float(parts[1])
                except ValueError:
                    continue
                for n, v in zip(names, parts[2:6]):
                    if v.lower().startswith("active"):
                        self.reasons.add(n)
            src = "nvidia-smi"
        else:
            return {"sm_mhz": None, "sm_max_mhz": None, "samples": 0,
                    "reasons": ["no clock source"]}
        sm = self.samples
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": self.smax,
                "sm_min_mhz": min(sm) if sm else None, "samples": len(sm),
                "reasons": sorted(self.reasons), "source": src}


def dist_init(n_gpus):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != n_gpus and world > 1:
        raise SystemExit(f"--gpus {n_gpus} but WORLD_SIZE={world}")
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x, world, device):
    if world == 1:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ------------------------------------------------------------ CPU oracle --

def oracle_prefill_sample(q, k, v, n_rows, seed=0):
    """Time the oracle on n_rows query rows of the prefill workload.

    Returns (seconds, algorithmic FLOPs of the rows, rows, outputs)."""
    import numpy as np
    from oracle import ref
    B, T, Hq, d = q.shape
    rng = np.random.default_rng(seed)
    rows = np.sort(rng.choice(B * Hq * T, size=n_rows, replace=False)).astype(np.int64)
    pos = rows % T
    flops = int(4 * d * (pos + 1).sum())                # causal: row i sees i+1 keys
    t = time.perf_counter()
    o, lse = ref.attn_fwd_rows(q, k, v, rows, causal=True)
    return time.perf_counter() - t, flops, rows, o


def calibrate_row_seconds(q, k, v, n=256):
    """Oracle seconds per random query row of the prefill workload."""
    secs, _, _, _ = oracle_prefill_sample(q, k, v, n, seed=12345)
    return max(secs / n, 1e-7)


def run_reference(args, world, rank):
    """The CPU oracle as the reference arm: rank 0 only, bounded samples."""
    if rank != 0:
        return
    from grouped_query_attention_attn_b200 import workloads
    from oracle import ref
    c = PREFILL
    q, k, v = workloads.prefill_inputs(c["B"], c["T"], c["Hq"], c["Hkv"], c["d"])
    ref.build_oracle()
    for i in range(args.warmup):
        oracle_prefill_sample(q, k, v, 64, seed=1000 + i)
    # rows per step sized so that all K steps take about args.ref_budget seconds
    per_row = calibrate_row_seconds(q, k, v)
    rows = int(min(max(args.ref_budget / args.steps / per_row, 16), c["B"] * c["Hq"] * c["T"]))
    secs, flops = 0.0, 0
    for i in range(args.steps):
        s, f, _, _ = oracle_prefill_sample(q, k, v, rows, seed=i)
        secs += s
        flops += f
    value = flops / secs / 1e12
    cores = ref.num_threads()
    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1000 * secs / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "impl": "reference",
        "config": {"workload": WORKLOAD, "prefill": c, "decode": DECODE,
                   "l2": "flushed before every timed launch (256 MB written, then read back: clean lines)",
                   "parallelism": "1 GPU"},
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                         "sample": f"{rows} random query rows of the causal T=4096 "
                                   f"prefill per step (C double oracle, OpenMP)"},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------- GPU path --

def visible_pairs(Tq, Tkv, causal=True, window=0, sinks=0):
    """Exact number of (query, key) pairs the mask leaves visible."""
    import numpy as np
    p = np.arange(Tq, dtype=np.int64) + (Tkv - Tq)
    if not causal:
        return Tq * Tkv
    n = np.clip(p + 1, 0, Tkv)
    if window > 0:
        lo = np.maximum(p - window + 1, 0)
        n = np.clip(np.minimum(p + 1, window), 0, Tkv) + np.minimum(sinks, lo)
    return int(n.sum())


class L2Flush:
    """Flushes L2 (126 MB) before a timed launch: writes a 256 MB buffer, then reads
    it back.  The read leaves L2 holding clean lines only, so the timed kernel does
    not pay for writing back the flush's dirty lines (a write-only flush left ~126 MB
    of them, which added ~15 us to the DRAM-bound decode and nothing to the prefill)."""

    def __init__(self, dev, nbytes=256 * 1024 * 1024):
        self.buf = torch.empty(nbytes, dtype=torch.uint8, device=dev)

    def __call__(self):
        self.buf.zero_()
        # read as fp32: one reduction over the 256 MB, no widening copy of the bytes
        return self.buf.view(torch.float32).sum()


def time_median(fn, flush, stream, reps):
    """Median CUDA-event time (ms) of fn() with L2 flushed before each launch."""
    for _ in range(3):
        fn()
    ts = []
    for _ in range(reps):
        flush()
        s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s0.record(stream)
        fn()
        s1.record(stream)
        torch.cuda.synchronize()
        ts.append(s0.elapsed_time(s1))
    return statistics.median(ts)


SWEEP = dict(B=4, Hq=32, T=2048, d=128, causal=True)          # Hkv in {32, 8, 1}
LONG = dict(B=1, Hq=64, Hkv=8, T=32768, d=128, causal=True, qk_std=8.0)
NEXT_ROWS = ("prefill_sweep_hkv32", "prefill_sweep_hkv8", "prefill_sweep_hkv1",
             "prefill_long_t32768", "prefill_window", "backward", "rope_qk", "prefill_rope_fused",
             "fold_kv", "decode_window", "decode_rope_fused")


def measure_next_rows(dev, stream, flush, peaks, peak_kind, reps, which=None):
    """Throughput of the other prefill workloads and of the rows built after the
    hot path, each on its own workload; ``which`` selects rows by name."""
    import grouped_query_attention_attn_b200 as gqa
    from grouped_query_attention_attn_b200 import workloads
    want = set(NEXT_ROWS if not which else which)

    def tensor_row(flops, ms, cfg):
        a = flops / (ms / 1e3) / 1e12
        return {"value": a, "unit": "TFLOP/s", "ms": ms, "config": cfg,
                "roofline": {"bound": "tensor", "achieved": a, "peak": peaks["bf16_tflops"],
                             "unit": "TFLOP/s", "frac": a / peaks["bf16_tflops"],
                             "frac_of_nominal_2250": a / 2250.0,
                             "peak_kind": f"{peak_kind} bf16 burst", "flops_per_launch": flops}}

    def hbm_row(nbytes, ms, cfg):
        a = nbytes / (ms / 1e3) / 1e9
        return {"value": a, "unit": "GB/s", "ms": ms, "config": cfg,
                "roofline": {"bound": "hbm", "achieved": a, "peak": peaks["hbm_gbs"],
                             "unit": "GB/s", "frac": a / peaks["hbm_gbs"],
                             "peak_kind": f"{peak_kind} copy", "bytes_per_launch": nbytes}}

    out = {}
    sampler = ClockSampler(dev)
    sampler.start()
    # the same-weights head-sharing sweep: one q, the Hkv=32 K/V and its GPU
    # folds to 8 and 1 heads; the FLOPs do not depend on Hkv
    if want & {"prefill_sweep_hkv32", "prefill_sweep_hkv8", "prefill_sweep_hkv1"}:
        c = SWEEP
        q, k32, v32 = (t.to(dev) for t in workloads.prefill_inputs(c["B"], c["T"], c["Hq"],
                                                                   32, c["d"]))
        o = torch.empty_like(q)
        flops = 4 * c["B"] * c["Hq"] * c["d"] * visible_pairs(c["T"], c["T"])
        for hkv in (32, 8, 1):
            name = f"prefill_sweep_hkv{hkv}"
            if name not in want:
                continue
            k, v = (k32, v32) if hkv == 32 else (gqa.fold_kv(k32, hkv), gqa.fold_kv(v32, hkv))
            ms = time_median(lambda: gqa.attn(q, k, v, causal=True, out=o), flush, stream, reps)
            out[name] = tensor_row(flops, ms, dict(c, Hkv=hkv, G=c["Hq"] // hkv,
                                                   kv="fold_kv of the Hkv=32 K/V"))
        del q, k32, v32, o
    # long-context causal prefill with q, k x 8 (logits of sigma ~ 64)
    if "prefill_long_t32768" in want:
        c = LONG
        q, k, v = (t.to(dev) for t in workloads.prefill_inputs(c["B"], c["T"], c["Hq"], c["Hkv"],
                                                              c["d"], qk_std=c["qk_std"]))
        o = torch.empty_like(q)
        ms = time_median(lambda: gqa.attn(q, k, v, causal=True, out=o), flush, stream,
                         max(3, reps // 4))
        out["prefill_long_t32768"] = tensor_row(
            4 * c["Hq"] * c["d"] * visible_pairs(c["T"], c["T"]), ms, c)
        del q, k, v, o
    # sliding window + sinks prefill (Mistral-like window over a long prompt)
    if "prefill_window" in want:
        cw = dict(B=1, Hq=32, Hkv=8, T=16384, d=128, window=4096, sinks=4)
        q, k, v = (t.to(dev) for t in workloads.prefill_inputs(1, cw["T"], cw["Hq"], cw["Hkv"],
                                                              128, seeds=(11, 12, 13)))
        o = torch.empty_like(q)
        ms = time_median(lambda: gqa.attn(q, k, v, causal=True, out=o, window=cw["window"],
                                          sinks=cw["sinks"]), flush, stream, reps)
        flops = 4 * cw["Hq"] * 128 * visible_pairs(cw["T"], cw["T"], True, cw["window"],
                                                   cw["sinks"])
        out["prefill_window"] = tensor_row(flops, ms, cw)
        del q, k, v, o
    # backward and RoPE on the headline prefill workload
    if want & {"backward", "rope_qk", "prefill_rope_fused"}:
        c = PREFILL
        q, k, v = (t.to(dev) for t in workloads.prefill_inputs(1, c["T"], c["Hq"], c["Hkv"], 128))
        if "backward" in want:
            do = workloads.randn((1, c["T"], c["Hq"], 128), 77).to(dev)
            o, lse = gqa.attn(q, k, v, causal=True, return_lse=True)
            ws = torch.empty(int(gqa._binding.gqa_attn_bwd_workspace_size(1, c["T"], c["Hq"])),
                             dtype=torch.uint8, device=dev)
            ms = time_median(lambda: gqa.attn_bwd(q, k, v, o, lse, do, workspace=ws), flush,
                             stream, reps)
            out["backward"] = tensor_row(10 * c["Hq"] * 128 * visible_pairs(c["T"], c["T"]), ms,
                                         dict(c, kernels="rowdot + dkdv (tcgen05) + dq (tcgen05)"))
            del o, lse, do, ws
        if "rope_qk" in want:
            # q and k rotated in place (read + write)
            ms = time_median(lambda: gqa.rope_qk_(q, k, 0), flush, stream, reps)
            out["rope_qk"] = hbm_row(2 * (q.numel() + k.numel()) * 2, ms, dict(c, theta=10000.0))
        if "prefill_rope_fused" in want:
            # rotary embedding + attention: k rotated once (as when it enters the
            # cache) and q rotated inside the prefill as its tiles are loaded,
            # against rotating q and k in one launch and then the plain prefill
            o = torch.empty_like(q)
            ms_f = time_median(lambda: (gqa.rope_(k, 0),
                                        gqa.attn(q, k, v, causal=True, out=o, rope_theta=10000.0)),
                               flush, stream, reps)
            ms_u = time_median(lambda: (gqa.rope_qk_(q, k, 0), gqa.attn(q, k, v, causal=True, out=o)),
                               flush, stream, reps)
            row = tensor_row(prefill_flops(c), ms_f, dict(c, theta=10000.0,
                                                          launches="rope(k) + prefill(rope q)"))
            row["unfused_ms"] = ms_u
            row["unfused"] = "rope_qk(q, k) + prefill"
            out["prefill_rope_fused"] = row
            del o
        del q, k, v
    # MHA -> GQA fold of the head-sharing sweep's K (32 -> 8 heads)
    if "fold_kv" in want:
        kv = workloads.randn((4, 2048, 32, 128), 2).to(dev)
        ms = time_median(lambda: gqa.fold_kv(kv, 8), flush, stream, reps)
        out["fold_kv"] = hbm_row(kv.numel() * 2 + kv.numel() // 4 * 2, ms,
                                 dict(B=4, T=2048, H=32, g=8, d=128))
        del kv
    # sliding-window decode on the batched-decode workload
    if "decode_window" in want:
        dc = DECODE
        dq_, kc, vc, sl = workloads.decode_inputs(dc["B"], dc["Hq"], dc["Hkv"], dc["d"],
                                                  dc["Lmin"], dc["Lmax"])
        W, S = 2048, 4
        rows = sum(min(int(L), W) + min(S, max(0, int(L) - W)) for L in sl)
        nbytes = rows * dc["Hkv"] * dc["d"] * 4 + 2 * dc["B"] * dc["Hq"] * dc["d"] * 2
        dq_, kc, vc, sl = dq_.to(dev), kc.to(dev), vc.to(dev), sl.to(dev)
        ws = torch.empty(gqa.decode_workspace_size(dc["B"], dc["Hq"], dc["Hkv"], dc["d"],
                                                   dc["Lmax"]), dtype=torch.uint8, device=dev)
        ms = time_median(lambda: gqa.decode(dq_, kc, vc, sl, workspace=ws, window=W, sinks=S),
                         flush, stream, reps)
        out["decode_window"] = hbm_row(nbytes, ms, dict(dc, window=W, sinks=S))
    if "decode_rope_fused" in want:
        dc = DECODE
        dq_, kc, vc, sl = workloads.decode_inputs(dc["B"], dc["Hq"], dc["Hkv"], dc["d"],
                                                  dc["Lmin"], dc["Lmax"])
        nbytes = decode_bytes(sl, dc)
        dq_, kc, vc, sl = dq_.to(dev), kc.to(dev), vc.to(dev), sl.to(dev)
        ws = torch.empty(gqa.decode_workspace_size(dc["B"], dc["Hq"], dc["Hkv"], dc["d"],
                                                   dc["Lmax"]), dtype=torch.uint8, device=dev)
        o = torch.empty_like(dq_)
        ms_f = time_median(lambda: gqa.decode(dq_, kc, vc, sl, workspace=ws, out=o,
                                              rope_theta=10000.0), flush, stream, reps)
        ms_u = time_median(lambda: (gqa.rope_decode_q_(dq_, sl),
                                    gqa.decode(dq_, kc, vc, sl, workspace=ws, out=o)),
                           flush, stream, reps)
        row = hbm_row(nbytes, ms_f, dict(dc, theta=10000.0, launches="decode(rope q)"))
        row["unfused_ms"] = ms_u
        row["unfused"] = "rope_decode_q + decode"
        out["decode_rope_fused"] = row
    out["clocks"] = sampler.stop()
    return out


def run_ours(args, world, rank, local):
    import grouped_query_attention_attn_b200 as gqa
    from grouped_query_attention_attn_b200 import workloads

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)
    do_pre = args.only in (None, "prefill")
    do_dec = args.only in (None, "decode")

    c, dc = PREFILL, DECODE
    stream = torch.cuda.current_stream(dev)
    flush = L2Flush(dev)
    if args.only == "next":
        # the rows beyond the hot path alone (profiling runs of their kernels)
        peaks, peak_kind = load_peaks()
        nxt = measure_next_rows(dev, stream, flush, peaks, peak_kind, args.next_reps,
                                args.rows.split(",") if args.rows else None)
        if rank == 0:
            print(json.dumps({"next_rows": nxt}), flush=True)
        return
    if do_pre:
        q_h, k_h, v_h = workloads.prefill_inputs(c["B"], c["T"], c["Hq"], c["Hkv"], c["d"])
        q, k, v = q_h.to(dev), k_h.to(dev), v_h.to(dev)
        o = torch.empty_like(q)
    if do_dec:
        dq_h, kc_h, vc_h, sl_h = workloads.decode_inputs(dc["B"], dc["Hq"], dc["Hkv"], dc["d"],
                                                         dc["Lmin"], dc["Lmax"])
        dq, kc, vc, sl = dq_h.to(dev), kc_h.to(dev), vc_h.to(dev), sl_h.to(dev)
        do = torch.empty_like(dq)
        ws = torch.empty(gqa.decode_workspace_size(dc["B"], dc["Hq"], dc["Hkv"], dc["d"],
                                                   dc["Lmax"]), dtype=torch.uint8, device=dev)

    def step(evs=None):
        if do_pre:
            flush()
            if evs:
                evs[0].record(stream)
            gqa.attn(q, k, v, causal=True, out=o)
            if evs:
                evs[1].record(stream)
        if do_dec:
            flush()
            if evs:
                evs[2].record(stream)
            gqa.decode(dq, kc, vc, sl, workspace=ws, out=do)
            if evs:
                evs[3].record(stream)

    for _ in range(args.warmup):
        step()
    gqa.device_status()
    K = args.steps
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(K)]
    sampler = ClockSampler(dev)
    sampler.start()
    barrier(world)
    torch.cuda.synchronize(dev)
    t_wall = time.perf_counter()
    for i in range(K):
        step(evs[i])
    torch.cuda.synchronize(dev)
    barrier(world)
    wall = time.perf_counter() - t_wall
    clocks = sampler.stop()
    gqa.device_status()
    pre_ms = sum(e[0].elapsed_time(e[1]) for e in evs) if do_pre else 0.0
    dec_ms = sum(e[2].elapsed_time(e[3]) for e in evs) if do_dec else 0.0
    pre_ms = max_over_ranks(pre_ms, world, dev)
    dec_ms = max_over_ranks(dec_ms, world, dev)
    peaks, peak_kind = load_peaks()

    value, roofline, e2e, cpu = None, None, None, None
    if do_pre:
        p_flops = prefill_flops(c)
        value = world * p_flops * K / (pre_ms / 1e3) / 1e12
        launch_ms = pre_ms / K
        roofline = {"bound": "tensor", "achieved": p_flops / (launch_ms / 1e3) / 1e12,
                    "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                    "peak_kind": f"{peak_kind} bf16 burst (kernel timed alone)",
                    "traffic": recorded_traffic("prefill_kernel",
                                                kernel_source_hash(["prefill.cu", "device.cuh"])),
                    "kernel": "prefill_kernel<128>", "flops_per_launch": p_flops,
                    "launch_ms": launch_ms}
        roofline["frac"] = roofline["achieved"] / roofline["peak"]
        roofline["frac_of_nominal_2250"] = roofline["achieved"] / 2250.0
        # time x median SM clock under load: the launch in SM cycles, which
        # separates a slow kernel from a slow clock
        if clocks.get("sm_mhz"):
            roofline["sm_cycles_per_launch"] = launch_ms * 1e3 * clocks["sm_mhz"]

        # ---- end to end through host buffers (the headline metric) ----
        if not args.no_e2e:
            # gqa_attn_fwd_host: pinned host q/k/v in, pinned host o out; the copies
            # run inside the call, overlapped with the attention chunk by chunk
            qp, kp, vp = q_h.pin_memory(), k_h.pin_memory(), v_h.pin_memory()
            op = torch.empty(o.shape, dtype=o.dtype).pin_memory()
            staging = gqa.host_staging(qp, kp, dev)
            done = torch.cuda.Event()
            n_e2e = max(3, min(K, 50))

            def e2e_step():
                # with a completion event, step i+1's copies up overlap step i's copies down
                gqa.attn_host(qp, kp, vp, out=op, causal=True, staging=staging, done=done)

            for _ in range(3):
                e2e_step()
            torch.cuda.synchronize(dev)
            barrier(world)
            s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            s0.record(stream)
            for _ in range(n_e2e):
                e2e_step()
            stream.wait_event(done)                     # the last step's o is on the host
            s1.record(stream)
            torch.cuda.synchronize(dev)
            e2e_ms = max_over_ranks(s0.elapsed_time(s1), world, dev)
            e2e = {"value": world * p_flops * n_e2e / (e2e_ms / 1e3) / 1e12, "unit": "TFLOP/s",
                   "h2d_bytes_per_step": sum(t.numel() * t.element_size() for t in (qp, kp, vp)),
                   "d2h_bytes_per_step": op.numel() * op.element_size(), "steps": n_e2e}

        if rank == 0 and not args.no_cpu:
            import numpy as np
            from oracle import ref
            ref.build_oracle()
            per_row = calibrate_row_seconds(q_h, k_h, v_h)
            n_rows = int(min(max(args.cpu_seconds / per_row, 256), c["B"] * c["Hq"] * c["T"]))
            secs, flops, rows, o_ref = oracle_prefill_sample(q_h, k_h, v_h, n_rows)
            T, Hq = c["T"], c["Hq"]
            r = torch.as_tensor(rows)
            got = o[(r // (T * Hq)).to(dev), (r % T).to(dev), ((r // T) % Hq).to(dev)]
            err = float(np.max(np.abs(got.float().cpu().numpy() - o_ref)))
            cpu = {"value": flops / secs / 1e12, "unit": "TFLOP/s", "cores": ref.num_threads(),
                   "kind": "oracle", "seconds": secs,
                   "sample": f"{n_rows} random query rows of the causal T=4096 prefill "
                             f"(C double oracle, OpenMP)",
                   "max_abs_err_vs_gpu": err}

    dec = None
    if do_dec:
        d_bytes = decode_bytes(sl_h, dc)
        launch_ms = dec_ms / K
        dec_roof = {"bound": "hbm", "achieved": d_bytes / (launch_ms / 1e3) / 1e9,
                    "peak": peaks["hbm_gbs"], "unit": "GB/s", "peak_kind": f"{peak_kind} copy",
                    "traffic": recorded_traffic("decode_split_kernel",
                                                kernel_source_hash(["decode.cu", "device.cuh"])),
                    "bytes_per_step": d_bytes, "launch_ms": launch_ms,
                    "kernels": "decode_split_kernel<128,1> (split merge fused)"}
        dec_roof["frac"] = dec_roof["achieved"] / dec_roof["peak"]
        dec_roof["frac_of_nominal_8000"] = dec_roof["achieved"] / 8000.0
        if clocks.get("sm_mhz"):
            dec_roof["sm_cycles_per_launch"] = launch_ms * 1e3 * clocks["sm_mhz"]
        dec = {"value": world * d_bytes * K / (dec_ms / 1e3) / 1e9, "unit": "GB/s",
               "roofline": dec_roof}

    # host time to enqueue one call through the C ABI from Python (ctypes
    # marshalling, argument checks, tensor maps, launch); outside the timed region
    enqueue = {}
    if not args.no_enqueue:
        from grouped_query_attention_attn_b200 import _binding as cabi
        st = stream.cuda_stream

        def per_call_us(fn, bursts=25, n=16):
            # bursts of n calls into an idle launch queue (a long queue of these
            # kernels would make each call wait for the GPU); median over bursts
            ts = []
            for _ in range(bursts):
                torch.cuda.synchronize(dev)
                t = time.perf_counter()
                for _ in range(n):
                    fn()
                ts.append(1e6 * (time.perf_counter() - t) / n)
            torch.cuda.synchronize(dev)
            return statistics.median(ts)

        if do_pre:
            enqueue["gqa_attn_fwd"] = per_call_us(lambda: cabi.gqa_attn_fwd(
                q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), c["B"], c["T"], c["T"],
                c["Hq"], c["Hkv"], c["d"], 1, c["d"] ** -0.5, st))
        if do_dec:
            enqueue["gqa_decode"] = per_call_us(lambda: cabi.gqa_decode(
                dq.data_ptr(), kc.data_ptr(), vc.data_ptr(), sl.data_ptr(), do.data_ptr(),
                dc["B"], dc["Hq"], dc["Hkv"], dc["d"], dc["Lmax"], dc["d"] ** -0.5,
                ws.data_ptr(), ws.numel(), st))
        gqa.device_status()

    nxt = None
    if args.only is None and not args.no_next:
        nxt = measure_next_rows(dev, stream, flush, peaks, peak_kind, args.next_reps)

    if rank == 0:
        line = {
            "metric": METRIC, "value": value if do_pre else (dec or {}).get("value"),
            "unit": "TFLOP/s" if do_pre else "GB/s", "n_gpus": world,
            "steps": K, "warmup": args.warmup, "ms_per_step": (pre_ms + dec_ms) / K,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic",
            "config": {"workload": WORKLOAD if args.only is None else args.only,
                       "prefill": c if do_pre else None, "decode": dc if do_dec else None,
                       "l2": "flushed before every timed launch (256 MB written, then read back: clean lines)",
                       "parallelism": f"{world} independent replicas" if world > 1 else "1 GPU"},
            "decode": dec,
            "roofline": roofline if do_pre else (dec or {}).get("roofline"),
            "clocks": clocks,
            "e2e": e2e,
            "gpu_launches": K * ((1 if do_pre else 0) + (1 if do_dec else 0)),
            "host_enqueue_us_per_call": enqueue or None,
            "wall_s_timed_region": wall,
            "cpu_baseline": cpu,
            "next_rows": nxt,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--cpu-seconds", type=float, default=15.0,
                    help="target seconds of oracle work for the CPU baseline")
    ap.add_argument("--ref-budget", type=float, default=90.0,
                    help="target seconds of oracle work for all steps of --impl reference")
    ap.add_argument("--only", choices=["prefill", "decode", "next"], default=None,
                    help="time one kernel family only (profiling runs)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-enqueue", action="store_true",
                    help="skip the host enqueue-time measurement")
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--no-next", action="store_true",
                    help="skip the measurements of the rows beyond the hot path")
    ap.add_argument("--next-reps", type=int, default=20)
    ap.add_argument("--rows", default=None,
                    help="with --only next: comma-separated row names (default: all of "
                         + ", ".join(NEXT_ROWS) + ")")
    args = ap.parse_args()
    if args.warmup < 3:
        raise SystemExit("--warmup must be >= 3")
    world, rank, local = dist_init(args.gpus)
    if args.impl == "reference":
        run_reference(args, world, rank)
        return
    run_ours(args, world, rank, local)


if __name__ == "__main__":
    main()
