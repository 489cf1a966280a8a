#!/usr/bin/env python
"""Benchmark of the B200 attention library on its seeded synthetic workloads.

Primary line (one JSON object on stdout, rank 0):
  paged GQA decode, bf16: B=32 sequences x 1 query token, Hq=32, Hkv=8, D=128,
  16-token pages, kv lengths ~ U[1, 8192], random block table over a
  20000-page pool.  value = algorithmic K/V (+Q, O, LSE, block-table) bytes per
  step / device time per step, in GB/s; one step = one attn_decode_paged call
  (split-KV kernel + combine kernel).
Carried in the same line (compact entries: value, unit, ms per step, and the
fraction of the measured peak "frac" and of the spec peak "frac_spec"):
  prefill       varlen paged GQA prefill, causal, 16 seqs, L ~ U[64, 4096],
                Hq=32, Hkv=8, D=128 -> TFLOP/s (4*D per allowed pair per head)
  prefill_fp8   fp8 e4m3 dense causal B=4, H=16, L=4096, D=128 -> TFLOP/s, with
                the bf16 kernel on the same data beside it
  window_softcap, kv_append, backward, only_qv, other_configs: the remaining
                hot-path rows on the same workloads.
  peaks         the denominators: measured HBM copy and bf16 GEMM rates (from
                MEASURED_PEAKS.json), the fp8 e4m3 GEMM rate measured here with
                torch._scaled_mm at 8192^3, and the spec figures.
  cpu_baseline  the fp64 oracle on the host cores: the decode sample (GB/s) and
                its wall seconds on bounded samples of every configuration.

Timing: W warm-up steps, then K steps each bracketed by CUDA events on the
launching stream, a 512 MiB L2 eviction between steps outside the events, and
a barrier + synchronize on both sides of the timed region; max over ranks.
The end-to-end decode leg times K steps as one region with host copies in it.
N > 1 runs N independent replicas (one process per GPU; no collective on the
data path).  --impl reference times the fp64 CPU oracle instead.
"""
from __future__ import annotations

import argparse
import json
import math
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

METRIC = "attn fwd TFLOP/s (prefill) & paged-decode KV GB/s on 1 B200, % of roofline"

# DRAM bytes read + written per launch of each timed kernel, from one ncu
# capture on its bench workload (full-size launch).  They hold only for the
# kernel sources they were taken on: when the sha256 prefix of those sources
# differs, the roofline reports traffic null.
KERNEL_SOURCES = {
    "decode": ["attention_paged_kv_gqa_b200/csrc/decode.cuh", "attention_paged_kv_gqa_b200/csrc/ptx.cuh"],
    "prefill": ["attention_paged_kv_gqa_b200/csrc/prefill.cuh", "attention_paged_kv_gqa_b200/csrc/ptx.cuh"],
}
MEASURED_TRAFFIC = {
    "decode": {"bytes": 579_056_128, "sources": "e1e056b670478940"},
    "decode_fp8": {"bytes": 294_267_904, "sources": "e1e056b670478940"},
    "prefill": {"bytes": 2_005_632_512, "sources": "53045763a6653a9a"},
    "prefill_fp8": {"bytes": 172_875_520, "sources": "53045763a6653a9a"},
}


def kernel_sources_sha(kind: str) -> str:
    import hashlib
    h = hashlib.sha256()
    for f in KERNEL_SOURCES[kind]:
        with open(os.path.join(ROOT, f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def measured_traffic(kind):
    rec = MEASURED_TRAFFIC.get(kind)
    if rec is None or rec["sources"] != kernel_sources_sha(kind.split("_")[0]):
        return None
    return rec["bytes"]


FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# The spec figures of a B200 (dense tensor rates; HBM3e bandwidth).
SPEC_PEAKS = {"hbm_gbs": 8000.0, "bf16_tflops": 2250.0, "fp8_tflops": 4500.0}


def measure_fp8_peak(dev, n=8192, reps=10):
    """Dense e4m3 GEMM rate (TFLOP/s): torch._scaled_mm at n^3, best of `reps`, CUDA events."""
    try:
        g = torch.Generator(device="cpu").manual_seed(0)
        a = torch.randn(n, n, generator=g).to(torch.float8_e4m3fn).to(dev)
        b = torch.randn(n, n, generator=g).to(torch.float8_e4m3fn).to(dev).t()   # column-major
        one = torch.ones((), dtype=torch.float32, device=dev)
        for _ in range(3):
            torch._scaled_mm(a, b, scale_a=one, scale_b=one, out_dtype=torch.bfloat16)
        best = float("inf")
        for _ in range(reps):
            s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            s.record()
            torch._scaled_mm(a, b, scale_a=one, scale_b=one, out_dtype=torch.bfloat16)
            e.record()
            torch.cuda.synchronize()
            best = min(best, s.elapsed_time(e))
        del a, b
        return 2.0 * n ** 3 / (best * 1e-3) / 1e12
    except Exception:
        return None


def entry(value, unit, ms, bound, peaks, dtype="bf16", digits=2):
    """A compact result: value, unit, ms per step, fraction of the measured and spec peaks."""
    key = "hbm_gbs" if bound == "hbm" else ("fp8_tflops" if dtype == "fp8" else "bf16_tflops")
    e = {"value": round(value, digits), "unit": unit, "ms": round(ms, 5)}
    if peaks.get(key):
        e["frac"] = round(value / peaks[key], 4)
    e["frac_spec"] = round(value / SPEC_PEAKS[key], 4)
    return e


def roofline(achieved, unit, bound, peaks, peak_kind, traffic, kernel, dtype="bf16"):
    key = "hbm_gbs" if bound == "hbm" else ("fp8_tflops" if dtype == "fp8" else "bf16_tflops")
    peak = peaks[key]
    return {"bound": bound if bound == "hbm" else "tensor", "achieved": round(achieved, 1),
            "peak": round(peak, 1), "unit": unit, "frac": round(achieved / peak, 4),
            "traffic": traffic, "kernel": kernel, "peak_kind": peak_kind,
            "peak_spec": SPEC_PEAKS[key], "frac_spec": round(achieved / SPEC_PEAKS[key], 4)}


def parse_args():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=50)
    p.add_argument("--warmup", type=int, default=5)
    p.add_argument("--impl", choices=["ours", "reference"], default="ours")
    p.add_argument("--no-prefill", action="store_true")
    p.add_argument("--workload", choices=["all", "decode", "prefill", "fp8", "window", "append",
                                          "backward", "only_qv", "patch"],
                   default="all",
                   help="run only one workload (profiling runs); the JSON line then carries "
                        "only what ran")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--seed", type=int, default=0)
    return p.parse_args()


# --------------------------------------------------------------------------- plumbing
def dist_setup(impl="ours"):
    """Process group for N > 1 (one process per GPU).  NCCL for the CUDA arm;
    gloo for the reference arm (CPU oracle) or when no GPU is present."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    use_cuda = torch.cuda.is_available() and impl == "ours"
    if world > 1:
        import datetime
        import torch.distributed as dist
        if use_cuda:
            torch.cuda.set_device(local)
            dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                    device_id=torch.device("cuda", local))
        else:
            dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=120))
    elif use_cuda:
        torch.cuda.set_device(0)
    return rank, world, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    if torch.cuda.is_available():
        torch.cuda.synchronize()


def max_over_ranks(x: float, world: int) -> float:
    """Largest value over all ranks (the slowest rank's time)."""
    if world == 1:
        return x
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return {k: float(d[k]) for k in ("hbm_gbs", "bf16_tflops", "bf16_tflops_sustained")}, "measured"
    except Exception:
        return dict(FALLBACK_PEAKS), "fallback"


class Clocks:
    """Samples SM clocks and throttle reasons with nvidia-smi during a timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.dev = device_index
        self.proc = None
        self.path = None

    def __enter__(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            # One query first, then the sampling loop with time to settle: the sampler's
            # start-up (NVML initialisation) once stalled a timed step to twice its time.
            subprocess.run(["nvidia-smi", "-i", str(self.dev), "--query-gpu=clocks.sm",
                            "--format=csv,noheader"], stdout=subprocess.DEVNULL,
                           stderr=subprocess.DEVNULL, timeout=30)
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.dev), "--query-gpu=" + self.FIELDS,
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
            time.sleep(1.0)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            time.sleep(0.2)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self):
        if self.proc is None or not self.path:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.path) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    sm.append(float(parts[1]))
                    smax.append(float(parts[2]))
                except ValueError:
                    continue
                for n, v in zip(names, parts[5:9]):
                    if v.lower() == "active":
                        reasons.add(n)
        os.unlink(self.path)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(smax), "samples": len(sm),
                "reasons": sorted(reasons)}


def flush_l2(flush):
    """Evicts L2 by reading a buffer 4x its size (outside the timed events).

    A read-only sweep leaves L2 full of clean lines of this buffer, so the next
    step starts cold without inheriting write-backs (a write sweep would leave
    ~126 MB of dirty lines for the next step's DRAM traffic to absorb).
    """
    flush.view(torch.int64).sum()


def time_steps(step_fn, steps, warmup, world, flush):
    """Per-step device times (ms) with CUDA events on the current stream, L2 flushed between steps."""
    stream = torch.cuda.current_stream()
    for _ in range(warmup):            # the warm-up steps are the timed steps' sequence, untimed
        flush_l2(flush)
        step_fn()
    barrier(world)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(steps)]
    # Keep the device busy (about 1 ms, outside the events) while the host queues the
    # first steps: otherwise the first step's events bracket the host's own time to
    # queue its kernels onto an idle device.
    torch.cuda._sleep(2_000_000)
    for s, e in ev:
        flush_l2(flush)
        s.record(stream)
        step_fn()
        e.record(stream)
    barrier(world)
    return [s.elapsed_time(e) for s, e in ev]


# --------------------------------------------------------------------------- algorithmic work
def decode_bytes(t, Hq, Hkv, D):
    lens = t["seqused_k"].numpy().astype(np.int64)
    B = len(lens)
    kv = int(lens.sum()) * Hkv * D * 2 * 2
    pages = int(((lens + 15) // 16).sum()) * 4
    return kv + B * Hq * D * 2 * 2 + B * Hq * 4 + pages + B * 4


def decode_bytes_fp8(t, Hq, Hkv, D):
    """decode_bytes with one-byte K, V and q (O stays bf16)."""
    lens = t["seqused_k"].numpy().astype(np.int64)
    B = len(lens)
    kv = int(lens.sum()) * Hkv * D * 2
    pages = int(((lens + 15) // 16).sum()) * 4
    return kv + B * Hq * D * (1 + 2) + B * Hq * 4 + pages + B * 4


def causal_flops(lens, Hq, D):
    lens = np.asarray(lens, np.int64)
    return float(4 * D * Hq * (lens * (lens + 1) // 2).sum())


def window_causal_flops(lens, Hq, D, window):
    """Allowed pairs of a causal sliding window: row i sees min(i + 1, window + 1) keys."""
    pairs = 0
    for L in np.asarray(lens, np.int64):
        full = min(int(L), window + 1)          # rows 0 .. full-1 see i + 1 keys
        pairs += full * (full + 1) // 2 + (int(L) - full) * (window + 1)
    return float(4 * D * Hq * pairs)


def window_decode_bytes(t, Hq, Hkv, D, window):
    """decode_bytes over the keys inside each sequence's window (newest query token)."""
    lens = np.minimum(t["seqused_k"].numpy().astype(np.int64), window + 1)
    B = len(lens)
    kv = int(lens.sum()) * Hkv * D * 2 * 2
    pages = int(((lens + 15) // 16).sum()) * 4
    return kv + B * Hq * D * 2 * 2 + B * Hq * 4 + pages + B * 4


# --------------------------------------------------------------------------- CPU oracle legs
def oracle_decode_sample(w, target_tokens=8192, offset=0):
    """Runs the fp64 oracle on a bounded sample of the decode batch; returns (seconds, bytes)."""
    import oracle
    t = w.tensors
    lens = t["seqused_k"].numpy()
    B = len(lens)
    idx, tok = [], 0
    for i in range(B):
        b = (offset + i) % B
        idx.append(b)
        tok += int(lens[b])
        if tok >= target_tokens:
            break
    q = t["q"][idx]
    k_parts, v_parts, bt_rows, maxp = [], [], [], 0
    base = 0
    for b in idx:
        n = (int(lens[b]) + 15) // 16
        pages = t["block_table"][b, :n].long()
        k_parts.append(t["k_cache"][pages])
        v_parts.append(t["v_cache"][pages])
        bt_rows.append(torch.arange(base, base + n, dtype=torch.int32))
        base += n
        maxp = max(maxp, n)
    bt = torch.zeros(len(idx), max(maxp, 1), dtype=torch.int32)
    for i, r in enumerate(bt_rows):
        bt[i, :len(r)] = r
    kc = torch.cat(k_parts) if k_parts else t["k_cache"][:1]
    vc = torch.cat(v_parts) if v_parts else t["v_cache"][:1]
    su = t["seqused_k"][idx]
    nthreads = os.cpu_count() or 1
    t0 = time.perf_counter()
    oracle.attn_decode(q, kc, vc, bt, su, scale=w.params["scale"], nthreads=nthreads)
    dt = time.perf_counter() - t0
    sub = {"seqused_k": su}
    return dt, decode_bytes(sub, w.params["Hq"], w.params["Hkv"], w.params["D"]), len(idx), int(su.sum())


def cpu_model():
    try:
        out = subprocess.run(["lscpu"], capture_output=True, text=True).stdout
        for line in out.splitlines():
            if line.startswith("Model name"):
                return line.split(":", 1)[1].strip()
    except Exception:
        pass
    return "unknown"


# --------------------------------------------------------------------------- arms
def run_reference(args, rank, world):
    """The oracle, as it stands, on the host cores (rank 0 only)."""
    if rank != 0:
        return
    from attention_paged_kv_gqa_b200 import workloads as W
    w = W.paged_decode(seed=args.seed)
    for i in range(args.warmup):
        oracle_decode_sample(w, offset=i)
    secs, nbytes, toks = 0.0, 0, 0
    for i in range(args.steps):
        dt, nb, _, tk = oracle_decode_sample(w, offset=args.warmup + i)
        secs += dt
        nbytes += nb
        toks += tk
    value = nbytes / secs / 1e9
    cores = os.cpu_count() or 1
    line = {
        "impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": "GB/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(secs / args.steps * 1e3, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": "paged_gqa_decode_bf16 (B=32, Hq=32, Hkv=8, D=128, 16-token pages, "
                               "L~U[1,8192], 20000-page pool); each step a sample of whole sequences "
                               "totalling >= 8192 keys", "parallelism": "replicas"},
        "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": cores, "kind": "oracle",
                         "sample": "%d steps, %d keys in total, all 32 heads" % (args.steps, toks),
                         "cpu": cpu_model()},
        "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def run_ours(args, rank, world, local):
    from attention_paged_kv_gqa_b200 import binding as A
    from attention_paged_kv_gqa_b200 import workloads as W
    dev = torch.device("cuda", local if world > 1 else 0)
    st = A.attn_check_device(dev.index)
    if st != 0:
        raise RuntimeError("device check failed: " + A.status_string(st))
    peaks, peak_kind = load_peaks()
    fp8 = measure_fp8_peak(dev)
    peaks["fp8_tflops"] = fp8 if fp8 else 2.0 * peaks["bf16_tflops"]
    fp8_kind = ("measured here: torch._scaled_mm e4m3 8192^3, best of 10" if fp8 else
                peak_kind + " bf16 x 2 (nominal fp8/bf16 ratio)")
    flush = torch.ones(512 << 20, dtype=torch.uint8, device=dev)

    line = {"metric": METRIC, "unit": "GB/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16"}
    ctx = dict(args=args, A=A, W=W, dev=dev, world=world, flush=flush, peaks=peaks,
               peak_kind=peak_kind, fp8_kind=fp8_kind, line=line, launches=0)
    w = None
    if args.workload in ("all", "decode"):
        w = run_decode(ctx)
    if args.workload in ("all", "prefill") and not args.no_prefill:
        run_prefill(ctx)
    if args.workload in ("all", "fp8") and not args.no_prefill:
        run_fp8(ctx)
    if args.workload in ("all", "window") and not args.no_prefill:
        run_window(ctx)
    if args.workload in ("all", "append"):
        run_append(ctx)
    if args.workload in ("all", "backward") and not args.no_prefill:
        run_backward(ctx)
    if args.workload in ("all", "only_qv") and not args.no_prefill:
        run_only_qv(ctx)
    if args.workload in ("all", "patch") and not args.no_prefill:
        run_patch_and_small(ctx)
    line["peaks"] = {"hbm_gbs": peaks["hbm_gbs"], "bf16_tflops": peaks["bf16_tflops"],
                     "fp8_tflops": round(peaks["fp8_tflops"], 1), "kind": peak_kind,
                     "fp8_kind": fp8_kind, "spec": SPEC_PEAKS}
    if args.workload in ("all", "decode") and rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(w)
    if rank == 0:
        print(json.dumps(line, separators=(",", ":")), flush=True)


def run_decode(c):
    # ---------------- decode (primary)
    args, A, W, dev, world, flush = c["args"], c["A"], c["W"], c["dev"], c["world"], c["flush"]
    peaks, line = c["peaks"], c["line"]
    w = W.paged_decode(seed=args.seed)
    t = w.tensors
    P = w.params
    d = {k: v.to(dev) for k, v in t.items()}
    ws = torch.empty(max(A.attn_decode_workspace_size(P["B"], P["Hq"], P["Hkv"], P["D"],
                                                      P["max_blocks_per_seq"]), 16),
                     dtype=torch.uint8, device=dev)
    o = torch.empty(P["B"], P["Hq"], P["D"], dtype=torch.bfloat16, device=dev)
    lse = torch.empty(P["B"], P["Hq"], dtype=torch.float32, device=dev)

    def dec_step():
        A.attn_decode_paged(d["q"], d["k_cache"], d["v_cache"], d["block_table"], d["seqused_k"],
                            scale=P["scale"], out=o, lse=lse, workspace=ws)

    nbytes = decode_bytes(t, P["Hq"], P["Hkv"], P["D"])
    with Clocks(dev.index) as clk:
        times = time_steps(dec_step, args.steps, args.warmup, world, flush)
    clocks = clk.summary()
    ms = statistics.mean(times)
    ms_max = max_over_ranks(sum(times), world) / args.steps
    value = nbytes * world / (ms_max * 1e-3) / 1e9
    kernel_gbs = nbytes / (ms * 1e-3) / 1e9
    ns = 1 if A.attn_decode_workspace_size(P["B"], P["Hq"], P["Hkv"], P["D"],
                                           P["max_blocks_per_seq"]) <= 16 else 2

    # End to end through the binding with host buffers: every step copies its q,
    # block_table and seqused_k in from pinned host memory (one packed buffer) and
    # its O and LSE out (one buffer); the paged cache is resident device state.  As
    # in a serving loop, the copies run on a second stream: step i+1's inputs go in
    # while step i's kernels run, and step i's outputs come back while step i+1's
    # run (two buffers each way).  The K steps are one timed region (device events);
    # the 574 MB of K/V read per step is larger than L2.
    def views_of(buf, like):
        out, off = [], 0
        for x in like:
            n = x.numel() * x.element_size()
            out.append(buf[off:off + n].view(x.dtype).view(x.shape))
            off += n
        return out

    ins = [t["q"], t["block_table"], t["seqused_k"]]
    n_in = sum(x.numel() * x.element_size() for x in ins)
    hin = torch.empty(n_in, dtype=torch.uint8).pin_memory()
    for v, x in zip(views_of(hin, ins), ins):
        v.copy_(x)
    n_out = o.numel() * o.element_size() + lse.numel() * lse.element_size()
    din = [torch.empty(n_in, dtype=torch.uint8, device=dev) for _ in range(2)]
    dout = [torch.empty(n_out, dtype=torch.uint8, device=dev) for _ in range(2)]
    hout = [torch.empty(n_out, dtype=torch.uint8).pin_memory() for _ in range(2)]
    vin = [views_of(b, ins) for b in din]
    vout = [views_of(b, [o, lse]) for b in dout]
    ks = torch.cuda.current_stream()
    cs = torch.cuda.Stream(device=dev)

    def e2e_run(n):
        ev_in = [torch.cuda.Event() for _ in range(2)]
        ev_k = [torch.cuda.Event() for _ in range(2)]
        ev_out = [torch.cuda.Event() for _ in range(2)]
        with torch.cuda.stream(cs):
            din[0].copy_(hin, non_blocking=True)
            ev_in[0].record(cs)
        for i in range(n):
            j = i % 2
            ks.wait_event(ev_in[j])
            if i >= 2:
                ks.wait_event(ev_out[j])            # step i-2's outputs have left buffer j
            qd, btd, sud = vin[j]
            od, ld = vout[j]
            A.attn_decode_paged(qd, d["k_cache"], d["v_cache"], btd, sud, scale=P["scale"],
                                out=od, lse=ld, workspace=ws, stream=ks)
            ev_k[j].record(ks)
            with torch.cuda.stream(cs):
                if i + 1 < n:
                    jn = (i + 1) % 2
                    if i >= 1:
                        cs.wait_event(ev_k[jn])     # step i-1 has consumed buffer jn
                    din[jn].copy_(hin, non_blocking=True)
                    ev_in[jn].record(cs)
                cs.wait_event(ev_k[j])
                hout[j].copy_(dout[j], non_blocking=True)
                ev_out[j].record(cs)
        ks.wait_event(ev_out[(n - 1) % 2])
        if n >= 2:
            ks.wait_event(ev_out[(n - 2) % 2])

    e2e_run(args.warmup)
    barrier(world)
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(ks)
    cs.wait_event(t0)
    e2e_run(args.steps)
    t1.record(ks)
    barrier(world)
    e2e_ms = max_over_ranks(t0.elapsed_time(t1), world) / args.steps
    c["launches"] += args.steps * ns * 2          # device-timed and end-to-end legs

    line.update({
        "value": round(value, 2), "ms_per_step": round(ms_max, 5),
        "data": "synthetic: seeded N(0,1) bf16 q/k/v, uniform kv lengths, permuted page pool",
        "config": {"workload": "paged_gqa_decode_bf16: B=32 x 1 query token, Hq=32, Hkv=8, "
                               "D=128, 16-token pages, kv len ~ U[1,8192] (seed %d: %d keys), "
                               "20000-page pool" % (args.seed, int(t["seqused_k"].sum())),
                   "global_batch": P["B"] * world, "seq_len": int(t["seqused_k"].max()),
                   "parallelism": "replicas" if world > 1 else "single",
                   "l2": "flushed between timed steps (read sweep of 512 MiB); 574 MB of K/V "
                         "per step, larger than L2",
                   "bytes_per_step": nbytes,
                   "step_us": {"mean": round(ms * 1e3, 2),
                               "median": round(statistics.median(times) * 1e3, 2),
                               "min": round(min(times) * 1e3, 2),
                               "max": round(max(times) * 1e3, 2)}},
        "roofline": roofline(kernel_gbs, "GB/s", "hbm", peaks, c["peak_kind"],
                             measured_traffic("decode"),
                             "decode_pages_kernel<128> + decode_pages_combine_kernel<128>"),
        "e2e": {"value": round(nbytes * world / (e2e_ms * 1e-3) / 1e9, 2), "unit": "GB/s",
                "h2d_bytes_per_step": n_in, "d2h_bytes_per_step": n_out,
                "ms_per_step": round(e2e_ms, 5),
                "note": "K steps in one timed region; each step copies q, block_table, "
                        "seqused_k in and O, LSE out (pinned host), on a copy stream "
                        "overlapping the neighbouring steps' kernels"},
        "clocks": clocks,
    })
    line["gpu_launches"] = c["launches"]
    return w


def run_prefill(c):
    args, A, W, dev, world, flush = c["args"], c["A"], c["W"], c["dev"], c["world"], c["flush"]
    peaks = c["peaks"]
    wp = W.varlen_paged_prefill(seed=args.seed)
    tp, Pp = wp.tensors, wp.params
    dp = {k: v.to(dev) for k, v in tp.items()}
    op = torch.empty(Pp["total_q"], Pp["Hq"], Pp["D"], dtype=torch.bfloat16, device=dev)
    lp = torch.empty(Pp["Hq"], Pp["total_q"], dtype=torch.float32, device=dev)

    def pf_step():
        A.attn_fwd_varlen_paged(dp["q"], dp["k_cache"], dp["v_cache"],
                                cu_seqlens_q=dp["cu_seqlens_q"], max_seqlen_q=Pp["max_seqlen_q"],
                                block_table=dp["block_table"], seqused_k=dp["seqused_k"],
                                mask=A.MASK_CAUSAL, scale=Pp["scale"], out=op, lse=lp)

    pms = statistics.mean(time_steps(pf_step, args.steps, args.warmup, world, flush))
    flops = causal_flops(tp["seqused_k"].numpy(), Pp["Hq"], Pp["D"])
    tf = flops / (pms * 1e-3) / 1e12
    e = entry(tf, "TFLOP/s", pms, "tensor", peaks)
    e["workload"] = "varlen paged GQA causal, %d tokens" % Pp["total_q"]
    e["flops_per_step"] = flops
    e["roofline"] = roofline(tf, "TFLOP/s", "tensor", peaks, c["peak_kind"],
                             measured_traffic("prefill"), "prefill_kernel<128,bf16>")
    c["line"]["prefill"] = e
    c["launches"] += args.steps
    c["line"]["gpu_launches"] = c["launches"]
    del dp


def run_fp8(c):
    args, A, W, dev, world, flush = c["args"], c["A"], c["W"], c["dev"], c["world"], c["flush"]
    peaks = c["peaks"]
    w8 = W.fp8_dense_causal(seed=args.seed)
    t8 = w8.tensors
    d8 = {k: v.to(dev) for k, v in t8.items()}
    o8 = torch.empty(4, 4096, 16, 128, dtype=torch.bfloat16, device=dev)
    l8 = torch.empty(4, 16, 4096, dtype=torch.float32, device=dev)

    def f8_step():
        A.attn_fwd_dense(d8["q_fp8"], d8["k_fp8"], d8["v_fp8"], causal=True,
                         scale=w8.params["scale"], descale_q=d8["descale_q"],
                         descale_k=d8["descale_k"], descale_v=d8["descale_v"], out=o8, lse=l8)

    def b16_step():
        A.attn_fwd_dense(d8["q"], d8["k"], d8["v"], causal=True, scale=w8.params["scale"],
                         out=o8, lse=l8)

    f8ms = statistics.mean(time_steps(f8_step, args.steps, args.warmup, world, flush))
    b16ms = statistics.mean(time_steps(b16_step, args.steps, args.warmup, world, flush))
    fl8 = causal_flops([4096] * 4, 16, 128)
    tf8, tf16 = fl8 / (f8ms * 1e-3) / 1e12, fl8 / (b16ms * 1e-3) / 1e12
    e = entry(tf8, "TFLOP/s", f8ms, "tensor", peaks, dtype="fp8")
    e["workload"] = "fp8 e4m3 dense causal B=4 H=16 L=4096 D=128"
    e["bf16_same_data"] = entry(tf16, "TFLOP/s", b16ms, "tensor", peaks)
    e["fp8_time_over_bf16_time"] = round(f8ms / b16ms, 4)
    e["roofline"] = roofline(tf8, "TFLOP/s", "tensor", peaks, c["fp8_kind"],
                             measured_traffic("prefill_fp8"), "prefill_kernel<128,fp8>",
                             dtype="fp8")
    c["line"]["prefill_fp8"] = e
    c["launches"] += 2 * args.steps
    c["line"]["gpu_launches"] = c["launches"]
    del d8

    # the paged decode workload with q and the cache in e4m3 (per-tensor descales)
    w = W.paged_decode(seed=args.seed)
    t, P = w.tensors, w.params
    d = {k: t[k].to(dev) for k in ("block_table", "seqused_k")}
    for name in ("q", "k_cache", "v_cache"):
        d[name], d["descale_" + name] = W.quantize_e4m3(t[name].to(dev))
        d["descale_" + name] = d["descale_" + name].to(dev)
    ws = torch.empty(max(A.attn_decode_workspace_size(P["B"], P["Hq"], P["Hkv"], P["D"],
                                                      P["max_blocks_per_seq"]), 16),
                     dtype=torch.uint8, device=dev)
    o = torch.empty(P["B"], P["Hq"], P["D"], dtype=torch.bfloat16, device=dev)
    lse = torch.empty(P["B"], P["Hq"], dtype=torch.float32, device=dev)

    def dec_step():
        A.attn_decode_paged(d["q"], d["k_cache"], d["v_cache"], d["block_table"], d["seqused_k"],
                            scale=P["scale"], descale_q=d["descale_q"],
                            descale_k=d["descale_k_cache"], descale_v=d["descale_v_cache"],
                            out=o, lse=lse, workspace=ws)

    dms = statistics.mean(time_steps(dec_step, args.steps, args.warmup, world, flush))
    nb = decode_bytes_fp8(t, P["Hq"], P["Hkv"], P["D"])
    e = entry(nb / (dms * 1e-3) / 1e9, "GB/s", dms, "hbm", peaks, dtype="fp8")
    e["workload"] = ("paged_gqa_decode with q and the cache in e4m3: B=32, Hq=32, Hkv=8, D=128, "
                     "kv len ~ U[1,8192]")
    e["bytes_per_step"] = nb
    e["keys_per_us"] = round(int(t["seqused_k"].sum()) / (dms * 1e3), 1)
    e["traffic"] = measured_traffic("decode_fp8")
    c["line"]["decode_fp8"] = e
    c["launches"] += 2 * args.steps
    c["line"]["gpu_launches"] = c["launches"]
    del d


WINDOW, SOFTCAP = 1024, 50.0


def run_window(c):
    """Decode and varlen prefill with a sliding window, a softcap, and both."""
    args, A, W, dev, world, flush = c["args"], c["A"], c["W"], c["dev"], c["world"], c["flush"]
    peaks = c["peaks"]
    w = W.paged_decode(seed=args.seed)
    t, P = w.tensors, w.params
    d = {k: v.to(dev) for k, v in t.items()}
    ws = torch.empty(max(A.attn_decode_workspace_size(P["B"], P["Hq"], P["Hkv"], P["D"],
                                                      P["max_blocks_per_seq"]), 16),
                     dtype=torch.uint8, device=dev)
    o = torch.empty(P["B"], P["Hq"], P["D"], dtype=torch.bfloat16, device=dev)
    lse = torch.empty(P["B"], P["Hq"], dtype=torch.float32, device=dev)
    out = {"window_left": WINDOW, "softcap": SOFTCAP}
    for name, wl, cap in (("decode_window", WINDOW, 0.0), ("decode_softcap", -1, SOFTCAP),
                          ("decode_window_softcap", WINDOW, SOFTCAP)):
        def dec_step():
            A.attn_decode_paged(d["q"], d["k_cache"], d["v_cache"], d["block_table"],
                                d["seqused_k"], scale=P["scale"], window_left=wl, softcap=cap,
                                out=o, lse=lse, workspace=ws)

        dms = statistics.mean(time_steps(dec_step, args.steps, args.warmup, world, flush))
        nb = (window_decode_bytes(t, P["Hq"], P["Hkv"], P["D"], wl) if wl >= 0
              else decode_bytes(t, P["Hq"], P["Hkv"], P["D"]))
        out[name] = entry(nb / (dms * 1e-3) / 1e9, "GB/s", dms, "hbm", peaks)
        c["launches"] += 2 * args.steps
    del d

    wp = W.varlen_paged_prefill(seed=args.seed)
    tp, Pp = wp.tensors, wp.params
    dp = {k: v.to(dev) for k, v in tp.items()}
    op = torch.empty(Pp["total_q"], Pp["Hq"], Pp["D"], dtype=torch.bfloat16, device=dev)
    lp = torch.empty(Pp["Hq"], Pp["total_q"], dtype=torch.float32, device=dev)
    lens = tp["seqused_k"].numpy()
    for name, wl, cap in (("prefill_window", WINDOW, 0.0), ("prefill_softcap", -1, SOFTCAP),
                          ("prefill_window_softcap", WINDOW, SOFTCAP)):
        def pf_step():
            A.attn_fwd_varlen_paged(dp["q"], dp["k_cache"], dp["v_cache"],
                                    cu_seqlens_q=dp["cu_seqlens_q"],
                                    max_seqlen_q=Pp["max_seqlen_q"],
                                    block_table=dp["block_table"], seqused_k=dp["seqused_k"],
                                    mask=A.MASK_CAUSAL, scale=Pp["scale"], window_left=wl,
                                    softcap=cap, out=op, lse=lp)

        pms = statistics.mean(time_steps(pf_step, args.steps, args.warmup, world, flush))
        fl = (window_causal_flops(lens, Pp["Hq"], Pp["D"], wl) if wl >= 0
              else causal_flops(lens, Pp["Hq"], Pp["D"]))
        out[name] = entry(fl / (pms * 1e-3) / 1e12, "TFLOP/s", pms, "tensor", peaks)
        c["launches"] += args.steps
    del dp
    out["note"] = "decode and varlen prefill workloads; work counted inside each window only"
    c["line"]["window_softcap"] = out
    c["line"]["gpu_launches"] = c["launches"]


def run_append(c):
    """Paged KV append at prefill size, and a decode step with its append."""
    args, A, W, dev, world, flush = c["args"], c["A"], c["W"], c["dev"], c["world"], c["flush"]
    peaks = c["peaks"]
    wp = W.varlen_paged_prefill(seed=args.seed)
    tp, Pp = wp.tensors, wp.params
    lens = tp["seqused_k"]
    total, Hkv, D = Pp["total_q"], Pp["Hkv"], Pp["D"]
    k_new = W.randn_bf16((total, Hkv, D), args.seed, 31).to(dev)   # every token's new K/V
    v_new = W.randn_bf16((total, Hkv, D), args.seed, 32).to(dev)
    kc, vc = tp["k_cache"].to(dev), tp["v_cache"].to(dev)
    bt = tp["block_table"].to(dev)
    zeros = torch.zeros_like(lens).to(dev)                   # sequences start empty
    cu = tp["cu_seqlens_k"].to(dev)
    after = torch.empty_like(zeros)

    def app_step():
        A.attn_kv_append_paged(k_new, v_new, kc, vc, bt, zeros, cu_seqlens_new=cu,
                               seqused_k_out=after)

    ams = statistics.mean(time_steps(app_step, args.steps, args.warmup, world, flush))
    nbytes = 2 * 2 * total * Hkv * D * 2 + int(lens.numel()) * 4 * 3 + 4 * (lens.numel() + 1)
    del k_new, v_new, kc, vc

    w = W.paged_decode(seed=args.seed)
    t, P = w.tensors, w.params
    d = {k: v.to(dev) for k, v in t.items()}
    g = torch.Generator().manual_seed(args.seed + 99)
    kn = torch.randn(P["B"], P["Hkv"], P["D"], generator=g).to(torch.bfloat16).to(dev)
    vn = torch.randn(P["B"], P["Hkv"], P["D"], generator=g).to(torch.bfloat16).to(dev)
    # lengths one short of the workload's, so the appended token is the last cached one
    before = (t["seqused_k"] - 1).clamp(min=0).to(dev)
    after = torch.empty_like(before)
    ws = torch.empty(max(A.attn_decode_workspace_size(P["B"], P["Hq"], P["Hkv"], P["D"],
                                                      P["max_blocks_per_seq"]), 16),
                     dtype=torch.uint8, device=dev)
    o = torch.empty(P["B"], P["Hq"], P["D"], dtype=torch.bfloat16, device=dev)
    lse = torch.empty(P["B"], P["Hq"], dtype=torch.float32, device=dev)

    def dec_step():
        A.attn_decode_paged_append(d["q"], kn, vn, d["k_cache"], d["v_cache"], d["block_table"],
                                   before, seqused_k_out=after, scale=P["scale"], out=o, lse=lse,
                                   workspace=ws)

    dms = statistics.mean(time_steps(dec_step, args.steps, args.warmup, world, flush))
    lens_after = (t["seqused_k"] - 1).clamp(min=0) + 1
    nb_dec = decode_bytes({"seqused_k": lens_after}, P["Hq"], P["Hkv"], P["D"]) + \
        2 * 2 * P["B"] * P["Hkv"] * P["D"] * 2
    del d
    e1 = entry(nbytes / (ams * 1e-3) / 1e9, "GB/s", ams, "hbm", peaks)
    e1["workload"] = "all %d prefill tokens into empty sequences" % total
    e2 = entry(nb_dec / (dms * 1e-3) / 1e9, "GB/s", dms, "hbm", peaks)
    e2["workload"] = "decode step with its one-token append (PDL chain)"
    c["line"]["kv_append"] = {"prefill_size": e1, "decode_step": e2}
    c["launches"] += 4 * args.steps
    c["line"]["gpu_launches"] = c["launches"]


def run_backward(c):
    """dQ, dK, dV of the varlen causal GQA workload (packed K/V)."""
    args, A, W, dev, world, flush = c["args"], c["A"], c["W"], c["dev"], c["world"], c["flush"]
    peaks = c["peaks"]
    wp = W.varlen_paged_prefill(seed=args.seed)
    Pp = wp.params
    lens = wp.tensors["seqused_k"]
    cu = W.cu_from_lens(lens).to(dev)
    total, Hq, Hkv, D = Pp["total_q"], Pp["Hq"], Pp["Hkv"], Pp["D"]
    q = W.randn_bf16((total, Hq, D), args.seed, 51).to(dev)
    k = W.randn_bf16((total, Hkv, D), args.seed, 52).to(dev)
    v = W.randn_bf16((total, Hkv, D), args.seed, 53).to(dev)
    do = W.randn_bf16((total, Hq, D), args.seed, 54).to(dev)
    maxlen = int(lens.max())
    o, lse = A.attn_fwd_varlen_paged(q, k, v, cu_seqlens_q=cu, cu_seqlens_k=cu,
                                     max_seqlen_q=maxlen, mask=A.MASK_CAUSAL, scale=Pp["scale"])
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    ws = torch.empty(A.lib().attn_bwd_workspace_size(Hq, total), dtype=torch.uint8, device=dev)

    def bwd_step():
        A.attn_bwd_varlen(q, k, v, o, do, lse, cu_seqlens_q=cu, cu_seqlens_k=cu,
                          max_seqlen_q=maxlen, max_seqlen_k=maxlen, mask=A.MASK_CAUSAL,
                          scale=Pp["scale"], dq=dq, dk=dk, dv=dv, workspace=ws)

    bms = statistics.mean(time_steps(bwd_step, args.steps, args.warmup, world, flush))
    flops = 2.5 * causal_flops(lens.numpy(), Hq, D)
    e = entry(flops / (bms * 1e-3) / 1e12, "TFLOP/s", bms, "tensor", peaks)
    e["workload"] = "varlen causal GQA backward, %d tokens, packed K/V" % total
    e["flops_convention"] = "10*D per allowed pair per query head (5 GEMMs; 7 run)"
    c["line"]["backward"] = e
    c["launches"] += 3 * args.steps
    c["line"]["gpu_launches"] = c["launches"]
    del q, k, v, do, o, dq, dk, dv


def run_only_qv(c):
    """The only_qv score path (score = scale * qv . v) on the decode and prefill workloads:
    the query tensor serves as qv and the value cache as the only KV store."""
    args, A, W, dev, world, flush = c["args"], c["A"], c["W"], c["dev"], c["world"], c["flush"]
    peaks = c["peaks"]
    w = W.paged_decode(seed=args.seed)
    t, P = w.tensors, w.params
    d = {k: v.to(dev) for k, v in t.items() if k != "k_cache"}
    ws = torch.empty(max(A.attn_decode_workspace_size(P["B"], P["Hq"], P["Hkv"], P["D"],
                                                      P["max_blocks_per_seq"]), 16),
                     dtype=torch.uint8, device=dev)
    o = torch.empty(P["B"], P["Hq"], P["D"], dtype=torch.bfloat16, device=dev)
    lse = torch.empty(P["B"], P["Hq"], dtype=torch.float32, device=dev)

    def dec_step():
        A.attn_decode_paged_only_qv(d["q"], d["v_cache"], d["block_table"], d["seqused_k"],
                                    scale=P["scale"], out=o, lse=lse, workspace=ws)

    dms = statistics.mean(time_steps(dec_step, args.steps, args.warmup, world, flush))
    # algorithmic bytes: decode_bytes with the V half of the K/V stream only
    lens = t["seqused_k"].numpy().astype(np.int64)
    nb = decode_bytes(t, P["Hq"], P["Hkv"], P["D"]) - int(lens.sum()) * P["Hkv"] * P["D"] * 2
    out = {"decode": entry(nb / (dms * 1e-3) / 1e9, "GB/s", dms, "hbm", peaks)}
    del d

    wp = W.varlen_paged_prefill(seed=args.seed)
    tp, Pp = wp.tensors, wp.params
    dp = {k: v.to(dev) for k, v in tp.items() if k != "k_cache"}
    op = torch.empty(Pp["total_q"], Pp["Hq"], Pp["D"], dtype=torch.bfloat16, device=dev)
    lp = torch.empty(Pp["Hq"], Pp["total_q"], dtype=torch.float32, device=dev)

    def pf_step():
        A.attn_fwd_varlen_paged_only_qv(dp["q"], dp["v_cache"], cu_seqlens_q=dp["cu_seqlens_q"],
                                        max_seqlen_q=Pp["max_seqlen_q"],
                                        block_table=dp["block_table"], seqused_k=dp["seqused_k"],
                                        mask=A.MASK_CAUSAL, scale=Pp["scale"], out=op, lse=lp)

    pms = statistics.mean(time_steps(pf_step, args.steps, args.warmup, world, flush))
    fl = causal_flops(tp["seqused_k"].numpy(), Pp["Hq"], Pp["D"])
    out["prefill"] = entry(fl / (pms * 1e-3) / 1e12, "TFLOP/s", pms, "tensor", peaks)
    del dp
    out["note"] = "q as qv, the value cache as the only store; decode bytes count V once"
    c["line"]["only_qv"] = out
    c["launches"] += 3 * args.steps
    c["line"]["gpu_launches"] = c["launches"]
    run_qv(c)


def run_qv(c):
    """The score with the extra Qv term, scale * (q.k + qv.v), on the decode and varlen prefill
    workloads (qv a second seeded bf16 tensor of q's shape)."""
    args, A, W, dev, world, flush = c["args"], c["A"], c["W"], c["dev"], c["world"], c["flush"]
    peaks = c["peaks"]
    w = W.paged_decode(seed=args.seed)
    t, P = w.tensors, w.params
    d = {k: v.to(dev) for k, v in t.items()}
    qv = W.randn_bf16(tuple(t["q"].shape), args.seed, 51).to(dev)
    ws = torch.empty(max(A.attn_decode_workspace_size(P["B"], P["Hq"], P["Hkv"], P["D"],
                                                      P["max_blocks_per_seq"]), 16),
                     dtype=torch.uint8, device=dev)
    o = torch.empty(P["B"], P["Hq"], P["D"], dtype=torch.bfloat16, device=dev)
    lse = torch.empty(P["B"], P["Hq"], dtype=torch.float32, device=dev)

    def dec_step():
        A.attn_decode_paged_qv(d["q"], qv, d["k_cache"], d["v_cache"], d["block_table"],
                               d["seqused_k"], scale=P["scale"], out=o, lse=lse, workspace=ws)

    dms = statistics.mean(time_steps(dec_step, args.steps, args.warmup, world, flush))
    nb = decode_bytes(t, P["Hq"], P["Hkv"], P["D"]) + int(qv.numel()) * 2
    out = {"decode": entry(nb / (dms * 1e-3) / 1e9, "GB/s", dms, "hbm", peaks)}
    del d

    wp = W.varlen_paged_prefill(seed=args.seed)
    tp, Pp = wp.tensors, wp.params
    dp = {k: v.to(dev) for k, v in tp.items()}
    qvp = W.randn_bf16(tuple(tp["q"].shape), args.seed, 52).to(dev)
    op = torch.empty(Pp["total_q"], Pp["Hq"], Pp["D"], dtype=torch.bfloat16, device=dev)
    lp = torch.empty(Pp["Hq"], Pp["total_q"], dtype=torch.float32, device=dev)

    def pf_step():
        A.attn_fwd_varlen_paged_qv(dp["q"], qvp, dp["k_cache"], dp["v_cache"],
                                   cu_seqlens_q=dp["cu_seqlens_q"], max_seqlen_q=Pp["max_seqlen_q"],
                                   block_table=dp["block_table"], seqused_k=dp["seqused_k"],
                                   mask=A.MASK_CAUSAL, scale=Pp["scale"], out=op, lse=lp)

    pms = statistics.mean(time_steps(pf_step, args.steps, args.warmup, world, flush))
    # three GEMMs per allowed pair (q.k, qv.v, P.V): 6 D flops per pair and query head
    fl = causal_flops(tp["seqused_k"].numpy(), Pp["Hq"], Pp["D"]) * 1.5
    out["prefill"] = entry(fl / (pms * 1e-3) / 1e12, "TFLOP/s", pms, "tensor", peaks)
    del dp
    out["note"] = ("score scale * (q.k + qv.v); decode bytes add qv, prefill flops count three "
                   "GEMMs (6 D per allowed pair and query head)")
    c["line"]["qv"] = out
    c["launches"] += 3 * args.steps
    c["line"]["gpu_launches"] = c["launches"]


def run_patch_and_small(c):
    """The two remaining configurations: patch cross-attention (memory-bound: GB/s against
    HBM) and the small dense causal case (launch-latency bound: microseconds per call)."""
    args, A, W, dev, world, flush = c["args"], c["A"], c["W"], c["dev"], c["world"], c["flush"]
    peaks = c["peaks"]
    w = W.patch_cross(seed=args.seed)
    t, P = w.tensors, w.params
    d = {k: v.to(dev) for k, v in t.items()}
    o = torch.empty(P["total_q"], P["Hq"], P["D"], dtype=torch.bfloat16, device=dev)
    lse = torch.empty(P["Hq"], P["total_q"], dtype=torch.float32, device=dev)

    def patch_step():   # patches are clipped to 16 bytes: the short-interval kernel
        A.attn_fwd_patch(d["q"], d["k"], d["v"], cu_seqlens_q=d["cu_seqlens_q"],
                         cu_seqlens_k=d["cu_seqlens_k"], patch_kv_range=d["patch_kv_range"],
                         max_seqlen_q=P["max_seqlen_q"], max_interval=16, scale=P["scale"], out=o,
                         lse=lse)

    def patch_tiled_step():
        A.attn_fwd_varlen_paged(d["q"], d["k"], d["v"], cu_seqlens_q=d["cu_seqlens_q"],
                                cu_seqlens_k=d["cu_seqlens_k"], max_seqlen_q=P["max_seqlen_q"],
                                mask=A.MASK_PATCH, patch_kv_range=d["patch_kv_range"],
                                scale=P["scale"], out=o, lse=lse)

    pms = statistics.mean(time_steps(patch_step, args.steps, args.warmup, world, flush))
    tms = statistics.mean(time_steps(patch_tiled_step, args.steps, args.warmup, world, flush))
    nb = patch_bytes(P)
    e = entry(nb / (pms * 1e-3) / 1e9, "GB/s", pms, "hbm", peaks)
    e["workload"] = "B=4 x 8192 bytes, %d patch queries, H=16, D=64" % P["total_q"]
    e["kernel"] = "patch_stream_kernel<64> (attn_fwd_patch)"
    e["tiled_kernel"] = entry(nb / (tms * 1e-3) / 1e9, "GB/s", tms, "hbm", peaks)
    out = {"patch": e}
    del d
    w1 = W.dense(seed=args.seed)
    t1 = {k: v.to(dev) for k, v in w1.tensors.items()}
    o1 = torch.empty_like(t1["q"])
    l1 = torch.empty(2, 2, 128, dtype=torch.float32, device=dev)

    def small_step():
        A.attn_fwd_dense(t1["q"], t1["k"], t1["v"], causal=True, scale=w1.params["scale"], out=o1, lse=l1)

    sms = statistics.mean(time_steps(small_step, args.steps, args.warmup, world, flush))
    out["dense_small"] = {"value": round(sms * 1e3, 2), "unit": "us per call",
                          "higher_is_better": False,
                          "note": "B=2 L=128 H=2 D=64 causal: 8.45 MFLOP, latency-bound"}
    c["line"]["other_configs"] = out
    c["launches"] += 3 * args.steps
    c["line"]["gpu_launches"] = c["launches"]


def patch_bytes(P):
    """Every key and value row once (each belongs to one patch), Q and O, LSE, the
    per-query ranges and the cumulative lengths."""
    return (2 * P["total_k"] * P["Hkv"] * P["D"] * 2 + 2 * P["total_q"] * P["Hq"] * P["D"] * 2
            + P["total_q"] * P["Hq"] * 4 + P["total_q"] * 8 + 2 * (P["B"] + 1) * 4)


def oracle_config_samples():
    """Wall seconds of the fp64 oracle, as it stands, on a bounded sample of each
    configuration (the small dense one whole), with the sample named and its work
    rate in the configuration's unit."""
    import oracle
    from attention_paged_kv_gqa_b200 import workloads as W
    n = os.cpu_count() or 1
    out = {}
    w = W.dense(seed=0)
    t = w.tensors
    t0 = time.perf_counter()
    oracle.attn_dense(t["q"], t["k"], t["v"], scale=w.params["scale"], causal=True, nthreads=n)
    out["dense_causal_small"] = {"seconds": round(time.perf_counter() - t0, 4),
                                 "sample": "whole (B=2, L=128, H=2, D=64)"}
    wp = W.varlen_paged_prefill(seed=0)
    tp = wp.tensors
    lens = tp["seqused_k"].numpy()
    b = int(np.argmax(lens))
    L = int(lens[b])
    cu = tp["cu_seqlens_q"].numpy()
    rows = 128
    q = tp["q"][cu[b + 1] - rows:cu[b + 1]]
    npg = (L + 15) // 16
    kc, vc = tp["k_cache"][tp["block_table"][b, :npg].long()], tp["v_cache"][tp["block_table"][b, :npg].long()]
    t0 = time.perf_counter()
    oracle.attn_varlen(q, kc, vc, cu_seqlens_q=np.array([0, rows], np.int32),
                       seqused_k=np.array([L], np.int32),
                       block_table=np.arange(npg, dtype=np.int32)[None], num_heads_kv=8,
                       scale=wp.params["scale"], mask=1, nthreads=n)
    dt = time.perf_counter() - t0
    pairs = sum(L - rows + i + 1 for i in range(rows))
    out["varlen_paged_prefill"] = {"seconds": round(dt, 3),
                                   "value": round(4 * 128 * 32 * pairs / dt / 1e9, 3),
                                   "unit": "GFLOP/s",
                                   "sample": "last %d rows of the %d-token sequence, 32 heads"
                                             % (rows, L)}
    wc = W.patch_cross(seed=0)
    tc = wc.tensors
    nq = 256
    r = tc["patch_kv_range"][:nq]
    t0 = time.perf_counter()
    oracle.attn_varlen(tc["q"][:nq], tc["k"][:8192], tc["v"][:8192],
                       cu_seqlens_q=np.array([0, nq], np.int32),
                       cu_seqlens_k=np.array([0, 8192], np.int32), num_heads_kv=16,
                       scale=wc.params["scale"], mask=2, patch_kv_range=r, nthreads=n)
    dt = time.perf_counter() - t0
    keys = int((r[:, 1] - r[:, 0]).sum())
    nbytes = 2 * keys * 16 * 64 * 2 + 2 * nq * 16 * 64 * 2 + nq * 16 * 4 + nq * 8
    out["patch_cross"] = {"seconds": round(dt, 3), "value": round(nbytes / dt / 1e9, 5),
                          "unit": "GB/s",
                          "sample": "first %d patch queries of sequence 0 (8192-key rows)" % nq}
    w8 = W.fp8_dense_causal(seed=0)
    t8 = w8.tensors
    rows = 128
    qd = oracle.dequant_e4m3(t8["q_fp8"][0:1, -rows:], t8["descale_q"])
    kd = oracle.dequant_e4m3(t8["k_fp8"][0:1], t8["descale_k"])
    vd = oracle.dequant_e4m3(t8["v_fp8"][0:1], t8["descale_v"])
    t0 = time.perf_counter()
    oracle.attn_varlen(qd[0], kd[0], vd[0], cu_seqlens_q=np.array([0, rows], np.int32),
                       cu_seqlens_k=np.array([0, 4096], np.int32), num_heads_kv=16,
                       scale=w8.params["scale"], mask=1, nthreads=n)
    dt = time.perf_counter() - t0
    pairs = sum(4096 - rows + i + 1 for i in range(rows))
    out["fp8_dense_causal"] = {"seconds": round(dt, 3),
                               "value": round(4 * 128 * 16 * pairs / dt / 1e9, 3),
                               "unit": "GFLOP/s",
                               "sample": "last %d rows of batch element 0, 16 heads" % rows}
    return out


def cpu_baseline(w):
    """The oracle on rank 0 at N=1: a bounded sample (about 10 s) of the decode batch, in
    the primary metric's unit, and its wall seconds on samples of every configuration."""
    secs, nb, nseq, tok = 0.0, 0, 0, 0
    t_start = time.perf_counter()
    i = 0
    while time.perf_counter() - t_start < 10.0 and i < 32:
        dt, b_, n_, tk = oracle_decode_sample(w, target_tokens=8192, offset=i * 3)
        secs += dt
        nb += b_
        nseq += n_
        tok += tk
        i += 1
    return {"value": round(nb / secs / 1e9, 4), "unit": "GB/s",
            "cores": os.cpu_count() or 1, "kind": "oracle",
            "sample": "%d oracle calls over %d whole sequences (%d keys, all "
                      "32 heads) of the decode batch" % (i, nseq, tok),
            "cpu": cpu_model(), "per_config": oracle_config_samples()}


def main():
    args = parse_args()
    rank, world, local = dist_setup(args.impl)
    try:
        if args.impl == "reference":
            run_reference(args, rank, world)
        else:
            run_ours(args, rank, world, local)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
