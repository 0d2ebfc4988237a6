#!/usr/bin/env python
"""Benchmark of the BitLinear forward on B200.

Headline workload (one JSON line on rank 0): decode GEMV — 1 token, K = 2560,
N = 6912, bf16 activations with 1 % ×20 outlier channels, 2-bit packed
ternary weights (pre-quantised), bf16 output. One step = 1000 BitLinear calls
(1 token each) chained on one stream with programmatic dependent launch,
replayed as a CUDA graph, each call against the next matrix of a rotating
pool of distinct packed weight matrices whose total size is ≥ 3× the L2
cache (so weights stream from HBM, no L2 flush needed). Metric: tokens/s.

Secondary workloads (key "extra"): small-batch decode (16 tokens, 4096 →
11008), prefill (2048 tokens, 4096 → 4096; INT8 tensor-core contraction timed
apart from the activation quantiser), the ternary FFN block (4096 → 11008 →
4096, M ∈ {1, 64, 512}) and the weight quantiser.

--impl reference times the CPU oracle (test infrastructure, the reference
arm) on the host cores on the decode workload.

Multi-GPU: one process per GPU (torchrun); every rank runs its own decode
stream (weak scaling, no data-path collective); time = max over ranks.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

import synth_inputs as si  # noqa: E402

METRIC = "BitLinear tokens/s; decode % of HBM roofline, prefill % of INT8 TC peak"
UNIT = "tokens/s"
EPS = 1e-5
DECODE = dict(M=1, K=2560, N=6912)
DECODE_WORKLOAD = "decode GEMV: 1 token, K=2560, N=6912, bf16 in/out, 1% x20 outlier channels"
CALLS_PER_STEP = 1000
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0
INT8_OVER_BF16 = 4.5 / 2.25  # nominal dense ratio (B200: 4.5 PFLOP/s fp8/int8, 2.25 bf16)
PROFILE_TRAFFIC = os.path.join(ROOT, "profiles", "gemv_decode_k2560_n6912.json")
GEMV_SOURCE = os.path.join(ROOT, "ternary_weight_linear_absmax_b200", "csrc", "gemv_kernel.cuh")


# ---------------------------------------------------------------------------
# distributed plumbing (also exercised on CPU with gloo by the tests)

def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def reduce_max(value: float, device=None) -> float:
    """Max of a float over all ranks (identity when not distributed)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate(per_rank_units: float, elapsed_max_s: float, world: int) -> float:
    """Whole-job throughput: units processed by all ranks ÷ the slowest rank's time."""
    return per_rank_units * world / elapsed_max_s


def barrier(device=None):
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        if device is not None and device.type == "cuda":
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


# ---------------------------------------------------------------------------
# measured peaks and profile-derived traffic

def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        return {"hbm_gbs": float(d["hbm_gbs"]), "bf16_tflops": float(d["bf16_tflops"]),
                "bf16_tflops_sustained": float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                "source": "measured"}
    except Exception:
        return {"hbm_gbs": FALLBACK_HBM_GBS, "bf16_tflops": FALLBACK_BF16_TFLOPS,
                "bf16_tflops_sustained": 1400.0, "source": "fallback"}


def sha256_file(path):
    h = hashlib.sha256()
    with open(path, "rb") as f:
        h.update(f.read())
    return h.hexdigest()


def profiled_traffic():
    """DRAM bytes per launch of the decode GEMV from the committed ncu
    summary (profiles/*.json), or None when missing or taken on a different
    kernel source."""
    try:
        with open(PROFILE_TRAFFIC) as f:
            d = json.load(f)
        if d.get("kernel_source_sha256") != sha256_file(GEMV_SOURCE):
            return None
        return float(d["dram_bytes_per_launch"])
    except Exception:
        return None


TRAFFIC_COMMAND = ("python bench.py --profile-case decode  (then) ncu --metrics "
                   "gpu__time_duration.sum,dram__bytes_read.sum,dram__bytes_write.sum "
                   "--clock-control none -k regex:gemv_ternary -s 5 -c 5 --csv "
                   "--log-file ncu_decode.csv python bench.py --profile-case decode")


def write_traffic_json(csv_path):
    """Summarise the decode GEMV's ncu capture (TRAFFIC_COMMAND) into the
    JSON that profiled_traffic() reads, stamped with the kernel source hash."""
    import csv
    per = {}
    with open(csv_path) as f:
        rows = [r for r in csv.reader(f) if len(r) > 10]
    head = rows[0]
    ki, ni, vi, ii = (head.index("Kernel Name"), head.index("Metric Name"),
                      head.index("Metric Value"), head.index("ID"))
    kernel = None
    for r in rows[1:]:
        if "gemv_ternary" not in r[ki]:
            continue
        kernel = r[ki].split("(")[0]
        per.setdefault(r[ni], {})[r[ii]] = float(r[vi].replace(",", ""))
    mean = {k: sum(v.values()) / len(v) for k, v in per.items()}
    n = len(per["dram__bytes_read.sum"])
    M, K, N = DECODE["M"], DECODE["K"], DECODE["N"]
    out = {"kernel": kernel,
           "workload": f"decode GEMV, {M} token, K={K}, N={N}, bf16 in/out",
           "command": TRAFFIC_COMMAND,
           "launches_averaged": n,
           "dram_bytes_read_per_launch": mean["dram__bytes_read.sum"],
           "dram_bytes_write_per_launch": mean["dram__bytes_write.sum"],
           "dram_bytes_per_launch": mean["dram__bytes_read.sum"] + mean["dram__bytes_write.sum"],
           "algorithmic_bytes_per_launch": N * K // 4 + 2 * K * M + 2 * N * M,
           "gpu_time_duration_ns_per_launch_cold_serialised": mean["gpu__time_duration.sum"],
           "kernel_source_sha256": sha256_file(GEMV_SOURCE)}
    with open(PROFILE_TRAFFIC, "w") as f:
        json.dump(out, f, indent=1)
        f.write("\n")
    print(json.dumps(out))
    return 0


# ---------------------------------------------------------------------------
# clocks sampler (during the timed region; reads only)

class ClockSampler:
    """SM clock and clock-event reasons while the timed region runs. NVML is
    polled every 5 ms from a thread (the decode step is tens of ms long);
    without NVML, `nvidia-smi -lms 100` is read instead. Entering waits for
    the first sample, so the sampler is running when the timing starts."""
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    REASON_BITS = (("hw_slowdown", 0x8), ("hw_thermal_slowdown", 0x40),
                   ("sw_thermal_slowdown", 0x20), ("sw_power_cap", 0x4))

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []
        self.samples = []  # (sm_mhz, reason bits) from NVML
        self.smax = None
        self.source = None
        self.thread = None
        self.stop = threading.Event()
        self.first = threading.Event()

    def _nvml_index(self):
        vis = os.environ.get("CUDA_VISIBLE_DEVICES", "")
        parts = [q.strip() for q in vis.split(",") if q.strip()]
        if self.gpu < len(parts) and parts[self.gpu].isdigit():
            return int(parts[self.gpu])
        return self.gpu

    def __enter__(self):
        try:
            import pynvml
            pynvml.nvmlInit()
            h = pynvml.nvmlDeviceGetHandleByIndex(self._nvml_index())
            self.smax = float(pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM))
            reasons = getattr(pynvml, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
                pynvml.nvmlDeviceGetCurrentClocksThrottleReasons
            self.source = "nvml, 5 ms"

            def poll():
                while not self.stop.is_set():
                    try:
                        self.samples.append((float(pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM)),
                                             int(reasons(h))))
                    except Exception:
                        pass
                    self.first.set()
                    time.sleep(0.005)
            self.thread = threading.Thread(target=poll, daemon=True)
            self.thread.start()
            self.first.wait(2.0)
            return self
        except Exception:
            self.samples = []
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.QUERY}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.source = "nvidia-smi, 100 ms"
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
            self.first.wait(5.0)
        except Exception:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())
            self.first.set()

    def __exit__(self, *a):
        self.stop.set()
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
        if self.thread is not None:
            self.thread.join(timeout=2)

    def summary(self):
        sm, smax, reasons = [], self.smax, set()
        for mhz, bits in self.samples:
            sm.append(mhz)
            for nm, bit in self.REASON_BITS:
                if bits & bit:
                    reasons.add(nm)
        names = [nm for nm, _ in self.REASON_BITS]
        for ln in self.lines:
            parts = [q.strip() for q in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax = float(parts[2])
            except ValueError:
                continue
            for nm, v in zip(names, parts[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(nm)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": smax, "reasons": [], "samples": 0,
                    "source": self.source}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": smax,
                "reasons": sorted(reasons), "samples": len(sm), "source": self.source}


# ---------------------------------------------------------------------------
# CUDA helpers

def l2_bytes(device_index: int) -> int:
    import torch
    try:
        return int(torch.cuda.get_device_properties(device_index).L2_cache_size)
    except Exception:
        return 126 * 1024 * 1024


def time_graph(graph, stream, reps: int):
    """Replay a captured graph `reps` times; device time in seconds."""
    import torch
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        start.record(stream)
        for _ in range(reps):
            graph.replay()
        end.record(stream)
    end.synchronize()
    return start.elapsed_time(end) / 1e3


def settled_time(graph, stream, reps: int, windows: int = 5):
    """Device seconds per replay of a captured graph for the secondary
    figures: after the caller's warm-up replays, synchronise, then time
    `windows` windows of `reps` replays and take the median window. (The
    first window after capture measured up to 1.6x slower than the rest.)"""
    import torch
    torch.cuda.synchronize()
    ts = [time_graph(graph, stream, reps) / reps for _ in range(windows)]
    return statistics.median(ts)


def capture(fn, stream):
    import torch
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(stream):
        fn()  # one eager call first (binds workspaces, sets kernel attributes)
        stream.synchronize()
        with torch.cuda.graph(g, stream=stream):
            fn()
    torch.cuda.synchronize()
    return g


def weight_pool(bl, N, K, seed, device, min_bytes, max_count=512):
    """Distinct packed matrices: one seeded bf16 matrix quantised by the
    library, then row-rotated copies (different contents, same statistics)."""
    import torch
    W = si.weights(N, K, seed=seed, dtype="bf16").torch(device)
    packed, gamma = bl.bl_quant_weights(W, EPS)
    del W
    count = max(1, min(max_count, math.ceil(min_bytes / packed.numel())))
    pool = [packed] + [torch.roll(packed, shifts=37 * i, dims=0).contiguous() for i in range(1, count)]
    return pool, gamma


# ---------------------------------------------------------------------------
# decode (headline)

def run_decode(bl, device, steps, warmup, peaks, world):
    import torch
    M, K, N = DECODE["M"], DECODE["K"], DECODE["N"]
    stream = torch.cuda.Stream(device)
    l2 = l2_bytes(device.index)
    pool, gamma = weight_pool(bl, N, K, 0, device, 3 * l2)
    tok = si.activations(CALLS_PER_STEP, K, seed=0, dtype="bf16").torch(device)
    Y = torch.empty((CALLS_PER_STEP, N), dtype=torch.bfloat16, device=device)

    def chain():
        for i in range(CALLS_PER_STEP):
            bl.bl_linear(tok[i:i + 1], pool[i % len(pool)], gamma, EPS, out=Y[i:i + 1],
                         pdl=True, stream=stream)

    graph = capture(chain, stream)
    for _ in range(max(3, warmup)):
        graph.replay()
    torch.cuda.synchronize()
    barrier(device)
    torch.cuda.synchronize()
    with ClockSampler(device.index) as clk:
        t = time_graph(graph, stream, steps)
    torch.cuda.synchronize()
    barrier(device)
    t_max = reduce_max(t, device)
    status = bl.bl_check_device_error(stream)
    if status != 0:
        raise RuntimeError(f"device error flag {status} after decode timing")

    launch_s = t / (steps * CALLS_PER_STEP)
    alg_bytes = N * K // 4 + M * K * 2 + M * N * 2
    achieved = alg_bytes / launch_s / 1e9
    res = {
        "value": aggregate(steps * CALLS_PER_STEP * M, t_max, world),
        "ms_per_step": t_max / steps * 1e3,
        "launch_us": launch_s * 1e6,
        "alg_bytes": alg_bytes,
        "achieved_gbs": achieved,
        "pool": {"matrices": len(pool), "bytes": len(pool) * pool[0].numel(), "l2_bytes": l2},
        "clocks": clk.summary(),
        "launches": steps * CALLS_PER_STEP,
    }

    # End to end through the public API: per step, copy the step's 1000
    # tokens from pinned host memory, run the chain, copy the 1000 outputs
    # back. Two device buffer sets (a graph captured on each) and separate
    # copy streams let step s+1's upload and step s-1's download run while
    # step s computes, as a serving loop would.
    h_tok = tok.cpu().pin_memory()
    h_out = [torch.empty(Y.shape, dtype=Y.dtype, pin_memory=True) for _ in range(2)]
    tok2 = torch.empty_like(tok)
    Y2 = torch.empty_like(Y)

    def chain2():
        for i in range(CALLS_PER_STEP):
            bl.bl_linear(tok2[i:i + 1], pool[i % len(pool)], gamma, EPS, out=Y2[i:i + 1],
                         pdl=True, stream=stream)

    graph2 = capture(chain2, stream)
    bufs = [(tok, Y, graph), (tok2, Y2, graph2)]
    up, down = torch.cuda.Stream(device), torch.cuda.Stream(device)
    e2e_steps = max(10, min(steps, 200))

    def e2e_run(n, timed):
        ev_in = [torch.cuda.Event() for _ in range(2)]
        ev_done = [torch.cuda.Event() for _ in range(2)]
        ev_free = [torch.cuda.Event() for _ in range(2)]
        s_ev, e_ev = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        if timed:
            barrier(device)
        s_ev.record(up)
        for k in range(n):
            b = k % 2
            d_tok, d_y, g = bufs[b]
            with torch.cuda.stream(up):
                if k >= 2:
                    up.wait_event(ev_free[b])
                d_tok.copy_(h_tok, non_blocking=True)
                ev_in[b].record(up)
            with torch.cuda.stream(stream):  # replay() launches on the current stream
                stream.wait_event(ev_in[b])
                g.replay()
                ev_done[b].record(stream)
            with torch.cuda.stream(down):
                down.wait_event(ev_done[b])
                h_out[b].copy_(d_y, non_blocking=True)
                ev_free[b].record(down)
        e_ev.record(down)
        e_ev.synchronize()
        return s_ev.elapsed_time(e_ev) / 1e3

    e2e_run(3, False)
    te = reduce_max(e2e_run(e2e_steps, True), device)
    res["e2e"] = {"value": aggregate(e2e_steps * CALLS_PER_STEP * M, te, world), "unit": UNIT,
                  "h2d_bytes_per_step": h_tok.numel() * h_tok.element_size(),
                  "d2h_bytes_per_step": h_out[0].numel() * h_out[0].element_size(),
                  "overlap": "uploads and downloads on two copy streams, two buffer sets"}
    del graph2

    # Single isolated call (no PDL overlap, weights cold in L2).
    flush = torch.empty(2 * l2, dtype=torch.uint8, device=device)
    lat = []
    with torch.cuda.stream(stream):
        for i in range(20):
            flush.fill_(i & 0xFF)
            s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            s.record(stream)
            bl.bl_linear(tok[0:1], pool[i % len(pool)], gamma, EPS, out=Y[0:1], stream=stream)
            e.record(stream)
            e.synchronize()
            lat.append(s.elapsed_time(e) * 1e3)
    res["single_call_us_median"] = statistics.median(lat[3:])
    del graph

    # Floor of a dependent chain with the same launch shape: empty kernels
    # (launch_dependents + wait only), 1000 per graph.
    def floor_chain():
        for _ in range(CALLS_PER_STEP):
            bl.bl_probe_pdl_floor(M, K, N, stream=stream)
    fg = capture(floor_chain, stream)
    for _ in range(3):
        fg.replay()
    tf = settled_time(fg, stream, max(3, min(steps, 10)))
    res["floor_us"] = tf / CALLS_PER_STEP * 1e6
    del fg
    res["pool_list"] = pool
    res["gamma"] = gamma
    res["tok"] = tok
    return res


def run_decode_storage_variants(bl, device, dec, peaks, reps=5):
    """The decode chain of the headline on the other two weight storages:
    radix-3 (5 weights per byte) and lookup-table index bytes. Same tokens,
    same matrices (converted), 1000 chained calls with PDL."""
    import torch
    M, K, N = DECODE["M"], DECODE["K"], DECODE["N"]
    stream = torch.cuda.Stream(device)
    pool, gamma, tok = dec["pool_list"], dec["gamma"], dec["tok"]
    Y = torch.empty((CALLS_PER_STEP, N), dtype=torch.bfloat16, device=device)
    out = {}
    r3 = [bl.bl_pack_radix3(w, K) for w in pool]
    lut = [bl.bl_pack_lut_index(w) for w in pool]
    torch.cuda.synchronize()
    rb = r3[0].shape[1]
    for name, mats, call, wbytes in (
            ("radix3", r3, bl.bl_linear_radix3, N * rb),
            ("lut_index", lut, bl.bl_linear_lut, N * K // 4)):
        def chain():
            for i in range(CALLS_PER_STEP):
                call(tok[i:i + 1], mats[i % len(mats)], gamma, EPS, out=Y[i:i + 1], pdl=True,
                     stream=stream)
        g = capture(chain, stream)
        for _ in range(3):
            g.replay()
        t = settled_time(g, stream, reps) / CALLS_PER_STEP
        alg = wbytes + M * K * 2 + M * N * 2
        out[name] = {"us_per_call": t * 1e6, "tokens_per_s": M / t, "weight_bytes": wbytes,
                     "gbs": alg / t / 1e9, "hbm_frac": alg / t / 1e9 / peaks["hbm_gbs"]}
        del g
    del r3, lut
    return out


def run_ste(bl, device, peaks, reps=10):
    """STE backward at the prefill shape (2048 tokens, 4096 → 4096): dA and dW,
    each 2·M·N·K flops on the bf16 tensor cores (layout kernels included)."""
    import torch
    M, N, K = 2048, 4096, 4096
    stream = torch.cuda.Stream(device)
    W = si.weights(N, K, seed=0, dtype="bf16").torch(device)
    packed, gamma = bl.bl_quant_weights(W, EPS)
    A = si.activations(M, K, seed=0, dtype="bf16").torch(device)
    Aq, gA, _ = bl.bl_quant_acts(A, EPS)
    dY = si.activations(M, N, seed=5, dtype="bf16").torch(device)
    torch.cuda.synchronize()
    flops = 2.0 * M * N * K
    res = {"workload": "dY [2048, 4096] bf16; W 4096x4096; A_q [2048, 4096]; fp32 gradients"}
    for name, fn in (("grad_input", lambda: bl.bl_ste_grad_input(dY, packed, gamma, stream=stream)),
                     ("grad_weight", lambda: bl.bl_ste_grad_weight(dY, Aq, gA, W, gamma, EPS,
                                                                   stream=stream))):
        t = rotating_time([fn], stream, reps)
        res[name] = {"us": t * 1e6, "tflops": flops / t / 1e12,
                     "frac_of_bf16_peak": flops / t / 1e12 / peaks["bf16_tflops"]}
    return res


# ---------------------------------------------------------------------------
# secondary workloads

def run_small_batch(bl, device, peaks, reps=200):
    import torch
    M, K, N = 16, 4096, 11008
    stream = torch.cuda.Stream(device)
    pool, gamma = weight_pool(bl, N, K, 0, device, 3 * l2_bytes(device.index))
    A = si.activations(M, K, seed=0, dtype="bf16").torch(device)
    Y = torch.empty((M, N), dtype=torch.bfloat16, device=device)
    ws = torch.empty(bl.workspace_bytes("linear", M, K, N), dtype=torch.uint8, device=device)
    calls = len(pool)

    def chain():
        for i in range(calls):
            bl.bl_linear(A, pool[i], gamma, EPS, out=Y, workspace=ws, pdl=True, stream=stream)

    g = capture(chain, stream)
    for _ in range(3):
        g.replay()
    t = settled_time(g, stream, max(1, reps // calls)) / calls
    alg = N * K // 4 + M * K * 2 + M * N * 2
    del g
    return {"workload": "16 tokens, K=4096 -> N=11008, bf16, rotating weight pool > L2, "
                        "chained calls with programmatic dependent launch",
            "tokens_per_s": M / t, "us_per_call": t * 1e6,
            "gbs": alg / t / 1e9, "hbm_frac": alg / t / 1e9 / peaks["hbm_gbs"],
            "tops": 2.0 * M * N * K / t / 1e12}


def rotating_time(calls, stream, reps):
    """Average device time (s) of one call in `calls`: all calls are captured
    in one CUDA graph (no host overhead between launches) and replayed
    `reps` times. Each call works on its own input set and the sets together
    exceed the L2 cache, so consecutive launches do not reuse cached inputs."""
    def run():
        for c in calls:
            c()
    g = capture(run, stream)
    for _ in range(3):
        g.replay()
    t = settled_time(g, stream, reps)
    del g
    return t / len(calls)


def n_sets(bytes_per_set, device_index, factor=1.1):
    return max(2, math.ceil(factor * l2_bytes(device_index) / bytes_per_set))


def run_prefill(bl, device, peaks, reps=10):
    import torch
    M, K, N = 2048, 4096, 4096
    stream = torch.cuda.Stream(device)
    W = si.weights(N, K, seed=0, dtype="bf16").torch(device)
    packed, gamma = bl.bl_quant_weights(W, EPS)
    del W
    A = si.activations(M, K, seed=0, dtype="bf16").torch(device)
    wsb = bl.workspace_bytes("linear", M, K, N)
    P = n_sets(N * K // 4 + M * K * 3 + M * N * 2 + wsb, device.index)
    sets = []
    for i in range(P):
        Ai = torch.roll(A, shifts=i, dims=0).contiguous()
        Aq, gA, rs = bl.bl_quant_acts(Ai, EPS)
        pk = torch.roll(packed, shifts=37 * i, dims=0).contiguous()
        Y = torch.empty((M, N), dtype=torch.bfloat16, device=device)
        ws = torch.empty(max(1, wsb), dtype=torch.uint8, device=device)
        sets.append((Ai, Aq, gA, rs, pk, Y, ws))
    torch.cuda.synchronize()
    tq = rotating_time([lambda s=s_: bl.bl_quant_acts(s[0], EPS, stream=stream) for s_ in sets],
                       stream, reps)
    tg = rotating_time([lambda s=s_: bl.bl_linear_q(s[1], s[2], s[4], gamma, rowsum=s[3], out=s[5],
                                                    pdl=True, stream=stream) for s_ in sets],
                       stream, reps)
    # The whole BitLinear forward (bf16 in, quantiser + contraction, bf16 out)
    # as a user calls it, chained with programmatic dependent launch.
    tl = rotating_time([lambda s=s_: bl.bl_linear(s[0], s[4], gamma, EPS, out=s[5], workspace=s[6],
                                                  pdl=True, stream=stream) for s_ in sets],
                       stream, reps)
    int8_peak = peaks["bf16_tflops"] * INT8_OVER_BF16
    ops = 2.0 * M * N * K
    return {"workload": "2048 tokens, K=4096 -> N=4096, int8 x ternary on tcgen05 kind::i8, bf16 out",
            "timing": f"CUDA graph over {P} rotating input sets (> L2), chained with programmatic dependent launch (static weights)",
            "gemm_us": tg * 1e6, "quant_acts_us": tq * 1e6, "linear_us": tl * 1e6,
            "tokens_per_s": M / tl, "tokens_per_s_separate_launches": M / (tg + tq),
            "gemm_tops": ops / tg / 1e12,
            "roofline": {"bound": "tensor", "achieved": ops / tg / 1e12, "peak": int8_peak,
                         "unit": "TOPS", "frac": ops / tg / 1e12 / int8_peak,
                         "peak_source": f"{peaks['source']} bf16 burst x {INT8_OVER_BF16:g} (nominal int8/bf16)"},
            "quant_acts_gbs": (M * K * 2 + M * K + 8 * M) / tq / 1e9}


def run_ffn(bl, device, peaks, Ms=(1, 64, 512), reps=10):
    import torch
    K, H = 4096, 11008
    stream = torch.cuda.Stream(device)
    Wu = si.weights(H, K, seed=1, dtype="bf16").torch(device)
    pu, gu = bl.bl_quant_weights(Wu, EPS)
    del Wu
    Wd = si.weights(K, H, seed=2, dtype="bf16").torch(device)
    pd, gd = bl.bl_quant_weights(Wd, EPS)
    del Wd
    out = {}
    for M in Ms:
        X = si.activations(M, K, seed=0, dtype="bf16").torch(device)
        wsb = max(1, bl.workspace_bytes("ffn", M, K, H))
        P = n_sets(2 * H * K // 4 + wsb + M * K * 4, device.index)
        sets = []
        for i in range(P):
            sets.append((torch.roll(X, shifts=i, dims=0).contiguous(),
                         torch.roll(pu, shifts=37 * i, dims=0).contiguous(),
                         torch.roll(pd, shifts=41 * i, dims=0).contiguous(),
                         torch.empty((M, K), dtype=torch.bfloat16, device=device),
                         torch.empty(wsb, dtype=torch.uint8, device=device)))
        t = rotating_time([lambda s=s_: bl.bl_ffn_relu2(s[0], s[1], gu, s[2], gd, EPS, out=s[3],
                                                        workspace=s[4], pdl=True, stream=stream)
                           for s_ in sets], stream, reps)
        wbytes = 2 * H * K // 4
        out[f"M{M}"] = {"us": t * 1e6, "tokens_per_s": M / t, "weight_gbs": wbytes / t / 1e9,
                        "tops": 4.0 * M * K * H / t / 1e12, "input_sets": P}
        del sets
    return out


def run_tp_ffn_shard(bl, device, worlds=(2, 4, 8), Ms=(1, 64, 512), reps=10):
    """One rank's compute in the tensor-parallel FFN block (4096 -> 11008 ->
    4096; the hidden dimension split over `world` ranks): the up step on its
    shard, the requantised down step and the final dequantisation, timed on
    one GPU over rotating weight shards larger than L2. The two all-reduces
    between them (MAX of M fp32, SUM of M x 4096 INT32) are not included;
    their payloads are reported."""
    import torch
    from ternary_weight_linear_absmax_b200.tp_ffn import shard_packed
    K, H = 4096, 11008
    stream = torch.cuda.Stream(device)
    pu, gu = bl.bl_quant_weights(si.weights(H, K, seed=1, dtype="bf16").torch(device), EPS)
    pd, gd = bl.bl_quant_weights(si.weights(K, H, seed=2, dtype="bf16").torch(device), EPS)
    out = {"note": "per-rank compute only; collectives excluded", "workload": "FFN 4096->11008->4096"}
    for world in worlds:
        pu_r, pd_r = shard_packed(pu, pd, H, world, 0)
        H_r = pu_r.shape[0]
        res = {"H_r": H_r}
        for M in Ms:
            X = si.activations(M, K, seed=0, dtype="bf16").torch(device)
            P = n_sets(pu_r.numel() + pd_r.numel() + M * H_r * 4, device.index)
            sets = [(torch.roll(pu_r, shifts=37 * i, dims=0).contiguous(),
                     torch.roll(pd_r, shifts=41 * i, dims=0).contiguous()) for i in range(P)]

            def step(s):
                acc, gx, rmax = bl.bl_ffn_tp_up(X, s[0], gu, EPS, stream=stream)
                part = bl.bl_ffn_tp_down(acc, gx, gu, rmax, s[1], EPS, stream=stream)
                bl.bl_dequant_i32(part, rmax, gd, stream=stream)
            t = rotating_time([lambda s=s_: step(s) for s_ in sets], stream, reps)
            res[f"M{M}"] = {"us": t * 1e6, "allreduce_bytes": M * 4 + M * K * 4, "input_sets": P}
            del sets
        out[f"world{world}"] = res
    return out


def run_quant_weights(bl, device, reps=5):
    import torch
    N, K = 11008, 4096
    stream = torch.cuda.Stream(device)
    W = si.weights(N, K, seed=0, dtype="bf16").torch(device)
    gamma = torch.empty((1,), dtype=torch.float32, device=device)
    ws = torch.empty(bl.workspace_bytes("quant_weights", 0, K, N), dtype=torch.uint8, device=device)
    sets = [(torch.roll(W, shifts=i, dims=0).contiguous(),
             torch.empty((N, K // 4), dtype=torch.uint8, device=device)) for i in range(2)]
    t = rotating_time([lambda s=s_: bl.bl_quant_weights(s[0], EPS, out=s[1], gamma=gamma,
                                                        workspace=ws, stream=stream)
                       for s_ in sets], stream, reps)
    alg = N * K * 2 * 2 + N * K // 4  # W read twice (γ pass, pack pass) + packed write
    return {"workload": "11008x4096 bf16 -> 2-bit packed", "us": t * 1e6,
            "gbs": alg / t / 1e9, "weights_per_s": N * K / t}


# ---------------------------------------------------------------------------
# CPU oracle timing (cpu_baseline and --impl reference)

def oracle_decode_rate(seconds: float = 12.0, max_calls: int | None = None):
    """Oracle BitLinear forward on the decode workload, one token per call,
    for about `seconds` (or `max_calls`). Returns (tokens/s, calls, threads)."""
    import oracle
    M, K, N = DECODE["M"], DECODE["K"], DECODE["N"]
    W = si.weights(N, K, seed=0, dtype="bf16").f32
    codes, g = oracle.quant_weights(W, EPS)
    tok = si.activations(64, K, seed=0, dtype="bf16").f32
    n, t0 = 0, time.perf_counter()
    while True:
        oracle.bitlinear(tok[n % 64:n % 64 + 1], codes, g, EPS)
        n += 1
        el = time.perf_counter() - t0
        if (max_calls is not None and n >= max_calls) or (max_calls is None and el >= seconds):
            break
    return n * M / el, n, oracle.max_threads()


# The five workloads, each timed on a bounded sample of its tokens (the
# oracle treats tokens independently, so tokens/s scales from the sample).
CPU_CONFIGS = [
    # name, kind, M (full), K, N (or H), tokens timed, dtype
    ("single_layer_4x512_256_f32", "linear", 4, 512, 256, 4, "f32"),
    ("decode_1x2560_6912", "linear", 1, 2560, 6912, 1, "bf16"),
    ("small_batch_16x4096_11008", "linear", 16, 4096, 11008, 2, "bf16"),
    ("prefill_2048x4096_4096", "linear", 2048, 4096, 4096, 2, "bf16"),
    ("ffn_4096_11008_M1", "ffn", 1, 4096, 11008, 1, "bf16"),
    ("ffn_4096_11008_M64", "ffn", 64, 4096, 11008, 1, "bf16"),
    ("ffn_4096_11008_M512", "ffn", 512, 4096, 11008, 1, "bf16"),
]


def oracle_per_config(min_seconds: float = 0.2):
    """Wall time of the oracle on every workload, single-threaded and on all
    host cores (OpenMP over output rows), on the same seeded inputs as the
    GPU. Returns {name: {...}} in tokens/s."""
    import oracle
    cores = oracle.max_threads()
    out, cache = {}, {}

    def codes_of(N, K, seed, dt):  # the three FFN workloads share their matrices
        if (N, K, seed, dt) not in cache:
            cache[(N, K, seed, dt)] = oracle.quant_weights(si.weights(N, K, seed=seed, dtype=dt).f32, EPS)
        return cache[(N, K, seed, dt)]

    for name, kind, M, K, N, T, dt in CPU_CONFIGS:
        X = si.activations(T, K, seed=0, outliers=(name != "single_layer_4x512_256_f32"),
                           dtype=dt).f32
        if kind == "linear":
            codes, g = codes_of(N, K, 0, dt)
            call = lambda: oracle.bitlinear(X, codes, g, EPS)  # noqa: E731
        else:
            cu, gu = codes_of(N, K, 1, dt)
            cd, gd = codes_of(K, N, 2, dt)
            call = lambda: oracle.ffn_relu2(X, cu, gu, cd, gd, EPS)  # noqa: E731
        row = {"tokens_timed": T, "tokens_full": M}
        for label, th in (("threads_1", 1), (f"threads_{cores}", cores)):
            oracle.set_threads(th)
            reps, t0 = 0, time.perf_counter()
            while True:
                call()
                reps += 1
                el = time.perf_counter() - t0
                if el >= min_seconds or reps >= 50:
                    break
            row[label] = {"tokens_per_s": reps * T / el, "s_per_call_full": el / reps * M / T,
                          "reps": reps}
        oracle.set_threads(cores)
        out[name] = row
    return out, cores


def lut_decode_rate(min_seconds: float = 1.0):
    """The host table-lookup BitLinear (libbitlinear_lut_cpu.so) on the decode
    workload, 1 thread and all cores. Returns {label: tokens/s} and the ISA."""
    import oracle
    from ternary_weight_linear_absmax_b200 import build as _b
    from ternary_weight_linear_absmax_b200 import lut_cpu
    _b.build_cpu()
    M, K, N = DECODE["M"], DECODE["K"], DECODE["N"]
    codes, g = oracle.quant_weights(si.weights(N, K, seed=0, dtype="bf16").f32, EPS)
    idx = lut_cpu.index_from_packed(oracle.pack_ternary(codes), K)
    tok = si.activations(64, K, seed=0, outliers=True, dtype="bf16").f32
    cores = oracle.max_threads()
    out = {}
    for th in (1, cores):
        lut_cpu.bitlinear_lut(tok[:1], idx, g, N, EPS, threads=th)
        n, t0 = 0, time.perf_counter()
        while time.perf_counter() - t0 < min_seconds:
            lut_cpu.bitlinear_lut(tok[n % 64:n % 64 + 1], idx, g, N, EPS, threads=th)
            n += 1
        out[f"threads_{th}"] = n * M / (time.perf_counter() - t0)
    return out, lut_cpu.ISA_NAMES[lut_cpu.best_isa()]


def run_reference(args):
    ws, rank, local = dist_env()
    if rank != 0:
        return 0
    import oracle
    oracle.build()
    import synth_inputs  # noqa: F401
    # warm-up calls, then the timed steps: one step = one decode call (1 token).
    oracle_decode_rate(max_calls=max(1, args.warmup))
    rate, n, cores = oracle_decode_rate(max_calls=max(1, args.steps))
    line = {
        "impl": "reference", "metric": METRIC, "value": rate, "unit": UNIT,
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 / rate, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "int8xternary->int32, fp32 scales", "data": "synthetic",
        "config": {"workload": DECODE_WORKLOAD,
                   "step": "one BitLinear call (1 token) of the CPU oracle"},
        "cpu_baseline": {"value": rate, "unit": UNIT, "cores": cores, "kind": "oracle",
                         "sample": f"{n} decode calls (1 token each) after {args.warmup} warm-up calls"},
        "e2e": {"value": rate, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------------------

# ---------------------------------------------------------------------------
# Small cases for ncu captures (one kernel each; the summaries under profiles/
# name these commands).

def profile_case(name: str) -> int:
    import torch
    import ternary_weight_linear_absmax_b200 as bl
    bl.load()
    device = torch.device("cuda", 0)
    torch.cuda.set_device(device)
    st = torch.cuda.Stream(device)
    if name in ("decode", "decode_radix3"):
        # 20 chained decode calls (1 token, 2560 -> 6912) over 6 distinct matrices
        K, N = DECODE["K"], DECODE["N"]
        mats = []
        for i in range(6):
            pk, g = bl.bl_quant_weights(si.weights(N, K, seed=i, dtype="bf16").torch(device), EPS)
            mats.append((bl.bl_pack_radix3(pk, K) if name == "decode_radix3" else pk, g))
        tok = si.activations(20, K, seed=0, dtype="bf16").torch(device)
        call = bl.bl_linear_radix3 if name == "decode_radix3" else bl.bl_linear
        torch.cuda.synchronize()
        for i in range(20):
            w, g = mats[i % 6]
            call(tok[i:i + 1], w, g, EPS, pdl=True, stream=st)
    elif name in ("skinny", "prefill"):
        M, K, N = (16, 4096, 11008) if name == "skinny" else (2048, 4096, 4096)
        pk, g = bl.bl_quant_weights(si.weights(N, K, seed=0, dtype="bf16").torch(device), EPS)
        Aq, gA, rs = bl.bl_quant_acts(si.activations(M, K, seed=0, dtype="bf16").torch(device), EPS)
        torch.cuda.synchronize()
        for _ in range(3):
            bl.bl_linear_q(Aq, gA, pk, g, rowsum=rs, pdl=True, stream=st)
    elif name in ("ffn1", "ffn64", "ffn512", "small_chain"):
        K, H = 4096, 11008
        if name.startswith("ffn"):
            M = int(name[3:])
            pu, gu = bl.bl_quant_weights(si.weights(H, K, seed=1, dtype="bf16").torch(device), EPS)
            pd, gd = bl.bl_quant_weights(si.weights(K, H, seed=2, dtype="bf16").torch(device), EPS)
            X = si.activations(M, K, seed=0, dtype="bf16").torch(device)
            ws = torch.empty(bl.workspace_bytes("ffn", M, K, H), dtype=torch.uint8, device=device)
            torch.cuda.synchronize()
            for _ in range(3):
                bl.bl_ffn_relu2(X, pu, gu, pd, gd, EPS, workspace=ws, pdl=True, stream=st)
        else:  # 10 chained 16-token calls over 5 distinct 11008 x 4096 matrices
            mats = [bl.bl_quant_weights(si.weights(H, K, seed=i, dtype="bf16").torch(device), EPS)
                    for i in range(5)]
            A = si.activations(16, K, seed=0, dtype="bf16").torch(device)
            ws = torch.empty(bl.workspace_bytes("linear", 16, K, H), dtype=torch.uint8, device=device)
            torch.cuda.synchronize()
            for i in range(10):
                w, g = mats[i % 5]
                bl.bl_linear(A, w, g, EPS, workspace=ws, pdl=True, stream=st)
    elif name == "ste":
        M, N, K = 2048, 4096, 4096
        W = si.weights(N, K, seed=0, dtype="bf16").torch(device)
        pk, g = bl.bl_quant_weights(W, EPS)
        dY = si.activations(M, N, seed=5, dtype="bf16").torch(device)
        torch.cuda.synchronize()
        A = si.activations(M, K, seed=0, dtype="bf16").torch(device)
        Aq, gA, _ = bl.bl_quant_acts(A, EPS)
        torch.cuda.synchronize()
        for _ in range(2):
            bl.bl_ste_grad_input(dY, pk, g, stream=st)
        for _ in range(2):
            bl.bl_ste_grad_weight(dY, Aq, gA, W, g, EPS, stream=st)
    else:
        raise SystemExit(f"unknown profile case {name}")
    st.synchronize()
    return int(bl.bl_check_device_error(st))


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-extra", action="store_true", help="skip the secondary workloads")
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--profile-case", choices=["decode", "decode_radix3", "skinny", "prefill", "ste",
                                               "ffn1", "ffn64", "ffn512", "small_chain"],
                    help="run one small case for an ncu capture and exit")
    ap.add_argument("--traffic-json", metavar="NCU_CSV",
                    help="write the decode GEMV traffic summary read by the bench line "
                         "from an ncu CSV of the --profile-case decode capture, and exit")
    args = ap.parse_args(argv)
    if args.traffic_json:
        return write_traffic_json(args.traffic_json)
    if args.profile_case:
        return profile_case(args.profile_case)
    if args.impl == "reference":
        return run_reference(args)
    args.warmup = max(3, args.warmup)

    import torch
    ws, rank, local = dist_env()
    if ws > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    import ternary_weight_linear_absmax_b200 as bl
    bl.load()
    peaks = load_peaks()

    dec = run_decode(bl, device, args.steps, args.warmup, peaks, ws)
    extra = {}
    # The secondary workloads run in single-GPU runs only: in a multi-GPU run
    # the other ranks would sit idle (holding their GPUs) while rank 0 works.
    if not args.no_extra and rank == 0 and ws == 1:
        extra["decode_single_call_us"] = dec["single_call_us_median"]
        extra["decode_pool"] = dec["pool"]
        extra["small_batch"] = run_small_batch(bl, device, peaks)
        extra["prefill"] = run_prefill(bl, device, peaks)
        extra["ffn"] = run_ffn(bl, device, peaks)
        extra["quant_weights"] = run_quant_weights(bl, device)
        extra["decode_storage_variants"] = run_decode_storage_variants(bl, device, dec, peaks)
        extra["ste_backward"] = run_ste(bl, device, peaks)
        extra["tp_ffn_shard"] = run_tp_ffn_shard(bl, device)
    cpu = None
    if rank == 0 and ws == 1:
        rate, n, cores = oracle_decode_rate(seconds=args.cpu_seconds)
        cpu = {"value": rate, "unit": UNIT, "cores": cores, "kind": "oracle",
               "sample": f"{n} decode calls (1 token, K=2560, N=6912) in ~{args.cpu_seconds:g} s"}
        if not args.no_extra:
            rates, isa = lut_decode_rate()
            cpu["lut_simd"] = {"unit": UNIT, "kind": "host table-lookup BitLinear (81 entries per "
                                                     "4 activations), not the oracle",
                               "isa": isa, **rates,
                               "sample": "decode calls (1 token, K=2560, N=6912) for 1 s each"}
            cpu["per_config"], _ = oracle_per_config()
            cpu["per_config_sample"] = ("each workload timed for >= 0.2 s on 'tokens_timed' of its "
                                        "tokens, 1 thread and all cores; s_per_call_full scales "
                                        "to the workload's full token count")
    if ws > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    if rank != 0:
        return 0
    traffic = profiled_traffic()
    line = {
        "metric": METRIC, "value": dec["value"], "unit": UNIT, "n_gpus": ws,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": dec["ms_per_step"],
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "int8 x ternary -> int32 (bf16 in/out, fp32 scales)", "data": "synthetic",
        "config": {"workload": DECODE_WORKLOAD,
                   "calls_per_step": CALLS_PER_STEP, "launch": "CUDA graph, programmatic dependent launch",
                   "l2": f"no flush: rotating pool of {dec['pool']['matrices']} packed matrices "
                         f"({dec['pool']['bytes'] / 1e6:.0f} MB) > 3x L2",
                   "parallelism": f"replicas x{ws}"},
        "roofline": {"bound": "hbm", "achieved": dec["achieved_gbs"], "peak": peaks["hbm_gbs"],
                     "unit": "GB/s", "frac": dec["achieved_gbs"] / peaks["hbm_gbs"],
                     "traffic": traffic, "kernel": "gemv_ternary_kernel",
                     "alg_bytes_per_launch": dec["alg_bytes"], "launch_us": dec["launch_us"],
                     "chain_floor_us": dec["floor_us"],
                     "above_floor_us": dec["launch_us"] - dec["floor_us"],
                     "peak_source": f"{peaks['source']} hbm_gbs"},
        "cpu_baseline": cpu,
        "e2e": dec["e2e"],
        "gpu_launches": dec["launches"],
        "clocks": dec["clocks"],
        "extra": extra,
    }
    print(json.dumps(line), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
