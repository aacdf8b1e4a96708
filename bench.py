"""Benchmark of the head-wise sparse attention layer (RTPurbo) on B200.

One JSON line on rank 0 (see --help).  By default a step is one decode token of the 128K workload:
B = 8 sequences of N = 131072 keys, 32 query / 4 KV heads (D = 128), 5 retrieval heads (r = 16,
p = 0.9) and 27 local heads (W = 8192, S = 4), seeded synthetic data shaped like the pages'
workloads.  Each step appends the token's K/V (RoPE + index keys) and runs the decode
(index stream, exact top-p, sparse attention, window + sink attention), through the C ABI.
Before every step the length is rolled back by one, so every step sees exactly N keys.

value   = decode microseconds per token (step time / B; all ranks' tokens / max rank time)
e2e     = the same through the C ABI with the step's q/k/v copied from pinned host memory
          and the output copied back, inside the timed region
roofline= the dominant kernel (fused index stream + top-p select): algorithmic bytes (the
          16-dim fp32 index keys, 64 B per key per retrieval head per sequence) per launch over
          its mean device time from CUDA events on its launch stream
--workload prefill_32k | prefill_1m: a step is one chunked-prefill call (the chunk's K/V
          appended, then every row's selection / window and attention), value in ms per chunk;
          the roofline is the chunk's longest kernel: the selection against the MUFU peak
          (one exp per causal (row, key) pair), or the local-head tcgen05 kernel (flops
          4 D sum_i |J_i| per head) or the retrieval attention kernel (4 D per selected pair)
          against the tensor peak
--impl reference: the fp64 CPU oracle as it stands, on this host's cores, same metric.

Multi-GPU: the layer does not shard; --gpus N runs N independent replicas (one per GPU).
"""
from __future__ import annotations

import argparse
import dataclasses
import hashlib
import json
import math
import os
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "RTPurbo attn layer: decode µs/token & prefill ms at 128K/1M; % of roofline"
DECODE_WORKLOADS = ("decode_128k", "decode_1m")
PREFILL_WORKLOADS = ("prefill_32k", "prefill_1m")


def _peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


def _tensor_peak():
    """Dense 16-bit tensor peak (TFLOP/s): the measured cuBLAS bf16 burst figure (fp16 runs at
    the same nominal rate), else the fallback."""
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            d = json.load(f)
        return float(d["bf16_tflops"]), "measured (bf16 burst; fp16 has the same nominal rate)"
    except Exception:
        return 1590.0, "fallback"


# MUFU (ex2) issue rate per SM per clock on B200, the unit the prefill selection's exponentials
# run on; the peak is this rate times the SM count times the sampled SM clock.
MUFU_EX2_PER_CLK_SM = 16


def _prefill_traffic(kernel: str, workload: str):
    """Per-launch DRAM bytes of the prefill retrieval kernels at the 32K and the 1M chunk, from
    the committed ncu summaries (each captured on its own workload), while their sources are
    unchanged since the capture (else None)."""
    files = {"prefill_32k": "prefill_kernels_32k.md", "prefill_1m": "prefill_kernels_1m.md"}
    if kernel not in ("prefill_select", "prefill_attn") or workload not in files:
        return None
    try:
        text = open(os.path.join(ROOT, "profiles", files[workload])).read()
    except OSError:
        return None
    traffic, srcs = None, None
    for line in text.splitlines():
        if line.startswith(f"- {kernel} dram bytes per launch (read + write):"):
            traffic = float(line.rsplit(":", 1)[1].strip().split()[0])
        if line.startswith(f"- {kernel} sources sha256[:16]:"):
            srcs = line.split("sha256[:16]:", 1)[1].strip()
    if traffic is None or srcs is None:
        return None
    for item in srcs.split(","):
        name, want = item.split()
        path = os.path.join(ROOT, "long_context_sparse_idx16_b200", "csrc", name)
        try:
            if hashlib.sha256(open(path, "rb").read()).hexdigest()[:16] != want:
                return None
        except OSError:
            return None
    return traffic


def _prefill_rooflines(kern: dict, flops: dict, exps: int, exp_peak: dict, sm_mhz, tensor_peak: float,
                       tensor_peak_kind: str) -> dict:
    """Roofline objects of the prefill chunk's kernels.

    prefill_select evaluates one exponential per causal (row, key) pair and is bound by the
    exp (MUFU) and integer pipes: "alu" against the exponential rate measured on this GPU by the
    ex2 probe (scaled to the SM clock sampled during the prefill).  prefill_attn and
    prefill_local are "tensor" against the dense 16-bit peak with algorithmic flops (4 D per
    attended pair).  "index_plus_sparse_attention" puts the retrieval heads' two kernels
    together against the tensor peak: 2 r flops per causal (row, key) index score plus the
    attention flops, over the two kernels' summed time."""
    out = {}
    if kern.get("prefill_select", {}).get("ms_per_launch", 0) > 0:
        ms = kern["prefill_select"]["ms_per_launch"]
        mhz = float(sm_mhz) if sm_mhz else float(exp_peak["sm_mhz"])
        peak = exp_peak["per_clk_per_sm"] * exp_peak["sms"] * mhz * 1e6 / 1e9
        achieved = exps / (ms * 1e-3) / 1e9
        out["prefill_select"] = {
            "bound": "alu", "kernel": "prefill_select", "achieved": achieved, "peak": peak,
            "peak_kind": (f"measured: ex2 probe {exp_peak['per_clk_per_sm']:.2f} per clock per SM x "
                          f"{exp_peak['sms']} SMs x {mhz:.0f} MHz ({'sampled' if sm_mhz else 'probe'} SM clock)"),
            "unit": "Gexp/s", "frac": achieved / peak, "traffic": None, "exps_per_launch": int(exps),
            "ms_per_launch": ms}
    for k, f in (("prefill_attn", flops["retrieval_attention"]), ("prefill_local", flops["local_attention"])):
        if kern.get(k, {}).get("ms_per_launch", 0) > 0:
            ms = kern[k]["ms_per_launch"]
            a = f / (ms * 1e-3) / 1e12
            out[k] = {"bound": "tensor", "kernel": k, "achieved": a, "peak": tensor_peak,
                      "peak_kind": tensor_peak_kind, "unit": "TFLOP/s", "frac": a / tensor_peak, "traffic": None,
                      "flops_per_launch": int(f), "ms_per_launch": ms}
    if "prefill_select" in out and "prefill_attn" in out:
        ms = out["prefill_select"]["ms_per_launch"] + out["prefill_attn"]["ms_per_launch"]
        f = flops["index_scores_flops"] + flops["retrieval_attention"]
        a = f / (ms * 1e-3) / 1e12
        out["index_plus_sparse_attention"] = {
            "bound": "tensor", "kernels": ["prefill_select", "prefill_attn"], "achieved": a, "peak": tensor_peak,
            "peak_kind": tensor_peak_kind, "unit": "TFLOP/s", "frac": a / tensor_peak, "flops_per_launch": int(f),
            "ms_per_launch": ms}
    return out


_TRAFFIC_KEYS = 40 * 131072  # keys streamed by the launch the committed traffic figure is for


def _profile_traffic(kernel_src: str):
    """Per-launch DRAM traffic of the select kernel from the committed ncu summary, if the
    kernel source has not changed since that capture (else None)."""
    path = os.path.join(ROOT, "profiles", "decode_select_128k.md")
    try:
        text = open(path).read()
    except OSError:
        return None
    want = hashlib.sha256(open(kernel_src, "rb").read()).hexdigest()[:16]
    traffic = None
    src_hash = None
    for line in text.splitlines():
        if line.startswith("- source sha256[:16]:"):
            src_hash = line.rsplit(":", 1)[1].strip()
        if line.startswith("- dram bytes per launch (read + write):"):
            traffic = float(line.split(":", 1)[1].strip().split()[0])
    return traffic if (src_hash == want and traffic) else None


class ClockSampler:
    """SM clock and throttle-reason sampling while a timed region runs (read-only).

    NVML (the library nvidia-smi reads) is polled from a thread about every half millisecond,
    so even a region of a few milliseconds gets samples; where NVML cannot be loaded,
    nvidia-smi is run in the background instead (50 ms period)."""

    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    # NVML clock-event reason bits, in the order of the names below
    REASONS = (("hw_slowdown", 0x8), ("hw_thermal_slowdown", 0x40), ("sw_thermal_slowdown", 0x20),
               ("sw_power_cap", 0x4))

    def __init__(self, gpu: int):
        self.gpu = gpu
        self.proc = None
        self.thread = None
        self.rows = []
        self.path = os.path.join("/tmp", f"rtp_clocks_{os.getpid()}.csv")

    def _nvml_handle(self):
        import pynvml
        import torch

        pynvml.nvmlInit()
        try:
            uuid = str(torch.cuda.get_device_properties(self.gpu).uuid)
            return pynvml.nvmlDeviceGetHandleByUUID(uuid if uuid.startswith("GPU-") else "GPU-" + uuid)
        except Exception:
            return pynvml.nvmlDeviceGetHandleByIndex(self.gpu)

    def start(self):
        import threading

        try:
            import pynvml

            h = self._nvml_handle()
            smax = pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM)
            self._stop = threading.Event()

            def poll():
                while not self._stop.is_set():
                    try:
                        sm = pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM)
                        rs = pynvml.nvmlDeviceGetCurrentClocksEventReasons(h)
                        self.rows.append((float(sm), float(smax), int(rs)))
                    except Exception:
                        pass
                    time.sleep(0.0005)

            self.thread = threading.Thread(target=poll, daemon=True)
            self.thread.start()
            return
        except Exception:
            self.thread = None
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.QUERY}", "--format=csv,noheader,nounits",
                 "-lms", "50"], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None

    def stop(self):
        if self.thread is not None:
            self._stop.set()
            self.thread.join(timeout=5)
            rows = self.rows
            if not rows:
                return None
            sm = sorted(r[0] for r in rows)
            reasons = sorted({n for r in rows for n, bit in self.REASONS if r[2] & bit})
            return {"sm_mhz": sm[len(sm) // 2], "sm_max_mhz": max(r[1] for r in rows), "reasons": reasons,
                    "samples": len(rows), "source": "nvml"}
        if self.proc is None:
            return None
        time.sleep(0.06)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        rows = []
        for line in open(self.path):
            f = [x.strip() for x in line.split(",")]
            if len(f) >= 9:
                rows.append(f)
        os.unlink(self.path)
        if not rows:
            return None
        sm = sorted(float(r[1]) for r in rows if r[1].replace(".", "").isdigit())
        smax = max(float(r[2]) for r in rows if r[2].replace(".", "").isdigit())
        names = [n for n, _ in self.REASONS]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower() == "active"})
        return {"sm_mhz": sm[len(sm) // 2] if sm else None, "sm_max_mhz": smax, "reasons": reasons,
                "samples": len(rows), "source": "nvidia-smi"}


def _dist():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def _max_over_ranks(x: float, world: int, device) -> float:
    if world == 1:
        return x
    import torch
    import torch.distributed as dist

    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def cpu_oracle_sample(x, seconds: float = 12.0):
    """Time the fp64 oracle (as it stands) on the decode step of whole sequences until about
    `seconds` of CPU work; returns (us per token, cores, description)."""
    import oracle

    s = x.spec
    t0 = time.perf_counter()
    done = 0
    for b in range(s.batch):
        for h in range(s.n_q_heads):
            oracle.layer_rows(x, b, h, [0], want_sel=False)
        done += 1
        if time.perf_counter() - t0 >= seconds:
            break
    dt = time.perf_counter() - t0
    return dt / done * 1e6, oracle.max_threads(), f"decode step of {done} of {s.batch} sequences, all {s.n_q_heads} heads"


def cpu_oracle_prefill_sample(x, seconds: float = 12.0):
    """Time the fp64 oracle (as it stands) on chunk rows spread over the chunk, one retrieval
    and one local head per row, until about `seconds`; returns (ms per chunk, cores,
    description), the chunk time being mean row time per class x rows x heads per class."""
    import numpy as np

    import oracle

    s = x.spec
    C = s.chunk
    Hr = len(s.retrieval_heads)
    loc = [h for h in range(s.n_q_heads) if h not in s.retrieval_heads]
    rows = np.linspace(0, C - 1, 64).astype(np.int64)
    tr = tl = 0.0
    n = 0
    t_start = time.perf_counter()
    for i, row in enumerate(rows):
        b = i % s.batch
        t0 = time.perf_counter()
        oracle.layer_rows(x, b, s.retrieval_heads[i % Hr], [int(row)], want_sel=False)
        t1 = time.perf_counter()
        if loc:
            oracle.layer_rows(x, b, loc[i % len(loc)], [int(row)], want_sel=False)
        t2 = time.perf_counter()
        tr += t1 - t0
        tl += t2 - t1
        n += 1
        if t2 - t_start >= seconds:
            break
    ms = (tr / n * Hr + tl / n * len(loc)) * C * s.batch * 1e3
    return ms, oracle.max_threads(), (f"{n} chunk rows spread over the chunk, one retrieval and one local head each; "
                                      f"chunk time = mean row time per class x {C} rows x heads per class x {s.batch}")


def run_reference(args):
    """The oracle arm.  Each step runs the oracle on one retrieval head and one local head of one
    sequence (cycling over all of them); the token time is estimated as
    mean(retrieval head) x Hr + mean(local head) x Hl, which is unbiased for any step count."""
    world, rank, _ = _dist()
    if rank != 0:
        return 0
    import oracle

    x = _generate(args)
    s = x.spec
    if args.workload in PREFILL_WORKLOADS:
        return _run_reference_prefill(args, x)
    ret = [(b, h) for b in range(s.batch) for h in s.retrieval_heads]
    loc = [(b, h) for b in range(s.batch) for h in range(s.n_q_heads) if h not in s.retrieval_heads]
    budget = 200.0

    def one(i):
        t = []
        for units in (ret, loc):
            if not units:
                t.append(0.0)
                continue
            b, h = units[i % len(units)]
            t0 = time.perf_counter()
            oracle.layer_rows(x, b, h, [0], want_sel=False)
            t.append(time.perf_counter() - t0)
        return t

    for i in range(args.warmup):
        one(i)
    tr = tl = 0.0
    n = 0
    t_start = time.perf_counter()
    for i in range(args.steps):
        a, b = one(args.warmup + i)
        tr += a
        tl += b
        n += 1
        if time.perf_counter() - t_start > budget:
            break
    dt = time.perf_counter() - t_start
    nr, nl = len(s.retrieval_heads), s.n_q_heads - len(s.retrieval_heads)
    us_token = (tr / n * nr + tl / n * nl) * 1e6
    line = {
        "impl": "reference", "metric": METRIC, "value": us_token, "unit": "us/token", "n_gpus": args.gpus,
        "steps": n, "warmup": args.warmup, "ms_per_step": dt / n * 1e3, "higher_is_better": False,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": _config(s, args.gpus),
        "cpu_baseline": {"value": us_token, "unit": "us/token", "cores": oracle.max_threads(), "kind": "oracle",
                         "sample": f"{n} steps of one retrieval head + one local head of one sequence, cycling over "
                                   f"all heads and sequences; token time = mean per class x heads per class"
                                   + (" (stopped at the time budget)" if n < args.steps else "")},
        "e2e": {"value": us_token, "unit": "us/token", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def _run_reference_prefill(args, x):
    """Oracle arm for a prefill workload: each step runs one retrieval-head row and one
    local-head row (rows and heads cycling over the chunk); chunk time = mean row time per
    class x rows x heads per class x sequences."""
    import numpy as np

    import oracle

    s = x.spec
    C = s.chunk
    Hr = len(s.retrieval_heads)
    loc = [h for h in range(s.n_q_heads) if h not in s.retrieval_heads]
    rows = np.linspace(0, C - 1, 97).astype(np.int64)
    budget = 200.0

    def one(i):
        row, b = int(rows[i % len(rows)]), i % s.batch
        t0 = time.perf_counter()
        oracle.layer_rows(x, b, s.retrieval_heads[i % Hr], [row], want_sel=False)
        t1 = time.perf_counter()
        if loc:
            oracle.layer_rows(x, b, loc[i % len(loc)], [row], want_sel=False)
        return t1 - t0, time.perf_counter() - t1

    for i in range(args.warmup):
        one(i)
    tr = tl = 0.0
    n = 0
    t_start = time.perf_counter()
    for i in range(args.steps):
        a, b = one(args.warmup + i)
        tr += a
        tl += b
        n += 1
        if time.perf_counter() - t_start > budget:
            break
    dt = time.perf_counter() - t_start
    ms = (tr / n * Hr + tl / n * len(loc)) * C * s.batch * 1e3
    line = {
        "impl": "reference", "metric": METRIC, "value": ms, "unit": "ms/chunk", "n_gpus": args.gpus,
        "steps": n, "warmup": args.warmup, "ms_per_step": dt / n * 1e3, "higher_is_better": False,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": _prefill_config(s, args.gpus),
        "cpu_baseline": {"value": ms, "unit": "ms/chunk", "cores": oracle.max_threads(), "kind": "oracle",
                         "sample": f"{n} steps of one retrieval-head row + one local-head row, cycling over rows "
                                   f"spread across the chunk; chunk time = mean row time per class x rows x heads"
                                   + (" (stopped at the time budget)" if n < args.steps else "")},
        "e2e": {"value": ms, "unit": "ms/chunk", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def _prefill_config(s, n_gpus):
    Hr = len(s.retrieval_heads)
    return {"workload": (f"{s.name}: chunked prefill, B={s.batch}, prefix={s.prefix}, chunk={s.chunk}, "
                         f"{s.n_q_heads} q / {s.n_kv_heads} kv heads, D={s.head_dim}, {Hr} retrieval heads "
                         f"r={s.index_dim} p={s.top_p}, local W={s.window} S={s.n_sink}"),
            "global_batch": s.batch * n_gpus, "seq_len": s.n_total, "parallelism": f"replicas x{n_gpus}",
            "l2": "inputs larger than L2 (q %.0f MB, q_rot %.0f MB and out %.0f MB per step)" % (
                s.batch * s.chunk * s.n_q_heads * s.head_dim * 2 / 1e6,
                s.batch * s.chunk * s.n_q_heads * s.head_dim * 4 / 1e6,
                s.batch * s.chunk * s.n_q_heads * s.head_dim * 4 / 1e6)}


def _generate(args):
    import synth

    return synth.generate(_spec(args))


def _spec(args, name=None):
    import synth

    name = name or args.workload
    ov = {}
    if args.batch and name == args.workload:
        base = synth.spec(name)
        ov["batch"] = args.batch
        if base.needles and len(base.needles) > 1:
            ov["needles"] = tuple(base.needles[i % len(base.needles)] for i in range(args.batch))
    return synth.spec(name, **ov)


def _config(s, n_gpus):
    return {"workload": (f"{s.name}: decode, B={s.batch}, N={s.n_total}, {s.n_q_heads} q / {s.n_kv_heads} kv heads, "
                         f"D={s.head_dim}, {len(s.retrieval_heads)} retrieval heads r={s.index_dim} p={s.top_p}, "
                         f"local W={s.window} S={s.n_sink}"),
            "global_batch": s.batch * n_gpus, "seq_len": s.n_total, "parallelism": f"replicas x{n_gpus}",
            "l2": "inputs larger than L2 (KV cache %.2f GiB + index keys %.0f MB per GPU)" % (
                2 * s.batch * s.n_kv_heads * s.n_total * s.head_dim * 2 / 2**30,
                s.batch * len(s.retrieval_heads) * s.n_total * s.index_dim * 4 / 1e6)}


def _bf16(a):
    import numpy as np
    import torch

    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16)


def measure_exp_rate(dev) -> dict:
    """The exponential (MUFU ex2) issue rate of this GPU, from the library's ex2 probe timed
    with CUDA events while nvidia-smi samples the SM clock: the peak the prefill selection's
    roofline divides by."""
    import torch

    from long_context_sparse_idx16_b200 import rtp_probe_ex2

    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    blocks, iters = sms * 8, 4096
    buf = torch.empty(blocks * 256, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream().cuda_stream
    for _ in range(3):
        rtp_probe_ex2(blocks, iters, buf.data_ptr(), stream)
    torch.cuda.synchronize()
    clocks = ClockSampler(dev.index or 0)
    clocks.start()
    best = None
    n = 0
    t_end = time.perf_counter() + 0.3
    while time.perf_counter() < t_end:
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        n = rtp_probe_ex2(blocks, iters, buf.data_ptr(), stream)
        e1.record()
        torch.cuda.synchronize()
        ms = e0.elapsed_time(e1)
        best = ms if best is None else min(best, ms)
    clk = clocks.stop()
    mhz = (clk or {}).get("sm_mhz") or 1965.0
    rate = n / (best * 1e-3)
    return {"gexp_s": rate / 1e9, "per_clk_per_sm": rate / (sms * mhz * 1e6), "sms": sms, "sm_mhz": mhz,
            "clock_source": "sampled" if clk and clk.get("sm_mhz") else "nominal max",
            "exps_per_launch": int(n), "ms_per_launch": best}


def _timed(step, steps: int, world: int, dev):
    """Device time (ms, max over ranks) of exactly `steps` calls of step(), bracketed by a
    barrier and a device synchronisation on both sides."""
    import torch

    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(steps):
        step()
    e1.record()
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    return _max_over_ranks(e0.elapsed_time(e1), world, dev)


def measure_decode(s, x, steps: int, warmup: int, world: int, dev, *, top_ps=None, cpu: bool = True,
                   cluster_k: int = 0, cluster_iters: int = 4):
    """Decode lines of workload s, one per p in top_ps (default: the workload's p), all on one
    layer.  A step appends the B new tokens and decodes their B queries; before every step the
    length is rolled back by one, so every step sees exactly N keys.  cluster_k > 0: the first
    N - 1 keys of every sequence are clustered into cluster_k clusters (timed once) and the
    steps select by clusters; the key each step appends is kept as one cached after the
    clustering."""
    import numpy as np
    import torch

    from long_context_sparse_idx16_b200 import Layer

    N, B = s.n_total, s.batch
    layer = Layer.from_spec(s, x, max_seq=N, max_chunk=1, n_clusters=cluster_k)
    for t0 in range(0, N - 1, 1 << 16):
        t1 = min(N - 1, t0 + (1 << 16))
        layer.append_kv(_bf16(x.k[:, t0:t1]).to(dev), _bf16(x.v[:, t0:t1]).to(dev))
    build = None
    if cluster_k:
        layer.cluster_build(cluster_iters)  # warm-up build
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        layer.cluster_build(cluster_iters)
        e1.record()
        torch.cuda.synchronize()
        assert layer.check() == 0
        layer.profile(True)
        layer.profile_read()
        layer.cluster_build(cluster_iters)
        torch.cuda.synchronize()
        bk = {}
        for k in ("cluster_init", "cluster_assign", "cluster_accum", "cluster_update"):
            kms, kn = layer.profile_read(k)
            bk[k] = {"us_per_launch": kms * 1e3 / max(kn, 1), "launches": kn}
        layer.profile(False)
        P_ = B * len(s.retrieval_heads)
        # fp64 work of one assignment pass: 16 subtractions + 16 fused multiply-adds per (key, centre)
        flops = P_ * (N - 1) * cluster_k * 16 * 3
        a_us = bk["cluster_assign"]["us_per_launch"]
        build = {"ms": e0.elapsed_time(e1), "n_clusters": cluster_k, "iters": cluster_iters,
                 "keys_per_problem": N - 1, "problems": P_, "kernels": bk,
                 "assign_fp64_tflops": flops / (a_us * 1e-6) / 1e12}
    k_tok = _bf16(x.k[:, N - 1:N]).to(dev).contiguous()
    v_tok = _bf16(x.v[:, N - 1:N]).to(dev).contiguous()
    q = _bf16(x.q[:, 0]).to(dev).contiguous()
    out = torch.empty((B, s.n_q_heads, 128), dtype=torch.float32, device=dev)
    # the step's inputs packed in one pinned host buffer (q | k | v), copied with one transfer
    # into one device buffer whose slices are the call's arguments (each a multiple of 128
    # elements, so every slice stays 16-byte aligned)
    nq, nk = q.numel(), k_tok.numel()
    in_h = torch.cat([q.reshape(-1), k_tok.reshape(-1), v_tok.reshape(-1)]).cpu().pin_memory()
    in_d = torch.empty_like(in_h, device=dev)
    q_d = in_d[:nq].view(q.shape)
    k_d = in_d[nq:nq + nk].view(k_tok.shape)
    v_d = in_d[nq + nk:].view(v_tok.shape)
    o_h = torch.empty(out.shape, dtype=out.dtype, pin_memory=True)

    def step():
        layer.truncate(N - 1)
        layer.append_kv(k_tok, v_tok)
        layer.decode(q, out)

    def e2e_step():  # the step's inputs from pinned host memory, the output back to the host
        in_d.copy_(in_h, non_blocking=True)
        layer.truncate(N - 1)
        layer.append_kv(k_d, v_d)
        layer.decode(q_d, out)
        o_h.copy_(out, non_blocking=True)

    peak, peak_kind = _peaks()
    P = B * len(s.retrieval_heads)
    key_bytes = 2 if getattr(s, "index_bf16", False) else 4
    sel_bytes = P * N * s.index_dim * key_bytes  # index keys streamed per launch (fp32 or bf16)
    traffic = _profile_traffic(os.path.join(ROOT, "long_context_sparse_idx16_b200", "csrc", "decode_select.cu"))
    lines = []
    for p in (top_ps or [s.top_p]):
        layer.set_top_p(p)
        for _ in range(warmup):
            step()
        torch.cuda.synchronize()
        assert layer.check() == 0
        _, st = layer.decode(q, out, stats=True)
        counts = st[0].cpu().numpy().ravel()
        clocks = ClockSampler(dev.index or 0)
        clocks.start()  # sampled during the timed region
        ms = _timed(step, steps, world, dev)
        clk = clocks.stop()
        assert layer.check() == 0
        # the same steps with a CUDA event pair around every kernel launch (on its launch
        # stream): per-kernel device time for the roofline and the launch count
        layer.profile(True)
        layer.profile_read()  # drop anything recorded before
        for _ in range(steps):
            step()
        torch.cuda.synchronize()
        sel_ms, sel_n = layer.profile_read("decode_select")
        kern = {"decode_select": {"us_per_launch": sel_ms * 1e3 / max(sel_n, 1), "launches": sel_n}}
        other_n = 0
        for k in ("append_kv", "q_prep", "decode_topk", "decode_gather", "decode_swa", "swa_merge", "dense_fill",
                  "cluster_select", "cluster_compact"):
            kms, kn = layer.profile_read(k)
            if kn:
                kern[k] = {"us_per_launch": kms * 1e3 / kn, "launches": kn}
            other_n += kn
        _, rest_n = layer.profile_read(None)
        layer.profile(False)
        for _ in range(warmup):
            e2e_step()
        torch.cuda.synchronize()
        e2e_ms = _timed(e2e_step, steps, world, dev)
        assert np.isfinite(o_h.numpy()).all()
        tokens = B * steps * world
        sel_us = sel_ms * 1e3 / max(sel_n, 1)
        achieved = sel_bytes / (sel_us * 1e-6) / 1e9 if sel_us > 0 else 0.0
        win_keys = min(N, s.window + s.n_sink)
        # whole-step algorithmic bytes: index keys + window/sink K/V rows + selected K/V rows
        step_bytes = sel_bytes + B * s.n_kv_heads * win_keys * 512 + int(counts.sum()) * 512
        roof = {"bound": "hbm", "kernel": "decode_select (fused index stream + exact top-p)",
                "achieved": achieved, "peak": peak, "peak_kind": peak_kind, "unit": "GB/s",
                "frac": achieved / peak,
                # the capture streams fp32 keys; its bytes scale with the keys streamed
                "traffic": (traffic * P * N / _TRAFFIC_KEYS if traffic and key_bytes == 4 else None),
                "bytes_per_launch": sel_bytes, "us_per_launch": sel_us}
        if cluster_k:
            # the clusters' keys replace the index stream: centres, one 2-byte assignment per
            # clustered key, then the selected K/V rows through the flat gather (the dominant kernel)
            g_us = kern["decode_gather"]["us_per_launch"]
            g_bytes = int(counts.sum()) * 512
            g_ach = g_bytes / (g_us * 1e-6) / 1e9
            roof = {"bound": "hbm", "kernel": "decode_gather (flat stream of the hit clusters' K/V rows)",
                    "achieved": g_ach, "peak": peak, "peak_kind": peak_kind, "unit": "GB/s", "frac": g_ach / peak,
                    "traffic": None, "bytes_per_launch": g_bytes, "us_per_launch": g_us}
            step_bytes = (P * cluster_k * s.index_dim * 8 + P * (N - 1) * 2 + B * s.n_kv_heads * win_keys * 512
                          + int(counts.sum()) * 512)
        lines.append({
            "value": ms * 1e3 / tokens, "unit": "us/token", "top_p": p, "steps": steps, "warmup": warmup,
            "ms_per_step": ms / steps, "config": _config(s, world),
            "roofline": roof,
            "step_roofline": {"bytes_per_step": step_bytes, "roofline_us_per_step": step_bytes / (peak * 1e9) * 1e6,
                              "frac": step_bytes / (peak * 1e9) / (ms / steps * 1e-3)},
            "e2e": {"value": e2e_ms * 1e3 / tokens, "unit": "us/token",
                    "h2d_bytes_per_step": int(q.numel() * 2 + k_tok.numel() * 2 * 2),
                    "d2h_bytes_per_step": int(out.numel() * 4)},
            "kernels": kern,
            "gpu_launches": int(sel_n + other_n + rest_n),
            "selected_tokens": {"min": int(counts.min()), "median": float(np.median(counts)),
                                "max": int(counts.max())},
            "clocks": clk,
        })
        if build:
            lines[-1]["cluster_build"] = build
    layer.close()
    if cpu and not cluster_k:
        v, cores, desc = cpu_oracle_sample(x)
        for ln in lines:
            ln["cpu_baseline"] = {"value": v, "unit": "us/token", "cores": cores, "kind": "oracle",
                                  "sample": desc + f" at p={s.top_p}"}
    return lines


def _local_pairs(s) -> int:
    """Sum over chunk rows of the local-head key count |J_i| (sinks + window, causal)."""
    import numpy as np

    pos = s.prefix + np.arange(s.chunk, dtype=np.int64)
    sinks = np.minimum(s.n_sink, pos + 1)
    w0 = np.maximum(s.n_sink, pos - s.window + 1)
    return int((sinks + np.maximum(0, pos - w0 + 1)).sum())


def measure_prefill(s, x, steps: int, warmup: int, world: int, dev, exp_peak: dict, *, cpu: bool = True):
    """A step is one chunked-prefill call of the workload: the chunk's K/V are appended (RoPE +
    index keys) after the length is rolled back to the prefix, then every row of the chunk runs
    its selection / window and attention."""
    import numpy as np
    import torch

    from long_context_sparse_idx16_b200 import Layer

    N, B, P, C = s.n_total, s.batch, s.prefix, s.chunk
    layer = Layer.from_spec(s, x, max_seq=N, max_chunk=C)
    for t0 in range(0, P, 1 << 16):
        t1 = min(P, t0 + (1 << 16))
        layer.append_kv(_bf16(x.k[:, t0:t1]).to(dev), _bf16(x.v[:, t0:t1]).to(dev))
    k_c = _bf16(x.k[:, P:N]).to(dev).contiguous()
    v_c = _bf16(x.v[:, P:N]).to(dev).contiguous()
    q = _bf16(x.q).to(dev).contiguous()
    out = torch.empty((B, C, s.n_q_heads, 128), dtype=torch.float32, device=dev)

    def step():
        layer.truncate(P)
        layer.append_kv(k_c, v_c)
        layer.prefill_chunk(q, out)

    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    assert layer.check() == 0
    _, st = layer.prefill_chunk(q, out, stats=True)
    counts = st[0].cpu().numpy()
    assert layer.check() == 0

    clocks = ClockSampler(dev.index or 0)
    clocks.start()  # sampled during the timed region
    ms = _timed(step, steps, world, dev)
    clk = clocks.stop()
    assert layer.check() == 0
    layer.profile(True)
    layer.profile_read()
    for _ in range(steps):
        step()
    torch.cuda.synchronize()
    per = {}
    for k in ("prefill_select", "prefill_attn", "prefill_local", "append_kv", "q_prep"):
        per[k] = layer.profile_read(k)
    _, rest_n = layer.profile_read(None)
    layer.profile(False)
    all_n = sum(n for _, n in per.values()) + rest_n

    # end to end: q and the chunk's K/V from pinned host memory, the output back to the host
    q_h = q.cpu().pin_memory()
    k_h = k_c.cpu().pin_memory()
    v_h = v_c.cpu().pin_memory()
    o_h = torch.empty(out.shape, dtype=out.dtype, pin_memory=True)
    q_d, k_d, v_d = torch.empty_like(q), torch.empty_like(k_c), torch.empty_like(v_c)

    def e2e_step():
        q_d.copy_(q_h, non_blocking=True)
        k_d.copy_(k_h, non_blocking=True)
        v_d.copy_(v_h, non_blocking=True)
        layer.truncate(P)
        layer.append_kv(k_d, v_d)
        layer.prefill_chunk(q_d, out)
        o_h.copy_(out, non_blocking=True)

    for _ in range(warmup):
        e2e_step()
    torch.cuda.synchronize()
    e2e_ms = _timed(e2e_step, steps, world, dev)
    layer.close()

    peak, peak_kind = _tensor_peak()
    Hr = len(s.retrieval_heads)
    Hl = s.n_q_heads - Hr
    pairs = Hr * B * (C * P + C * (C + 1) // 2)  # causal (row, key) index scores, all retrieval heads
    flops = {"local_attention": 4 * s.head_dim * _local_pairs(s) * Hl * B,
             "retrieval_attention": 4 * s.head_dim * int(counts.sum()),
             "index_scores": pairs, "index_scores_flops": 2 * s.index_dim * pairs}
    kern = {k: {"ms_per_launch": kms / max(kn, 1), "launches": kn} for k, (kms, kn) in per.items()}
    roofs = _prefill_rooflines(kern, flops, pairs, exp_peak, (clk or {}).get("sm_mhz"), peak, peak_kind)
    if "prefill_select" in roofs:
        roofs["prefill_select"]["traffic"] = _prefill_traffic("prefill_select", s.name)
    if "prefill_attn" in roofs:
        roofs["prefill_attn"]["traffic"] = _prefill_traffic("prefill_attn", s.name)
    # the chunk's dominant kernel is the headline roofline
    dom = max((k for k in ("prefill_select", "prefill_attn", "prefill_local") if k in roofs),
              key=lambda k: roofs[k]["ms_per_launch"])
    line = {
        "value": ms / steps, "unit": "ms/chunk", "steps": steps, "warmup": warmup, "ms_per_step": ms / steps,
        "config": _prefill_config(s, world),
        "roofline": roofs[dom],
        "rooflines": roofs,
        "kernels": kern,
        "flops": flops,
        "e2e": {"value": e2e_ms / steps, "unit": "ms/chunk",
                "h2d_bytes_per_step": int((q.numel() + k_c.numel() + v_c.numel()) * 2),
                "d2h_bytes_per_step": int(out.numel() * 4)},
        "gpu_launches": int(all_n),
        "selected_tokens": {"min": int(counts.min()), "median": float(np.median(counts)), "max": int(counts.max()),
                            "mean": float(counts.mean())},
        "clocks": clk,
    }
    if cpu:
        v, cores, desc = cpu_oracle_prefill_sample(x)
        line["cpu_baseline"] = {"value": v, "unit": "ms/chunk", "cores": cores, "kind": "oracle", "sample": desc}
    return line


# the workloads measured besides the headline one: (record name, workload, layer options,
# the steps each takes at most -- a 1M prefill chunk takes about a second -- and the p values)
# Layer-only options: cluster_k (K-cache clustering with that many clusters; K = 128 is the
# page's example, 256 at 1M keeps about 4K keys per cluster).
SUB_WORKLOADS = (("decode_1m", "decode_1m", {}, None, None),
                 ("decode_1m_bf16_index", "decode_1m", {"index_bf16": True}, None, (0.9,)),
                 ("decode_1m_clustered", "decode_1m", {"index_bf16": True, "cluster_k": 256}, None, (0.9,)),
                 ("decode_128k_clustered", "decode_128k", {"index_bf16": True, "cluster_k": 128}, None, None),
                 ("prefill_32k", "prefill_32k", {}, 5, None),
                 ("prefill_1m", "prefill_1m", {}, 3, None))


def run_gpu(args):
    import torch

    import synth

    world, rank, local = _dist()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime

        import torch.distributed as dist

        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300), device_id=dev)
    cpu = rank == 0 and not args.no_cpu_baseline
    exp_peak = measure_exp_rate(dev)
    decode_wl = args.workload in DECODE_WORKLOADS

    generated = {}

    def one(name, steps, opts=None, ps=None):
        opts = dict(opts or {})
        layer_opts = {k: opts.pop(k) for k in list(opts) if k.startswith("cluster_")}
        s = _spec(args, name)
        if opts:
            s = dataclasses.replace(s, **opts)
        key = (name, tuple(sorted(opts.items())))
        if key not in generated:  # inputs shared by the records of one spec
            generated.clear()
            generated[key] = synth.generate(s)
        x = generated[key]
        if name in PREFILL_WORKLOADS:
            return [measure_prefill(s, x, steps, args.warmup, world, dev, exp_peak, cpu=cpu)]
        ps = ps or (list(s.p_sweep) if s.p_sweep else None)
        return measure_decode(s, x, steps, args.warmup, world, dev, top_ps=list(ps) if ps else None, cpu=cpu,
                              **layer_opts)

    head = one(args.workload, args.steps,
               {"index_bf16": True, "cluster_k": args.cluster_k} if args.cluster_k and decode_wl else None)
    main = head[len(head) // 2] if args.workload == "decode_1m" else head[0]  # p = 0.9 of a sweep
    decode = args.workload in DECODE_WORKLOADS
    line = {"metric": METRIC, "value": main["value"], "unit": main["unit"], "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": main["ms_per_step"], "higher_is_better": False,
            "scaling": "weak", "vs_baseline": None, "dtype": "f32" if decode else "f16 mma / f32",
            "data": "synthetic"}
    line.update({k: v for k, v in main.items() if k not in ("value", "unit", "steps", "warmup", "ms_per_step")})
    if args.workload == "decode_1m":
        line["p_sweep"] = {f"p={ln['top_p']}": ln for ln in head}
    if args.cluster_k and decode_wl:
        line["layer_options"] = {"index_bf16": True, "n_clusters": args.cluster_k}
    line["exp_peak"] = exp_peak
    if not args.only:
        subs = {}
        total = line["gpu_launches"]
        for rec, name, opts, cap, ps in SUB_WORKLOADS:
            if name == args.workload and not opts:
                continue
            steps = args.steps if cap is None else max(1, min(args.steps, cap))
            for ln in one(name, steps, opts, ps):
                key = rec if name not in DECODE_WORKLOADS else f"{rec}_p{ln['top_p']}"
                if opts:
                    ln["layer_options"] = opts
                subs[key] = ln
                total += ln["gpu_launches"]
        line["workloads"] = subs
        line["gpu_launches_all_workloads"] = int(total)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        torch.distributed.destroy_process_group()
    return 0


def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=DECODE_WORKLOADS + PREFILL_WORKLOADS, default="decode_128k",
                    help="headline workload (the default is the one the value is quoted on)")
    ap.add_argument("--only", action="store_true",
                    help="measure the headline workload alone (no sub-records for the other workloads)")
    ap.add_argument("--batch", type=int, default=0, help="override the sequence count (profiling cases)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cluster-k", type=int, default=0,
                    help="decode workloads: K-cache clustering with K clusters (bf16 index keys) for the headline "
                         "workload (profiling cases)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.impl == "reference":
        return run_reference(args)
    return run_gpu(args)


if __name__ == "__main__":
    sys.exit(main())
