#!/usr/bin/env python
"""Benchmark of exact ring blockwise attention (forward + backward) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl native|reference]

A step is one pass of the hot path over one batch of synthetic input:
ring forward (ringattn_fwd) and ring backward (ringattn_bwd's three phases)
of the attention workload, plus, for the layer workload, the blockwise SwiGLU
feed-forward.  Inputs are resident in HBM when the timed region starts and
are larger than the 126 MB L2.  The timed region is bracketed by a barrier and
a device synchronise on both sides and timed with CUDA events on the launch
stream; with several GPUs every rank runs its own batch (weak scaling, no
data-path collective) and the maximum time over ranks is taken.

Under ``--impl reference`` the fp64 CPU oracle is timed instead (rank 0
only), on a bounded sample of the same workload.

Prints one JSON line on rank 0.
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

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "ring-attn fwd+bwd TFLOP/s & tokens/s on 1 B200; % of BF16 tensor peak"

# DRAM traffic per launch of the dominant kernel, from one ncu capture
# (dram__bytes_read.sum + dram__bytes_write.sum), valid only for the kernel
# code it was taken on: the sha256 of the source file with its comments and
# blank lines removed (code_fingerprint), so that any change to the code
# voids the figure and a change to a comment does not.
# n32k_d128: captured on 8 heads of the workload and scaled x4 to its 32
# heads (heads are independent units); n8k_d64_causal: the whole workload.
NCU_TRAFFIC = {
    ("bwd_fused_kernel", "n32k_d128"): {
        "bytes": 4 * (418.488064e6 + 236.270592e6),
        "code_sha256": "4a7e542d5ea8f821cedeb8f71d9f4428d80b751d8e8d7b1e4fe037036d5a7de9"},
    ("bwd_fused_kernel", "n8k_d64_causal"): {
        "bytes": 206.973696e6 + 93.997568e6,
        "code_sha256": "4a7e542d5ea8f821cedeb8f71d9f4428d80b751d8e8d7b1e4fe037036d5a7de9"},
    ("fwd_tc2_kernel", "n32k_d128"): {
        "bytes": 4 * (202.440192e6 + 50.114304e6),
        "code_sha256": "c488625a208af031ae2481df9d6dd97427efc681e42ec2e1e105e4c354ca19e5"},
}


def code_fingerprint(path: str) -> str:
    """sha256 of a C/C++/CUDA source with // and /* */ comments and blank
    lines removed and trailing blanks stripped (string and character
    literals are kept as they are)."""
    src = open(path, encoding="utf-8").read()
    out, i, n = [], 0, len(src)
    while i < n:
        c = src[i]
        if c in "\"'":  # literal: copy up to the matching unescaped quote
            j = i + 1
            while j < n and src[j] != c:
                j += 2 if src[j] == "\\" else 1
            out.append(src[i:j + 1])
            i = j + 1
        elif src.startswith("//", i):
            j = src.find("\n", i)
            i = n if j < 0 else j
        elif src.startswith("/*", i):
            j = src.find("*/", i + 2)
            i = n if j < 0 else j + 2
        else:
            out.append(c)
            i += 1
    lines = [ln.rstrip() for ln in "".join(out).split("\n")]
    return hashlib.sha256("\n".join(ln for ln in lines if ln).encode()).hexdigest()


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=40)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", default="n32k_d128",
                    choices=["n32k_d128", "n8k_d64_causal", "n8k_d64_full", "layer7b", "layer7b_full",
                             "n1m_d128", "n32k_d128_gqa8", "decode_n128k", "n32k_d128_step", "merge_n32k"])
    ap.add_argument("--impl", default="native", choices=["native", "reference"])
    ap.add_argument("--ring", action="store_true",
                    help="run the multi-device ring (one sequence shard per rank, key/value blocks passed "
                         "rank to rank) on the workload's whole sequence instead of one batch per rank")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--heads", type=int, default=0, help="override the head count (smaller profiling cases)")
    ap.add_argument("--tokens", type=int, default=0,
                    help="override the sequence length of layer7b_full or the cache length of decode_n128k")
    return ap.parse_args()


# ---------------------------------------------------------------------------
# workload description and FLOP counts
# ---------------------------------------------------------------------------

def workload(name):
    from exact_blockwise_long_b200.synthetic import FFN_WORKLOADS, WORKLOADS
    if name == "layer7b":
        return WORKLOADS["layer7b_attn"], FFN_WORKLOADS["layer7b_ffn"]
    return WORKLOADS[name], None


def attn_fwd_flops(w):
    """4 B H N^2 d, halved under the causal mask (causal FLOPs counted once)."""
    f = 4.0 * w.B * w.H * w.N * w.N * w.D
    return f * 0.5 if w.causal else f


def attn_step_flops(w):
    return attn_fwd_flops(w) * (3.5 if w.bwd else 1.0)  # backward = 2.5 x forward (5 MMAs vs 2)


def ffn_flops(f):
    """Forward (three GEMMs) plus backward (dh, dx from dg and du, dw1, dw3,
    dw2: six GEMMs; the backward's recomputation of g and u is not counted)."""
    return 18.0 * f.T * f.d_model * f.d_ff


def max_over_ranks(x: float, dist=None, device=None) -> float:
    """The largest value of x over all ranks (a no-op with one process)."""
    if dist is None or not dist.is_initialized() or dist.get_world_size() == 1:
        return float(x)
    import torch
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_tflops(flops_per_rank: float, world: int, ms_step: float) -> float:
    """Weak scaling: every rank did flops_per_rank in (at most) ms_step."""
    return flops_per_rank * world / (ms_step * 1e-3) / 1e12


def describe(aw, fw):
    d = {"workload": f"{aw.name}: ring attention {'fwd+bwd' if aw.bwd else 'fwd'}, B={aw.B}, H={aw.H}, "
                     + (f"Hkv={aw.kv_heads}, " if aw.kv_heads != aw.H else "")
                     + f"N={aw.N}, d={aw.D}, S={aw.S}, q_chunk={aw.q_chunk}, k_chunk={aw.k_chunk}, "
                     f"{'causal' if aw.causal else 'non-causal'}"
                     + (f"; blockwise SwiGLU FFN {fw.d_model}->{fw.d_ff}->{fw.d_model} fwd+bwd, chunk {fw.chunk}"
                        if fw else ""),
         "B": aw.B, "H": aw.H, "seq_len": aw.N, "head_dim": aw.D, "shards": aw.S,
         "q_chunk": aw.q_chunk, "k_chunk": aw.k_chunk, "causal": aw.causal,
         "l2": "inputs larger than L2 (no flush between steps)"}
    return d


# ---------------------------------------------------------------------------
# peaks, clocks
# ---------------------------------------------------------------------------

def tensor_peak(pk, region_ms):
    """The bf16 peak a timed region is held against: the burst figure for a
    region shorter than the seconds a power-capped steady state takes to set
    in, the sustained one for a longer region.  Returns (peak, description,
    the other figure)."""
    if region_ms >= 3000.0:
        return pk["bf16_sustained"], f"bf16 dense, sustained ({pk['source']}; timed region >= 3 s)", pk["bf16_burst"]
    return pk["bf16_burst"], f"bf16 dense, burst ({pk['source']}; timed region < 3 s)", pk["bf16_sustained"]


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            j = json.load(f)
        return {"bf16_burst": float(j["bf16_tflops"]), "bf16_sustained": float(j["bf16_tflops_sustained"]),
                "hbm_gbs": float(j["hbm_gbs"]), "source": "measured"}
    except Exception:
        return {"bf16_burst": 1590.0, "bf16_sustained": 1400.0, "hbm_gbs": 6650.0, "source": "fallback"}


class ClockSampler:
    """SM clock, power and clock-event reasons of one GPU while the timed
    region runs: NVML polled every 10 ms from a thread (nvidia-smi's 100 ms
    loop is the fallback), so even a short timed region gets samples."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    # NVML clock-event reason bits
    REASON_BITS = {"sw_power_cap": 0x4, "hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20,
                   "hw_thermal_slowdown": 0x40}

    def __init__(self, index):
        self.index = index
        self.proc = None
        self.thread = None
        self.samples = []  # (sm_mhz, power_w, reason_bits)
        self.max_mhz = None
        self.path = os.path.join("/tmp", f"ra_clocks_{os.getpid()}.csv")

    def start(self):
        try:
            import threading
            import pynvml
            pynvml.nvmlInit()
            h = None
            try:  # the CUDA device by PCI address (CUDA and NVML numbering can differ)
                pr = torch.cuda.get_device_properties(self.index)
                bus = f"{pr.pci_domain_id:08x}:{pr.pci_bus_id:02x}:{pr.pci_device_id:02x}.0"
                h = pynvml.nvmlDeviceGetHandleByPciBusId(bus.encode())
            except Exception:
                h = None
            if h is None:
                h = pynvml.nvmlDeviceGetHandleByIndex(self.index)
            self.max_mhz = float(pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM))
            reasons_fn = getattr(pynvml, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
                pynvml.nvmlDeviceGetCurrentClocksThrottleReasons
            self.stop_evt = threading.Event()

            def poll():
                while not self.stop_evt.is_set():
                    try:
                        self.samples.append((float(pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM)),
                                             pynvml.nvmlDeviceGetPowerUsage(h) / 1000.0, int(reasons_fn(h))))
                    except Exception:
                        pass
                    self.stop_evt.wait(0.01)

            self.thread = threading.Thread(target=poll, daemon=True)
            self.thread.start()
            return
        except Exception:
            self.thread = None
        try:
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=self.f, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def _summary(self, sm, power, reasons, mx, source):
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": mx, "reasons": sorted(reasons), "samples": 0, "source": source}
        loaded = [s for s, p in zip(sm, power) if p > 300] or sm
        return {"sm_mhz": statistics.median(loaded), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm), "samples_under_load": len(loaded), "source": source}

    def stop(self):
        if self.thread is not None:
            self.stop_evt.set()
            self.thread.join(timeout=5)
            reasons = {nm for nm, bit in self.REASON_BITS.items() if any(r & bit for _, _, r in self.samples)}
            return self._summary([x[0] for x in self.samples], [x[1] for x in self.samples], reasons,
                                 self.max_mhz, "nvml, 10 ms")
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.f.close()
        sm, mx, reasons, power = [], None, set(), []
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx = float(parts[2])
                power.append(float(parts[3]))
            except ValueError:
                continue
            for nm, val in zip(names, parts[5:9]):
                if val.lower().startswith("active"):
                    reasons.add(nm)
        os.unlink(self.path)
        return self._summary(sm, power, reasons, mx, "nvidia-smi, 100 ms")


REJECT_REASONS = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown")


def clocks_rejected(clk, dist=None, dev=None):
    """True (on every rank alike) if any rank's timed region saw a hardware or
    thermal slowdown, or SM clocks below 75% of their maximum with no reason
    active (a leftover clock lock)."""
    bad = any(r in REJECT_REASONS for r in clk.get("reasons", []))
    mhz, mx = clk.get("sm_mhz"), clk.get("sm_max_mhz")
    if mhz is not None and mx and mhz < 0.75 * mx and not clk.get("reasons"):
        bad = True
    if dist is not None:
        import torch
        t = torch.tensor([1.0 if bad else 0.0], device=dev)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        bad = bool(t.item() > 0)
    return bad


# ---------------------------------------------------------------------------
# the oracle on a bounded sample (cpu_baseline and the reference arm)
# ---------------------------------------------------------------------------

def oracle_sample(aw, fw, n_tokens=4096, min_seconds=0.0, max_heads=32):
    """Time the fp64 oracle on heads of the workload cut to their first
    n_tokens tokens (a causal prefix is a complete sub-problem), adding heads
    until min_seconds of CPU time have been spent.

    Returns (seconds, counted FLOPs, description, threads)."""
    import oracle
    from dataclasses import replace
    from exact_blockwise_long_b200.synthetic import attention_inputs, to_f64
    n = min(aw.N, n_tokens)
    small = replace(aw, B=1, H=1, N=n)
    dt, heads = 0.0, 0
    while heads < max_heads and (heads == 0 or dt < min_seconds):
        q, k, v, do = attention_inputs(replace(small, seed=aw.seed + 7919 * heads), device="cpu",
                                       with_dout=aw.bwd)
        q, k, v = to_f64(q), to_f64(k), to_f64(v)
        t0 = time.perf_counter()
        oracle.attention_forward(q, k, v, aw.causal)
        if aw.bwd:
            oracle.attention_backward(q, k, v, to_f64(do), aw.causal)
        dt += time.perf_counter() - t0
        heads += 1
    flops = attn_step_flops(small) * heads
    desc = (f"fp64 oracle (numpy) {'forward+backward' if aw.bwd else 'forward'} of {heads} head(s) cut to "
            f"their first {n} tokens, same workload recipe; causal FLOPs counted once")
    if fw is not None:
        from exact_blockwise_long_b200.synthetic import ffn_inputs
        tf = 256
        x, w1, w2, w3, dy = (to_f64(t) for t in ffn_inputs(replace(fw, chunk=tf), device="cpu", T=tf,
                                                          with_dy=True))
        t0 = time.perf_counter()
        oracle.blockwise_ffn(x, w1, w2, w3, tf)
        oracle.blockwise_ffn_backward(x, w1, w2, w3, dy, tf)
        dt += time.perf_counter() - t0
        flops += ffn_flops(replace(fw, T=tf))
        desc += f"; plus the SwiGLU FFN forward+backward of {tf} tokens at the layer's full width"
    try:
        from threadpoolctl import threadpool_info
        threads = max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    except Exception:
        threads = os.cpu_count()
    return dt, flops, desc, threads


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    from dataclasses import replace
    if args.workload.startswith("decode"):
        from exact_blockwise_long_b200.synthetic import DECODE_WORKLOADS
        dw = DECODE_WORKLOADS[args.workload]
        sampler = lambda: decode_oracle_sample(dw)  # noqa: E731
        config = {"workload": f"{dw.name}: decode, one new token per head against a cache of N={dw.N}, B={dw.B}, "
                              f"H={dw.H}, Hkv={dw.Hkv}, d={dw.D}"}
    elif args.workload == "layer7b_full":
        from exact_blockwise_long_b200.synthetic import LAYER_WORKLOADS
        lw = LAYER_WORKLOADS[args.workload]
        aw = fw = None
        sampler = lambda: layer_oracle_sample(lw)  # noqa: E731
        config = {"workload": f"{lw.name}: one blockwise transformer layer fwd+bwd, N={lw.N}, H={lw.H}, "
                              f"d={lw.D}, d_ff={lw.d_ff}, S={lw.S}"}
    elif args.workload == "merge_n32k":
        sampler = merge_oracle_sample
        config = {"workload": "merge_n32k: exact merge of two fp32 partials per row, d=128"}
    else:
        name = "n32k_d128" if args.workload == "n32k_d128_step" else args.workload
        aw, fw = workload(name)
        if args.workload == "n32k_d128_step":
            aw = replace(aw, bwd=False)  # the step-mode workload is the forward
        if args.heads:
            aw = replace(aw, H=args.heads)
        sampler = lambda: oracle_sample(aw, fw)  # noqa: E731
        config = describe(aw, fw)
    times, flops, desc, threads = [], 0.0, "", 1
    for i in range(args.warmup + args.steps):
        dt, flops, desc, threads = sampler()
        if i >= args.warmup:
            times.append(dt)
    t = sum(times) / len(times)
    value = flops / t / 1e12
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": t * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": config,
            "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
                             "sample": desc + f"; {args.steps} timed samples"},
            "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------------------
# the native arm
# ---------------------------------------------------------------------------

def run_step_mode(args, ra, dev, rank, world, dist):
    """Auxiliary workloads of the 32k shapes.

    n32k_d128_step: the causal forward as S ring steps (ringattn_fwd_step,
    each merging its partial exactly into fp32 accumulators in HBM), the
    per-step building block of a multi-device ring; compare its TFLOP/s with
    the fused whole-ring forward.  merge_n32k: the standalone exact merge
    (ringattn_merge) of two fp32 partials of every row, HBM-bound."""
    import torch
    from dataclasses import replace
    from exact_blockwise_long_b200.synthetic import WORKLOADS, attention_inputs
    w = replace(WORKLOADS["n32k_d128"], bwd=False)
    q, k, v, _ = attention_inputs(replace(w, seed=w.seed + 1000 * rank), device=dev)
    B, H, N, D = q.shape
    stream = torch.cuda.current_stream()
    o_acc = torch.empty((B, H, N, D), device=dev, dtype=torch.float32)
    lse_acc = torch.empty((B, H, N), device=dev, dtype=torch.float32)
    if args.workload == "n32k_d128_step":
        def step():
            o_acc.zero_()
            lse_acc.fill_(float("-inf"))
            for t in range(w.S):
                ra.ringattn_fwd_step(q, k, v, o_acc, lse_acc, w.S, w.q_chunk, w.k_chunk, w.causal, t)
        launches = w.S
    else:
        o_b = torch.randn((B, H, N, D), device=dev)
        l_b = torch.randn((B, H, N), device=dev)
        o_acc.normal_()
        lse_acc.normal_()

        def step():
            ra.ringattn_merge(o_acc, lse_acc, o_b, l_b)
        launches = 1
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    clocks = ClockSampler(dev.index)
    clocks.start()
    time.sleep(0.3)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(args.steps):
        step()
    b.record(stream)
    torch.cuda.synchronize()
    clk = clocks.stop()
    if ra.ringattn_get_error() != 0:
        raise RuntimeError("device status word set during the timed region")
    ms = max_over_ranks(a.elapsed_time(b) / args.steps, dist if world > 1 else None, dev)
    pk = peaks()
    if args.workload == "n32k_d128_step":
        fl = attn_fwd_flops(w)
        tf = whole_job_tflops(fl, world, ms)
        return {"metric": METRIC, "value": tf, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
                "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
                "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
                "config": {"workload": f"n32k_d128_step: causal forward as {w.S} ring steps merged into fp32 "
                                       f"HBM accumulators, B={B}, H={H}, N={N}, d={D}"},
                "roofline": {"bound": "tensor", "kernel": "fwd_tc2_kernel (step mode)", "achieved": tf,
                             "peak": tensor_peak(pk, ms * args.steps)[0], "unit": "TFLOP/s",
                             "frac": tf / tensor_peak(pk, ms * args.steps)[0], "traffic": None,
                             "peak_kind": tensor_peak(pk, ms * args.steps)[1]},
                "gpu_launches": launches * args.steps, "clocks": clk}
    rows = B * H * N
    nbytes = rows * (3 * D * 4 + 3 * 4)  # read o_a, o_b, lse_a, lse_b; write o_a, lse_a
    gbs = nbytes / (ms * 1e-3) / 1e9
    return {"metric": "ringattn_merge HBM throughput (auxiliary)", "value": gbs * world, "unit": "GB/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "config": {"workload": f"merge_n32k: exact merge of two fp32 partials of {rows} rows, d={D}"},
            "roofline": {"bound": "hbm", "kernel": "merge_kernel", "achieved": gbs, "peak": pk["hbm_gbs"],
                         "unit": "GB/s", "frac": gbs / pk["hbm_gbs"], "traffic": None,
                         "peak_kind": f"HBM copy ({pk['source']})"},
            "gpu_launches": launches * args.steps, "clocks": clk}


def run_decode(args, ra, dev, rank, world, dist):
    """One decode step (new token per head against the sharded cache) per
    bench step; HBM-bound, so the roofline is bandwidth."""
    import torch
    from dataclasses import replace
    from exact_blockwise_long_b200.synthetic import DECODE_WORKLOADS, decode_inputs
    w = DECODE_WORKLOADS[args.workload]
    if args.tokens:  # a shorter cache (smaller profiling cases)
        w = replace(w, N=args.tokens)
    q, k, v = decode_inputs(replace(w, seed=w.seed + 1000 * rank), device=dev)
    out = torch.empty_like(q)
    lse = torch.empty((w.B, w.H), device=dev, dtype=torch.float32)
    ws = torch.empty(ra.ringattn_decode_workspace_size(w.B, w.H, w.N, w.D, w.S, w.k_chunk), device=dev,
                     dtype=torch.uint8)
    stream = torch.cuda.current_stream()
    for _ in range(args.warmup):
        ra.ringattn_decode(q, k, v, out, lse, w.S, w.k_chunk, ws)
    clocks = ClockSampler(dev.index)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    clocks.start()
    time.sleep(0.3)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(args.steps):
        ra.ringattn_decode(q, k, v, out, lse, w.S, w.k_chunk, ws)
    b.record(stream)
    torch.cuda.synchronize()
    clk = clocks.stop()
    if ra.ringattn_get_error() != 0:
        raise RuntimeError("device status word set during the timed region")
    ms = max_over_ranks(a.elapsed_time(b) / args.steps, dist if world > 1 else None, dev)
    flops = 4.0 * w.B * w.H * w.N * w.D
    cache_bytes = 2.0 * w.B * w.Hkv * w.N * w.D * 2
    pk = peaks()
    gbs = cache_bytes / (ms * 1e-3) / 1e9
    return {"metric": METRIC, "value": whole_job_tflops(flops, world, ms), "unit": "TFLOP/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": f"{w.name}: decode, one new token per head against a cache of N={w.N} in "
                                   f"S={w.S} shards, B={w.B}, H={w.H}, Hkv={w.Hkv}, d={w.D}, k_chunk={w.k_chunk}",
                       "l2": "cache larger than L2 (no flush between steps)"},
            "tokens_per_s": w.B * world / (ms * 1e-3),
            "roofline": {"bound": "hbm", "kernel": "decode_partial_kernel+decode_merge_kernel",
                         "achieved": gbs, "peak": pk["hbm_gbs"], "unit": "GB/s", "frac": gbs / pk["hbm_gbs"],
                         "traffic": None, "peak_kind": f"HBM copy ({pk['source']})"},
            "gpu_launches": 2 * args.steps, "clocks": clk}


def layer_flops(w):
    """Algorithmic FLOPs of one layer step (forward + backward):
    projections 8 T dm^2 forward and 16 T dm^2 backward (dO, dWo, dxn from
    three weights, dWq/dWk/dWv); attention 3.5 x its causal forward; the
    feed-forward 18 T dm d_ff (forward 6, backward 12).  RMS norms are not
    counted."""
    from exact_blockwise_long_b200.synthetic import AttnWorkload
    aw = AttnWorkload("x", w.B, w.H, w.N, w.D, w.S, w.q_chunk, w.k_chunk, w.causal, 0)
    proj = 24.0 * w.T * w.d_model * w.d_model
    ffn = 18.0 * w.T * w.d_model * w.d_ff
    return proj, attn_fwd_flops(aw), ffn


def layer_oracle_sample(w, tokens=1024):
    """The fp64 oracle layer (forward, then backward) on `tokens` tokens of
    one sequence at the layer's full widths.  Returns (seconds, FLOPs, desc, threads)."""
    import oracle
    from dataclasses import replace
    from exact_blockwise_long_b200.synthetic import layer_inputs, to_f64
    small = replace(w, B=1, N=tokens, S=1, q_chunk=tokens, k_chunk=tokens, ffn_chunk=tokens)
    x, params, dy = layer_inputs(small, device="cpu")
    xf, pf, dyf = to_f64(x), [to_f64(p_) for p_ in params], to_f64(dy)
    t0 = time.perf_counter()
    oracle.layer_forward(xf, pf, 1, tokens, w.H, w.D, w.causal, w.eps)
    oracle.layer_backward(xf, pf, dyf, 1, tokens, w.H, w.D, w.causal, w.eps)
    dt = time.perf_counter() - t0
    proj, af, ffn = layer_flops(small)
    try:
        from threadpoolctl import threadpool_info
        threads = max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    except Exception:
        threads = os.cpu_count()
    desc = (f"fp64 oracle (numpy) layer forward+backward of one {tokens}-token sequence at the layer's widths "
            f"(H={w.H}, d={w.D}, d_ff={w.d_ff}), same recipe; causal FLOPs counted once")
    return dt, proj + 3.5 * af + ffn, desc, threads


def decode_oracle_sample(w, min_seconds=2.0):
    """The fp64 oracle decode on whole (batch, key/value head) groups of the
    workload's cache, adding groups until min_seconds of CPU time.
    Returns (seconds, FLOPs, desc, threads)."""
    import oracle
    from dataclasses import replace
    from exact_blockwise_long_b200.synthetic import decode_inputs, to_f64
    G = w.H // w.Hkv
    dt, groups = 0.0, 0
    while groups == 0 or (dt < min_seconds and groups < w.B * w.Hkv):
        q, k, v = decode_inputs(replace(w, B=1, H=G, Hkv=1, seed=w.seed + 7919 * groups), device="cpu")
        q, k, v = to_f64(q), to_f64(k), to_f64(v)
        t0 = time.perf_counter()
        oracle.attention_decode(q, k, v)
        dt += time.perf_counter() - t0
        groups += 1
    try:
        from threadpoolctl import threadpool_info
        threads = max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    except Exception:
        threads = os.cpu_count()
    desc = f"fp64 oracle (numpy) decode of {groups} (batch, key/value head) group(s) of {G} query heads, N={w.N}"
    return dt, 4.0 * G * w.N * w.D * groups, desc, threads


def merge_oracle_sample(rows=1 << 18, D=128):
    """The fp64 oracle's exact merge on `rows` rows of random partials (about
    a quarter of the merge workload's rows).  Returns (seconds, the merge's
    FLOPs counted as 3 per output element, desc, threads)."""
    import numpy as np
    import oracle
    rng = np.random.default_rng(11)
    o_a, o_b = rng.standard_normal((rows, D)), rng.standard_normal((rows, D))
    l_a, l_b = rng.standard_normal(rows) * 5, rng.standard_normal(rows) * 5
    t0 = time.perf_counter()
    oracle.lse_merge(o_a, l_a, o_b, l_b)
    dt = time.perf_counter() - t0
    try:
        from threadpoolctl import threadpool_info
        threads = max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    except Exception:
        threads = os.cpu_count()
    return dt, 3.0 * rows * D, f"fp64 oracle (numpy) lse_merge of {rows} rows of d={D}", threads


def run_layer(args, ra, dev, rank, world, dist):
    """One training step of the whole blockwise layer: blockwise_layer_fwd then
    blockwise_layer_bwd, with per-step events from the library's marks."""
    import torch
    from dataclasses import replace
    from exact_blockwise_long_b200.synthetic import LAYER_WORKLOADS, layer_inputs
    w = LAYER_WORKLOADS[args.workload]
    if args.tokens:  # a shorter sequence with the same shard length (smaller profiling cases)
        w = replace(w, N=args.tokens, S=max(1, args.tokens // (w.N // w.S)))
    x, params, dy = layer_inputs(replace(w, seed=w.seed + 1000 * rank), device=dev)
    saved = torch.empty(ra.blockwise_layer_saved_size(w.B, w.N, w.H, w.D), device=dev, dtype=torch.uint8)
    fws = torch.empty(ra.blockwise_layer_fwd_workspace_size(w.ffn_chunk, w.d_ff), device=dev, dtype=torch.uint8)
    bws = torch.empty(ra.blockwise_layer_bwd_workspace_size(w.B, w.N, w.H, w.D, w.d_ff, w.ffn_chunk), device=dev,
                      dtype=torch.uint8)
    y, dx = torch.empty_like(x), torch.empty_like(x)
    grads = tuple(torch.empty(p_.shape, device=dev, dtype=torch.float32) for p_ in params)
    stream = torch.cuda.current_stream()
    dims = (w.B, w.N, w.H, w.D, w.S, w.q_chunk, w.k_chunk, w.causal, w.ffn_chunk)
    n_chunks = w.T // w.ffn_chunk
    # forward: norm, 3 projections, attention, o projection, norm, 2 GEMMs per FFN chunk;
    # backward: 6 GEMMs per FFN chunk, norm (3), dO, dWo, attention (3), dxn, 3 dW, norm (3)
    launches_per_step = (7 + 2 * n_chunks) + (6 * n_chunks + 3 + 1 + 1 + 3 + 1 + 3 + 3)

    def event():
        return torch.cuda.Event(enable_timing=True)

    spans = []

    def step(xx, gy, yy, gx, gr, timed=False):
        fm = [event() for _ in range(6)] if timed else None
        bm = [event() for _ in range(10)] if timed else None
        if timed:
            s0 = event()
            s0.record(stream)
        ra.blockwise_layer_fwd(xx, params, yy, saved, *dims, fws, eps=w.eps, marks=fm)
        ra.blockwise_layer_bwd(xx, params, saved, gy, gx, gr, *dims, bws, marks=bm)
        if timed:
            spans.append((s0, fm, bm))

    for _ in range(args.warmup):
        step(x, dy, y, dx, grads)
    torch.cuda.synchronize()
    if ra.ringattn_get_error() != 0:
        raise RuntimeError("device status word set during warm-up")
    clocks = ClockSampler(dev.index)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    clocks.start()
    time.sleep(0.3)
    a, b = event(), event()
    a.record(stream)
    for _ in range(args.steps):
        step(x, dy, y, dx, grads, timed=True)
    b.record(stream)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    clk = clocks.stop()
    if ra.ringattn_get_error() != 0:
        raise RuntimeError("device status word set during the timed region")
    ms = max_over_ranks(a.elapsed_time(b) / args.steps, dist if world > 1 else None, dev)
    proj, af, ffn = layer_flops(w)
    flops = proj + 3.5 * af + ffn
    value = whole_job_tflops(flops, world, ms)

    def avg(fn):
        return sum(fn(s0, fm, bm) for s0, fm, bm in spans) / len(spans)

    fwd_name = ra.ringattn_kernel_plan(0, w.N, w.D, torch.bfloat16, w.S)
    bwd_plan = ra.ringattn_kernel_plan(1, w.N, w.D, torch.bfloat16, w.S)
    # the layer records a mark after the attention backward's preprocess, its
    # main pass and its last launch (the dQ conversion, or the split dQ pass)
    main, last = (("bwd_fused_kernel", 2.5), ("bwd_dq_convert_kernel", 0.0)) if "bwd_fused_kernel" in bwd_plan \
        else (("bwd_kv_kernel", 2.0), ("bwd_q_kernel", 0.5))
    kernels = {
        fwd_name: (avg(lambda s0, fm, bm: fm[1].elapsed_time(fm[2])), af, "fwd_tc.cu"),
        main[0]: (avg(lambda s0, fm, bm: bm[4].elapsed_time(bm[5])), main[1] * af, "bwd_tc.cu"),
        last[0]: (avg(lambda s0, fm, bm: bm[5].elapsed_time(bm[6])), last[1] * af, "bwd_tc.cu"),
        "gemm_kernel[projections]": (avg(lambda s0, fm, bm: fm[0].elapsed_time(fm[1]) + fm[2].elapsed_time(fm[3]) +
                                         bm[1].elapsed_time(bm[3]) + bm[6].elapsed_time(bm[8])), proj,
                                     "gemm_tc.cu"),
        "gemm_kernel[ffn fwd+bwd]": (avg(lambda s0, fm, bm: fm[4].elapsed_time(fm[5]) +
                                         fm[5].elapsed_time(bm[0])), ffn, "gemm_tc.cu"),
    }
    kname = max(kernels, key=lambda k_: kernels[k_][0])
    kms, kflops, ksrc = kernels[kname]
    pk = peaks()
    achieved = kflops / (kms * 1e-3) / 1e12
    src = os.path.join(ROOT, "exact_blockwise_long_b200", "csrc", ksrc)
    sha = code_fingerprint(src)
    tr = NCU_TRAFFIC.get((kname, args.workload))
    peak, peak_kind, other = tensor_peak(pk, ms * args.steps)
    roof = {"bound": "tensor", "kernel": kname, "achieved": achieved, "peak": peak,
            "unit": "TFLOP/s", "frac": achieved / peak,
            "traffic": tr["bytes"] if tr and tr["code_sha256"] == sha else None,
            "peak_kind": peak_kind, "frac_of_other_peak": achieved / other,
            "kernel_ms": kms,
            "kernels": {k_: {"ms": v_[0], "algorithmic_tflops": v_[1] / (v_[0] * 1e-3) / 1e12}
                        for k_, v_ in kernels.items()}}
    line = {"metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": f"{w.name}: one blockwise transformer layer fwd+bwd (RMS norms, q/k/v/o "
                                   f"projections, ring attention, SwiGLU FFN), B={w.B}, N={w.N}, H={w.H}, d={w.D}, "
                                   f"d_ff={w.d_ff}, S={w.S}, q_chunk={w.q_chunk}, k_chunk={w.k_chunk}, "
                                   f"ffn_chunk={w.ffn_chunk}, {'causal' if w.causal else 'non-causal'}",
                       "B": w.B, "seq_len": w.N, "H": w.H, "head_dim": w.D, "d_ff": w.d_ff, "shards": w.S,
                       "l2": "inputs larger than L2 (no flush between steps)"},
            "tokens_per_s": w.T * world / (ms * 1e-3), "pct_of_bf16_peak": 100.0 * value / world / peak,
            "roofline": roof, "gpu_launches": launches_per_step * args.steps, "clocks": clk}

    if not args.no_e2e:
        # end to end: x and dy in from pinned host memory, y, dx and the nine
        # parameter gradients back, on copy streams overlapped with compute
        hin = [t.cpu().pin_memory() for t in (x, dy)]
        outs0 = [y, dx] + list(grads)
        hout = [torch.empty(t.shape, dtype=t.dtype, pin_memory=True) for t in outs0]
        ins = [[x, dy], [torch.empty_like(x), torch.empty_like(dy)]]
        outs = [outs0, [torch.empty_like(t) for t in outs0]]
        h2d = sum(t.numel() * t.element_size() for t in hin)
        d2h = sum(t.numel() * t.element_size() for t in hout)
        e2e_steps = max(3, min(args.steps, 5))
        s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
        in_ready, done, copied = [event(), event()], [event(), event()], [event(), event()]
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        ea, eb = event(), event()
        ea.record(stream)
        s_in.wait_event(ea)
        for j in range(e2e_steps):
            bi = j % 2
            if j >= 2:
                s_in.wait_event(done[bi])
            with torch.cuda.stream(s_in):
                for h_, d_ in zip(hin, ins[bi]):
                    d_.copy_(h_, non_blocking=True)
            in_ready[bi].record(s_in)
            stream.wait_event(in_ready[bi])
            if j >= 2:
                stream.wait_event(copied[bi])
            o_ = outs[bi]
            step(ins[bi][0], ins[bi][1], o_[0], o_[1], tuple(o_[2:]))
            done[bi].record(stream)
            s_out.wait_event(done[bi])
            with torch.cuda.stream(s_out):
                for h_, d_ in zip(hout, outs[bi]):
                    h_.copy_(d_, non_blocking=True)
            copied[bi].record(s_out)
        stream.wait_event(copied[(e2e_steps - 1) % 2])
        stream.wait_event(copied[(e2e_steps - 2) % 2])
        eb.record(stream)
        torch.cuda.synchronize()
        if ra.ringattn_get_error() != 0:
            raise RuntimeError("device status word set during the end-to-end run")
        e_ms = max_over_ranks(ea.elapsed_time(eb) / e2e_steps, dist if world > 1 else None, dev)
        line["e2e"] = {"value": whole_job_tflops(flops, world, e_ms), "unit": "TFLOP/s", "h2d_bytes_per_step": h2d,
                       "d2h_bytes_per_step": d2h, "ms_per_step": e_ms, "steps": e2e_steps,
                       "copies": "pinned host, overlapped with compute on two copy streams"}
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        dt, fl, desc, threads = layer_oracle_sample(w)
        line["cpu_baseline"] = {"value": fl / dt / 1e12, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
                                "sample": desc, "seconds": dt}
    return line


def run_ring(args, ra, dev, rank, world, dist):
    """The workload's sequence cut into `world` contiguous shards, one per
    rank; forward and backward by exact_blockwise_long_b200.ring (key/value
    blocks and the dK/dV accumulators passed rank to rank by NCCL send/receive,
    overlapped with each shard pair's compute).  The total work is fixed
    (strong scaling)."""
    import torch
    from dataclasses import replace
    from exact_blockwise_long_b200 import ring
    from exact_blockwise_long_b200.synthetic import attention_inputs
    aw, _ = workload(args.workload)
    if args.heads:
        aw = replace(aw, H=args.heads)
    if aw.N % world or (aw.N // world) % aw.q_chunk or (aw.N // world) % aw.k_chunk:
        raise SystemExit(f"--ring: {aw.N} tokens do not split into {world} shards of whole chunks")
    L = aw.N // world
    q, k, v, do = attention_inputs(aw, device=dev)  # the same full-sequence draw on every rank
    sl = slice(rank * L, (rank + 1) * L)
    q, k, v, do = (t[:, :, sl].contiguous() for t in (q, k, v, do))
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream()

    def step():
        out, lse = ring.ring_attention_forward(q, k, v, aw.causal, q_chunk=aw.q_chunk, k_chunk=aw.k_chunk)
        ring.ring_attention_backward(q, k, v, out, lse, do, aw.causal, q_chunk=aw.q_chunk, k_chunk=aw.k_chunk)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if ra.ringattn_get_error() != 0:
        raise RuntimeError("device status word set during warm-up")
    clocks = ClockSampler(dev.index)
    dist.barrier()
    torch.cuda.synchronize()
    clocks.start()
    time.sleep(0.3)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(args.steps):
        step()
    b.record(stream)
    torch.cuda.synchronize()
    dist.barrier()
    clk = clocks.stop()
    if ra.ringattn_get_error() != 0:
        raise RuntimeError("device status word set during the timed region")
    ms = max_over_ranks(a.elapsed_time(b) / args.steps, dist, dev)
    flops = attn_step_flops(aw)
    value = flops / (ms * 1e-3) / 1e12
    pk = peaks()
    peak, peak_kind, _ = tensor_peak(pk, ms * args.steps)
    # this rank's launches per step: forward pairs and the cast; backward
    # preparation, pairs, the accumulator additions after the first step, casts
    vis = sum(1 for t in range(world) if not (aw.causal and (rank - t) % world > rank))
    per_pair = 1 if "bwd_fused_kernel" in ra.ringattn_kernel_plan(1, L, aw.D, torch.bfloat16, 1) else 2
    launches = (vis + 1) + (1 + per_pair * vis + 2 * (vis - 1) + 3)
    return {"metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "strong",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": dict(describe(aw, None), workload=f"{aw.name} as a device ring: {world} shard(s) of {L} "
                                                        f"tokens, one per rank, causal FLOPs counted once",
                           parallelism=f"ring{world}"),
            "tokens_per_s": aw.B * aw.N / (ms * 1e-3), "pct_of_bf16_peak": 100.0 * value / world / peak,
            "roofline": {"bound": "tensor", "kernel": "ring (all per-pair launches)", "achieved": value / world,
                         "peak": peak, "unit": "TFLOP/s", "frac": value / world / peak, "traffic": None,
                         "peak_kind": peak_kind},
            "gpu_launches": launches * args.steps, "clocks": clk, "e2e": None}


def main():
    args = parse()
    if args.impl == "reference":
        return run_reference(args)

    import torch
    import torch.distributed as dist

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        from datetime import timedelta
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(0)
        if args.ring:  # a ring of one rank still runs through the process-group calls
            import socket
            from datetime import timedelta
            sk = socket.socket()
            sk.bind(("127.0.0.1", 0))
            os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
            os.environ.setdefault("MASTER_PORT", str(sk.getsockname()[1]))
            sk.close()
            dist.init_process_group("nccl", rank=0, world_size=1, timeout=timedelta(seconds=120),
                                    device_id=torch.device("cuda", 0))
    dev = torch.device("cuda", torch.cuda.current_device())

    from exact_blockwise_long_b200 import build
    if rank == 0:
        build.build()
    if world > 1:
        dist.barrier()
    import exact_blockwise_long_b200 as ra
    from dataclasses import replace
    from exact_blockwise_long_b200.synthetic import attention_inputs, ffn_inputs

    if args.ring or args.workload.startswith("decode") or args.workload in ("layer7b_full", "n32k_d128_step",
                                                                            "merge_n32k"):
        runner = (run_ring if args.ring else run_decode if args.workload.startswith("decode") else
                  run_layer if args.workload == "layer7b_full" else run_step_mode)
        line = runner(args, ra, dev, rank, world, dist)
        if dist.is_initialized():
            dist.barrier()
            dist.destroy_process_group()
        if rank == 0:
            print(json.dumps(line), flush=True)
        return 0

    aw, fw = workload(args.workload)
    if args.heads:
        aw = replace(aw, H=args.heads)
    # each rank draws its own batch (weak scaling): seed offset by rank
    aw_r = replace(aw, seed=aw.seed + 1000 * rank)
    q, k, v, do = attention_inputs(aw_r, device=dev)
    B, H, N, D = q.shape
    o = torch.empty_like(q)
    lse = torch.empty((B, H, N), device=dev, dtype=torch.float32)
    if aw.bwd:
        dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
        ws = torch.empty(ra.ringattn_bwd_workspace_size(B, H, N, D), device=dev, dtype=torch.uint8)
    if fw is not None:
        x, w1, w2, w3, dy = ffn_inputs(replace(fw, seed=fw.seed + 1000 * rank), device=dev, with_dy=True)
        y, dx = torch.empty_like(x), torch.empty_like(x)
        dw1, dw3 = (torch.empty(w1.shape, device=dev, dtype=torch.float32) for _ in range(2))
        dw2 = torch.empty(w2.shape, device=dev, dtype=torch.float32)
        ffn_ws = torch.empty(ra.blockwise_ffn_workspace_size(fw.chunk, fw.d_ff), device=dev, dtype=torch.uint8)
        ffn_bws = torch.empty(ra.blockwise_ffn_bwd_workspace_size(fw.chunk, fw.d_ff), device=dev,
                              dtype=torch.uint8)
    stream = torch.cuda.current_stream()
    cfg = (aw.S, aw.q_chunk, aw.k_chunk, aw.causal)
    gqa = aw.kv_heads != aw.H
    # the kernels the library launches for this shape on this device
    fwd_name = ra.ringattn_kernel_plan(0, aw.N, aw.D, torch.bfloat16, aw.S)
    bwd_plan = ra.ringattn_kernel_plan(1, aw.N, aw.D, torch.bfloat16, aw.S) if aw.bwd else ""
    fused = "bwd_fused_kernel" in bwd_plan
    # backward phases timed one by one: preprocess, main pass, last pass
    bwd_phases = (1, 8, 16) if fused else (1, 2, 4)
    bwd_names = ("bwd_fused_kernel", "bwd_dq_convert_kernel") if fused else ("bwd_kv_kernel", "bwd_q_kernel")

    def fwd_call(qq, kk, vv, oo, ll):
        if gqa:
            ra.ringattn_fwd_gqa(qq, kk, vv, oo, ll, *cfg)
        else:
            ra.ringattn_fwd(qq, kk, vv, oo, ll, *cfg)

    def bwd_call(qq, kk, vv, oo, ll, dd, gq, gk, gv):
        if gqa:
            ra.ringattn_bwd_gqa(qq, kk, vv, oo, ll, dd, gq, gk, gv, *cfg, ws)
        else:
            ra.ringattn_bwd(qq, kk, vv, oo, ll, dd, gq, gk, gv, *cfg, ws)

    ev = {}

    def event():
        return torch.cuda.Event(enable_timing=True)

    def step(timed=False):
        if timed:
            e = [event() for _ in range(7)]
            e[0].record(stream)
        fwd_call(q, k, v, o, lse)
        launches = 1
        if timed:
            e[1].record(stream)
        if aw.bwd and gqa:
            bwd_call(q, k, v, o, lse, do, dq, dk, dv)
            if timed:
                e[2].record(stream)
                e[4].record(stream)
            launches += 3
        elif aw.bwd:
            for i, m in enumerate(bwd_phases):
                ra.ringattn_bwd_phase(q, k, v, o, lse, do, dq, dk, dv, *cfg, ws, m)
                if timed:
                    e[2 + i].record(stream)
            launches += 3
        if fw is not None:
            if timed:
                e[5].record(stream)
            ra.blockwise_ffn(x, w1, w2, w3, y, fw.chunk, ffn_ws)
            ra.blockwise_ffn_bwd(x, w1, w2, w3, dy, dx, dw1, dw2, dw3, fw.chunk, ffn_bws)
            launches += 8 * (fw.T // fw.chunk)  # forward: 2 GEMMs per chunk, backward: 6 per chunk
            if timed:
                e[6].record(stream)
                ev.setdefault("ffn", []).append((e[5], e[6]))
        if timed:
            ev.setdefault("fwd", []).append((e[0], e[1]))
            if aw.bwd and gqa:
                ev.setdefault("bwd", []).append((e[1], e[4]))
            elif aw.bwd:
                ev.setdefault("bwd_main", []).append((e[2], e[3]))
                ev.setdefault("bwd_last", []).append((e[3], e[4]))
        return launches

    for _ in range(args.warmup):
        step()
    if ra.ringattn_get_error() != 0:
        raise RuntimeError("device status word set during warm-up")

    def timed_region():
        ev.clear()
        clocks = ClockSampler(dev.index)
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        clocks.start()
        time.sleep(0.3)
        t_start, t_stop = event(), event()
        t_start.record(stream)
        n_launch = 0
        for _ in range(args.steps):
            n_launch += step(timed=True)
        t_stop.record(stream)
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        c = clocks.stop()
        if ra.ringattn_get_error() != 0:
            raise RuntimeError("device status word set during the timed region")
        ms_total = max_over_ranks(t_start.elapsed_time(t_stop), dist if world > 1 else None, dev)
        return ms_total / args.steps, c, n_launch

    ms_step, clk, launches = timed_region()
    # a timed region that saw a hardware or thermal slowdown, or clocks well
    # below their maximum with no reason given, is measured once more
    if clocks_rejected(clk, dist if world > 1 else None, dev):
        first = clk
        ms_step, clk, launches = timed_region()
        clk = dict(clk, remeasured_after={"sm_mhz": first.get("sm_mhz"), "reasons": first.get("reasons")})

    flops_step = attn_step_flops(aw) + (ffn_flops(fw) if fw else 0.0)
    value = whole_job_tflops(flops_step, world, ms_step)
    tokens_s = aw.B * aw.N * world / (ms_step * 1e-3)
    pk = peaks()

    # dominant kernel: the backward main loop when there is a backward
    def mean_ms(pairs):
        return sum(a.elapsed_time(b) for a, b in pairs) / len(pairs)

    # Algorithmic FLOPs per launch: the forward's two matmuls (S, PV); the
    # fused backward pass's five (S, dP, dV, dK, dQ); or, split, the dK/dV
    # kernel's four and the dQ kernel's one (its S and dP are recomputation,
    # not credited): 2 + 5 = 7 = 3.5 x the forward's 2 either way.
    fwd_fl = attn_fwd_flops(aw)
    kernels = {fwd_name: (mean_ms(ev["fwd"]), fwd_fl, "fwd_tc.cu")}
    hbm = {}
    if aw.bwd and gqa:
        # one call: all the backward's launches, timed together
        kernels[bwd_plan.replace("bwd_preprocess_kernel+", "")] = (mean_ms(ev["bwd"]), 2.5 * fwd_fl, "bwd_tc.cu")
    elif aw.bwd and fused:
        kernels["bwd_fused_kernel"] = (mean_ms(ev["bwd_main"]), 2.5 * fwd_fl, "bwd_tc.cu")
        # the conversion reads the fp32 accumulator and writes bf16 dq
        conv_ms = mean_ms(ev["bwd_last"])
        conv_bytes = aw.B * aw.H * aw.N * aw.D * 6.0
        hbm["bwd_dq_convert_kernel"] = {"ms": conv_ms, "gbs": conv_bytes / (conv_ms * 1e-3) / 1e9}
    elif aw.bwd:
        kernels["bwd_kv_kernel"] = (mean_ms(ev["bwd_main"]), 2.0 * fwd_fl, "bwd_tc.cu")
        kernels["bwd_q_kernel"] = (mean_ms(ev["bwd_last"]), 0.5 * fwd_fl, "bwd_tc.cu")
    kname = max(kernels, key=lambda k_: kernels[k_][0])
    if fw is not None:
        # the feed-forward's forward and backward GEMMs, timed together
        kernels["gemm_kernel[ffn fwd+bwd]"] = (mean_ms(ev["ffn"]), ffn_flops(fw), "gemm_tc.cu")
    kms, kflops, ksrc = kernels[kname]
    achieved = kflops / (kms * 1e-3) / 1e12
    src = os.path.join(ROOT, "exact_blockwise_long_b200", "csrc", ksrc)
    sha = code_fingerprint(src)
    tr = NCU_TRAFFIC.get((kname, args.workload))
    traffic = tr["bytes"] if tr and tr["code_sha256"] == sha else None
    peak, peak_kind, other = tensor_peak(pk, ms_step * args.steps)
    roof = {"bound": "tensor", "kernel": kname, "achieved": achieved, "peak": peak,
            "unit": "TFLOP/s", "frac": achieved / peak, "traffic": traffic, "peak_kind": peak_kind,
            "frac_of_other_peak": achieved / other, "kernel_ms": kms,
            "kernels": {k_: {"ms": v_[0], "algorithmic_tflops": v_[1] / (v_[0] * 1e-3) / 1e12}
                        for k_, v_ in kernels.items()}}
    if hbm:
        roof["hbm_kernels"] = hbm

    line = {"metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic", "config": describe(aw, fw),
            "tokens_per_s": tokens_s, "pct_of_bf16_peak": 100.0 * value / world / peak,
            "roofline": roof, "gpu_launches": launches, "clocks": clk,
            "kernel_plan": {"fwd": fwd_name, "bwd": bwd_plan or None}}

    # End to end through the C ABI's host-buffer step (plain attention
    # workloads): every step's inputs come from pinned host memory and its
    # results go back to it inside ringattn_step_host; two device buffer sets
    # are used in turn.  A set's inputs are refilled once the backward that
    # read them has run (its consumed event) and its results overwritten once
    # they are on the host (its done event), so one step's copies overlap the
    # neighbouring steps' compute.
    if not args.no_e2e and aw.bwd and fw is None and not gqa:
        hin = [t.cpu().pin_memory() for t in (q, k, v, do)]
        hout = [[torch.empty(t.shape, dtype=t.dtype, pin_memory=True) for t in (o, lse, dq, dk, dv)]
                for _ in range(2)]
        devs = [torch.empty(ra.ringattn_step_host_size(B, H, N, D), device=dev, dtype=torch.uint8) for _ in range(2)]
        h2d = sum(t.numel() * t.element_size() for t in hin)
        d2h = sum(t.numel() * t.element_size() for t in hout[0])
        e2e_steps = max(3, args.steps)
        s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
        done, consumed = [event(), event()], [event(), event()]
        for e_ in done + consumed:
            e_.record(stream)  # create the events before their handles are passed on
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        a, b = event(), event()
        a.record(stream)
        s_in.wait_event(a)
        s_out.wait_event(a)
        for j in range(e2e_steps):
            bi = j % 2
            ra.ringattn_step_host(*hin, *hout[bi], devs[bi], *cfg, stream, s_in, s_out,
                                  inputs_free_event=consumed[bi] if j >= 2 else None,
                                  outputs_free_event=done[bi] if j >= 2 else None,
                                  consumed_event=consumed[bi], done_event=done[bi])
        stream.wait_event(done[(e2e_steps - 1) % 2])
        stream.wait_event(done[(e2e_steps - 2) % 2])
        b.record(stream)
        torch.cuda.synchronize()
        if ra.ringattn_get_error() != 0:
            raise RuntimeError("device status word set during the end-to-end run")
        e_ms = max_over_ranks(a.elapsed_time(b) / e2e_steps, dist if world > 1 else None, dev)
        line["e2e"] = {"value": whole_job_tflops(flops_step, world, e_ms), "unit": "TFLOP/s",
                       "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e_ms,
                       "steps": e2e_steps, "api": "ringattn_step_host (C ABI, host buffers)",
                       "copies": "pinned host, on two copy streams inside the C call, overlapped with compute"}

    # End to end through the public API (the other workloads): every step
    # copies its inputs from pinned host memory and reads its results back.  Two device buffer sets
    # let step j+1's host-to-device copies and step j-1's device-to-host
    # copies run on their own streams while step j computes.  Each tensor
    # moves as soon as it can: q, k, v first and dO (and the FFN's x, dy)
    # behind them while the forward runs; O and LSE go back while the
    # backward runs, dK and dV while the dQ pass runs, dQ last.
    if not args.no_e2e and "e2e" not in line:
        in_f0 = [q, k, v]
        in_b0 = ([do] if aw.bwd else []) + ([x, dy] if fw is not None else [])
        out_f0 = [o, lse]
        out_kv0 = [dk, dv] if aw.bwd else []
        out_b0 = ([dq] if aw.bwd else []) + ([y, dx, dw1, dw2, dw3] if fw is not None else [])
        groups0 = [in_f0, in_b0, out_f0, out_kv0, out_b0]
        hgrp = [[t.cpu().pin_memory() for t in g_] for g_ in groups0[:2]] + \
               [[torch.empty(t.shape, dtype=t.dtype, pin_memory=True) for t in g_] for g_ in groups0[2:]]
        dev_sets = [groups0, [[torch.empty_like(t) for t in g_] for g_ in groups0]]
        h2d = sum(t.numel() * t.element_size() for g_ in hgrp[:2] for t in g_)
        d2h = sum(t.numel() * t.element_size() for g_ in hgrp[2:] for t in g_)
        e2e_steps = max(3, args.steps)  # as many as the device-timed loop: pipeline fill and drain amortise alike
        s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
        f_in, b_in, f_done, kv_done, done, copied = ([event(), event()] for _ in range(6))
        split_bwd = aw.bwd and not gqa
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        a, b = event(), event()
        a.record(stream)
        s_in.wait_event(a)

        def to_host(dev_group, host_group):
            with torch.cuda.stream(s_out):
                for h, d_ in zip(host_group, dev_group):
                    h.copy_(d_, non_blocking=True)

        for j in range(e2e_steps):
            bi = j % 2
            in_f, in_b, out_f, out_kv, out_b = dev_sets[bi]
            if j >= 2:
                s_in.wait_event(done[bi])  # step j-2 no longer reads these inputs
            with torch.cuda.stream(s_in):
                for h, d_ in zip(hgrp[0], in_f):
                    d_.copy_(h, non_blocking=True)
                f_in[bi].record(s_in)
                for h, d_ in zip(hgrp[1], in_b):
                    d_.copy_(h, non_blocking=True)
                b_in[bi].record(s_in)
            stream.wait_event(f_in[bi])
            if j >= 2:
                stream.wait_event(copied[bi])  # step j-2's results have been read back
            qq, kk, vv = in_f
            oo, ll = out_f
            fwd_call(qq, kk, vv, oo, ll)
            f_done[bi].record(stream)
            s_out.wait_event(f_done[bi])
            to_host(out_f, hgrp[2])
            stream.wait_event(b_in[bi])
            if split_bwd:
                # dk, dv are final after the main pass: they go back while the last pass runs
                ra.ringattn_bwd_phase(qq, kk, vv, oo, ll, in_b[0], out_b[0], out_kv[0], out_kv[1], *cfg, ws,
                                      bwd_phases[0] | bwd_phases[1])
                kv_done[bi].record(stream)
                s_out.wait_event(kv_done[bi])
                to_host(out_kv, hgrp[3])
                ra.ringattn_bwd_phase(qq, kk, vv, oo, ll, in_b[0], out_b[0], out_kv[0], out_kv[1], *cfg, ws,
                                      bwd_phases[2])
            elif aw.bwd:
                bwd_call(qq, kk, vv, oo, ll, in_b[0], out_b[0], out_kv[0], out_kv[1])
            if fw is not None:
                xx, gy = in_b[-2], in_b[-1]
                ra.blockwise_ffn(xx, w1, w2, w3, out_b[-5], fw.chunk, ffn_ws)
                ra.blockwise_ffn_bwd(xx, w1, w2, w3, gy, *out_b[-4:], fw.chunk, ffn_bws)
            done[bi].record(stream)
            s_out.wait_event(done[bi])
            if not split_bwd:
                to_host(out_kv, hgrp[3])
            to_host(out_b, hgrp[4])
            copied[bi].record(s_out)
        stream.wait_event(copied[(e2e_steps - 1) % 2])
        if e2e_steps > 1:
            stream.wait_event(copied[(e2e_steps - 2) % 2])
        b.record(stream)
        torch.cuda.synchronize()
        if ra.ringattn_get_error() != 0:
            raise RuntimeError("device status word set during the end-to-end run")
        e_ms = max_over_ranks(a.elapsed_time(b) / e2e_steps, dist if world > 1 else None, dev)
        line["e2e"] = {"value": whole_job_tflops(flops_step, world, e_ms), "unit": "TFLOP/s",
                       "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e_ms,
                       "steps": e2e_steps, "copies": "pinned host, overlapped with compute on two copy streams"}

    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        if not args.no_cpu_baseline and world == 1:
            dt, fl, desc, threads = oracle_sample(aw, fw, n_tokens=8192, min_seconds=10.0)
            line["cpu_baseline"] = {"value": fl / dt / 1e12, "unit": "TFLOP/s", "cores": threads,
                                    "kind": "oracle", "sample": desc, "seconds": dt}
        print(json.dumps(line), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
