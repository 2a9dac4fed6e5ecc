"""Benchmark of the quantized attention prefill path on B200.

One step = the whole hot path on the canonical call of the "Exact Numerical
Contract" page: B=1, N=37,810, H=56, D=128, interleaved BF16 QKV [N, 21504]:
  qattn_prep_quant (RMSNorm + RoPE, K mean, INT8 Q/K, FP8 V; two HBM passes)
  -> qattn_fwd (tcgen05 INT8 QK^T, online softmax, FP8 P.V, BF16 out).
Value = effective TFLOP/s = 4*B*H*N^2*D per step (all ranks) / step time
(max over ranks).  Each rank runs its own independent problem (weak scaling,
no data-path collective).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]

--impl reference times the CPU oracle (the plain reference implementation of
the method written for this repository) on a bounded sample of the same
workload, on the host cores.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "ms/call and effective TFLOPS at N=37810 H=56 D=128; % of INT8/FP8 tensor peak"
WORKLOAD = {"workload": "canonical interleaved-QKV quantized attention prefill",
            "B": 1, "N": 37810, "H": 56, "D": 128, "qkv_row_width": 21504,
            "rotary_dim": 96, "causal": False,
            "l2": "inputs larger than L2 (1.63 GB QKV, 126 MB L2); no flush needed"}
NOMINAL_FP8_OVER_BF16 = 2.0          # 4.5 / 2.25 PFLOP/s dense (nominal ratio)
# DRAM bytes per canonical attention launch: ncu dram__bytes_read + write of one
# attention launch on the B1 N16384 H32 D128 case, scaled by the units processed
# (N*H: 2117360 / 524288 = 4.0386).  Valid only for the attention kernel the
# capture was taken on; None until it is re-taken after a kernel change.
ATTN_TRAFFIC_BYTES = int((203279616 + 102831360) * 2117360 / 524288)
ATTN_TRAFFIC_SOURCE = ("ncu dram__bytes_read.sum + dram__bytes_write.sum of one attn_fwd_kernel<128,2,0> "
                       "launch on B1 N16384 H32 D128 (306.1 MB), scaled by the units processed "
                       "N*H (x4.0386) to the canonical launch")
SPEC_FP8_TFLOPS = 4500.0
PROBE_MMA_MACS = 128 * 256 * 32      # multiply-adds of one probe MMA (M128 N256 K32)


# ------------------------------------------------------------------ distributed plumbing
def dist_env():
    """(rank, world, local_rank) from the torchrun environment (1 rank if absent)."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


def init_dist(world: int, backend: str):
    import torch.distributed as dist
    if world > 1 and not dist.is_initialized():
        import datetime
        dist.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=120))
    return dist if world > 1 else None


def percentile(values, q: float) -> float:
    """The q-quantile (0..1) of a list by the nearest-rank rule on the sorted values."""
    v = sorted(values)
    if not v:
        raise ValueError("no values")
    return v[min(len(v) - 1, max(0, round(q * (len(v) - 1))))]


def max_over_ranks(x: float, dist, device=None) -> float:
    """Largest value of x over all ranks (x itself with one rank)."""
    if dist is None:
        return x
    import torch
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(x: float, dist, device=None) -> float:
    if dist is None:
        return x
    import torch
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


from quantized_exact_attention_qattn_b200.shard import kv_shard, shard_heads  # noqa: E402,F401


# ------------------------------------------------------------------ clocks
class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons during a region."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.Q}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except OSError:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *a):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            self.t.join(timeout=5)

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx = float(f[2])
            except ValueError:
                continue
            for nm, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(nm)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": mx, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


def prep_quant_bytes(w) -> int:
    """Algorithmic HBM bytes of one qattn_prep_quant call (or, for the rotated
    variant, of qattn_quant_hadamard): every tensor read or written once per pass
    that touches it.  Fused path: raw Q, K, V read and INT8 Q written (pass 1),
    FP64 K sums and FP32 V maxima per 64-row block written and read back, raw K and
    V read again and INT8 K and E4M3 V (padded to 64-row blocks) written (pass 2)."""
    nk = -(-w.Nkv // 64)
    q_in = 2 * w.B * w.Nq * w.Hq * w.D
    kv_in = 2 * w.B * w.Nkv * w.Hkv * w.D
    q8 = w.B * w.Nq * w.Hq * w.D
    k8 = w.B * w.Nkv * w.Hkv * w.D
    v8 = w.B * w.Hkv * w.D * 64 * nk
    partials = 2 * 12 * w.B * nk * w.Hkv * w.D
    if w.hadamard:   # V statistics pass, then Q, K and V quantized
        return kv_in + 4 * w.B * nk * w.Hkv * w.D * 2 + q_in + 2 * kv_in + q8 + k8 + v8
    return (q_in + 2 * kv_in + q8) + partials + (2 * kv_in + k8 + v8)


def tc_probe(dev, kind: int, iters: int = 8192):
    """The library's tensor-core peak probe (one CTA per SM, back-to-back M128 N256
    K32 MMAs from shared memory): event-timed TFLOP/s and multiply-adds per clock
    per SM from the in-kernel cycle count."""
    import torch
    import quantized_exact_attention_qattn_b200 as qa
    n_sm = torch.cuda.get_device_properties(dev).multi_processor_count
    cycles = torch.zeros(1, dtype=torch.int64, device=dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    qa.qattn_tc_probe(kind, 256, n_sm, cycles, err)
    qa.qattn_check(err)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    qa.qattn_tc_probe(kind, iters, n_sm, cycles, err)
    e1.record()
    qa.qattn_check(err)
    ms = e0.elapsed_time(e1)
    macs_clk = iters * PROBE_MMA_MACS / int(cycles.item())
    return {"tflops": 2.0 * n_sm * iters * PROBE_MMA_MACS / (ms / 1e3) / 1e12,
            "macs_per_clk_per_sm": macs_clk, "n_sm": n_sm, "iters": iters}


# ------------------------------------------------------------------ workloads
def make_workload(name: str):
    from quantized_exact_attention_qattn_b200 import synth
    if name == "profile16k":   # B1 N16384 H32 D128: > L2 inputs, small enough to profile
        return synth.custom(16, 1, 16384, 32, 128, name="profile16k")
    return synth.make(name)


def workload_config(w) -> dict:
    if w.name == "canonical":
        return dict(WORKLOAD)
    return {"workload": f"{w.name} quantized attention prefill", "B": w.B, "Nq": w.Nq,
            "Nkv": w.Nkv, "Hq": w.Hq, "Hkv": w.Hkv, "D": w.D, "hadamard": w.hadamard}


# ------------------------------------------------------------------ CPU oracle sample
def oracle_sample(w, heads, q_tiles):
    """Run the CPU oracle on `heads` x `q_tiles` of workload `w` (all keys).
    Returns (seconds, attention flops of the sample)."""
    import numpy as np
    from oracle import qattn_oracle as O
    t0 = time.perf_counter()
    hs = list(heads)
    rows = np.concatenate([np.arange(128 * t, min(w.Nq, 128 * t + 128)) for t in q_tiles])
    k = w.k[:, :, hs]
    v = w.v[:, :, hs]
    q = w.q[:, rows][:, :, hs]
    kp = O.prep(k, w.k_weight, w.eps, w.rotary_dim, w.theta)
    mu = O.k_mean(kp)
    k8, ks = O.quant_k(kp, mu)
    v8t, vs = O.quant_v(v)
    qp = O.prep(q, w.q_weight, w.eps, w.rotary_dim, w.theta, positions=rows)
    q8, qs = O.quant_q(qp)
    O.attention(q8, qs, k8, ks, v8t, vs, w.Nkv)
    dt = time.perf_counter() - t0
    return dt, 4.0 * len(hs) * len(rows) * w.Nkv * w.D


def blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:
        return os.cpu_count() or 1


def cpu_baseline_line(w, heads=(0, 1, 2, 3), q_tiles=tuple(range(8))):
    dt, flops = oracle_sample(w, heads, q_tiles)
    return {"value": flops / dt / 1e12, "unit": "TFLOP/s", "cores": blas_threads(), "kind": "oracle",
            "seconds": dt,
            "sample": (f"heads {list(heads)} x query tiles {list(q_tiles)} (128 rows each) against "
                       f"all {w.Nkv} keys, including prep/K-mean/quant of those heads; numpy "
                       "oracle, BLAS matmul multithreaded, elementwise single-threaded")}


# ------------------------------------------------------------------ reference arm
def run_reference(args):
    rank, world, _ = dist_env()
    if rank != 0:
        return 0
    from quantized_exact_attention_qattn_b200 import synth
    w = synth.make("canonical")
    times, flops = [], 0.0
    for i in range(args.warmup + args.steps):
        dt, fl = oracle_sample(w, heads=(i % w.Hq,), q_tiles=(i % 296,))
        if i >= args.warmup:
            times.append(dt)
            flops = fl
    ms = 1e3 * statistics.mean(times)
    val = flops / (ms / 1e3) / 1e12
    line = {"impl": "reference", "metric": METRIC, "value": val, "unit": "TFLOP/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64/f32 (numpy oracle)", "data": "synthetic",
            "config": dict(WORKLOAD),
            "cpu_baseline": {"value": val, "unit": "TFLOP/s", "cores": blas_threads(),
                             "kind": "oracle",
                             "sample": "per step: one head x one 128-row query tile against all "
                                       "37810 keys, with that head's prep/K-mean/quant"},
            "e2e": {"value": val, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------------ side workloads
def side_workloads(dev, reps: int = 20):
    """Attention-call times of the pages' other workloads (not the benchmark
    line's metric): the GQA prefill chunk with rotated int8 K (Nq1024 x Nkv32768,
    16/4 heads, D256) and the 729-key encoder batch (B32 N729 H16 D64), each on
    seeded device-generated inputs of the workload's shape, CUDA events, median."""
    import torch
    import quantized_exact_attention_qattn_b200 as qa
    out = {}
    g = torch.Generator(device=dev)
    g.manual_seed(7)
    for name, (B, Nq, Nkv, Hq, Hkv, D, had, rot) in {
            "gqa_chunk": (1, 1024, 32768, 16, 4, 256, True, 0),
            "encoder": (32, 729, 729, 16, 16, 64, False, 0)}.items():
        q = torch.randn((B, Nq, Hq, D), device=dev, generator=g).to(torch.bfloat16)
        k = torch.randn((B, Nkv, Hkv, D), device=dev, generator=g).to(torch.bfloat16)
        v = torch.randn((B, Nkv, Hkv, D), device=dev, generator=g).to(torch.bfloat16)
        pipe = qa.Pipeline(B, Nq, Nkv, Hq, Hkv, D, hadamard=had, device=dev)
        w = (1 + 0.1 * torch.randn(D, device=dev, generator=g)).to(torch.bfloat16)
        pipe.run(q, k, v, w, w, 1e-5, rot)
        for _ in range(3):
            pipe.run_fwd()
        ts = []
        for _ in range(reps):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            pipe.run_fwd()
            b.record()
            b.synchronize()
            ts.append(a.elapsed_time(b))
        pipe.check()
        ms = percentile(ts, 0.5)
        out[name] = {"fwd_ms": ms, "tflops": pipe.attn_ops / (ms / 1e3) / 1e12,
                     "shape": {"B": B, "Nq": Nq, "Nkv": Nkv, "Hq": Hq, "Hkv": Hkv, "D": D,
                               "rotated_int8_k": had}}
    return out


# ------------------------------------------------------------------ GPU arm
def run_gpu(args):
    import torch
    import quantized_exact_attention_qattn_b200 as qa
    from quantized_exact_attention_qattn_b200 import synth

    rank, world, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    dist = init_dist(world, "nccl")

    w = make_workload(args.config)
    import numpy as np
    if args.shard_heads and world > 1:
        # one problem split over the ranks by heads: each rank holds the column
        # slice of the inputs with its heads (no exchange is needed anywhere)
        (h0, h1), (k0, k1) = kv_shard(w.Hq, w.Hkv, world, rank)
        if w.qkv is not None:
            full = w.qkv.reshape(w.B, w.Nq, 3, w.Hq, w.D)
            w.qkv = np.ascontiguousarray(full[:, :, :, h0:h1]).reshape(w.B * w.Nq, -1)
            w.q = w.k = w.v = None
        else:
            w.q = np.ascontiguousarray(w.q[:, :, h0:h1])
            w.k = np.ascontiguousarray(w.k[:, :, k0:k1])
            w.v = np.ascontiguousarray(w.v[:, :, k0:k1])
        w.Hq, w.Hkv = h1 - h0, k1 - k0
    if w.qkv is not None:
        host_qkv = torch.from_numpy(w.qkv).view(torch.bfloat16).pin_memory()
    else:   # contiguous workloads: one pinned buffer holding q | k | v
        host_qkv = torch.from_numpy(np.concatenate([w.q.ravel(), w.k.ravel(), w.v.ravel()])
                                    ).view(torch.bfloat16).pin_memory()
    qkv = host_qkv.to(dev)
    if w.qkv is not None:
        view = qkv.view(w.B, w.Nq, 3, w.Hq, w.D)
        q, k, v = view[:, :, 0], view[:, :, 1], view[:, :, 2]
    else:
        nq, nk = w.q.size, w.k.size
        q = qkv[:nq].view(w.q.shape)
        k = qkv[nq:nq + nk].view(w.k.shape)
        v = qkv[nq + nk:].view(w.v.shape)
    qw = kw = None
    if w.q_weight is not None:
        qw = torch.from_numpy(w.q_weight).view(torch.bfloat16).to(dev)
        kw = torch.from_numpy(w.k_weight).view(torch.bfloat16).to(dev)
    pipe = qa.Pipeline(w.B, w.Nq, w.Nkv, w.Hq, w.Hkv, w.D, hadamard=w.hadamard,
                       fused=not w.hadamard, rotary_dim=w.rotary_dim, device=dev)
    stream = torch.cuda.current_stream(dev)
    flops = pipe.attn_ops

    def step(ev=None):
        if ev is not None:
            ev[0].record(stream)
        if w.hadamard:
            pipe.run_quant_hadamard(q, k, v)
        else:
            pipe.run_prep_quant(q, k, v, qw, kw, w.eps, w.theta)
        if ev is not None:
            ev[1].record(stream)
        pipe.run_fwd()
        if ev is not None:
            ev[2].record(stream)

    probe = {}
    if rank == 0 and not args.no_probe:
        with ClockSampler(local) as pclk:
            probe = {"i8": tc_probe(dev, 0), "e4m3": tc_probe(dev, 1)}
        probe["clocks"] = pclk.summary()

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    pipe.check()

    # ---- device-timed region
    fwd_events = [tuple(torch.cuda.Event(enable_timing=True) for _ in range(3))
                  for _ in range(args.steps)]
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        time.sleep(0.3)
        t_start.record(stream)
        for i in range(args.steps):
            step(fwd_events[i])
        t_end.record(stream)
        torch.cuda.synchronize()
    if dist:
        dist.barrier()
    pipe.check()
    ms_total = t_start.elapsed_time(t_end)
    ms_total = max_over_ranks(ms_total, dist, dev)
    ms_step = ms_total / args.steps
    fwd_all = [b.elapsed_time(c) for a, b, c in fwd_events]
    fwd_ms = statistics.mean(fwd_all)
    pq_ms = statistics.mean([a.elapsed_time(b) for a, b, c in fwd_events])
    value = sum_over_ranks(flops, dist, dev) / (ms_step / 1e3) / 1e12

    # ---- end-to-end: pinned host QKV in, host output back, every step, through
    # qattn_attention_host (chunks of KV heads overlap PCIe with compute)
    out_host = torch.empty(pipe.out.shape, dtype=torch.bfloat16).pin_memory()
    if w.qkv is not None:
        hview = host_qkv.view(w.B, w.Nq, 3, w.Hq, w.D)
        hq, hk, hv = hview[:, :, 0], hview[:, :, 1], hview[:, :, 2]
    else:
        nq, nk = w.q.size, w.k.size
        hq = host_qkv[:nq].view(w.q.shape)
        hk = host_qkv[nq:nq + nk].view(w.k.shape)
        hv = host_qkv[nq + nk:].view(w.v.shape)
    runner = None if args.no_e2e else qa.HostRunner(
        w.B, w.Nq, w.Nkv, w.Hq, w.Hkv, w.D, hadamard=w.hadamard,
        kv_heads_per_chunk=args.e2e_chunk, device=dev)

    def e2e_step():
        runner.run(hq, hk, hv, out_host, qw, kw, w.eps, w.rotary_dim, w.theta, stream=stream)

    e2e_ms = None
    if not args.no_e2e:
        for _ in range(max(1, args.warmup)):
            e2e_step()
        torch.cuda.synchronize()
        if dist:
            dist.barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(args.steps):
            e2e_step()
        e1.record(stream)
        torch.cuda.synchronize()
        e2e_ms = max_over_ranks(e0.elapsed_time(e1), dist, dev) / args.steps
        runner.check(stream)

    if rank == 0:
        peaks = {}
        try:
            with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
                peaks = json.load(f)
        except OSError:
            pass
        clocks = clk.summary()
        # burst figure when the attention kernel ran at the maximum SM clock (it does
        # not reach the power cap), the sustained one when the clock sagged
        at_max = (clocks.get("sm_mhz") and clocks.get("sm_max_mhz") and
                  clocks["sm_mhz"] >= 0.97 * clocks["sm_max_mhz"])
        if "bf16_tflops" in peaks and at_max:
            peak = peaks["bf16_tflops"] * NOMINAL_FP8_OVER_BF16
            peak_src = ("of measured: MEASURED_PEAKS bf16 burst x nominal fp8/bf16 ratio 2 "
                        "(SM clock at max during the timed region)")
        elif "bf16_tflops_sustained" in peaks:
            peak = peaks["bf16_tflops_sustained"] * NOMINAL_FP8_OVER_BF16
            peak_src = ("of measured: MEASURED_PEAKS bf16 sustained x nominal fp8/bf16 ratio 2 "
                        "(SM clock below max during the timed region)")
        else:
            peak = 1590.0 * NOMINAL_FP8_OVER_BF16
            peak_src = "of fallback: bf16 burst 1.59 PFLOP/s x nominal ratio 2"
        hbm = peaks.get("hbm_gbs", 6650.0)
        hbm_src = "of measured" if "hbm_gbs" in peaks else "of fallback"
        achieved = flops / (fwd_ms / 1e3) / 1e12
        pq_bytes = prep_quant_bytes(w)
        probe_line = None
        if probe:
            mhz = clocks.get("sm_mhz") or clocks.get("sm_max_mhz")
            i8_peak = 2.0 * probe["i8"]["macs_per_clk_per_sm"] * probe["i8"]["n_sm"] * mhz * 1e6 / 1e12
            probe_line = {
                "i8_tflops_event_timed": probe["i8"]["tflops"],
                "e4m3_tflops_event_timed": probe["e4m3"]["tflops"],
                "i8_macs_per_clk_per_sm": probe["i8"]["macs_per_clk_per_sm"],
                "e4m3_macs_per_clk_per_sm": probe["e4m3"]["macs_per_clk_per_sm"],
                "probe_clocks": probe["clocks"],
                "i8_peak_at_attention_clock": i8_peak,
                "frac_of_probe_peak": achieved / i8_peak,
                "kernel": "qattn_tc_probe: one CTA per SM, back-to-back M128 N256 K32 MMAs "
                          "from shared memory"}
        line = {
            "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
            "higher_is_better": True,
            "scaling": "strong" if (args.shard_heads and world > 1) else "weak",
            "vs_baseline": None,
            "dtype": "int8 QK / e4m3 PV (f32 accumulate), bf16 in/out", "data": "synthetic",
            "config": dict(workload_config(w),
                           parallelism=(f"one problem, heads split over {world} GPUs (no exchange)"
                                        if (args.shard_heads and world > 1) else
                                        f"{world} independent problems (one per GPU)")),
            "fwd_ms_per_call": fwd_ms,
            "fwd_ms_p10": percentile(fwd_all, 0.1),
            "fwd_ms_p90": percentile(fwd_all, 0.9),
            "fwd_tflops": achieved,
            "fwd_frac_of_spec_4500": achieved / SPEC_FP8_TFLOPS,
            "prep_quant_ms": pq_ms,
            "prep_quant": {"call": "qattn_quant_hadamard" if w.hadamard else "qattn_prep_quant",
                           "ms": pq_ms, "algorithmic_bytes": pq_bytes,
                           "gbs": pq_bytes / (pq_ms / 1e3) / 1e9,
                           "frac_of_hbm": pq_bytes / (pq_ms / 1e3) / 1e9 / hbm,
                           "hbm_gbs": hbm, "hbm_source": hbm_src},
            "tensor_probe": probe_line,
            "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                         "frac": achieved / peak,
                         "traffic": ATTN_TRAFFIC_BYTES if args.config == "canonical" else None,
                         "traffic_source": ATTN_TRAFFIC_SOURCE if args.config == "canonical" else None,
                         "kernel": "attn_fwd_kernel<%d,%d,%d>" % (w.D, {64: 3, 128: 2}.get(w.D, 1),
                                                                  1 if w.hadamard else 0),
                         "peak_source": peak_src,
                         "algorithmic_work": "4*B*H*N^2*D = %.4e ops per launch" % flops},
            "e2e": {"value": flops * world / (e2e_ms / 1e3) / 1e12 if e2e_ms else None,
                    "unit": "TFLOP/s", "ms_per_step": e2e_ms,
                    "call": "qattn_attention_host, %d KV heads per chunk" % (runner.chunk if runner else 0),
                    "h2d_bytes_per_step": host_qkv.numel() * 2,
                    "d2h_bytes_per_step": out_host.numel() * 2},
            # rope table (when R > 0), pass 1, finalize, pass 2, attention; rotated
            # path: V statistics (2), rotation + quant, V quant, attention
            "gpu_launches": (5 if w.hadamard else (5 if w.rotary_dim > 0 else 4)) * args.steps,
            "clocks": clocks,
        }
        if world == 1 and not args.no_cpu_baseline and args.config == "canonical":
            line["cpu_baseline"] = cpu_baseline_line(w)
        if world == 1 and args.config == "canonical" and not args.no_side:
            line["side_workloads"] = side_workloads(dev)
        print(json.dumps(line), flush=True)
    if dist:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-probe", action="store_true", help="skip the tensor-core peak probe")
    ap.add_argument("--no-side", action="store_true",
                    help="skip the side timings of the GQA-chunk and encoder attention calls")
    ap.add_argument("--shard-heads", action="store_true",
                    help="with N > 1 ranks: split one problem's heads over the ranks "
                         "(strong scaling) instead of one whole problem per rank")
    ap.add_argument("--e2e-chunk", type=int, default=None,
                    help="KV heads per chunk of the end-to-end call (default Hkv // 8)")
    ap.add_argument("--config", default="canonical",
                    choices=["canonical", "small", "mid", "encoder", "gqa_chunk", "profile16k"],
                    help="workload; only 'canonical' is the benchmark line, the others are "
                         "for profiling and checks")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.impl == "reference":
        return run_reference(args)
    return run_gpu(args)


if __name__ == "__main__":
    sys.exit(main())
