#!/usr/bin/env python
"""Throughput of the gated delta-rule chunked forward on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--workload NAME]

One step is one gdr_fwd_chunked call over the whole workload (every chunk's
UT/WY transform, the state scan, the outputs and the final state), on
synthetic seeded inputs already resident in HBM. The default workload is the
nanochat-scale GDN layer: B=8, T=2048, Hk=Hv=16, Dk=Dv=128, bf16 q/k/v/o,
fp32 scalar gates, beta and state, h0 ~ 0.02 N(0,1).

Prints one JSON line (rank 0). ``value`` is B*T*Hv head-tokens per second over
all ranks (each rank runs its own full workload: weak scaling, no data-path
collective), timed on the device with CUDA events, max over ranks. ``e2e`` is
the same metric through the public Python API with pinned host buffers, the
host<->device copies of every step's inputs and results inside the timed
region. ``roofline`` compares algorithmic HBM bytes per launch with the
measured HBM copy bandwidth. ``cpu_baseline`` times the fp64 CPU oracle on a
bounded sample of the same workload on this host's cores.

Other workloads (``--workload``): ``gva_gdn_bf16`` and ``kda_bf16`` (the same
step on the grouped-value and per-channel-gate shapes), ``decode_bf16`` (one
``gdr_decode_step`` over the batch per step), ``gdn_layer_bf16`` (three short
convolutions plus the forward with its q/k and output norms) and ``gdn_bwd_bf16``
(one ``gdr_bwd_chunked`` call per step, the tensor-core chunked backward, against
the measured tensor-core peak; the fp32 ``gdr_bwd`` is timed beside it). ``--T``
shortens a workload's sequences for profiling small cases.

``--impl reference`` times that oracle alone (the reference arm): each step is
a bounded sample of the workload on the host cores.
"""
import argparse
import hashlib
import json
import math
import os
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "gated-delta fwd tokens/s (B·T·Hv per sec) bf16 d=128; % of roofline"
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0
L2_BYTES = 126 * 2 ** 20


def parse_args(argv=None):
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=20)
    p.add_argument("--warmup", type=int, default=5)
    p.add_argument("--impl", choices=["ours", "reference"], default="ours")
    p.add_argument("--workload", default="gdn_bf16")
    p.add_argument("--no-e2e", action="store_true")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--T", type=int, default=None,
                   help="override the workload's sequence length (small cases for profiling)")
    p.add_argument("--B", type=int, default=None,
                   help="override the workload's batch size (small cases for profiling)")
    a = p.parse_args(argv)
    a.warmup = max(a.warmup, 3)
    return a


# ----------------------------------------------------------------------------- accounting
def algorithmic_bytes(w):
    """HBM bytes the method must move per call: q, k, v, o, g, beta, h0 and hT. For the
    decode workload, per step: the state read and written once, and one token's inputs
    and output for every (batch row, value head)."""
    es = 2 if w.dtype == "bf16" else 4
    if w.layer:
        return layer_conv_bytes(w) + algorithmic_bytes(w.with_(layer=False)) + w.B * w.T * w.Hv * w.Dv * es
    if w.decode:
        tok = w.B * (2 * w.Hk * w.Dk * es + 2 * w.Hv * w.Dv * es
                     + w.Hv * (w.Dk if w.gate == "channel" else 1) * 4 + w.Hv * 4)
        return 2 * w.B * w.Hv * w.Dk * w.Dv * 4 + tok
    qk = 2 * w.B * w.T * w.Hk * w.Dk * es
    vo = 2 * w.B * w.T * w.Hv * w.Dv * es
    g = w.B * w.T * w.Hv * (w.Dk if w.gate == "channel" else 1) * 4
    beta = w.B * w.T * w.Hv * 4
    states = (2 if w.h0_std > 0 else 1) * w.B * w.Hv * w.Dk * w.Dv * 4
    return qk + vo + g + beta + states


def layer_conv_bytes(w):
    """The short convolution reads the q/k/v projections once and writes them once."""
    es = 2 if w.dtype == "bf16" else 4
    return 2 * w.B * w.T * (2 * w.Hk * w.Dk + w.Hv * w.Dv) * es


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def measured_tensor_peak():
    """Dense bf16 tensor-core peak (TFLOP/s) measured by a cuBLAS GEMM burst on this machine's B200s;
    fp16 runs at the same nominal rate."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["bf16_tflops"]), "measured (bf16 cuBLAS burst; fp16 at the same nominal rate)"
    except Exception:
        return FALLBACK_BF16_TFLOPS, "fallback"


# The sources each captured kernel is built from: a recorded DRAM figure stands only while
# these files are unchanged.
KERNEL_SOURCES = {
    "tc_fwd_kernel": ("chunk_tc.cu", "tc_util.cuh", "mma_util.cuh", "common.cuh", "kernels.h"),
    "fused_fwd_kernel": ("chunk_mma.cu", "mma_util.cuh", "common.cuh", "kernels.h"),
    "bwd_kernel": ("bwd.cu", "common.cuh", "kernels.h"),
    "decode_kernel": ("decode.cu", "common.cuh", "kernels.h"),
    "bwdc_tc_kernel": ("bwd_chunk.cu", "mma_util.cuh", "tc_util.cuh", "common.cuh", "kernels.h"),
    # the chunked backward's step: its forward pass, scan and chunk kernels together
    "bwdc_step": ("bwd_chunk.cu", "chunk_tc.cu", "mma_util.cuh", "tc_util.cuh", "common.cuh", "kernels.h"),
}


def kernel_sources_sha(kernel=None):
    csrc = os.path.join(ROOT, "gated_delta_rule_68_b200", "csrc")
    names = sorted(n for n in os.listdir(csrc) if n.endswith((".cu", ".cuh", ".h")))
    if kernel is not None:
        names = sorted(KERNEL_SOURCES[kernel.split("<")[0]])
    h = hashlib.sha256()
    for n in names:
        h.update(n.encode())
        with open(os.path.join(csrc, n), "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def recorded_traffic(workload):
    """DRAM bytes per launch from a committed ncu capture, if the kernels are unchanged since."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            d = json.load(f)[workload]
    except Exception:
        return None, None
    if d.get("kernel_sources_sha256") != kernel_sources_sha(d.get("kernel")):
        return None, d.get("kernel")
    return float(d["dram_bytes_per_launch"]), d.get("kernel")


# ----------------------------------------------------------------------------- ranks
def rank_workload(w, rank):
    """Each rank runs the whole workload on its own inputs: the seed is offset by the rank."""
    return w.with_(seed=w.seed + rank)


def max_over_ranks(x, device=None):
    """The largest of every rank's value (the step time of the whole job)."""
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_tokens_per_s(units_per_rank, world, ms_max):
    """Whole-job throughput: the units all ranks processed over the slowest rank's time."""
    return world * units_per_rank / (ms_max / 1e3)


# ----------------------------------------------------------------------------- clocks
class ClockSampler:
    """Samples SM clock and clock-event reasons with NVML every few ms while running."""

    REASONS = {
        "gpu_idle": 0x1, "applications_clocks_setting": 0x2, "sw_power_cap": 0x4,
        "hw_slowdown": 0x8, "sync_boost": 0x10, "sw_thermal_slowdown": 0x20,
        "hw_thermal_slowdown": 0x40, "hw_power_brake_slowdown": 0x80,
    }

    def __init__(self, device_index, period_s=0.005):
        self.samples, self.reasons = [], set()
        self.ok = False
        self.period = period_s
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nvml = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception as e:  # NVML unavailable: report that instead of clocks
            self.err = str(e)
        self._stop = threading.Event()

    def _run(self):
        nv = self.nvml
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
                r = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                for name, bit in self.REASONS.items():
                    if r & bit:
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.ok:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *exc):
        if self.ok:
            self._stop.set()
            self.t.join()

    def summary(self):
        if not self.ok:
            return {"error": getattr(self, "err", "nvml unavailable")}
        s = sorted(self.samples)
        med = s[len(s) // 2] if s else None
        return {"sm_mhz": med, "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons - {"gpu_idle"}),
                "samples": len(s)}


# ----------------------------------------------------------------------------- CPU oracle
def cpu_oracle_sample(w, target_s=12.0, seed_rank=0):
    """Time the fp64 oracle on a bounded sample of the workload: whole sequences of some
    (b, h) units, chosen so the run takes about target_s seconds on this host."""
    import oracle
    from gated_delta_rule_68_b200.workloads import make_inputs

    small = w.with_(B=1, Hk=1, Hv=1)
    inp = make_inputs(small.with_(seed=w.seed + seed_rank), "cpu")
    cores = oracle.threads_used(0, 1 << 30)
    t0 = time.perf_counter()
    oracle.recurrent(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], inp["h0"], nthreads=1)
    t_unit = time.perf_counter() - t0
    units = max(cores, min(w.B * w.Hv, int(target_s * cores / max(t_unit, 1e-6))))
    units = min(units, w.B * w.Hv)
    sample = w.with_(B=units, Hk=1, Hv=1)
    inp = make_inputs(sample, "cpu")
    q, k, v, g, beta, h0 = (inp[n] for n in ("q", "k", "v", "g", "beta", "h0"))
    qd, kd, vd, gd, bd = (x.double().numpy() for x in (q, k, v, g, beta))
    hd = None if h0 is None else h0.double().numpy()
    reps, dt = 0, 0.0
    while reps == 0 or (dt < target_s and reps < 1000):
        t0 = time.perf_counter()
        oracle.recurrent(qd, kd, vd, gd, bd, hd, nthreads=0)
        dt += time.perf_counter() - t0
        reps += 1
    return {
        "value": reps * units * w.T / dt, "unit": "tokens/s", "cores": oracle.threads_used(0, units),
        "kind": "oracle",
        "sample": f"{units} whole (batch row, value head) sequences of T={w.T}, Dk=Dv={w.Dk}, "
                  f"{w.gate} gate, fp64 token recurrence, run {reps} times; {dt:.1f} s",
        "seconds": dt,
    }


def layer_oracle_unit(inp, b, h):
    """The oracle composition for one (b, h) unit of the layer: the short convolution of the
    unit's q, k and v channels, L2 norms of q and k, the fp64 recurrence, the gated RMSNorm."""
    import oracle
    from oracle import prologue
    D = inp["z"].shape[-1]
    Hk, Hv = inp["xq"].shape[-1] // D, inp["z"].shape[2]
    hk = h // (Hv // Hk)
    sl = lambda n, hh: inp[n][b:b + 1, :, hh * D:(hh + 1) * D]
    wsl = lambda n, hh: inp[n][hh * D:(hh + 1) * D]
    q, _ = prologue.causal_conv_silu(sl("xq", hk), wsl("wq", hk))
    k, _ = prologue.causal_conv_silu(sl("xk", hk), wsl("wk", hk))
    v, _ = prologue.causal_conv_silu(sl("xv", h), wsl("wv", h))
    q, k = prologue.l2norm(q), prologue.l2norm(k)
    h0 = None if inp["h0"] is None else inp["h0"][b:b + 1, h:h + 1]
    o, hT = oracle.recurrent(q[:, :, None], k[:, :, None], v[:, :, None], inp["g"][b:b + 1, :, h:h + 1],
                             inp["beta"][b:b + 1, :, h:h + 1], h0, nthreads=1)
    return prologue.rmsnorm_gated(o[0, :, 0], inp["z"][b, :, h], inp["nw"]), hT


def layer_cpu_sample(w, target_s=12.0, seed_rank=0):
    """Time the oracle composition on whole sequences of (b, h) units for about target_s."""
    from gated_delta_rule_68_b200.workloads import make_layer_inputs
    inp = make_layer_inputs(w.with_(seed=w.seed + seed_rank), "cpu")
    units, dt = 0, 0.0
    while units == 0 or (dt < target_s and units < w.B * w.Hv):
        b, h = divmod(units, w.Hv)
        t0 = time.perf_counter()
        layer_oracle_unit(inp, b, h)
        dt += time.perf_counter() - t0
        units += 1
    return {"value": units * w.T / dt, "unit": "tokens/s", "cores": 1, "kind": "oracle",
            "sample": f"{units} whole (batch row, value head) sequences of T={w.T}: conv + SiLU, L2 norms, "
                      f"fp64 token recurrence, gated RMSNorm, one thread; {dt:.1f} s",
            "seconds": dt}


def run_layer_bench(args, w, wr, rank, world, local, dev):
    """One step = the layer's recurrence block: three short convolutions (+ SiLU) of the q/k/v
    projections, then the fused chunked forward with in-kernel q/k L2 norms and the gated
    output RMSNorm."""
    import torch
    import torch.distributed as dist
    import gated_delta_rule_68_b200 as gdr
    from gated_delta_rule_68_b200.workloads import make_layer_inputs

    inp_cpu = make_layer_inputs(wr, "cpu")
    inp = {n: (None if t is None else t.to(dev)) for n, t in inp_cpu.items()}
    yq, yk, yv = (torch.empty_like(inp[n]) for n in ("xq", "xk", "xv"))
    o = torch.empty((w.B, w.T, w.Hv, w.Dv), dtype=w.torch_dtype, device=dev)
    hT = torch.empty((w.B, w.Hv, w.Dk, w.Dv), dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)
    shp_k, shp_v = (w.B, w.T, w.Hk, w.Dk), (w.B, w.T, w.Hv, w.Dv)

    def convs(x):
        gdr.gdr_causal_conv_silu(x["xq"], x["wq"], y=yq, stream=stream)
        gdr.gdr_causal_conv_silu(x["xk"], x["wk"], y=yk, stream=stream)
        gdr.gdr_causal_conv_silu(x["xv"], x["wv"], y=yv, stream=stream)

    def layer(x):
        convs(x)
        gdr.gdr_fwd_chunked_norm(yq.view(shp_k), yk.view(shp_k), yv.view(shp_v), x["g"], x["beta"], x["h0"],
                                 qk_l2norm=True, z=x["z"], norm_weight=x["nw"], o=o, hT=hT, stream=stream)

    def barrier():
        if world > 1:
            dist.barrier()

    def timed(fn, steps):
        barrier()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(steps):
            fn()
        e1.record(stream)
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / steps

    for _ in range(args.warmup):
        layer(inp)
    torch.cuda.synchronize()
    n0 = gdr.gdr_kernel_launches()
    with ClockSampler(local) as clk:
        ms = timed(lambda: layer(inp), args.steps)
    launches = gdr.gdr_kernel_launches() - n0
    ms_max = max_over_ranks(ms, dev)
    conv_ms = timed(lambda: convs(inp), args.steps)
    fwd_ms = ms - conv_ms

    e2e = None
    if not args.no_e2e:
        host = {n: (None if x is None else x.pin_memory()) for n, x in inp_cpu.items()}
        dbuf = {n: (None if x is None else torch.empty_like(x, device=dev)) for n, x in inp_cpu.items()}
        o_h = torch.empty(o.shape, dtype=o.dtype).pin_memory()
        hT_h = torch.empty(hT.shape, dtype=hT.dtype).pin_memory()
        h2d = sum(x.numel() * x.element_size() for x in host.values() if x is not None)
        d2h = o_h.numel() * o_h.element_size() + hT_h.numel() * hT_h.element_size()

        def e2e_step():
            for n, x in host.items():
                if x is not None:
                    dbuf[n].copy_(x, non_blocking=True)
            layer(dbuf)
            o_h.copy_(o, non_blocking=True)
            hT_h.copy_(hT, non_blocking=True)

        e2e_step()
        e2e_steps = max(3, min(args.steps, 10))
        te = max_over_ranks(timed(e2e_step, e2e_steps), dev)
        e2e = {"value": job_tokens_per_s(w.head_tokens, world, te), "unit": "tokens/s",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": e2e_steps, "ms_per_step": te}

    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return 0
    peak, peak_kind = measured_peaks()
    alg, conv_alg = algorithmic_bytes(w), layer_conv_bytes(w)
    fwd_alg = alg - conv_alg
    traffic, traffic_kernel = recorded_traffic(w.name)
    cpu = layer_cpu_sample(w) if world == 1 and not args.no_cpu_baseline else None
    line = {
        "metric": METRIC, "value": job_tokens_per_s(w.head_tokens, world, ms_max), "unit": "tokens/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_max,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": w.dtype,
        "data": "synthetic (seeded CPU generator; q/k/v projections N(0,1), conv taps 0.5 N(0,1); "
                f"g logsigmoid(N({w.g_mu:g},1)); beta sigmoid(N(0,1)); h0 0.02 N(0,1); z N(0,1))",
        "config": workload_config(w, world),
        "roofline": {"bound": "hbm", "achieved": fwd_alg / (fwd_ms / 1e3) / 1e9, "peak": peak, "unit": "GB/s",
                     "frac": fwd_alg / (fwd_ms / 1e3) / 1e9 / peak, "peak_source": peak_kind,
                     "algorithmic_bytes_per_launch": fwd_alg, "traffic": traffic, "traffic_kernel": traffic_kernel,
                     "kernel": "gdr_fwd_chunked_norm (q/k L2 norm and gated output norm fused)"},
        "step_roofline": {"achieved": alg / (ms / 1e3) / 1e9, "frac": alg / (ms / 1e3) / 1e9 / peak,
                          "algorithmic_bytes": alg},
        "conv": {"ms_per_step": conv_ms, "launches_per_step": 3, "algorithmic_bytes": conv_alg,
                 "achieved_gbs": conv_alg / (conv_ms / 1e3) / 1e9,
                 "frac": conv_alg / (conv_ms / 1e3) / 1e9 / peak},
        "cpu_baseline": cpu, "e2e": e2e, "gpu_launches": launches, "launches_per_step": launches / args.steps,
        "clocks": clk.summary(),
    }
    print(json.dumps(line), flush=True)
    return 0


def run_reference(args, w, rank, world):
    if rank != 0:
        return 0
    import oracle
    from gated_delta_rule_68_b200.workloads import make_inputs

    if w.layer:
        return run_layer_reference(args, w, world)
    if w.bwd:
        return run_bwd_reference(args, w, world)
    if w.decode:
        return run_decode_reference(args, w, world)
    cores = oracle.threads_used(0, 1 << 30)
    units = max(cores, 8)
    sample = w.with_(B=units, Hk=1, Hv=1)
    inp = make_inputs(sample, "cpu")
    arrs = [None if inp[n] is None else inp[n].double().numpy()
            for n in ("q", "k", "v", "g", "beta", "h0")]
    times = []
    for it in range(args.warmup + args.steps):
        t0 = time.perf_counter()
        oracle.recurrent(*arrs, nthreads=0)
        dt = time.perf_counter() - t0
        if it >= args.warmup:
            times.append(dt)
    per_step = sum(times) / len(times)
    value = units * w.T / per_step
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": per_step * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded, same recipe as the GPU arm)",
        "config": workload_config(w, world),
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": oracle.threads_used(0, units),
                         "kind": "oracle",
                         "sample": f"each step: {units} whole (batch row, value head) sequences of "
                                   f"T={w.T} of the workload, fp64 token recurrence"},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def run_layer_reference(args, w, world):
    """The reference arm on the layer workload: each step is the oracle composition on two whole
    (b, h) sequences, on one host core."""
    from gated_delta_rule_68_b200.workloads import make_layer_inputs
    inp = make_layer_inputs(w, "cpu")
    units = 2
    times = []
    for it in range(args.warmup + args.steps):
        t0 = time.perf_counter()
        for u in range(units):
            layer_oracle_unit(inp, *divmod(u, w.Hv))
        if it >= args.warmup:
            times.append(time.perf_counter() - t0)
    per_step = sum(times) / len(times)
    value = units * w.T / per_step
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": per_step * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded, same recipe as the GPU arm)", "config": workload_config(w, world),
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": 1, "kind": "oracle",
                         "sample": f"each step: {units} whole (batch row, value head) sequences of T={w.T}: "
                                   "conv + SiLU, L2 norms, fp64 token recurrence, gated RMSNorm"},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ----------------------------------------------------------------------------- backward
BWD_METRIC = "gated-delta bwd tokens/s (B·T·Hv per sec) bf16 d=128; % of roofline"


def bwd_bytes(w):
    """HBM bytes the backward must move per call: q, k, v, do, g, beta, h0 and dhT read once;
    dq, dk, dv, dg, dbeta and dh0 (fp32) written once."""
    es = 2 if w.dtype == "bf16" else 4
    gw = w.Dk if w.gate == "channel" else 1
    ins = 2 * w.B * w.T * w.Hk * w.Dk * es + 2 * w.B * w.T * w.Hv * w.Dv * es + w.B * w.T * w.Hv * (gw + 1) * 4
    outs = 2 * w.B * w.T * w.Hk * w.Dk * 4 + w.B * w.T * w.Hv * (w.Dv + gw + 1) * 4
    states = 3 * w.B * w.Hv * w.Dk * w.Dv * 4
    return ins + outs + states


def bwd_flops(w):
    """fp32 flops per call of the token-level backward: per (batch row, value head, token) and
    state element, 5 to rebuild the decayed state and the delta step (decay, k-projection,
    rank-one update) and 15 for the adjoint (the q do^T and k dp^T rank-one terms, the
    k-projection of dS, dq, the two dk terms, the gate's row sums and the decay of dS)."""
    return 20 * w.B * w.T * w.Hv * w.Dk * w.Dv


def bwdc_flops(w):
    """Tensor-core flops per call of the chunked backward, per (unit, 64-token chunk): the
    forward pass's products (Gram [K; Q] K^T, W and U, R, Qh, Uh, P and the state batch),
    the reverse scan's dS^T P and dO^T Qh, and the chunk kernel's products (Grams, W, U, U', dU',
    dM, dQ, dK3, dW, T^T dU', T^T dW, dT, T^T dT T^T, the dK terms: 26.2 MFLOP, 6400 tiles of
    16 x 8 x 16). Rows and blocks that the tensor-core shapes compute beyond these are not counted."""
    fwd = 5 * 2 * 128 * 64 * 128 + 2 * 128 * 64 * 64 + 2 * 128 * 128 * 128 + 2 * 128 * 64 * 128
    scan = 2 * 128 * 128 * 128 + 2 * 128 * 128 * 64
    chunk = 6400 * 2 * 16 * 8 * 16
    return w.B * w.Hv * ((w.T + 63) // 64) * (fwd + scan + chunk)


def alu_peak_tflops(sm_mhz):
    """fp32 FMA peak of the CUDA cores: 148 SMs x 128 lanes x 2 flops per clock."""
    return 148 * 128 * 2 * sm_mhz * 1e6 / 1e12


def bwd_cpu_sample(w, target_s=12.0):
    """Time the fp64 oracle backward on whole (b, h) sequences of the workload (Hk = Hv = 1 units)."""
    import oracle
    from gated_delta_rule_68_b200.workloads import make_inputs, make_upstream
    cores = oracle.threads_used(0, 1 << 30)
    one = w.with_(B=1, Hk=1, Hv=1)
    inp, up = make_inputs(one, "cpu"), make_upstream(one, "cpu")
    t0 = time.perf_counter()
    oracle.backward(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], inp["h0"], up["do"], up["dhT"],
                    nthreads=1)
    t_unit = time.perf_counter() - t0
    units = max(1, min(w.B * w.Hv, int(target_s * cores / max(t_unit, 1e-6))))
    sample = w.with_(B=units, Hk=1, Hv=1)
    inp, up = make_inputs(sample, "cpu"), make_upstream(sample, "cpu")
    t0 = time.perf_counter()
    oracle.backward(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], inp["h0"], up["do"], up["dhT"],
                    nthreads=0)
    dt = time.perf_counter() - t0
    return {"value": units * w.T / dt, "unit": "tokens/s", "cores": oracle.threads_used(0, units),
            "kind": "oracle",
            "sample": f"{units} whole (batch row, value head) sequences of T={w.T}, Dk=Dv={w.Dk}: fp64 token "
                      f"recurrence forward and its adjoint; {dt:.1f} s", "seconds": dt}


def run_bwd_bench(args, w, wr, rank, world, local, dev):
    """One step = one backward call over the whole workload, every gradient written: the
    tensor-core chunked backward (gdr_bwd_chunked: forward pass storing the chunk maps, reverse
    scan of the state gradient, per-chunk gradients) for the scalar gate with bf16 inputs and
    d = 128, else the fp32 token-level gdr_bwd (checkpointing forward pass and reverse sweep).
    The chunked line also times the fp32 path on the same inputs, outside the timed region."""
    import torch
    import torch.distributed as dist
    import gated_delta_rule_68_b200 as gdr
    from gated_delta_rule_68_b200.workloads import make_inputs, make_upstream

    inp_cpu = make_inputs(wr, "cpu")
    inp_cpu.update(make_upstream(wr, "cpu"))
    inp = {n: (None if t is None else t.to(dev)) for n, t in inp_cpu.items()}
    f32 = dict(dtype=torch.float32, device=dev)
    out = {"dq": torch.empty(inp["q"].shape, **f32), "dk": torch.empty(inp["k"].shape, **f32),
           "dv": torch.empty(inp["v"].shape, **f32), "dg": torch.empty(inp["g"].shape, **f32),
           "dbeta": torch.empty(inp["beta"].shape, **f32), "dh0": torch.empty((w.B, w.Hv, w.Dk, w.Dv), **f32)}
    dt = gdr.GDR_BF16 if w.dtype == "bf16" else gdr.GDR_FP32
    chunked = w.dtype == "bf16" and w.gate == "scalar" and w.Dk == 128 and w.Dv == 128
    ws_size = gdr.gdr_bwd_chunked_workspace_size if chunked else gdr.gdr_bwd_workspace_size
    need = ws_size(w.B, w.T, w.Hk, w.Hv, w.Dk, w.Dv, w.gate_mode, dt)
    ws = torch.empty(max(need, 1), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    bwd_fn = gdr.gdr_bwd_chunked if chunked else gdr.gdr_bwd

    def step(x):
        bwd_fn(x["q"], x["k"], x["v"], x["g"], x["beta"], x["h0"], x["do"], x["dhT"], workspace=ws,
               stream=stream, out=out)

    def barrier():
        if world > 1:
            dist.barrier()

    for _ in range(args.warmup):
        step(inp)
    torch.cuda.synchronize()
    barrier()
    torch.cuda.synchronize()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    n0 = gdr.gdr_kernel_launches()
    with ClockSampler(local) as clk:
        ev0.record(stream)
        for _ in range(args.steps):
            step(inp)
        ev1.record(stream)
        torch.cuda.synchronize()
    launches = gdr.gdr_kernel_launches() - n0
    barrier()
    ms = ev0.elapsed_time(ev1) / args.steps
    ms_max = max_over_ranks(ms, dev)

    fp32_path = None
    if chunked:   # the fp32 token-level path on the same inputs, for comparison (not the timed region)
        need32 = gdr.gdr_bwd_workspace_size(w.B, w.T, w.Hk, w.Hv, w.Dk, w.Dv, w.gate_mode, dt)
        ws32 = torch.empty(max(need32, 1), dtype=torch.uint8, device=dev)
        out32 = {n: torch.empty_like(t) for n, t in out.items()}

        def step32():
            gdr.gdr_bwd(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], inp["h0"], inp["do"], inp["dhT"],
                        workspace=ws32, stream=stream, out=out32)

        step32()
        torch.cuda.synchronize()
        barrier()
        f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        f0.record(stream)
        for _ in range(3):
            step32()
        f1.record(stream)
        torch.cuda.synchronize()
        fp32_path = {"ms_per_step": max_over_ranks(f0.elapsed_time(f1) / 3, dev), "steps": 3,
                     "kernel": "gdr_bwd (bwd_ckpt_kernel + bwd_kernel, fp32)"}
        del ws32, out32

    e2e = None
    if not args.no_e2e:
        host = {n: (None if x is None else x.pin_memory()) for n, x in inp_cpu.items()}
        dbuf = {n: (None if x is None else torch.empty_like(x, device=dev)) for n, x in inp_cpu.items()}
        out_h = {n: torch.empty(t.shape, dtype=t.dtype).pin_memory() for n, t in out.items()}
        h2d = sum(x.numel() * x.element_size() for x in host.values() if x is not None)
        d2h = sum(x.numel() * x.element_size() for x in out_h.values())
        e2e_steps = max(3, min(args.steps, 5))

        def e2e_step():
            for n, x in host.items():
                if x is not None:
                    dbuf[n].copy_(x, non_blocking=True)
            step(dbuf)
            for n, x in out_h.items():
                x.copy_(out[n], non_blocking=True)

        e2e_step()
        torch.cuda.synchronize()
        barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(e2e_steps):
            e2e_step()
        e1.record(stream)
        torch.cuda.synchronize()
        te = max_over_ranks(e0.elapsed_time(e1) / e2e_steps, dev)
        e2e = {"value": job_tokens_per_s(w.head_tokens, world, te), "unit": "tokens/s",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": e2e_steps, "ms_per_step": te}

    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return 0
    clocks = clk.summary()
    peak_mhz = clocks.get("sm_max_mhz") or 1965
    hbm, hbm_kind = measured_peaks()
    alg = bwd_bytes(w)
    traffic, traffic_kernel = recorded_traffic(w.name)
    cpu = bwd_cpu_sample(w) if world == 1 and not args.no_cpu_baseline else None
    if chunked:
        # tensor-bound at the measured dense bf16 peak (fp16 runs at the same rate): the products'
        # time there is above the HBM time of the backward's algorithmic bytes
        flops = bwdc_flops(w)
        tpk, tkind = measured_tensor_peak()
        achieved = flops / (ms / 1e3) / 1e12
        roofline = {"bound": "tensor", "achieved": achieved, "peak": tpk, "unit": "TFLOP/s",
                    "frac": achieved / tpk, "peak_source": tkind, "algorithmic_flops_per_launch": flops,
                    "traffic": traffic, "traffic_kernel": traffic_kernel,
                    "kernel": "gdr_bwd_chunked step (tc_fwd_kernel storing the chunk maps + bwdc_scan_kernel "
                              "+ bwdc_tc_kernel)"}
    else:
        peak = alu_peak_tflops(peak_mhz)
        flops = bwd_flops(w)
        achieved = flops / (ms / 1e3) / 1e12
        roofline = {"bound": "alu", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                    "frac": achieved / peak,
                    "peak_source": f"derived: 148 SMs x 128 fp32 lanes x 2 x {peak_mhz} MHz",
                    "algorithmic_flops_per_launch": flops, "traffic": traffic, "traffic_kernel": traffic_kernel,
                    "kernel": "gdr_bwd step (bwd_ckpt_kernel + bwd_kernel)"}
    line = {
        "metric": BWD_METRIC, "value": job_tokens_per_s(w.head_tokens, world, ms_max), "unit": "tokens/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_max,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f16" if chunked else "f32",
        "data": "synthetic (seeded CPU generator; inputs as the gdn_bf16 recipe; do N(0,1) bf16, "
                "dhT 0.1 N(0,1) fp32)",
        "config": workload_config(w, world),
        "roofline": roofline, "fp32_token_path": fp32_path,
        "hbm_roofline": {"algorithmic_bytes": alg, "achieved": alg / (ms / 1e3) / 1e9, "peak": hbm,
                         "frac": alg / (ms / 1e3) / 1e9 / hbm, "peak_source": hbm_kind},
        "cpu_baseline": cpu, "e2e": e2e, "gpu_launches": launches, "launches_per_step": launches / args.steps,
        "clocks": clocks,
    }
    print(json.dumps(line), flush=True)
    return 0


def run_bwd_reference(args, w, world):
    """The reference arm on the backward workload: each step is the fp64 oracle backward on
    whole (b, h) sequences, on the host cores."""
    import oracle
    from gated_delta_rule_68_b200.workloads import make_inputs, make_upstream
    units = max(oracle.threads_used(0, 1 << 30), 4)
    sample = w.with_(B=units, Hk=1, Hv=1)
    inp, up = make_inputs(sample, "cpu"), make_upstream(sample, "cpu")
    times = []
    for it in range(args.warmup + args.steps):
        t0 = time.perf_counter()
        oracle.backward(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], inp["h0"], up["do"], up["dhT"],
                        nthreads=0)
        if it >= args.warmup:
            times.append(time.perf_counter() - t0)
    per_step = sum(times) / len(times)
    value = units * w.T / per_step
    line = {
        "impl": "reference", "metric": BWD_METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": per_step * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded, same recipe as the GPU arm)", "config": workload_config(w, world),
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": oracle.threads_used(0, units),
                         "kind": "oracle",
                         "sample": f"each step: {units} whole (batch row, value head) sequences of T={w.T}, "
                                   "fp64 forward and adjoint"},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def workload_config(w, world):
    ab = bwd_bytes(w) if w.bwd else algorithmic_bytes(w)
    return {"workload": w.name, "B": w.B, "T": w.T, "Hk": w.Hk, "Hv": w.Hv, "Dk": w.Dk, "Dv": w.Dv,
            "gate": w.gate, "chunk": 64, "global_batch": w.B * world,
            "parallelism": f"dp{world} (independent batch shards, no collective)",
            "l2": ("inputs exceed L2, no flush" if ab > L2_BYTES else "L2 flushed between steps")}


# ----------------------------------------------------------------------------- decode
def decode_oracle_sample(w, target_s=12.0):
    """Time the fp64 oracle's decode steps on a bounded sample: `units` (batch row, value
    head) states stepped through `steps` tokens, chosen to take about target_s seconds."""
    import oracle
    from gated_delta_rule_68_b200.workloads import make_inputs
    cores = oracle.threads_used(0, 1 << 30)
    units, steps = max(cores, 8), 8
    sample = w.with_(B=units, Hk=1, Hv=1, T=steps)
    inp = make_inputs(sample, "cpu")
    arrs = [inp[n].double().numpy() for n in ("q", "k", "v", "g", "beta", "h0")]
    reps, dt = 0, 0.0
    while reps == 0 or (dt < target_s and reps < 1000):
        t0 = time.perf_counter()
        oracle.decode_steps(*arrs)
        dt += time.perf_counter() - t0
        reps += 1
    return {"value": reps * units * steps / dt, "unit": "tokens/s", "cores": oracle.threads_used(0, units),
            "kind": "oracle", "seconds": dt,
            "sample": f"{units} (batch row, value head) states of Dk=Dv={w.Dk} through {steps} decode steps, "
                      f"fp64, run {reps} times; {dt:.1f} s"}


def run_decode_reference(args, w, world):
    """The reference arm on the decode workload: each step is one fp64 decode step of a sample
    of (batch row, value head) states on the host cores."""
    import oracle
    from gated_delta_rule_68_b200.workloads import make_inputs
    units = max(oracle.threads_used(0, 1 << 30), 8)
    sample = w.with_(B=units, Hk=1, Hv=1, T=args.warmup + args.steps)
    inp = make_inputs(sample, "cpu")
    q, k, v, g, beta = (inp[n].double().numpy() for n in ("q", "k", "v", "g", "beta"))
    S = inp["h0"].double().numpy()
    times = []
    for it in range(args.warmup + args.steps):
        t0 = time.perf_counter()
        _, S = oracle.decode_steps(q[it:it + 1], k[it:it + 1], v[it:it + 1], g[it:it + 1], beta[it:it + 1], S)
        if it >= args.warmup:
            times.append(time.perf_counter() - t0)
    per_step = sum(times) / len(times)
    value = units / per_step
    metric = "gated-delta decode tokens/s (B·Hv per sec per step) bf16 d=128; % of roofline"
    line = {
        "impl": "reference", "metric": metric, "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": per_step * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded, same recipe as the GPU arm)", "config": workload_config(w, world),
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": oracle.threads_used(0, units),
                         "kind": "oracle",
                         "sample": f"each step: one fp64 decode step of {units} (batch row, value head) states"},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def run_decode_bench(args, w, wr, rank, world, local, dev):
    """One step = one gdr_decode_step over the whole batch: every (batch row, value head)
    state is read and written once. Each step takes the next pre-generated token."""
    import torch
    import torch.distributed as dist
    import gated_delta_rule_68_b200 as gdr
    from gated_delta_rule_68_b200.workloads import make_inputs

    n_tok = args.warmup + args.steps
    inp_cpu = make_inputs(wr.with_(T=n_tok), "cpu")
    inp = {n: t.to(dev) for n, t in inp_cpu.items()}
    state = inp["h0"].clone()
    o = torch.empty((w.B, w.Hv, w.Dv), dtype=w.torch_dtype, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step(s):
        gdr.gdr_decode_step(inp["q"][s], inp["k"][s], inp["v"][s], inp["g"][s], inp["beta"][s], state, o=o,
                            stream=stream)

    def barrier():
        if world > 1:
            dist.barrier()

    for s in range(args.warmup):
        step(s)
    torch.cuda.synchronize()
    barrier()
    torch.cuda.synchronize()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    n0 = gdr.gdr_kernel_launches()
    with ClockSampler(local) as clk:
        ev0.record(stream)
        for s in range(args.warmup, n_tok):
            step(s)
        ev1.record(stream)
        torch.cuda.synchronize()
    launches = gdr.gdr_kernel_launches() - n0
    barrier()
    ms = ev0.elapsed_time(ev1) / args.steps
    ms_max = max_over_ranks(ms, dev)

    # The same steps captured in a CUDA graph and replayed (the entry point allocates nothing
    # and does not synchronise), at this batch and at a serving batch of 4 rows where launch
    # overhead shows; outside the timed region.
    def graph_ms(bw):
        winp = make_inputs(wr.with_(B=bw, T=args.steps), "cpu")
        winp = {n: t.to(dev) for n, t in winp.items()}
        st = winp["h0"].clone()
        ob = torch.empty((args.steps, bw, w.Hv, w.Dv), dtype=w.torch_dtype, device=dev)
        cap = torch.cuda.Stream(dev)
        cap.wait_stream(stream)

        def run(strm):
            for s in range(args.steps):
                gdr.gdr_decode_step(winp["q"][s], winp["k"][s], winp["v"][s], winp["g"][s], winp["beta"][s], st,
                                    o=ob[s], stream=strm)

        run(stream)   # eager, warm
        torch.cuda.synchronize()
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        t0.record(stream)
        run(stream)
        t1.record(stream)
        torch.cuda.synchronize()
        eager = t0.elapsed_time(t1) / args.steps
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=cap):
            run(cap)
        graph.replay()
        torch.cuda.synchronize()
        t0.record(stream)
        graph.replay()
        t1.record(stream)
        torch.cuda.synchronize()
        return {"batch": bw, "eager_ms_per_step": eager, "graph_ms_per_step": t0.elapsed_time(t1) / args.steps}

    cuda_graph = [graph_ms(w.B), graph_ms(4)] if world == 1 else None

    e2e = None
    if not args.no_e2e:   # one token's inputs up, its outputs down, every step
        host = {n: inp_cpu[n][0].pin_memory() for n in ("q", "k", "v", "g", "beta")}
        dbuf = {n: torch.empty_like(x, device=dev) for n, x in host.items()}
        o_h = torch.empty(o.shape, dtype=o.dtype).pin_memory()
        h2d = sum(x.numel() * x.element_size() for x in host.values())
        d2h = o_h.numel() * o_h.element_size()

        def e2e_step():
            for n, x in host.items():
                dbuf[n].copy_(x, non_blocking=True)
            gdr.gdr_decode_step(dbuf["q"], dbuf["k"], dbuf["v"], dbuf["g"], dbuf["beta"], state, o=o,
                                stream=stream)
            o_h.copy_(o, non_blocking=True)

        e2e_step()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(args.steps):
            e2e_step()
        e1.record(stream)
        torch.cuda.synchronize()
        te = max_over_ranks(e0.elapsed_time(e1) / args.steps, dev)
        e2e = {"value": job_tokens_per_s(w.B * w.Hv, world, te), "unit": "tokens/s",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": args.steps,
               "ms_per_step": te}
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return 0
    peak, peak_kind = measured_peaks()
    alg = algorithmic_bytes(w)
    achieved = alg / (ms / 1e3) / 1e9
    traffic, traffic_kernel = recorded_traffic(w.name)
    line = {
        "metric": "gated-delta decode tokens/s (B·Hv per sec per step) bf16 d=128; % of roofline",
        "value": job_tokens_per_s(w.B * w.Hv, world, ms_max), "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_max, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": w.dtype,
        "data": "synthetic (seeded CPU generator, one fresh token per step; state 0.02 N(0,1))",
        "config": workload_config(w, world),
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                     "frac": achieved / peak, "peak_source": peak_kind, "algorithmic_bytes_per_launch": alg,
                     "traffic": traffic, "traffic_kernel": traffic_kernel, "kernel": "gdr_decode_step"},
        "cpu_baseline": decode_oracle_sample(w) if world == 1 and not args.no_cpu_baseline else None,
        "e2e": e2e, "gpu_launches": launches,
        "launches_per_step": launches / args.steps, "clocks": clk.summary(), "cuda_graph": cuda_graph,
    }
    print(json.dumps(line), flush=True)
    return 0


# ----------------------------------------------------------------------------- GPU arm
def main(argv=None):
    args = parse_args(argv)
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))

    from gated_delta_rule_68_b200.workloads import WORKLOADS, make_inputs
    w = WORKLOADS[args.workload]
    if args.T is not None:
        w = w.with_(name=f"{w.name}_T{args.T}", T=args.T)
    if args.B is not None:
        w = w.with_(name=f"{w.name}_B{args.B}", B=args.B)
    if args.impl == "reference":
        return run_reference(args, w, rank, world)

    import torch
    import torch.distributed as dist
    from datetime import timedelta

    import gated_delta_rule_68_b200 as gdr

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        dist.init_process_group("nccl", timeout=timedelta(seconds=300), device_id=dev)

    wr = rank_workload(w, rank)
    if w.decode:
        return run_decode_bench(args, w, wr, rank, world, local, dev)
    if w.layer:
        return run_layer_bench(args, w, wr, rank, world, local, dev)
    if w.bwd:
        return run_bwd_bench(args, w, wr, rank, world, local, dev)
    inp_cpu = make_inputs(wr, "cpu")
    inp = {n: (None if t is None else t.to(dev)) for n, t in inp_cpu.items()}
    o = torch.empty((w.B, w.T, w.Hv, w.Dv), dtype=w.torch_dtype, device=dev)
    hT = torch.empty((w.B, w.Hv, w.Dk, w.Dv), dtype=torch.float32, device=dev)
    need = gdr.gdr_fwd_workspace_size(w.B, w.T, w.Hk, w.Hv, w.Dk, w.Dv, w.gate_mode,
                                      gdr.GDR_BF16 if w.dtype == "bf16" else gdr.GDR_FP32)
    ws = torch.empty(max(need, 1), dtype=torch.uint8, device=dev)
    flush = None if algorithmic_bytes(w) > L2_BYTES else torch.empty(256 * 2 ** 20, dtype=torch.uint8,
                                                                      device=dev)
    stream = torch.cuda.current_stream(dev)

    def step():
        if flush is not None:
            flush.add_(1)
        gdr.gdr_fwd_chunked(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], inp["h0"], o=o, hT=hT,
                            workspace=ws, stream=stream)

    def barrier():
        if world > 1:
            dist.barrier()

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()

    # ---- device-timed region
    barrier()
    torch.cuda.synchronize()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    n0 = gdr.gdr_kernel_launches()
    with ClockSampler(local) as clk:
        ev0.record(stream)
        for _ in range(args.steps):
            step()
        ev1.record(stream)
        torch.cuda.synchronize()
    launches = gdr.gdr_kernel_launches() - n0
    barrier()
    ms = ev0.elapsed_time(ev1) / args.steps
    ms_max = max_over_ranks(ms, dev)

    # ---- end to end through the public API with host buffers
    e2e = None
    if not args.no_e2e:
        host = {n: (None if x is None else x.pin_memory()) for n, x in inp_cpu.items()}
        names = [n for n, x in host.items() if x is not None]
        h2d = sum(host[n].numel() * host[n].element_size() for n in names)
        d2h = o.numel() * o.element_size() + hT.numel() * hT.element_size()
        e2e_steps = max(3, min(args.steps, 10))
        # Two sets of device and pinned result buffers: step i's inputs go in on s_in and its
        # results out on s_out while step i - 1 computes, as a pipelined caller would run it.
        dbufs = [{n: torch.empty_like(host[n], device=dev) for n in names} for _ in range(2)]
        obufs = [(torch.empty_like(o), torch.empty_like(hT)) for _ in range(2)]
        hbufs = [(torch.empty(o.shape, dtype=o.dtype).pin_memory(), torch.empty(hT.shape, dtype=hT.dtype).pin_memory())
                 for _ in range(2)]
        s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        in_ready, comp_done, out_done = ([torch.cuda.Event() for _ in range(2)] for _ in range(3))
        used = [False, False]

        def e2e_step(i):
            j = i % 2
            d, (od, hd), (oh, hh) = dbufs[j], obufs[j], hbufs[j]
            if used[j]:
                s_in.wait_event(comp_done[j])     # step i - 2 has read this input set
            with torch.cuda.stream(s_in):
                for n in names:
                    d[n].copy_(host[n], non_blocking=True)
                in_ready[j].record(s_in)
            stream.wait_event(in_ready[j])
            if used[j]:
                stream.wait_event(out_done[j])    # step i - 2's results have left this output set
            gdr.gdr_fwd_chunked(d["q"], d["k"], d["v"], d["g"], d["beta"], d.get("h0"), o=od, hT=hd,
                                workspace=ws, stream=stream)
            comp_done[j].record(stream)
            s_out.wait_event(comp_done[j])
            with torch.cuda.stream(s_out):
                oh.copy_(od, non_blocking=True)
                hh.copy_(hd, non_blocking=True)
                out_done[j].record(s_out)
            used[j] = True

        def serial_step():
            d = dbufs[0]
            for n in names:
                d[n].copy_(host[n], non_blocking=True)
            gdr.gdr_fwd_chunked(d["q"], d["k"], d["v"], d["g"], d["beta"], d.get("h0"), o=o, hT=hT,
                                workspace=ws, stream=stream)
            hbufs[0][0].copy_(o, non_blocking=True)
            hbufs[0][1].copy_(hT, non_blocking=True)

        for i in range(2):
            e2e_step(i)
        torch.cuda.synchronize()
        barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(s_in)                      # before the first copy in
        for i in range(2, 2 + e2e_steps):
            e2e_step(i)
        e1.record(s_out)                     # after the last copy out
        torch.cuda.synchronize()
        te = max_over_ranks(e0.elapsed_time(e1) / e2e_steps, dev)
        # the same steps one after another on one stream, for reference
        serial_step()
        torch.cuda.synchronize()
        e2, e3 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e2.record(stream)
        for _ in range(e2e_steps):
            serial_step()
        e3.record(stream)
        torch.cuda.synchronize()
        ts = max_over_ranks(e2.elapsed_time(e3) / e2e_steps, dev)
        e2e = {"value": job_tokens_per_s(w.head_tokens, world, te), "unit": "tokens/s",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": e2e_steps,
               "ms_per_step": te, "pipelined": "inputs of step i+1 and results of step i-1 cross the "
               "host link while step i computes (two copy streams, two buffer sets)",
               "serial_ms_per_step": ts}

    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return 0

    peak, peak_kind = measured_peaks()
    alg = algorithmic_bytes(w)
    achieved = alg / (ms / 1e3) / 1e9
    traffic, traffic_kernel = recorded_traffic(w.name)
    cpu = None
    if world == 1 and not args.no_cpu_baseline:
        cpu = cpu_oracle_sample(w)
    line = {
        "metric": METRIC,
        "value": job_tokens_per_s(w.head_tokens, world, ms_max),
        "unit": "tokens/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": ms_max,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": w.dtype,
        "data": "synthetic (seeded CPU generator; q,k L2-normalised N(0,1); v N(0,1); "
                f"g logsigmoid(N({w.g_mu:g},1)); beta sigmoid(N(0,1)); h0 0.02 N(0,1))",
        "config": workload_config(w, world),
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                     "frac": achieved / peak, "peak_source": peak_kind,
                     "algorithmic_bytes_per_launch": alg,
                     "traffic": traffic, "traffic_kernel": traffic_kernel,
                     "kernel": "gdr_fwd_chunked step"},
        "cpu_baseline": cpu,
        "e2e": e2e,
        "gpu_launches": launches,
        "launches_per_step": launches / args.steps,
        "clocks": clk.summary(),
    }
    print(json.dumps(line), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
