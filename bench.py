"""Benchmark of the KLA hot path on B200 (one JSON line on stdout, rank 0).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl kla|reference]
    torchrun --nproc-per-node N bench.py --gpus N ...      (N > 1: independent replicas)

Headline (`value`): prefill tokens/s of kla_chunk_fwd on the 0.4B-layer-shaped workload
(B=8, T=2048, H=8, Dk=Dv=128, bf16 inputs, fp32 state), inputs resident in HBM, L2 flushed
between timed steps.  One step = one kla_chunk_fwd call over the whole batch.  The same line
carries the decode workload (B=64, H=16, 1024 sequential kla_decode_step calls), the
training workload (B=4, T=4096, H=16: kla_chunk_fwd + kla_chunk_bwd) and the long-context
prefill (B=1, T=65536, H=16) as sub-objects, each with its own roofline.

Multi-GPU: the (batch, head) pairs are independent problems, so every rank runs its own
replica of the workload (different seed), with no collective on the data path; the timed
region is bracketed by barriers and the time taken is the max over ranks ("weak" scaling).

`--impl reference` times the fp64 CPU oracle (the slow, obviously correct reference) on a
bounded sample of the same workload, on the host cores; only rank 0 runs it.
"""
import argparse
import hashlib
import json
import math
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "prefill tokens/s & decode tokens/s at 1 B200; % of tensor-core/HBM roofline"
PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
L2_FLUSH_BYTES = 256 << 20  # > 2x the 126 MB L2


# ---------------------------------------------------------------------------------------
# algorithmic work (fixed at chunk C = 64, whatever the kernel does internally)
# ---------------------------------------------------------------------------------------
def fwd_flops_per_token_head(d, C=64):
    # 10 C d (KK^T, QK^T, the two UT-transform products, (A o QK^T) U) + 6 d^2 (W S, Q S,
    # K^T U) + (2/3) C^2 (forward substitution)
    return 10 * C * d + 6 * d * d + (2.0 / 3.0) * C * C


def fwd_bytes(B, T, H, Dk, Dv, elt, s0, s_out=True, out_elt=4):
    per_tok = (2 * Dk + Dv) * elt + Dv * out_elt + 8  # q, k, v in; o out (fp32); eta, g
    state = B * H * Dk * Dv * 4 * ((1 if s0 else 0) + (1 if s_out else 0))
    return B * T * H * per_tok + state


def attainable(flops, nbytes, tc_peak_tflops, hbm_peak_gbs, seconds):
    """Floors of a call's algorithmic work on the measured peaks, and the measured time's
    fraction of the slower one (the attainable roofline)."""
    t_tc = flops / (tc_peak_tflops * 1e12)
    t_hbm = nbytes / (hbm_peak_gbs * 1e9)
    return {"t_tensor_us": t_tc * 1e6, "t_hbm_us": t_hbm * 1e6, "bound": "hbm" if t_hbm >= t_tc else "tensor",
            "frac": max(t_tc, t_hbm) / seconds}


def decode_bytes(B, H, Dk, Dv, elt, out_elt=4):
    return B * H * (2 * Dk * Dv * 4 + (2 * Dk + Dv) * elt + Dv * out_elt + 8)


def bwd_bytes(B, T, H, Dk, Dv, elt, out_elt=4):
    # reads q, k, v, dO, eta, g; writes dq, dk, dv (fp32), deta, dg; plus the dS0 write
    per_tok = (2 * Dk + Dv) * elt + Dv * elt + 8 + (2 * Dk + Dv) * out_elt + 8
    return B * T * H * per_tok + B * H * Dk * Dv * 4


# ---------------------------------------------------------------------------------------
# helpers
# ---------------------------------------------------------------------------------------
def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(PEAKS_FALLBACK), "fallback"


def kernel_source_hash(files=None):
    """Hash of the CUDA sources a kernel is built from (all of csrc/ when `files` is None);
    recorded ncu traffic is only valid for the same sources."""
    h = hashlib.sha256()
    cdir = os.path.join(ROOT, "gated_delta_rule_kla_b200", "csrc")
    for f in sorted(files if files is not None else os.listdir(cdir)):
        with open(os.path.join(cdir, f), "rb") as fh:
            h.update(f.encode() + fh.read())
    return h.hexdigest()[:16]


def recorded_traffic(kernel_key):
    """DRAM bytes per launch from the committed ncu summary, or None if stale/absent.  An entry
    names the source files of its kernels (`sources`) and their hash at capture time."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    e = d.get(kernel_key)
    if not e or e.get("source_hash") != kernel_source_hash(e.get("sources")):
        return None
    return e.get("dram_bytes_per_launch")


class ClockSampler:
    """Samples SM clock, power and throttle reasons through NVML while the GPU is busy."""

    def __init__(self, device_index, period=0.05):
        self.samples = []
        self.period = period
        self._stop = threading.Event()
        self._thr = None
        self.max_mhz = None
        self.ok = False
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            vis = os.environ.get("CUDA_VISIBLE_DEVICES")
            idx = device_index
            if vis:
                ids = [x for x in vis.split(",") if x.strip()]
                if device_index < len(ids) and ids[device_index].strip().isdigit():
                    idx = int(ids[device_index])
            self.h = pynvml.nvmlDeviceGetHandleByIndex(idx)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:
            self.ok = False

    def _run(self):
        nv = self.nv
        while not self._stop.is_set():
            try:
                clk = nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM)
                util = nv.nvmlDeviceGetUtilizationRates(self.h).gpu
                reasons = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                self.samples.append((clk, util, reasons))
            except Exception:
                pass
            self._stop.wait(self.period)

    def __enter__(self):
        if self.ok:
            self._thr = threading.Thread(target=self._run, daemon=True)
            self._thr.start()
        return self

    def __exit__(self, *exc):
        self._stop.set()
        if self._thr:
            self._thr.join()

    def summary(self):
        if not self.ok:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvml unavailable"], "samples": 0}
        nv = self.nv
        names = {
            "gpu_idle": getattr(nv, "nvmlClocksEventReasonGpuIdle", 0x1),
            "applications_clocks_setting": getattr(nv, "nvmlClocksEventReasonApplicationsClocksSetting", 0x2),
            "sw_power_cap": getattr(nv, "nvmlClocksEventReasonSwPowerCap", 0x4),
            "hw_slowdown": getattr(nv, "nvmlClocksEventReasonHwSlowdown", 0x8),
            "sync_boost": getattr(nv, "nvmlClocksEventReasonSyncBoost", 0x10),
            "sw_thermal_slowdown": getattr(nv, "nvmlClocksEventReasonSwThermalSlowdown", 0x20),
            "hw_thermal_slowdown": getattr(nv, "nvmlClocksEventReasonHwThermalSlowdown", 0x40),
            "hw_power_brake_slowdown": getattr(nv, "nvmlClocksEventReasonHwPowerBrakeSlowdown", 0x80),
        }
        loaded = [s for s in self.samples if s[1] > 0] or self.samples
        reasons = set()
        for _, _, r in loaded:
            for n, bit in names.items():
                if n != "gpu_idle" and r & bit:
                    reasons.add(n)
        med = statistics.median([s[0] for s in loaded]) if loaded else None
        return {"sm_mhz": med, "sm_max_mhz": self.max_mhz, "reasons": sorted(reasons),
                "samples": len(loaded)}


def dist_env():
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
            int(os.environ.get("LOCAL_RANK", "0")))


def max_over_ranks(value, world):
    """Max of a float over all ranks (device-timed numbers are combined this way)."""
    if world <= 1:
        return value
    import torch
    import torch.distributed as dist
    dev = torch.device("cuda", torch.cuda.current_device()) if dist.get_backend() == "nccl" else torch.device("cpu")
    t = torch.tensor([value], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(value, world):
    if world <= 1:
        return value
    import torch
    import torch.distributed as dist
    dev = torch.device("cuda", torch.cuda.current_device()) if dist.get_backend() == "nccl" else torch.device("cpu")
    t = torch.tensor([value], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


# ---------------------------------------------------------------------------------------
# GPU arm
# ---------------------------------------------------------------------------------------
class Flusher:
    """Evicts L2 between timed steps by writing a buffer larger than L2.  The timed kernel then
    starts with no useful line in L2 and an L2 full of dirty lines, so the write-backs its own
    traffic forces are paid inside its timing (as in a loop over many layers' states)."""

    def __init__(self, dev):
        import torch
        self.a = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
        self.k = 0

    def __call__(self):
        self.k += 1
        self.a.fill_(float(self.k))


def time_steps(fn, steps, flush, stream):
    """Run fn `steps` times, L2 flushed before each; returns per-step device ms (events on
    the launching stream, recorded around the kernel launches only)."""
    import torch
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    for i in range(steps):
        flush()
        evs[i][0].record(stream)
        fn()
        evs[i][1].record(stream)
    torch.cuda.synchronize()
    return [a.elapsed_time(b) for a, b in evs]


def gpu_arm(args, rank, world, local_rank):
    import torch
    import gated_delta_rule_kla_b200 as kla
    from gated_delta_rule_kla_b200.workloads import WORKLOADS, make_inputs

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    kla.lib()
    stream = torch.cuda.current_stream(dev)
    peaks, peaks_kind = load_peaks()
    hbm_peak = peaks["hbm_gbs"]
    tc_peak = peaks["bf16_tflops"]
    flush = Flusher(dev)

    # ---------------- prefill (headline) ----------------
    w = WORKLOADS[args.workload]
    w = w.with_(seed=w.seed + 1000 * rank)
    inp = make_inputs(w)
    d = {k: (v.to(dev) if v is not None else None) for k, v in inp.items()}
    o = torch.empty(w.B, w.T, w.H, w.Dv, device=dev, dtype=torch.float32)
    ST = torch.empty(w.B, w.H, w.Dk, w.Dv, device=dev, dtype=torch.float32)
    ws = kla.fwd_workspace(d["k"], d["v"])  # the split path's per-chunk records, allocated once
    launches = kla.fwd_kernel_launches(d["k"], d["v"])  # 4: two slabs (prep + state pass each)

    def prefill():
        kla.chunk_fwd(d["q"], d["k"], d["v"], d["eta"], d["g"], w.eps, d["S0"], o=o, S_T=ST, workspace=ws)

    sampler = ClockSampler(local_rank)
    for _ in range(args.warmup):
        flush()
        prefill()
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    with sampler:
        ms = time_steps(prefill, args.steps, flush, stream)
        torch.cuda.synchronize()
        barrier(world)
        torch.cuda.synchronize()
        total_ms = max_over_ranks(sum(ms), world)
        tokens = sum_over_ranks(float(w.B * w.T), world) * args.steps
        elt = d["q"].element_size()
        alg_bytes = fwd_bytes(w.B, w.T, w.H, w.Dk, w.Dv, elt, d["S0"] is not None)
        alg_bytes_bf16_o = fwd_bytes(w.B, w.T, w.H, w.Dk, w.Dv, elt, d["S0"] is not None, out_elt=2)
        alg_flops = fwd_flops_per_token_head(w.Dk) * w.B * w.T * w.H
        mean_s = statistics.mean(ms) / 1e3
        achieved_gbs = alg_bytes / mean_s / 1e9
        achieved_tf = alg_flops / mean_s / 1e12
        stages = time_fwd_stages(kla, d, w, ws, o, ST, flush, stream, 3 if args.quick else 10)

        extra = {}
        parts = set(args.parts.split(",")) if not args.skip_extra else set()
        if "decode" in parts:
            extra["decode"] = bench_decode(kla, WORKLOADS, make_inputs, dev, stream, flush, rank, world,
                                           hbm_peak, args)
        if "train" in parts:
            extra["train"] = bench_train(kla, WORKLOADS, make_inputs, dev, stream, flush, rank, world,
                                         hbm_peak, tc_peak, args)
        if "long" in parts:
            extra["long_context"] = bench_long(kla, WORKLOADS, make_inputs, dev, stream, rank, world,
                                               hbm_peak, tc_peak, args)
        if "direct" in parts:
            extra["direct_beta"] = bench_direct(kla, w, d, ws, o, ST, flush, stream, world, hbm_peak, args)
        if "diag" in parts:
            extra["diagonal_gating"] = bench_diag(kla, WORKLOADS, make_inputs, dev, stream, flush, rank, world,
                                                  hbm_peak, peaks, args)
        if "gates" in parts:
            extra["gate_prologue"] = bench_gates(kla, dev, stream, flush, rank, world, hbm_peak, args)

    # ---------------- end-to-end through the public API with host buffers ----------------
    e2e = None if args.skip_e2e else bench_e2e(kla, w, inp, dev, stream, rank, world, args)
    clocks = sampler.summary()

    line = {
        "metric": METRIC,
        "value": tokens / (total_ms / 1e3),
        "unit": "tokens/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": total_ms / args.steps,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16" if w.dtype == "bf16" else "f32",
        "data": "synthetic (seeded; shapes of the paper's 0.4B model, App. C)",
        "config": {"workload": w.name, "B": w.B, "T": w.T, "H": w.H, "Dk": w.Dk, "Dv": w.Dv,
                   "chunk": w.chunk, "state": "fp32", "l2": "flushed between timed steps",
                   "parallelism": f"{world} independent replica(s), no collective"},
        "roofline": {"bound": "hbm", "achieved": achieved_gbs, "peak": hbm_peak, "unit": "GB/s",
                     "frac": achieved_gbs / hbm_peak, "peak_kind": peaks_kind,
                     "scope": ("one kla_chunk_fwd call: chunk_prep_kernel + chunk_state_kernel"
                               + (", as two slabs (slab 1's state pass concurrent with slab 2's"
                                  " preparation)" if launches == 4 else "")),
                     "traffic": recorded_traffic("chunk_fwd_prefill_b8_t2048_h8_d128"),
                     "alg_bytes_per_launch": alg_bytes, "kernel_us": mean_s * 1e6, "stages": stages,
                     # the same call counted with a bf16 o (1032 B per token-head): the output
                     # store the scope table fixes, below the fp32 o this call writes
                     "alg_bytes_bf16_o": alg_bytes_bf16_o,
                     "frac_bf16_o": alg_bytes_bf16_o / mean_s / 1e9 / hbm_peak,
                     "tensor": {"achieved": achieved_tf, "peak": tc_peak, "unit": "TFLOP/s",
                                "frac": achieved_tf / tc_peak, "alg_flops_per_launch": alg_flops},
                     # the attainable roofline: the slower of the tensor-core and HBM floors of
                     # the call's algorithmic work (fp32 o as written), over the measured time
                     "attainable": attainable(alg_flops, alg_bytes, tc_peak, hbm_peak, mean_s)},
        "e2e": e2e,
        "gpu_launches": launches * args.steps,
        "clocks": clocks,
    }
    line.update(extra)
    return line


def time_fwd_stages(kla, d, w, ws, o, ST, flush, stream, nsteps):
    """Each stage of the split forward timed on its own with CUDA events on the launching
    stream (L2 flushed before every step): the preparation kernel and the state pass -- with
    parallel segments, the state pass's transition pass, segment scan and output pass apart."""
    import torch
    nseg = kla.fwd_state_segments(d["k"], d["v"])
    parts = [("chunk_state_kernel", 0)] if nseg <= 1 else [
        ("transition_pass", 1), ("seg_scan_kernel", 2), ("output_pass", 3)]
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2 + len(parts))] for _ in range(nsteps)]
    for i in range(nsteps):
        flush()
        ev[i][0].record(stream)
        kla.chunk_fwd_prep(d["q"], d["k"], d["v"], d["eta"], d["g"], w.eps, ws)
        ev[i][1].record(stream)
        for j, (_, stage) in enumerate(parts):
            kla.chunk_fwd_state(d["q"], d["v"], d["g"], d["S0"], ws, o=o, S_T=ST, stage=stage)
            ev[i][2 + j].record(stream)
    torch.cuda.synchronize()
    us = {"chunk_prep_kernel": statistics.median(e[0].elapsed_time(e[1]) for e in ev) * 1e3}
    for j, (name, _) in enumerate(parts):
        us[name] = statistics.median(e[1 + j].elapsed_time(e[2 + j]) for e in ev) * 1e3
    tot = sum(us.values())
    out = {k: {"us": v, "share": v / tot} for k, v in us.items()}
    if nseg > 1:
        out["segments_per_head"] = nseg
        out["transition_pass"]["what"] = ("chunk_state_kernel, two runs per segment (from zero and from the "
                                          "identity), no outputs")
        out["output_pass"]["what"] = "chunk_state_kernel, one run per segment from its start state, with o"
    out["dominant"] = max(us, key=us.get)
    return out


def bench_decode(kla, WORKLOADS, make_inputs, dev, stream, flush, rank, world, hbm_peak, args,
                 wname="decode_b64_h16_d128_x1024", step_fn=None, traffic_key="decode_b64_h16_d128"):
    import torch
    step_fn = step_fn or kla.decode_step
    w = WORKLOADS[wname]
    w = w.with_(seed=w.seed + 1000 * rank)
    inp = make_inputs(w)
    q, k, v = inp["q"].to(dev), inp["k"].to(dev), inp["v"].to(dev)
    eta, g = inp["eta"].to(dev), inp["g"].to(dev)
    # The state (67 MB) fits in L2.  Inputs larger than L2 instead of a flush between steps:
    # NSETS independent groups of B sequences, each with its own state, decode in turn (step t
    # advances group t % NSETS by one token), so every step finds its state evicted by the
    # other groups' traffic and moves exactly its own read and write through HBM -- as a
    # server with more live sequences than L2 holds would.  (A write flush between steps
    # leaves dirty lines whose write-back lands inside the next timed step.)
    NSETS = 4
    S_sets = [inp["S0"].to(dev).clone() for _ in range(NSETS)]
    o = torch.empty(w.B, w.H, w.Dv, device=dev, dtype=torch.float32)
    steps = w.T if not args.quick else 64
    for t in range(8):
        step_fn(q[t], k[t], v[t], eta[t], g[t], S_sets[0], w.eps, o=o)
    S_sets[0].copy_(inp["S0"].to(dev))
    torch.cuda.synchronize()
    barrier(world)

    def all_steps():
        for t in range(steps):
            tok = t // NSETS
            step_fn(q[tok], k[tok], v[tok], eta[tok], g[tok], S_sets[t % NSETS], w.eps, o=o)

    # The steps are captured once in a CUDA graph and replayed, as a serving loop would run
    # them: one host launch per step costs about as much as the step itself, so timed eagerly
    # the number would follow the host CPU.  Events bracket the whole replay.
    timing = "one CUDA graph of every step, events around its second replay"
    try:
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=torch.cuda.Stream(dev)):  # captured off the default stream
            all_steps()
    except Exception as exc:  # capture unavailable: per-step events on eager launches
        graph, timing = None, f"per-step events on eager launches (graph capture failed: {type(exc).__name__})"
    for S_, S0_ in zip(S_sets, [inp["S0"]] * NSETS):
        S_.copy_(S0_.to(dev))
    torch.cuda.synchronize()
    barrier(world)
    if graph is not None:
        graph.replay()  # the first replay also uploads the graph: untimed (the states decode on)
        torch.cuda.synchronize()
        ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        ev0.record(stream)
        graph.replay()
        ev1.record(stream)
        torch.cuda.synchronize()
        ms = [ev0.elapsed_time(ev1) / steps] * steps
        del graph
    else:
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
        for t in range(steps):
            tok = t // NSETS
            evs[t][0].record(stream)
            step_fn(q[tok], k[tok], v[tok], eta[tok], g[tok], S_sets[t % NSETS], w.eps, o=o)
            evs[t][1].record(stream)
        torch.cuda.synchronize()
        ms = [a.elapsed_time(b) for a, b in evs]
    barrier(world)
    total_ms = max_over_ranks(sum(ms), world)
    tokens = sum_over_ranks(float(w.B), world) * steps
    mean_s = statistics.mean(ms) / 1e3
    alg = decode_bytes(w.B, w.H, w.Dk, w.Dv, q.element_size())
    if g.dim() == 4:  # diagonal gating: one log-decay per key channel
        alg += w.B * w.H * (w.Dk - 1) * 4
    gbs = alg / mean_s / 1e9
    return {"workload": w.name, "value": tokens / (total_ms / 1e3), "unit": "tokens/s",
            "steps": steps, "us_per_step": total_ms * 1e3 / steps, "gpu_launches": steps, "timing": timing,
            "l2": "inputs larger than L2 (4 sequence groups' states cycled, 268 MB)",
            "roofline": {"bound": "hbm", "achieved": gbs, "peak": hbm_peak, "unit": "GB/s",
                         "frac": gbs / hbm_peak, "alg_bytes_per_launch": alg,
                         "traffic": recorded_traffic(traffic_key)}}


def bench_train(kla, WORKLOADS, make_inputs, dev, stream, flush, rank, world, hbm_peak, tc_peak, args):
    import torch
    w = WORKLOADS["train_b4_t4096_h16_d128"]
    w = w.with_(seed=w.seed + 1000 * rank)
    inp = make_inputs(w)
    d = {k: (v.to(dev) if v is not None else None) for k, v in inp.items()}
    dO = d["dO"].to(d["q"].dtype)
    # one workspace shared by the training forward and the backward (kla_chunk_fwd_train,
    # kla_chunk_bwd_after_train): the backward reuses the forward's records and tiles
    ws = kla.train_workspace(d["k"], d["v"])
    o = torch.empty(w.B, w.T, w.H, w.Dv, device=dev, dtype=torch.float32)
    ST = torch.empty(w.B, w.H, w.Dk, w.Dv, device=dev, dtype=torch.float32)

    def step():
        kla.chunk_fwd_train(d["q"], d["k"], d["v"], d["eta"], d["g"], w.eps, d["S0"], workspace=ws, o=o, S_T=ST)
        kla.chunk_bwd_after_train(d["q"], d["k"], d["v"], d["eta"], d["g"], dO, ws, w.eps)

    nsteps = 2 if args.quick else 5
    # + the reverse state pass and the gradient kernel, each twice when the reverse pass runs as
    # two slabs (the gradient kernel of the newest chunks beside the reverse pass over the rest)
    slab = kla.lib().kla_chunk_bwd_reverse_slab_chunks(w.B, w.T, w.H, w.Dk, w.Dv, 64, 1)
    launches = kla.fwd_kernel_launches(d["k"], d["v"]) + (4 if slab > 0 else 2)
    step()
    torch.cuda.synchronize()
    barrier(world)
    ms = time_steps(step, nsteps, flush, stream)
    barrier(world)
    total_ms = max_over_ranks(sum(ms), world)
    tokens = sum_over_ranks(float(w.B * w.T), world) * nsteps
    mean_s = statistics.mean(ms) / 1e3
    flops = 3 * fwd_flops_per_token_head(w.Dk) * w.B * w.T * w.H
    elt = d["q"].element_size()
    alg = fwd_bytes(w.B, w.T, w.H, w.Dk, w.Dv, elt, False) + bwd_bytes(w.B, w.T, w.H, w.Dk, w.Dv, elt)
    return {"workload": w.name, "value": tokens / (total_ms / 1e3), "unit": "tokens/s",
            "steps": nsteps, "ms_per_step": total_ms / nsteps,
            # forward: preparation + state pass (each twice with two slabs); backward: reverse
            # state pass + gradient kernel (each twice with two slabs)
            "gpu_launches_per_step": launches,
            "reverse_slab_newest_chunks": slab,
            "roofline": {"bound": "tensor", "achieved": flops / mean_s / 1e12, "peak": tc_peak,
                         "unit": "TFLOP/s", "frac": flops / mean_s / 1e12 / tc_peak,
                         "hbm_frac": alg / mean_s / 1e9 / hbm_peak, "alg_flops_per_step": flops,
                         "alg_bytes_per_step": alg,
                         "attainable": attainable(flops, alg, tc_peak, hbm_peak, mean_s)}}


def bench_long(kla, WORKLOADS, make_inputs, dev, stream, rank, world, hbm_peak, tc_peak, args):
    import torch
    w = WORKLOADS["prefill_b1_t65536_h16_d128"]
    w = w.with_(seed=w.seed + 1000 * rank)
    inp = make_inputs(w)
    d = {k: (v.to(dev) if v is not None else None) for k, v in inp.items()}
    o = torch.empty(w.B, w.T, w.H, w.Dv, device=dev, dtype=torch.float32)
    ST = torch.empty(w.B, w.H, w.Dk, w.Dv, device=dev, dtype=torch.float32)
    # few heads, long sequences: the split path with a segmented state pass (workspace
    # allocated once here)
    ws = kla.fwd_workspace(d["k"], d["v"])

    def run():
        kla.chunk_fwd(d["q"], d["k"], d["v"], d["eta"], d["g"], w.eps, d["S0"], o=o, S_T=ST, workspace=ws)

    run()
    torch.cuda.synchronize()
    barrier(world)
    nsteps = 2 if args.quick else 3
    ms = time_steps(run, nsteps, lambda: None, stream)  # inputs (403 MB) exceed L2
    # the preparation and the segmented state pass (transition pass, segment scan, output pass)
    # timed on their own
    stages = time_fwd_stages(kla, d, w, ws, o, ST, lambda: None, stream, nsteps)
    del ws
    # the long-context training step: kla_chunk_fwd_train + kla_chunk_bwd_after_train sharing
    # one workspace (records and tile images: about 5 GB here)
    dO = torch.randn(w.B, w.T, w.H, w.Dv, device=dev).to(d["q"].dtype)
    wst = kla.train_workspace(d["k"], d["v"])

    def fwd_t():
        kla.chunk_fwd_train(d["q"], d["k"], d["v"], d["eta"], d["g"], w.eps, d["S0"], workspace=wst, o=o, S_T=ST)

    def bwd_t():
        kla.chunk_bwd_after_train(d["q"], d["k"], d["v"], d["eta"], d["g"], dO, wst, w.eps)

    fwd_t()
    bwd_t()
    torch.cuda.synchronize()
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(2)]
    for e in ev:
        e[0].record(stream)
        fwd_t()
        e[1].record(stream)
        bwd_t()
        e[2].record(stream)
    torch.cuda.synchronize()
    f_ms = statistics.mean(e[0].elapsed_time(e[1]) for e in ev)
    b_ms = statistics.mean(e[1].elapsed_time(e[2]) for e in ev)
    del wst
    train = {"ms_per_step": f_ms + b_ms, "forward_ms": f_ms, "backward_ms": b_ms,
             "value": w.B * w.T / ((f_ms + b_ms) / 1e3), "unit": "tokens/s",
             "what": "kla_chunk_fwd_train + kla_chunk_bwd_after_train (reverse state pass over 1024 chunks per head, "
                     "as parallel segments when kla_chunk_bwd_reverse_segments > 1; then the chunk-parallel "
                     "gradient kernel)",
             "reverse_segments": kla.lib().kla_chunk_bwd_reverse_segments(w.B, w.T, w.H, w.Dk, w.Dv, 64, 1)}
    barrier(world)
    total_ms = max_over_ranks(sum(ms), world)
    tokens = sum_over_ranks(float(w.B * w.T), world) * nsteps
    mean_s = statistics.mean(ms) / 1e3
    alg = fwd_bytes(w.B, w.T, w.H, w.Dk, w.Dv, d["q"].element_size(), True)
    flops = fwd_flops_per_token_head(w.Dk) * w.B * w.T * w.H
    return {"workload": w.name, "value": tokens / (total_ms / 1e3), "unit": "tokens/s",
            "steps": nsteps, "ms_per_step": total_ms / nsteps, "l2": "inputs larger than L2",
            # preparation, transition pass, segment scan, output pass
            "gpu_launches_per_step": 4, "stages": stages, "train": train,
            "roofline": {"bound": "hbm", "achieved": alg / mean_s / 1e9, "peak": hbm_peak, "unit": "GB/s",
                         "frac": alg / mean_s / 1e9 / hbm_peak,
                         "tensor_frac": flops / mean_s / 1e12 / tc_peak,
                         "attainable": attainable(flops, alg, tc_peak, hbm_peak, mean_s)}}


def bench_direct(kla, w, d, ws, o, ST, flush, stream, world, hbm_peak, args):
    """The headline prefill with the direct write strength (beta_t = eta_t as given: the
    Gated DeltaNet update, KLA_BETA_DIRECT): the same kernels, the coefficient map changed."""
    import torch
    eta = (d["eta"] / ((d["k"].float() ** 2).sum(-1) + 1.0)).contiguous()  # contractive writes

    def prefill():
        kla.chunk_fwd(d["q"], d["k"], d["v"], eta, d["g"], w.eps, d["S0"], o=o, S_T=ST, workspace=ws,
                      beta="direct")

    for _ in range(3):
        flush()
        prefill()
    torch.cuda.synchronize()
    nsteps = 5 if args.quick else 20
    ms = time_steps(prefill, nsteps, flush, stream)
    total_ms = max_over_ranks(sum(ms), world)
    tokens = sum_over_ranks(float(w.B * w.T), world) * nsteps
    mean_s = statistics.mean(ms) / 1e3
    alg = fwd_bytes(w.B, w.T, w.H, w.Dk, w.Dv, d["q"].element_size(), d["S0"] is not None)
    return {"workload": w.name, "beta": "direct", "value": tokens / (total_ms / 1e3), "unit": "tokens/s",
            "steps": nsteps, "ms_per_step": total_ms / nsteps, "l2": "flushed between timed steps",
            "gpu_launches_per_step": kla.fwd_kernel_launches(d["k"], d["v"]),
            "roofline": {"bound": "hbm", "achieved": alg / mean_s / 1e9, "peak": hbm_peak, "unit": "GB/s",
                         "frac": alg / mean_s / 1e9 / hbm_peak}}


def fp32_alu_peak_tflops(peaks):
    """fp32 FMA peak of the CUDA cores: 148 SMs x 128 fp32 lanes x 2 FLOP per FMA at the
    maximum SM clock (the unit counts and clock of the part; no measured figure exists)."""
    return 148 * 128 * 2 * peaks.get("sm_max_mhz", 1965.0) * 1e6 / 1e12


def bench_diag(kla, WORKLOADS, make_inputs, dev, stream, flush, rank, world, hbm_peak, peaks, args):
    """Diagonal (per-key-channel) gating (App. A.5, B.5): the headline prefill shape through
    kla_chunk_fwd_diag, its backward kla_chunk_bwd_diag, and the decode shape through
    kla_decode_step_diag (same timing as the scalar decode leg)."""
    import torch
    w = WORKLOADS["prefill_diag_b8_t2048_h8_d128"]
    w = w.with_(seed=w.seed + 1000 * rank)
    inp = make_inputs(w)
    d = {k: (v.to(dev) if v is not None else None) for k, v in inp.items()}
    o = torch.empty(w.B, w.T, w.H, w.Dv, device=dev, dtype=torch.float32)
    ST = torch.empty(w.B, w.H, w.Dk, w.Dv, device=dev, dtype=torch.float32)
    dO = torch.randn(w.B, w.T, w.H, w.Dv, device=dev).to(d["q"].dtype)
    L = kla.lib()
    wsb = torch.empty(L.kla_chunk_bwd_diag_workspace(w.B, w.T, w.H, w.Dk, w.Dv, 64, 1), device=dev,
                      dtype=torch.uint8)

    def fwd():
        kla.chunk_fwd_diag(d["q"], d["k"], d["v"], d["eta"], d["g"], w.eps, d["S0"], o=o, S_T=ST)

    def bwd():
        kla.chunk_bwd_diag(d["q"], d["k"], d["v"], d["eta"], d["g"], dO, w.eps, d["S0"], workspace=wsb)

    for _ in range(3):
        flush()
        fwd()
    bwd()
    torch.cuda.synchronize()
    barrier(world)
    nf = 3 if args.quick else 10
    ms_f = time_steps(fwd, nf, flush, stream)
    ms_b = time_steps(bwd, 2 if args.quick else 3, flush, stream)
    barrier(world)
    tf_f = max_over_ranks(sum(ms_f), world) / nf
    tf_b = max_over_ranks(sum(ms_b), world) / len(ms_b)
    tokens = sum_over_ranks(float(w.B * w.T), world)
    elt = d["q"].element_size()
    # bytes as for scalar gating, plus the per-channel log-decays (Dk fp32 per token-head)
    alg = fwd_bytes(w.B, w.T, w.H, w.Dk, w.Dv, elt, False) + w.B * w.T * w.H * (w.Dk - 1) * 4
    flops = fwd_flops_per_token_head(w.Dk) * w.B * w.T * w.H
    mean_f = statistics.mean(ms_f) / 1e3
    nl = L.kla_chunk_fwd_diag_kernel_launches(w.B, w.T, w.H, w.Dk, w.Dv, 64, 1)
    # bf16 at Dk = Dv = 128: preparation and state pass on the tensor cores (the bound as for the
    # headline forward: HBM on the algorithmic bytes, with the tensor-core fraction beside it)
    out = {"workload": w.name, "value": tokens / (tf_f / 1e3), "unit": "tokens/s", "steps": nf,
           "ms_per_step": tf_f, "l2": "flushed between timed steps", "gpu_launches_per_step": nl,
           "path": "tensor cores: chunk_prep_diag_kernel + chunk_state_kernel (64-token chunks)",
           "roofline": {"bound": "hbm", "achieved": alg / mean_f / 1e9, "peak": hbm_peak, "unit": "GB/s",
                        "frac": alg / mean_f / 1e9 / hbm_peak, "alg_bytes_per_launch": alg,
                        "tensor": {"achieved": flops / mean_f / 1e12, "peak": peaks["bf16_tflops"],
                                   "unit": "TFLOP/s", "frac": flops / mean_f / 1e12 / peaks["bf16_tflops"],
                                   "alg_flops_per_launch": flops}},
           "backward": {"value": tokens / (tf_b / 1e3), "unit": "tokens/s", "ms_per_step": tf_b,
                        "gpu_launches_per_step": 4,
                        # CUDA cores, fp32: twice the forward's FLOPs (the training step's 3x
                        # convention) against the fp32 FMA peak
                        "roofline": {"bound": "alu", "achieved": 2 * flops / (tf_b / 1e3) / 1e12,
                                     "peak": fp32_alu_peak_tflops(peaks), "unit": "TFLOP/s",
                                     "frac": 2 * flops / (tf_b / 1e3) / 1e12 / fp32_alu_peak_tflops(peaks),
                                     "peak_kind": "derived: 148 SMs x 128 fp32 FMA lanes x 2 x max SM clock"},
                        "what": "kla_chunk_bwd_diag: forward state recompute, reverse pass, finish, dg scan"}}
    out["decode"] = bench_decode(kla, WORKLOADS, make_inputs, dev, stream, flush, rank, world, hbm_peak, args,
                                 wname="decode_diag_b64_h16_d128_x1024", step_fn=kla.decode_step_diag,
                                 traffic_key="decode_diag_b64_h16_d128")
    return out


def bench_gates(kla, dev, stream, flush, rank, world, hbm_peak, args):
    """The gate prologue on the headline's tokens (N = B T = 16384, D = 1024 = 8 heads x 128,
    H = 8, q normalised for Dk = 128): kla_gate_prologue and kla_gate_prologue_bwd."""
    import torch
    from gated_delta_rule_kla_b200.workloads import make_gate_inputs
    N, D, H, Dk = 8 * 2048, 1024, 8, 128
    gi = make_gate_inputs(N, D, H, Dk, "bf16", seed=31 + 1000 * rank, device=dev)
    deta = torch.randn(N, H, device=dev)
    dg = torch.randn(N, H, device=dev)
    dqh = torch.randn(N, H, Dk, device=dev)
    res = {}

    def fwd():
        res["f"] = kla.gate_prologue(gi["x"], gi["W"], gi["bias"], gi["q"])

    fwd()

    def bwd():
        kla.gate_prologue_bwd(gi["x"], gi["W"], res["f"][0], res["f"][1], deta, dg, gi["q"], dqh)

    for _ in range(3):
        flush()
        fwd()
        bwd()
    torch.cuda.synchronize()
    barrier(world)
    n = 5 if args.quick else 20
    ms_f = time_steps(fwd, n, flush, stream)
    ms_b = time_steps(bwd, n, flush, stream)
    barrier(world)
    tf = max_over_ranks(sum(ms_f), world) / n
    tb = max_over_ranks(sum(ms_b), world) / n
    # forward: x, W, q in; eta, g, qhat out.  backward: x, W, q, eta, g, deta, dg, dqhat in;
    # dx, dq, dW, dbias out (fp32), plus the per-tile partial sums written and read once
    fb = N * D * 2 + 2 * H * D * 2 + 2 * N * H * Dk * 2 + 2 * N * H * 4
    bb = N * D * 2 + N * H * Dk * 2 + 4 * N * H * 4 + N * H * Dk * 4 + N * D * 4 + N * H * Dk * 4
    tokens = sum_over_ranks(float(N), world)
    return {"shape": {"N": N, "D": D, "H": H, "Dk": Dk, "dtype": "bf16"},
            "value": tokens / (tf / 1e3), "unit": "tokens/s", "us_per_call": tf * 1e3,
            "gpu_launches_per_step": 2, "l2": "flushed between timed steps",
            "roofline": {"bound": "hbm", "achieved": fb / (tf / 1e3) / 1e9, "peak": hbm_peak, "unit": "GB/s",
                         "frac": fb / (tf / 1e3) / 1e9 / hbm_peak, "alg_bytes_per_launch": fb},
            "backward": {"us_per_call": tb * 1e3, "gpu_launches_per_step": 3,
                         "roofline": {"bound": "hbm", "achieved": bb / (tb / 1e3) / 1e9, "peak": hbm_peak,
                                      "unit": "GB/s", "frac": bb / (tb / 1e3) / 1e9 / hbm_peak,
                                      "alg_bytes_per_launch": bb}}}


def bench_e2e(kla, w, inp, dev, stream, rank, world, args):
    """Same metric through the public API from pinned host buffers: every step's inputs go
    host -> device, kla_chunk_fwd runs, and o and S_T come back device -> host, all inside the
    timed region.  Steps are pipelined the way a serving loop would run them: two buffer sets,
    inputs of step i + 1 copied on their own stream while step i computes and its results
    are copied back, so the two copy directions and the kernels overlap."""
    import torch
    names = ["q", "k", "v", "eta", "g"]
    host = {n: inp[n].pin_memory() for n in names}
    nbuf = 2
    devb = [{n: torch.empty_like(host[n], device=dev) for n in names} for _ in range(nbuf)]
    outs = [(torch.empty(w.B, w.T, w.H, w.Dv, device=dev), torch.empty(w.B, w.H, w.Dk, w.Dv, device=dev))
            for _ in range(nbuf)]
    o_h = [torch.empty(w.B, w.T, w.H, w.Dv, dtype=torch.float32).pin_memory() for _ in range(nbuf)]
    ST_h = [torch.empty(w.B, w.H, w.Dk, w.Dv, dtype=torch.float32).pin_memory() for _ in range(nbuf)]
    ws = kla.fwd_workspace(devb[0]["k"], devb[0]["v"])
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev = lambda: torch.cuda.Event()
    in_ready = [ev() for _ in range(nbuf)]
    in_free = [ev() for _ in range(nbuf)]    # the step that used this input set has computed
    out_ready = [ev() for _ in range(nbuf)]  # o, S_T of this set computed
    out_free = [ev() for _ in range(nbuf)]   # o, S_T of this set copied back

    def run(nsteps):
        for i in range(nsteps):
            j = i % nbuf
            with torch.cuda.stream(s_in):
                if i >= nbuf:
                    s_in.wait_event(in_free[j])
                for n in names:
                    devb[j][n].copy_(host[n], non_blocking=True)
                in_ready[j].record(s_in)
            stream.wait_event(in_ready[j])
            if i >= nbuf:
                stream.wait_event(out_free[j])
            o, ST = outs[j]
            kla.chunk_fwd(devb[j]["q"], devb[j]["k"], devb[j]["v"], devb[j]["eta"], devb[j]["g"], w.eps, None,
                          o=o, S_T=ST, workspace=ws, stream=stream)
            in_free[j].record(stream)
            out_ready[j].record(stream)
            with torch.cuda.stream(s_out):
                s_out.wait_event(out_ready[j])
                o_h[j].copy_(o, non_blocking=True)
                ST_h[j].copy_(ST, non_blocking=True)
                out_free[j].record(s_out)
        stream.wait_stream(s_in)
        stream.wait_stream(s_out)

    run(2)
    torch.cuda.synchronize()
    barrier(world)
    nsteps = 4 if args.quick else 12
    st, en = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    st.record(stream)
    s_in.wait_stream(stream)
    s_out.wait_stream(stream)
    run(nsteps)
    en.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    ms = max_over_ranks(st.elapsed_time(en), world)
    tokens = sum_over_ranks(float(w.B * w.T), world) * nsteps
    h2d = sum(host[n].numel() * host[n].element_size() for n in names)
    d2h = o_h[0].numel() * o_h[0].element_size() + ST_h[0].numel() * 4
    return {"value": tokens / (ms / 1e3), "unit": "tokens/s", "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h, "steps": nsteps,
            "pipelining": "2 buffer sets; H2D, kernels and D2H on separate streams"}


def oracle_sample(workload_name, npairs, seed_offset=0):
    """Inputs of `npairs` (b, h) pairs of the workload, as fp64 arrays [npairs, T, 1, D]."""
    import numpy as np
    from gated_delta_rule_kla_b200.workloads import WORKLOADS, make_inputs
    w = WORKLOADS[workload_name]
    w = w.with_(seed=w.seed + seed_offset)
    inp = make_inputs(w)
    pairs = [(i % w.B, (i * 5) % w.H) for i in range(npairs)]

    def sel(x, state=False):
        if x is None:
            return None
        x = x.double().numpy()
        if state:
            return np.ascontiguousarray(np.stack([x[b, h] for b, h in pairs])[:, None])
        return np.ascontiguousarray(np.stack([x[b, :, h] for b, h in pairs])[:, :, None])

    return w, [sel(inp[n]) for n in ("q", "k", "v", "eta", "g")], sel(inp["S0"], True)


def cpu_baseline(workload_name, npairs):
    import oracle
    w, args, S0 = oracle_sample(workload_name, npairs)
    oracle.forward(*[a[:1, :64] for a in args], w.eps, None if S0 is None else S0[:1])  # load
    t0 = time.perf_counter()
    oracle.forward(*args, w.eps, S0)
    dt = time.perf_counter() - t0
    tokens = npairs * w.T / w.H  # (b, h) pairs -> whole-token equivalents
    return {"value": tokens / dt, "unit": "tokens/s", "cores": oracle.threads(), "kind": "oracle",
            "sample": f"{npairs} of {w.B * w.H} (batch, head) pairs of {w.name}, full T={w.T}, "
                      f"fp64 token recurrence; {dt:.2f} s"}


def reference_arm(args, world):
    import oracle
    w, inputs, S0 = oracle_sample(args.workload, args.ref_pairs)
    oracle.forward(*[a[:1, :64] for a in inputs], w.eps, None)
    for _ in range(args.warmup if args.warmup <= 1 else 1):
        oracle.forward(*[a[:1] for a in inputs], w.eps, None)
    times = []
    for _ in range(args.steps):
        t0 = time.perf_counter()
        oracle.forward(*inputs, w.eps, S0)
        times.append(time.perf_counter() - t0)
    tokens = args.ref_pairs * w.T / w.H * args.steps
    value = tokens / sum(times)
    sample = (f"{args.ref_pairs} of {w.B * w.H} (batch, head) pairs of {w.name} per step, "
              f"full T={w.T}, fp64 token recurrence")
    return {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": 1e3 * sum(times) / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic (seeded; shapes of the paper's 0.4B model, App. C)",
            "config": {"workload": w.name, "B": w.B, "T": w.T, "H": w.H, "Dk": w.Dk, "Dv": w.Dv},
            "impl": "reference",
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": oracle.threads(),
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


# ---------------------------------------------------------------------------------------
def parse(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["kla", "reference"], default="kla")
    ap.add_argument("--workload", default="prefill_b8_t2048_h8_d128")
    ap.add_argument("--ref-pairs", type=int, default=16,
                    help="(b,h) pairs per reference step (at least the host's cores, so none idles)")
    ap.add_argument("--cpu-pairs", type=int, default=64, help="(b,h) pairs in the CPU baseline sample")
    ap.add_argument("--skip-extra", action="store_true", help="headline prefill only")
    ap.add_argument("--parts", default="decode,train,long,direct,diag,gates",
                    help="sub-measurements after the headline prefill (comma list of "
                         "decode,train,long,direct,diag,gates)")
    ap.add_argument("--skip-e2e", action="store_true", help="omit the host-buffer end-to-end leg")
    ap.add_argument("--skip-cpu", action="store_true", help="omit the CPU baseline")
    ap.add_argument("--quick", action="store_true", help="fewer decode/train steps (smoke runs)")
    return ap.parse_args(argv)


def main(argv=None):
    args = parse(argv)
    rank, world, local_rank = dist_env()
    if args.warmup < 3 and args.impl == "kla":
        args.warmup = 3  # timing rule: at least 3 warm-up steps
    if args.impl == "reference":
        if rank != 0:
            return 0
        print(json.dumps(reference_arm(args, world)), flush=True)
        return 0
    import torch
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    try:
        line = gpu_arm(args, rank, world, local_rank)
        if rank == 0:
            if not args.skip_cpu:
                line["cpu_baseline"] = cpu_baseline(args.workload, args.cpu_pairs)
            print(json.dumps(line), flush=True)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
