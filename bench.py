#!/usr/bin/env python
"""Benchmark of the capacity-limited MoE layer forward on B200.

One step = one ``moe_forward`` call (router logits, softmax/top-k, capacity selection and
dispatch, expert GEMM1 + SiLU, expert GEMM2, combine) over one batch of synthetic tokens whose
inputs are already in HBM.  Default workload: the skewed E=64 top-6 layer (T=16384,
d_model=2048, d_ff=1408, capacity factor 1.0).  Under torchrun each rank runs its own batch
(independent problems, no data-path collective): weak scaling, time = max over ranks.

``--impl reference`` times the CPU oracle on the host cores instead (a bounded sample of the
same workload per step, extrapolated to the whole batch).
"""
import argparse
import dataclasses
import datetime
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from expert_ffn_layer_router_b200 import inputs  # noqa: E402

METRIC = "MoE-layer tokens/s; expert grouped-GEMM TFLOP/s as % of B200 bf16 dense peak"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
L2_FLUSH_BYTES = 256 << 20


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="cuda", choices=["cuda", "reference"])
    ap.add_argument("--config", default="skewed_e64_top6", choices=inputs.CONFIG_ORDER)
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--cpu-seconds", type=float, default=15.0,
                    help="target CPU time of the oracle baseline sample")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--min-warmup-s", type=float, default=0.5,
                    help="warm-up lasts at least this long (clock sampler coverage)")
    ap.add_argument("--tokens", type=int, default=None,
                    help="override the workload's token count (profiling of smaller cases)")
    ap.add_argument("--gated", action="store_true",
                    help="gated experts (SiLU(gate) * up, W1 twice as tall) on the same shapes")
    ap.add_argument("--drop-policy", default="weight", choices=["weight", "arrival"],
                    help="capacity selection: lowest router weight dropped first (default) or"
                         " the first K pairs of each expert in token order kept")
    ap.add_argument("--ep", action="store_true",
                    help="expert-parallel layer: experts split over the ranks, NCCL all-to-all")
    ap.add_argument("--renormalize", action="store_true",
                    help="top-k weights renormalised to sum to 1 before the capacity selection")
    return ap.parse_args()


def max_over_ranks(value, dist=None, device=None):
    """Largest per-rank value (times are taken as the slowest rank); identity on one rank."""
    if dist is None or not dist.is_available() or not dist.is_initialized() or \
            dist.get_world_size() == 1:
        return float(value)
    import torch
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def layer_flags(spec, args):
    """The layer's flag word (same bit values in the library and the oracle): 1 renormalised
    top-k weights, 2 arrival-order capacity, 4 gated experts."""
    return ((1 if getattr(args, "renormalize", False) else 0)
            | (2 if getattr(args, "drop_policy", "weight") == "arrival" else 0)
            | (4 if spec.gated else 0))


def workload_desc(spec, flags=0):
    C = "dropless" if math.isinf(spec.C) else "C=%g" % spec.C
    return "%s: T=%d, d_model=%d, d_ff=%d, E=%d, top-%d, %s, %s%s%s%s" % (
        spec.name, spec.T, spec.d_model, spec.d_ff, spec.E, spec.k, C, spec.dtype,
        ", gated experts" if spec.gated else "",
        ", arrival-order capacity" if flags & 2 else "",
        ", renormalised top-k weights" if flags & 1 else "")


# ------------------------------------------------------------------------------------------------
# CPU oracle timing (the reference arm and the cpu_baseline object)
# ------------------------------------------------------------------------------------------------
def oracle_step(L, spec, sample, nthreads, flags=0):
    """Time the oracle on one bounded sample; returns (seconds extrapolated to T tokens, info)."""
    import oracle
    T = spec.T
    rng = np.random.default_rng(sample)
    toks = np.sort(rng.choice(T, size=sample, replace=False)).astype(np.int32)
    t0 = time.perf_counter()
    Ls = oracle.logits(L["x"][toks], L["Wr"], L["br"], nthreads) if L["logits"] is None else \
        L["logits"][toks]
    t_logits = time.perf_counter() - t0
    # Routing needs the whole batch (capacity competition is per batch): logits of the batch
    # are formed once outside the timing, and the route itself is timed on all T tokens.
    full = L["_full_logits"]
    t0 = time.perf_counter()
    K = oracle.capacity(T, spec.E, spec.k, spec.C)
    r = oracle.route(full, spec.k, K, flags & (oracle.RENORMALIZE | oracle.ARRIVAL_ORDER))
    t_route = time.perf_counter() - t0
    t0 = time.perf_counter()
    oracle.combine_tokens(L["x"], L["W1"], L["b1"], L["W2"], L["b2"], r, toks, nthreads,
                          flags=flags & oracle.GATED)
    t_ffn = time.perf_counter() - t0
    del Ls
    est = (t_logits + t_ffn) * T / sample + t_route
    return est, dict(t_logits=t_logits, t_route=t_route, t_ffn=t_ffn,
                     measured=t_logits + t_route + t_ffn)


def prepare_oracle_inputs(L, spec, nthreads):
    import oracle
    if L["logits"] is not None:
        L["_full_logits"] = L["logits"]
    else:
        L["_full_logits"] = oracle.logits(L["x"], L["Wr"], L["br"], nthreads)


def calibrate_sample(L, spec, target_s, nthreads, flags=0):
    """Tokens per sample so that one oracle step takes about target_s seconds."""
    s = max(1, min(spec.T, 8))
    est, info = oracle_step(L, spec, s, nthreads, flags)
    per_tok = max((info["t_logits"] + info["t_ffn"]) / s, 1e-6)
    budget = max(target_s - info["t_route"], 0.05)
    return int(max(1, min(spec.T, budget / per_tok)))


def cpu_cores():
    try:
        return len(os.sched_getaffinity(0))
    except Exception:
        return os.cpu_count() or 1


def bench_spec(args):
    """The workload of this run: the named configuration with --tokens and --gated applied."""
    spec = inputs.CONFIGS[args.config]
    if args.tokens:
        spec = dataclasses.replace(spec, T=args.tokens)
    if args.gated:
        spec = dataclasses.replace(spec, gated=True)
    return spec


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    spec = bench_spec(args)
    flags = layer_flags(spec, args)
    L = inputs.make_layer(spec, seed=args.seed)
    cores = cpu_cores()
    prepare_oracle_inputs(L, spec, cores)
    step_budget = max(0.2, min(8.0, 150.0 / max(1, args.steps + args.warmup)))
    sample = calibrate_sample(L, spec, step_budget, cores, flags)
    for _ in range(args.warmup):
        oracle_step(L, spec, sample, cores, flags)
    ests, meas = [], []
    for _ in range(args.steps):
        est, info = oracle_step(L, spec, sample, cores, flags)
        ests.append(est)
        meas.append(info["measured"])
    t = statistics.mean(ests)
    value = spec.T / t
    desc = ("oracle on %d of %d tokens per step (logits + expert FFN + combine, scaled by T/%d)"
            " plus routing of all %d tokens" % (sample, spec.T, sample, spec.T))
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": t * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": workload_desc(spec, flags), "seed": args.seed},
            "cpu_baseline": {"kind": "oracle", "cores": cores, "sample": desc, "value": value,
                             "unit": "tokens/s"},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0},
            "measured_seconds_per_step": statistics.mean(meas),
            "sample_tokens_per_step": sample,
            "timing_note": "ms_per_step extrapolates each step's timed sample to all T tokens;"
                           " measured_seconds_per_step is the time actually spent per step"}
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------------------------------------------
# Clock sampling during the timed region
# ------------------------------------------------------------------------------------------------
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, uuid):
        self.uuid = uuid
        self.proc = None
        self.f = tempfile.TemporaryFile(mode="w+")

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", self.uuid, "--query-gpu=" + self.FIELDS,
                 "--format=csv,noheader,nounits", "-lms", "50"], stdout=self.f,
                stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.f.seek(0)
        sm, smax, reasons, power = [], [], set(), []
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in self.f.read().splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax.append(float(parts[2]))
                power.append(float(parts[3]))
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(smax),
                "reasons": sorted(reasons), "samples": len(sm),
                "power_w_max": max(power) if power else None}


# ------------------------------------------------------------------------------------------------
# The CUDA arm
# ------------------------------------------------------------------------------------------------
def to_dev(a, torch, dev):
    if a is None:
        return None
    if a.dtype == np.uint16:
        return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).to(dev)
    return torch.from_numpy(np.ascontiguousarray(a)).to(dev)


def kernel_source_hash():
    """sha256[:16] over the GEMM kernel's sources (gemm_tc.cu, then common.cuh)."""
    csrc = os.path.join(ROOT, "expert_ffn_layer_router_b200", "csrc")
    h = hashlib.sha256()
    for name in ("gemm_tc.cu", "common.cuh"):
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def traffic_record(kernel, workload):
    """dram bytes per launch from the committed ncu summary, if taken on the current source and
    on this workload."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        rec = json.load(f)
    h = kernel_source_hash()
    r = rec.get(kernel)
    if not r or r.get("source_sha256_16") != h or r.get("workload") != workload:
        return None
    return r.get("bytes_per_launch")


def run_cuda(args):
    import torch
    import torch.distributed as dist

    from expert_ffn_layer_router_b200 import moe

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        raise SystemExit("--gpus %d but WORLD_SIZE=%d" % (args.gpus, world))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=dev)

    spec = bench_spec(args)
    flags = layer_flags(spec, args)
    L = inputs.make_layer(spec, seed=args.seed + rank)
    layer = moe.MoELayer(spec.T, spec.d_model, spec.d_ff, spec.E, spec.k, spec.C, spec.dtype,
                         device=dev, flags=flags)
    names = ("x", "Wr", "br", "W1", "b1", "W2", "b2")
    d = {n: to_dev(L[n], torch, dev) for n in names}
    # The router weights are constant: their two bf16 terms are formed once, as a serving
    # deployment forms them when it loads the weights (a no-op where the router does not use them).
    layer.prepare_router(d["Wr"])
    out = torch.empty_like(d["x"])
    counts = torch.empty(2 * spec.E, dtype=torch.int32, device=dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()

    def step(ev=None):
        moe.moe_forward(layer.p, d["x"], d["Wr"], d["br"], d["W1"], d["b1"], d["W2"], d["b2"],
                        out, layer.ws, counts_out=counts)

    uuid = str(torch.cuda.get_device_properties(dev).uuid)
    sampler = ClockSampler(uuid if uuid.startswith("GPU-") else "GPU-" + uuid)
    # The clock sampler runs from the warm-up through the timed steps (same load); warm-up lasts
    # at least W steps and at least half a second so the sampler sees the part under load.
    # Timed region: K steps, L2 flushed before each (outside the step's events).  The headline
    # steps carry only a start and an end event; a second, instrumented run of K steps records
    # an event between every stage (moe_set_stage_events) for the per-kernel durations.  Stage
    # events cost the GPU about 2.5 us each, so the headline is taken without them.  All events
    # are created before the warm-up (torch creates a CUDA event at its first record), so the GPU
    # idles only for the synchronisation and barrier between the warm-up and the timed steps.
    K = args.steps
    ev_sets = {inst: [[torch.cuda.Event(enable_timing=True)
                       for _ in range(moe.STAGE_EVENTS if inst else 2)] for _ in range(K)]
               for inst in (False, True)}
    for rows in ev_sets.values():
        for row in rows:
            for e in row:
                e.record(stream)
    torch.cuda.synchronize()

    sampler.start()
    t_end = time.perf_counter() + args.min_warmup_s
    n_warm = 0
    while n_warm < max(args.warmup, 3) or time.perf_counter() < t_end:
        flush.zero_()
        step()
        n_warm += 1
        if n_warm % 8 == 0:
            torch.cuda.synchronize()
    launches_per_step = moe.moe_last_launch_count()

    def timed_steps(instrumented):
        evs = ev_sets[instrumented]
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        for i in range(K):
            flush.zero_()
            if instrumented:
                moe.moe_set_stage_events(evs[i])
                step()
            else:
                evs[i][0].record(stream)
                step()
                evs[i][1].record(stream)
        if instrumented:
            moe.moe_set_stage_events(None)
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        return evs

    evs_plain = timed_steps(False)
    evs = timed_steps(True)
    clocks = sampler.stop()
    kept = int(counts[spec.E:].sum().item())
    received = int(counts[:spec.E].sum().item())
    stage_ms = np.zeros((K, moe.STAGE_EVENTS - 1))
    for i in range(K):
        for s in range(moe.STAGE_EVENTS - 1):
            stage_ms[i, s] = evs[i][s].elapsed_time(evs[i][s + 1])
    step_ms = np.array([evs_plain[i][0].elapsed_time(evs_plain[i][1]) for i in range(K)])
    instr_ms = np.array([evs[i][0].elapsed_time(evs[i][-1]) for i in range(K)])
    total_ms = max_over_ranks(float(step_ms.sum()), dist if world > 1 else None, dev)
    ms_per_step = total_ms / K
    value = world * spec.T / (ms_per_step / 1e3)
    # End to end through the C ABI with host buffers, as a serving loop runs it: every step
    # copies its x from pinned host memory to the device, runs the layer and copies its output
    # back to pinned host memory.  Copy-in, compute and copy-out run on three streams with
    # double-buffered device x/out, so step i's copies overlap steps i-1 and i+1.
    x_host = d["x"].cpu().pin_memory()
    out_host = [torch.empty_like(x_host).pin_memory() for _ in range(2)]
    xd = [torch.empty_like(d["x"]) for _ in range(2)]
    od = [torch.empty_like(d["x"]) for _ in range(2)]
    s_in, s_cmp, s_out = (torch.cuda.Stream(device=dev) for _ in range(3))
    ev = lambda: torch.cuda.Event(enable_timing=False)
    h2d_done = [ev() for _ in range(K)]
    cmp_done = [ev() for _ in range(K)]
    d2h_done = [ev() for _ in range(K)]
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    e0.record(s_in)
    for i in range(K):
        b = i % 2
        if i >= 2:
            s_in.wait_event(cmp_done[i - 2])             # xd[b] no longer read
        with torch.cuda.stream(s_in):
            xd[b].copy_(x_host, non_blocking=True)
        h2d_done[i].record(s_in)
        s_cmp.wait_event(h2d_done[i])
        if i >= 2:
            s_cmp.wait_event(d2h_done[i - 2])            # od[b] already copied out
        moe.moe_forward(layer.p, xd[b], d["Wr"], d["br"], d["W1"], d["b1"], d["W2"], d["b2"],
                        od[b], layer.ws, stream=s_cmp)
        cmp_done[i].record(s_cmp)
        s_out.wait_event(cmp_done[i])
        with torch.cuda.stream(s_out):
            out_host[b].copy_(od[b], non_blocking=True)
        d2h_done[i].record(s_out)
    s_in.wait_event(d2h_done[K - 1])
    e1.record(s_in)
    e1.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), dist if world > 1 else None, dev)
    e2e_value = world * spec.T / (e2e_ms / K / 1e3)
    # The last step's output must equal the device-timed path's output (same inputs).
    assert torch.equal(out_host[(K - 1) % 2], out.cpu()), "e2e output differs"
    assert moe.moe_get_device_status(layer.ws) == 0, "device status word reports an error"

    # Roofline bookkeeping (algorithmic work per launch).
    pk, pk_kind = peaks()
    esz = 2 if spec.dtype == "bf16" else 4
    T, dm, F, E, k = spec.T, spec.d_model, spec.d_ff, spec.E, spec.k
    st_avg = stage_ms.mean(axis=0)
    names6 = moe.STAGE_NAMES
    gemm_flop_each = 2.0 * kept * dm * F
    g1_flop = gemm_flop_each * (2 if spec.gated else 1)
    # Algorithmic work per stage (the method's, not the implementation's): the router's flops
    # are 2 T d E; bytes count every input read once and every output written once.  Small bf16
    # batches with the single-block dispatch (T <= 1024, T k <= 1024) compute logits and routing
    # in one launch: the router stage reads x and Wr and writes ids and weights, and the top-k
    # stage is empty.  Otherwise the logits round-trip through HBM between the two stages.
    router_routes = (spec.dtype == "bf16" and T <= 1024 and E <= 256 and dm <= 12288
             and T * k <= 1024)
    router_out = T * k * 8 if router_routes else T * E * 4
    by = {
        "router_logits": dict(flop=2.0 * T * dm * E, bytes=T * dm * esz + dm * E * 4 + router_out),
        "route_topk": dict(bytes=0 if router_routes else T * E * 4 + T * k * 8),
        "capacity_dispatch": dict(bytes=T * k * 8 + T * k * 5 + kept * 4 + E * 16),
        "expert_gemm1": dict(flop=g1_flop,
                             bytes=T * dm * esz + E * F * dm * esz * (2 if spec.gated else 1)
                             + kept * F * esz),
        "expert_gemm2": dict(flop=gemm_flop_each,
                             bytes=kept * F * esz + E * dm * F * esz + kept * dm * esz),
        "combine": dict(bytes=2 * T * dm * esz + kept * dm * esz + T * k * 12 + (E + 1) * 4),
    }
    input_bytes = sum(int(t.numel() * t.element_size()) for t in d.values() if t is not None)
    traffic_key = spec.name + (" gated" if spec.gated else "") + \
        (" T=%d" % spec.T if args.tokens else "") + (" flags=%d" % (flags & 3) if flags & 3 else "")
    kernels = {}
    for i, n in enumerate(names6):
        ms = float(st_avg[i])
        rec = {"ms": ms}
        if "flop" in by[n]:
            rec["tflops"] = by[n]["flop"] / (ms * 1e-3) / 1e12 if ms > 0 else None
        rec["gbs"] = by[n]["bytes"] / (ms * 1e-3) / 1e9 if ms > 0 else None
        kernels[n] = rec
    tensor_peak = pk.get("bf16_tflops_sustained", pk.get("bf16_tflops"))
    g1, g2 = kernels["expert_gemm1"], kernels["expert_gemm2"]
    dom = "expert_gemm1" if g1["ms"] >= g2["ms"] else "expert_gemm2"
    # The dominant kernel's bound: tensor cores when its flops per algorithmic byte exceed the
    # ridge point of the two peaks (cfg3: ~780 flop/B against a ridge of ~210), HBM otherwise
    # (decode: each expert's weights serve ~8 rows, ~8 flop/B).
    ridge = tensor_peak * 1e12 / (pk["hbm_gbs"] * 1e9)
    hbm_bound = by[dom]["flop"] / by[dom]["bytes"] < ridge
    if hbm_bound:
        roofline = {"bound": "hbm", "kernel": dom, "achieved": kernels[dom]["gbs"],
                    "peak": pk["hbm_gbs"], "unit": "GB/s",
                    "frac": kernels[dom]["gbs"] / pk["hbm_gbs"] if kernels[dom]["gbs"] else None,
                    "peak_source": "%s hbm_gbs (copy bandwidth)" % pk_kind,
                    "algorithmic_bytes_per_launch": by[dom]["bytes"]}
    else:
        achieved = kernels[dom]["tflops"]
        roofline = {"bound": "tensor", "kernel": dom, "achieved": achieved,
                    "peak": tensor_peak, "unit": "TFLOP/s",
                    "frac": achieved / tensor_peak if achieved else None,
                    "peak_source": "%s bf16_tflops_sustained (kernel timed inside a long"
                                   " loop of steps)" % pk_kind,
                    "algorithmic_flop_per_launch": by[dom]["flop"]}
    roofline["traffic"] = traffic_record(dom, traffic_key)
    gemm_ms = g1["ms"] + g2["ms"]
    gemm_tflops = (g1_flop + gemm_flop_each) / (gemm_ms * 1e-3) / 1e12
    rdc_stages = ("router_logits", "route_topk", "capacity_dispatch", "combine")
    rdc_bytes = sum(by[n]["bytes"] for n in rdc_stages)
    rdc_ms = sum(kernels[n]["ms"] for n in rdc_stages)
    rdc_gbs = rdc_bytes / (rdc_ms * 1e-3) / 1e9
    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": K,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16" if spec.dtype == "bf16" else "f32",
        "data": "synthetic (seeded numpy draws; random-init weights of the stated shape)",
        "config": {"workload": workload_desc(spec, flags), "seed": args.seed + rank,
                   "per_rank_tokens": T, "parallelism": "dp%d (independent batches)" % world,
                   "l2": "flushed before every timed step (256 MiB write, outside the step's"
                         " events); per-step inputs %.0f MB" % (input_bytes / 1e6),
                   "timing": "value: K steps with start/end events only; kernels and roofline:"
                             " a second run of K steps with an event between stages; the timed"
                             " steps follow the warm-up with no idle gap (sustained,"
                             " power-capped state)",
                   "router_weights": "split into two bf16 terms once, before the timed steps"
                                     " (moe_prepare_router)",
                   "kept_pairs": kept, "received_pairs": received,
                   "dropped_pairs": received - kept},
        "gpu_launches": launches_per_step * K,
        "warmup_steps_run": n_warm,
        "gpu_launches_per_step": launches_per_step,
        "clocks": clocks,
        "e2e": {"value": e2e_value, "unit": "tokens/s",
                "h2d_bytes_per_step": int(x_host.numel() * x_host.element_size()),
                "d2h_bytes_per_step": int(out_host[0].numel() * out_host[0].element_size()),
                "ms_per_step": e2e_ms / K,
                "pipeline": "copy-in / compute / copy-out streams, double-buffered device x and"
                            " out; pinned host buffers"},
        "roofline": roofline,
        "expert_gemm": {"tflops": gemm_tflops, "frac_of_peak": gemm_tflops / tensor_peak,
                        "frac_of_burst_peak": gemm_tflops / pk.get("bf16_tflops", tensor_peak),
                        "flop_per_step": g1_flop + gemm_flop_each},
        "route_dispatch_combine": {"gbs": rdc_gbs, "frac_of_hbm": rdc_gbs / pk["hbm_gbs"],
                                   "bytes_per_step": rdc_bytes, "hbm_peak_gbs": pk["hbm_gbs"],
                                   "stages": list(rdc_stages),
                                   "router_stage_routes": router_routes},
        "kernels": kernels,
        "step_ms_min": float(step_ms.min()), "step_ms_median": float(np.median(step_ms)),
        "step_ms_each": [round(float(v), 4) for v in step_ms],
        "instrumented_ms_per_step": float(instr_ms.mean()),
    }
    if world == 1 and rank == 0 and not args.no_cpu_baseline:
        cores = cpu_cores()
        prepare_oracle_inputs(L, spec, cores)
        sample = calibrate_sample(L, spec, max(1.0, args.cpu_seconds / 3), cores, flags)
        ests = [oracle_step(L, spec, sample, cores, flags)[0] for _ in range(3)]
        cv = spec.T / statistics.mean(ests)
        line["cpu_baseline"] = {
            "value": cv, "unit": "tokens/s", "cores": cores, "kind": "oracle",
            "sample": "3 runs of the oracle on %d of %d tokens (logits + expert FFN + combine, "
                      "scaled by T/%d) plus routing of all %d tokens" % (sample, T, sample, T)}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def run_ep(args):
    """--ep: the expert-parallel layer (expert_ffn_layer_router_b200/ep.py).  Every rank routes its
    own T tokens and owns E/N experts; candidates, x rows and expert outputs cross ranks by NCCL
    all-to-all.  The capacity is that of the whole N*T-token batch, so the result equals one
    device running the union of the batches.  Timed like the default mode (flush, events, max
    over ranks); value = N*T / step time."""
    import torch
    import torch.distributed as dist

    from expert_ffn_layer_router_b200 import moe
    from expert_ffn_layer_router_b200.ep import ExpertParallelLayer

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        raise SystemExit("--gpus %d but WORLD_SIZE=%d" % (args.gpus, world))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
    os.environ.setdefault("MASTER_PORT", "29533")
    dist.init_process_group("nccl", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=300), device_id=dev)
    spec = bench_spec(args)
    flags = layer_flags(spec, args)
    if spec.E % world:
        raise SystemExit("--ep needs E (%d) to be a multiple of the number of GPUs" % spec.E)
    T = spec.T
    # One global layer of world*T tokens: rank r holds tokens [rT, (r+1)T) and experts
    # [r E/N, (r+1) E/N).
    L = inputs.make_layer(dataclasses.replace(spec, T=world * T), seed=args.seed)
    El = spec.E // world
    ts, es = slice(rank * T, (rank + 1) * T), slice(rank * El, (rank + 1) * El)
    d = {"x": to_dev(L["x"][ts], torch, dev), "Wr": to_dev(L["Wr"], torch, dev),
         "br": to_dev(L["br"], torch, dev)}
    for n in ("W1", "b1", "W2", "b2"):
        d[n] = to_dev(L[n][es], torch, dev)
    del L
    ep = ExpertParallelLayer(dist.group.WORLD, T, spec.d_model, spec.d_ff, spec.E, spec.k, spec.C,
                             spec.dtype, dev, flags)
    ep.steps.router.prepare_router(d["Wr"])
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()

    def step():
        return ep.forward(d["x"], d["Wr"], d["br"], d["W1"], d["b1"], d["W2"], d["b2"])

    uuid = str(torch.cuda.get_device_properties(dev).uuid)
    sampler = ClockSampler(uuid if uuid.startswith("GPU-") else "GPU-" + uuid)
    K = args.steps
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(K)]
    for row in evs:                       # created before the warm-up, as in the default mode
        for e in row:
            e.record(stream)
    sampler.start()
    for _ in range(max(args.warmup, 3)):
        flush.zero_()
        step()
    torch.cuda.synchronize()
    dist.barrier()
    torch.cuda.synchronize()
    l0 = ep.steps.launches
    for i in range(K):
        flush.zero_()
        evs[i][0].record(stream)
        out, r = step()
        evs[i][1].record(stream)
    torch.cuda.synchronize()
    dist.barrier()
    clocks = sampler.stop()
    launches = ep.steps.launches - l0
    step_ms = np.array([evs[i][0].elapsed_time(evs[i][1]) for i in range(K)])
    total_ms = max_over_ranks(float(step_ms.sum()), dist if world > 1 else None, dev)
    ms_per_step = total_ms / K
    kept = int((r["slot"] >= 0).sum().item())
    line = {
        "metric": METRIC, "value": world * T / (ms_per_step / 1e3), "unit": "tokens/s",
        "n_gpus": world, "steps": K, "warmup": args.warmup, "ms_per_step": ms_per_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16" if spec.dtype == "bf16" else "f32",
        "data": "synthetic (seeded numpy draws; random-init weights of the stated shape)",
        "mode": "expert-parallel",
        "config": {"workload": workload_desc(spec, flags), "seed": args.seed,
                   "per_rank_tokens": T, "experts_per_rank": El,
                   "parallelism": "ep%d (experts split over ranks; candidates, x rows and expert"
                                  " outputs by NCCL all-to-all; the whole batch's capacity)" % world,
                   "l2": "flushed before every timed step (256 MiB write, outside the step's"
                         " events)",
                   "kept_pairs_of_rank0_tokens": kept},
        "gpu_launches": launches,
        "gpu_launches_per_step": launches / K,
        "clocks": clocks,
        "step_ms_min": float(step_ms.min()), "step_ms_median": float(np.median(step_ms)),
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    dist.destroy_process_group()
    return 0


def main():
    args = parse()
    if args.impl == "reference":
        return run_reference(args)
    if args.ep:
        return run_ep(args)
    return run_cuda(args)


if __name__ == "__main__":
    sys.exit(main())
