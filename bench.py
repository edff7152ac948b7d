#!/usr/bin/env python
"""Throughput of the Dreamer depth-recurrent core forward on B200.

Metric: token-depth-steps per second (one unit = one token through one depth step) of the
full L-depth forward, bf16, and its fraction of the roofline
T_roof = max(F_alg / tensor peak, B_alg / HBM peak) with both peaks measured on B200: the HBM
copy bandwidth, and the bf16 GEMM rate sustained under the power cap for a timed loop of a
second or more (the burst rate for a shorter one; the other one is reported beside it).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--config large|medium|small|decode|...]

The default workload is the large one (b 2, s 8192, h 2048, 16x128 heads, L 64, E 2048,
k 8, m 64, 16 linear-MoE projection experts): the largest that runs on one GPU.
  python bench.py --impl reference ...     # the CPU oracle, timed on the host cores

N > 1 runs one replica per GPU (torchrun, one rank per GPU): sequences are independent,
each rank runs the whole configured batch (weak scaling), nothing crosses ranks on the data
path; the timed region is the max over ranks.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

from depth_recurrent_attention_b200 import configs, inputs  # noqa: E402

METRIC = "Dreamer core fwd token·depth-steps/s (bf16, 1×B200) and % of roofline"
UNIT = "token-depth-steps/s"
L2_BYTES = 126 * 1024 * 1024


# ----------------------------------------------------------------------------------------
# roofline accounting (algorithmic work of one forward)

def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return dict(hbm=float(p["hbm_gbs"]), tc=float(p["bf16_tflops"]),
                    tc_sust=float(p["bf16_tflops_sustained"]), source="measured")
    except Exception:
        return dict(hbm=6650.0, tc=1590.0, tc_sust=1400.0, source="fallback")


def tensor_peaks(pk, timed_ms: float):
    """(peak held to, the other peak, its kind) in TFLOP/s: the sustained GEMM figure when the
    timed region is a loop of a second or more (the GPU then runs at its power cap, as the
    sustained figure was measured), the burst figure for a shorter one."""
    if timed_ms >= 1000.0:
        return pk["tc_sust"], pk["tc"], "sustained"
    return pk["tc"], pk["tc_sust"], "burst"


def algorithmic(cfg, counts=None):
    """Per-stage algorithmic FLOPs and HBM bytes of one full forward (or decode step), by the
    accounting of the roofline: every multiply-add of a contraction counted twice at tensor
    rate (SA over the causal half only; routers 2 h d_r + 2 E d_r per token; non-tensor math
    not counted); bytes with perfect on-chip reuse inside a depth step and none across depths:
    weights once per depth (every projection expert; only the routed experts the run's own
    route counts touch), the residual x read and written once a depth, the DA keys/values
    written once (4h bytes a token) and re-read by every later depth (4h l), the SA keys/values
    written and read once (prefill) or the decode cache read once (4h per cached token).
    Bytes are attributed to the stage that moves them: qkv (x^ in, projection weights, DA and
    SA K/V out), da (earlier depths' K/V), sa (K/V in or the cache), o_proj and routers (their
    weights), experts (touched expert weights), finish (x out).  2-byte bf16 values."""
    b, s, h, L = cfg.batch, cfg.seq, cfg.hidden, cfg.depth
    E, k, m, dr, P = cfg.n_experts, cfg.top_k, cfg.expert_hidden, cfg.router_dim, cfg.n_proj_experts
    T = cfg.tokens
    es = 2 if cfg.dtype == "bf16" else 4
    G = max(P, 1)
    st = {}

    def add(name, fl, by):
        f0, b0 = st.get(name, (0.0, 0.0))
        st[name] = (f0 + fl, b0 + by)

    no_da = cfg.variant == 3
    nq = 3 if no_da else 6                                        # projection widths / h
    ko = 1 if no_da else 2                                        # O contraction width / h
    for l in range(L):
        if P > 0:
            add("proj_route", 2.0 * T * h * dr + 2.0 * T * P * dr, (h * dr + P * dr) * es)
        kv_out = (0 if no_da else 2 * T * h * es) + 2 * T * h * es   # DA and SA keys/values
        add("qkv", 2.0 * T * h * nq * h, T * h * es + G * nq * h * h * es + kv_out)
        if not no_da:
            ctx = l + 1 if cfg.da_window <= 0 else min(l + 1, cfg.da_window)
            add("da", 4.0 * T * h * ctx, 2.0 * T * h * es * (ctx - 1))
        if cfg.is_decode:
            n_ctx = cfg.cache_len + 1
            add("sa", 4.0 * T * h * n_ctx, 2.0 * T * h * es * cfg.cache_len)
        else:
            add("sa", 4.0 * h * b * s * (s + 1) / 2, 2.0 * T * h * es)
        add("o_proj", 2.0 * T * ko * h * h, G * ko * h * h * es)
        add("ea_route", 2.0 * T * h * dr + 2.0 * T * E * dr, (h * dr + E * dr) * es)
        touched = E
        if counts is not None:
            touched = int((np.asarray(counts)[l] > 0).sum())
        add("experts", 4.0 * T * k * h * m, 2.0 * touched * h * m * es)
        add("finish", 0.0, T * h * es)
    tot_f = sum(v[0] for v in st.values())
    tot_b = sum(v[1] for v in st.values())
    return st, tot_f, tot_b


# ----------------------------------------------------------------------------------------
# clocks sampled during the timed region

class ClockSampler:
    PERIOD_MS = 100
    MIN_SAMPLES = 10   # fewer samples than this over the timed region: flagged as too short
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
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.dev}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", str(self.PERIOD_MS)],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *a):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self):
        rows = []
        try:
            for line in open(self.path):
                parts = [p.strip() for p in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        except Exception:
            pass
        finally:
            try:
                os.unlink(self.path)
            except Exception:
                pass
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"]}

        def num(x):
            try:
                return float(x)
            except ValueError:
                return None
        sm = [num(r[1]) for r in rows if num(r[1]) is not None]
        mx = [num(r[2]) for r in rows if num(r[2]) is not None]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4)
                          if r[5 + i].lower() in ("active", "1")})
        out = {"sm_mhz": statistics.median(sm) if sm else None,
               "sm_max_mhz": max(mx) if mx else None, "reasons": reasons,
               "samples": len(rows), "period_ms": self.PERIOD_MS}
        if len(rows) < self.MIN_SAMPLES:
            out["too_short"] = True   # the median says little about the timed kernels' clock
        return out


# ----------------------------------------------------------------------------------------
# our arm

def measured_traffic(workload: str, stage: str):
    """DRAM bytes (read + write) per launch of the stage's kernel from the committed ncu
    summary (profiles/dram_traffic.json), or None where none was taken."""
    try:
        with open(os.path.join(ROOT, "profiles", "dram_traffic.json")) as f:
            return json.load(f).get(workload, {}).get(stage)
    except Exception:
        return None


# ----------------------------------------------------------------------------------------
# multi-rank host logic (one replica per GPU; tested on CPU with gloo ranks)

def rank_seed(cfg, rank: int) -> int:
    """Seed of rank `rank`'s input batch: every rank draws its own batch, weights are shared."""
    return cfg.seed + 1000 * rank


def max_over_ranks(x: float, dist, device) -> float:
    """The slowest rank's time: all-reduce MAX (no-op on one rank)."""
    if dist is None:
        return float(x)
    import torch
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_value(cfg, world: int, ms_per_step: float):
    """(units of the whole job per step, whole-job units/s): all ranks' units over the
    slowest rank's step time."""
    units = cfg.units * world
    return units, units / (ms_per_step / 1e3)


def device_setup(cfg, torch, rank):
    W = inputs.device_weights(cfg)
    X = inputs.device_inputs(cfg)
    if rank:
        X = {s.name: inputs.device_tensor(s, rank_seed(cfg, rank)) for s in inputs.input_specs(cfg)}
    return W, X


def run_ours(args, cfg, rank, world, torch, dist):
    from depth_recurrent_attention_b200.dreamer import Dreamer

    dev = torch.device("cuda", torch.cuda.current_device())
    W, X = device_setup(cfg, torch, rank)
    model = Dreamer(cfg, W)
    x_in = X["x0"]
    x_out = torch.empty_like(x_in)
    decode = cfg.is_decode
    if decode:
        lens = torch.full((cfg.batch,), cfg.cache_len, dtype=torch.int32, device=dev)
        kc, vc = X["k_cache"], X["v_cache"]

    def step(xi=x_in, xo=x_out):
        if decode:
            model.decode_step(xi, kc, vc, lens, x_out=xo)
        else:
            model.forward(xi, x_out=xo)

    flush = torch.empty(2 * L2_BYTES // 4, dtype=torch.float32, device=dev)
    resident = (sum(t.numel() * t.element_size() for t in W.values()) +
                sum(t.numel() * t.element_size() for t in X.values()))
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()

    def barrier():
        if dist is not None:
            dist.barrier()

    # ---- timed region: K steps, L2 flushed before each (flush not timed)
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    model.stats(reset=True)
    barrier()
    torch.cuda.synchronize()
    with ClockSampler(torch.cuda.current_device()) as clk:
        for i in range(args.steps):
            flush.fill_(float(i))
            starts[i].record()
            step()
            ends[i].record()
        torch.cuda.synchronize()
    barrier()
    launches = model.stats(reset=True)["launches"]
    ms_steps = [s.elapsed_time(e) for s, e in zip(starts, ends)]
    ms_total = max_over_ranks(float(sum(ms_steps)), dist, dev)
    ms_step = ms_total / args.steps
    units, value = job_value(cfg, world, ms_step)
    clocks = clk.summary()

    # ---- per-stage device times (same workload, profiling events on, separate run)
    model.set_profiling(True)
    for i in range(args.steps):
        flush.fill_(float(i))
        step()
    st = model.stats(reset=True)
    model.set_profiling(False)
    counts = model.route_counts(on_host=True).numpy()
    stage_alg, F, B = algorithmic(cfg, counts)
    pk = peaks()
    # the tensor peak a kernel is held to (tensor_peaks); the other figure is reported beside it
    tc_peak, tc_other, tc_kind = tensor_peaks(pk, ms_total)
    long_loop = tc_kind == "sustained"
    t_roof = max(F / (tc_peak * 1e12), B / (pk["hbm"] * 1e9))
    t_roof_other = max(F / (tc_other * 1e12), B / (pk["hbm"] * 1e9))
    per_stage = {}
    for name, ms in st["ms"].items():
        n = max(st["count"][name], 1)
        per_stage[name] = ms / max(args.steps, 1)
    # the dominant stage: the slowest of all stages of the depth step
    timed = [k for k in per_stage if per_stage[k] > 0 and k in stage_alg]
    dominant = max(timed, key=lambda k: per_stage[k])
    fl, by = stage_alg.get(dominant, (0.0, 0.0))
    t_dom = per_stage[dominant] / 1e3  # s per forward
    bound_tensor = fl / (tc_peak * 1e12) > by / (pk["hbm"] * 1e9)
    launches_per_fwd = max(st["count"][dominant] // max(args.steps, 1), 1)
    if bound_tensor:
        achieved = fl / t_dom / 1e12
        roof = dict(bound="tensor", achieved=achieved, peak=tc_peak, unit="TFLOP/s",
                    frac=achieved / tc_peak,
                    peak_kind="sustained" if long_loop else "burst",
                    other_peak={"kind": "burst" if long_loop else "sustained",
                                "peak": tc_other, "frac": achieved / tc_other})
    else:
        achieved = by / t_dom / 1e9
        roof = dict(bound="hbm", achieved=achieved, peak=pk["hbm"], unit="GB/s",
                    frac=achieved / pk["hbm"])
    roof.update(kernel=dominant, kernels=STAGE_KERNELS.get(dominant, dominant),
                launches_per_step=launches_per_fwd,
                traffic=None if args.reduced else measured_traffic(cfg.name, dominant),
                alg_bytes_per_launch=by / launches_per_fwd,
                peak_source=("measured (MEASURED_PEAKS.json)" if pk["source"] == "measured"
                             else "fallback (no MEASURED_PEAKS.json: 6650 GB/s copy; bf16 GEMM "
                                  "1590 TFLOP/s burst, 1400 TFLOP/s sustained under the power "
                                  "cap; earlier B200 measurements)"))

    # ---- end to end through the public API with host buffers
    e2e = None
    if not decode:
        host_in = torch.empty(x_in.shape, dtype=x_in.dtype, pin_memory=True)
        host_in.copy_(x_in)
        host_out = torch.empty(x_in.shape, dtype=x_in.dtype, pin_memory=True)
        xi = torch.empty_like(x_in)
        for _ in range(2):
            xi.copy_(host_in, non_blocking=True)
            step(xi, x_out)
            host_out.copy_(x_out, non_blocking=True)
        torch.cuda.synchronize()
        barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for i in range(args.steps):
            xi.copy_(host_in, non_blocking=True)
            step(xi, x_out)
            host_out.copy_(x_out, non_blocking=True)
        e1.record()
        torch.cuda.synchronize()
        ms_e2e = max_over_ranks(e0.elapsed_time(e1), dist, dev)
        nbytes = x_in.numel() * x_in.element_size()
        e2e = {"value": units / (ms_e2e / args.steps / 1e3), "unit": UNIT,
               "h2d_bytes_per_step": nbytes, "d2h_bytes_per_step": nbytes,
               "note": "includes the L2-resident reuse of weights across steps"}
    else:
        # decode: new token embeddings in, outputs out
        host_in = torch.empty(x_in.shape, dtype=x_in.dtype, pin_memory=True)
        host_in.copy_(x_in)
        host_out = torch.empty(x_in.shape, dtype=x_in.dtype, pin_memory=True)
        xi = torch.empty_like(x_in)
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for i in range(args.steps):
            xi.copy_(host_in, non_blocking=True)
            step(xi, x_out)
            host_out.copy_(x_out, non_blocking=True)
        e1.record()
        torch.cuda.synchronize()
        ms_e2e = max_over_ranks(e0.elapsed_time(e1), dist, dev)
        nbytes = x_in.numel() * x_in.element_size()
        e2e = {"value": units / (ms_e2e / args.steps / 1e3), "unit": UNIT,
               "h2d_bytes_per_step": nbytes, "d2h_bytes_per_step": nbytes}

    out = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16" if cfg.dtype == "bf16" else "f32",
        "data": "synthetic (seeded N(0,1) inputs, N(0,1/fan_in) weights)",
        "config": dict(config_dict(cfg, world), resident_bytes_per_gpu=resident),
        "roofline": roof,
        "roofline_step": {"t_roof_ms": t_roof * 1e3, "t_meas_ms": ms_step,
                          "frac": t_roof * 1e3 / ms_step, "F_alg": F, "B_alg": B,
                          "peaks": {"tensor_tflops": tc_peak,
                                    "tensor_kind": "sustained" if long_loop else "burst",
                                    "hbm_gbs": pk["hbm"], "source": pk["source"]},
                          "frac_other_tensor_peak": {"tensor_tflops": tc_other,
                                                     "frac": t_roof_other * 1e3 / ms_step}},
        "stage_ms_per_step": per_stage,
        "e2e": e2e,
        "gpu_launches": launches,
        "clocks": clocks,
    }
    return out, model


# kernels of each stage (bf16 path)
STAGE_KERNELS = {
    "qkv": "tc_gemm_kernel<EpiQKV>", "o_proj": "tc_gemm_kernel<EpiO>",
    "sa": "tc_sa_kernel (prefill) / dec_bulk_kernel + attn_merge_kernel (decode)",
    "da": "da_fast_kernel", "proj_route": "tc_gemm_kernel<EpiProjRoute> + permute_kernel",
    "ea_route": "tc_gemm_kernel<EpiRouterQ> + tc_gemm_kernel<EpiTopK> or route_q_topk_kernel "
                "(decode: route_cluster_kernel)",
    "permute": "permute_kernel",
    "experts": "tc_gemm_kernel<EpiUp> + tc_gemm_kernel<EpiDownStore>, or tc_ffn_kernel "
               "(decode: expert_rows_kernel)",
    "finish": "combine_norm_kernel", "norm": "rmsnorm_kernel",
}


def config_dict(cfg, world=1):
    """The `config` object of the JSON line (both arms)."""
    return {"workload": workload_name(cfg), "global_batch": cfg.batch * world,
            "seq_len": cfg.seq, "depth": cfg.depth, "hidden": cfg.hidden,
            "heads": f"{cfg.n_heads}x{cfg.head_dim}", "experts": cfg.n_experts,
            "top_k": cfg.top_k, "expert_hidden": cfg.expert_hidden,
            "proj_experts": cfg.n_proj_experts, "units_per_step": cfg.units * world,
            "parallelism": f"dp{world} (replicas)",
            "l2": "flushed before every timed step (256 MB write, not timed)"}


def workload_name(cfg):
    base = f"{cfg.name}: b={cfg.batch} s={cfg.seq} h={cfg.hidden} {cfg.n_heads}x{cfg.head_dim} " \
           f"L={cfg.depth} E={cfg.n_experts} k={cfg.top_k} m={cfg.expert_hidden} P={cfg.n_proj_experts}"
    if cfg.is_decode:
        base += f" decode cache={cfg.cache_len}"
    if cfg.variant:
        base += {1: " serial DA->SA->EA", 2: " fully parallel", 3: " without DA"}[cfg.variant]
    if cfg.da_window:
        base += f" DA window {cfg.da_window}"
    return base


# ----------------------------------------------------------------------------------------
# the oracle on the host cores (cpu_baseline leg and the --impl reference arm)

class OracleSampler:
    """The oracle on the host cores (all of them, OpenMP), on a bounded sample of the
    workload: for prefill the first S' <= 1024 tokens of one sequence (causal SA makes them an
    exact part of the workload) through its first depths, for decode one sequence's whole
    step.  Weights are drawn once; sample() returns (units/s, description)."""

    def __init__(self, cfg, threads=None):
        sys.path.insert(0, os.path.join(ROOT, "oracle"))
        import oracle as O
        self.cfg = cfg
        self.threads = threads or os.cpu_count() or 1
        W = inputs.host_weights(cfg)
        self.one = cfg.with_(batch=1) if cfg.is_decode else cfg.with_(batch=1, seq=min(cfg.seq, 1024))
        self.o = O.Oracle(self.one, W, threads=self.threads)

    def sample(self, seconds_hint=20.0):
        cfg, one, o = self.cfg, self.one, self.o
        if cfg.is_decode:
            L, H, d = cfg.depth, cfg.n_heads, cfg.head_dim
            cap = cfg.cache_len + 1
            kc = np.zeros((L, H, cap, d))
            vc = np.zeros((L, H, cap, d))
            x = inputs.draw([s for s in inputs.input_specs(cfg) if s.name == "x0"][0], cfg.seed,
                            0, cfg.hidden)
            t0 = time.perf_counter()
            o.decode_seq(x, kc, vc, cfg.cache_len)
            dt = time.perf_counter() - t0
            return cfg.depth / dt, f"one sequence's decode step (all {cfg.depth} depths, " \
                                   f"cache {cfg.cache_len}, zero cache contents)"
        x = inputs.host_inputs(one)["x0"]
        t0 = time.perf_counter()
        depths = 0
        da = np.zeros((one.tokens, cfg.depth, 2, cfg.hidden))
        while depths < cfg.depth:
            r = o.forward(x, depths, depths + 1, da_kv=da, trace=False)
            x = inputs.round_to(r["x_out"], cfg.dtype)
            da = r["da_kv"]
            depths += 1
            if time.perf_counter() - t0 > seconds_hint:
                break
        dt = time.perf_counter() - t0
        return one.tokens * depths / dt, f"the first {one.tokens} of {cfg.seq} tokens of one " \
                                         f"sequence through depths 0..{depths - 1} of {cfg.depth}"


def run_reference(args, cfg):
    """The reference arm: the oracle, as it stands, on the host cores; each of the K timed steps
    is one bounded sample of the workload (W untimed warm-up samples first)."""
    smp = OracleSampler(cfg)
    hint = max(2.0, 60.0 / max(args.steps + args.warmup, 1))
    for _ in range(args.warmup):
        smp.sample(seconds_hint=hint)
    vals = []
    for _ in range(max(args.steps, 1)):
        v, sample = smp.sample(seconds_hint=hint)
        vals.append(v)
    cores = smp.threads
    value = statistics.median(vals)
    return {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": None,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f64", "data": "synthetic", "impl": "reference",
        "config": config_dict(cfg, 1),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


# ----------------------------------------------------------------------------------------

def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--config", default="large", choices=sorted(configs.CONFIGS))
    ap.add_argument("--no-cpu-baseline", action="store_true")
    for k in ("depth", "batch", "seq"):
        ap.add_argument(f"--{k}", type=int, default=0,
                        help=f"run the workload with this {k} instead of its own (reduced cases "
                             "for ncu captures of single kernels); the line's config names it")
    args = ap.parse_args()
    cfg = configs.CONFIGS[args.config]
    args.reduced = {k: getattr(args, k) for k in ("depth", "batch", "seq") if getattr(args, k)}
    if args.reduced:
        cfg = cfg.with_(**args.reduced)
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))

    if args.impl == "reference":
        if rank != 0:
            return 0
        print(json.dumps(run_reference(args, cfg)))
        return 0

    import torch
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        local = int(os.environ.get("LOCAL_RANK", "0"))
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    else:
        torch.cuda.set_device(0)
    out, model = run_ours(args, cfg, rank, world, torch, dist)
    if rank == 0:
        if world == 1 and not args.no_cpu_baseline:
            smp = OracleSampler(cfg)
            v, sample = smp.sample()
            out["cpu_baseline"] = {"value": v, "unit": UNIT, "cores": smp.threads,
                                   "kind": "oracle", "sample": sample}
        print(json.dumps(out))
    model.close()
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
