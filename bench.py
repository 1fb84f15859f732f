#!/usr/bin/env python
"""Throughput of the DeepSeek-V3 MoE layer forward on B200 (one JSON line).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

A step is one pass of the whole path over one batch of synthetic tokens:
gate GEMM + routing, permutation, routed SwiGLU experts (two grouped GEMMs),
the shared expert, combine, and the aux-loss-free bias update. The default
workload is the V3-shaped layer (T=8192 tokens, H=7168, 256 routed experts
with I=2048, 1 shared expert, top-8 of 8 groups keeping 4, sigmoid scoring
with a selection bias, renormalised weights x2.5), bf16 weights and
activations, fp32 accumulation. Inputs are larger than L2 (22.5 GB of expert
weights stream through every step), so no L2 flush is done between steps.

N > 1 (launched under torchrun): every rank runs an independent replica on
its own tokens (weak scaling); the expert counts are summed over ranks before
the bias step so all replicas keep the same bias.

--impl reference times the CPU oracle (the plain float64 statement of the
layer) on the host cores, on a bounded sample of tokens per step.
"""
import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "MoE-layer fwd tokens/s and achieved TFLOP/s vs B200 peak at V3 shape"
PROFILE_DIR = os.path.join(ROOT, "profiles")      # *_traffic.txt: DRAM bytes of one launch per workload
GEMM_SOURCES = ["grouped_gemm.cu", "common.cuh", "kernels.cuh"]


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--config", default="v3")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-sample-tokens", type=int, default=1024,
                    help="tokens of the CPU baseline's sample (at least; it always holds every token "
                         "of the hottest and the coldest expert)")
    ap.add_argument("--fuse-combine", action="store_true",
                    help="run the combine inside the down GEMM (atomic fp32 scatter-add) instead of after it")
    ffn = ap.add_mutually_exclusive_group()
    ffn.add_argument("--split-ffn", action="store_true",
                     help="always run the experts' two GEMMs as two launches (gate/up, then down)")
    ffn.add_argument("--fuse-ffn", action="store_true",
                     help="always run them as one launch (default: one launch from 512 routed rows per expert)")
    ap.add_argument("--routing-sweep", action="store_true",
                    help="instead of the throughput line: load CV, aux loss and router time for "
                         "topk_group 8/4/2/1 of 8 groups on the V3 and skewed inputs (one line each)")
    return ap.parse_args()


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained", d["bf16_tflops"]),
                "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
            "source": "fallback"}


def workload_name(cfg):
    return (f"{cfg.name} MoE layer fwd: T={cfg.T} tokens, H={cfg.H}, {cfg.E} routed experts "
            f"(I={cfg.I}) + shared (I_s={cfg.I_s}), top-{cfg.k}, n_group={cfg.n_group}/"
            f"topk_group={cfg.topk_group}, {cfg.scoring}, {cfg.dtype}")


def config_block(cfg, world):
    return {"workload": workload_name(cfg), "T_per_gpu": cfg.T, "global_tokens": cfg.T * world,
            "H": cfg.H, "E": cfg.E, "I": cfg.I, "I_s": cfg.I_s, "k": cfg.k,
            "n_group": cfg.n_group, "topk_group": cfg.topk_group, "scoring": cfg.scoring,
            "norm_topk_prob": cfg.norm_topk_prob, "routed_scaling_factor": cfg.scale,
            "weights_dtype": cfg.dtype, "parallelism": f"replicas x{world} (token-sharded)",
            "l2": "inputs larger than L2 (all expert weights stream each step); no flush"}


# ------------------------------------------------------------ clock sampling
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index):
        self.proc = None
        self.sel = None
        try:
            import torch
            p = torch.cuda.get_device_properties(device_index)
            self.sel = f"{p.pci_domain_id:08X}:{p.pci_bus_id:02X}:{p.pci_device_id:02X}.0"
        except Exception:
            self.sel = None

    def start(self):
        cmd = ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "100"]
        if self.sel:
            cmd += ["-i", self.sel]
        try:
            self.proc = subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"], "samples": 0}
        time.sleep(0.25)
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except Exception:
            self.proc.kill()
            out, _ = self.proc.communicate()
        sm, smax, power, reasons = [], [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.strip().splitlines():
            f = [c.strip() for c in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                smax.append(float(f[2]))
                power.append(float(f[3]))
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        # samples under load: SM clock above the idle floor
        load = [s for s in sm if s > 0.3 * max(smax)] or sm
        return {"sm_mhz": statistics.median(load), "sm_max_mhz": max(smax), "reasons": sorted(reasons),
                "samples": len(sm), "power_w_max": max(power)}


# ------------------------------------------------------------ CPU oracle arm
def oracle_tokens_per_s(cfg, inp, tokens, threads):
    """Times the float64 oracle on the given tokens: logits, routing, every
    routed expert they use, the shared expert and the combine. Expert weights
    are fetched from device memory one expert at a time as the oracle asks
    for them; the fetches are not counted in the time."""
    import numpy as np
    import torch
    import oracle
    toks = torch.as_tensor(tokens, device=inp.x.device)
    x = inp.x[toks].float().cpu().numpy()
    gate = inp.gate.float().cpu().numpy()
    bias = inp.bias.float().cpu().numpy() if inp.bias is not None else None
    shared = (inp.sw13.float().cpu().numpy(), inp.sw2.float().cpu().numpy()) if inp.sw13 is not None else None
    fetch = [0.0]

    def expert(e):
        f0 = time.perf_counter()
        w = (inp.w13[e].float().cpu().numpy(), inp.w2[e].float().cpu().numpy())
        fetch[0] += time.perf_counter() - f0
        return w

    t0 = time.perf_counter()
    L = oracle.gate_logits(x, gate).astype(np.float32)
    r = oracle.route_from_logits(L, cfg.k, cfg.n_group, cfg.topk_group, cfg.scoring,
                                 cfg.norm_topk_prob, cfg.scale, bias)
    oracle.moe_forward(x, r, expert, shared, fp8=(cfg.dtype == "e4m3"))
    dt = time.perf_counter() - t0 - fetch[0]
    return len(tokens) / dt, dt


def cpu_sample_tokens(layer, cfg, n_min, seed=7):
    """The CPU baseline's sample: every token routed to the hottest expert and
    to the coldest expert that received any, then random tokens up to n_min
    (from the layer's last forward on the bench's inputs)."""
    import numpy as np
    off = layer.offsets.cpu().numpy().astype(np.int64)
    src = layer.src_token[:cfg.T * cfg.k].cpu().numpy()
    counts = np.diff(off)
    hot = int(np.argmax(counts))
    cold = int(np.argmin(np.where(counts > 0, counts, np.iinfo(np.int64).max)))
    toks = set(src[off[hot]:off[hot + 1]].tolist()) | set(src[off[cold]:off[cold + 1]].tolist())
    rng = np.random.default_rng(seed)
    rest = [t for t in rng.permutation(cfg.T).tolist() if t not in toks]
    toks |= set(rest[:max(0, n_min - len(toks))])
    return np.array(sorted(toks)), hot, int(counts[hot]), cold, int(counts[cold])


def oracle_bias_loop_s(name="v3_skewed"):
    """Host time of the oracle's bias loop on the skewed layer: fp64 logits of
    all T tokens once, then per step the routing of every token and the bias
    update from its counts (steps + 1 routing passes)."""
    import numpy as np
    import torch
    import oracle
    from moe_inputs import get_config, make_inputs
    cfg = get_config(name)
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    inp = make_inputs(cfg, device=dev, experts=False, shared=False)
    x = inp.x.float().cpu().numpy()
    gate = inp.gate.float().cpu().numpy()
    bias = inp.bias.float().cpu().numpy()
    del inp
    t0 = time.perf_counter()
    L = oracle.gate_logits(x, gate).astype(np.float32)
    for step in range(cfg.bias_steps + 1):
        r = oracle.route_from_logits(L, cfg.k, cfg.n_group, cfg.topk_group, cfg.scoring,
                                     cfg.norm_topk_prob, cfg.scale, bias)
        if step < cfg.bias_steps:
            bias = oracle.bias_update(r.counts, bias, cfg.gamma, cfg.T, cfg.k)
    return time.perf_counter() - t0, cfg


def host_threads():
    try:
        return len(os.sched_getaffinity(0))
    except Exception:
        return os.cpu_count() or 1


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    import numpy as np
    import torch
    from moe_inputs import get_config, make_inputs
    cfg = get_config(args.config)
    threads = host_threads()
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    inp = make_inputs(cfg, device=dev)
    rng = np.random.default_rng(2024)
    per_step = 1
    times, ntok = [], 0
    for i in range(args.warmup + args.steps):
        toks = rng.choice(cfg.T, per_step, replace=False)
        _, dt = oracle_tokens_per_s(cfg, inp, toks, threads)
        if i >= args.warmup:
            times.append(dt)
            ntok += per_step
    total = sum(times)
    value = ntok / total
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1e3 * total / max(1, len(times)), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": config_block(cfg, 1),
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": threads, "kind": "oracle",
                             "sample": f"{per_step} random token(s) of {cfg.T} per step: fp64 logits, "
                                       "routing, its experts, shared expert, combine"},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line))
    return 0


# ------------------------------------------------------------ our arm
def gemm_source_hash():
    h = hashlib.sha256()
    for f in GEMM_SOURCES:
        h.update(open(os.path.join(ROOT, "mixture_experts_layer_limited_b200", "csrc", f), "rb").read())
    return h.hexdigest()[:16]


def profiled_traffic(stage, workload):
    """DRAM bytes per launch of a stage's GEMM from the committed ncu
    summaries (profiles/*_traffic.txt), only from one taken of this stage's
    launch on this workload, and only while the GEMM source is the one
    captured."""
    if not os.path.isdir(PROFILE_DIR):
        return None
    for name in sorted(os.listdir(PROFILE_DIR)):
        if not name.endswith("_traffic.txt"):
            continue
        kv = {}
        for line in open(os.path.join(PROFILE_DIR, name)):
            if ":" in line and not line.startswith("#"):
                k, v = line.split(":", 1)
                kv[k.strip()] = v.strip()
        if (kv.get("gemm_source_sha256_16") != gemm_source_hash() or kv.get("stage") != stage
                or kv.get("workload") != workload):
            continue
        try:
            return float(kv["traffic_bytes_per_launch_full_size"])
        except (KeyError, ValueError):
            return None
    return None


LAUNCHES = {"route": 1, "permute": 3, "gate_up_routed": 1, "down_routed": 1,
            "gate_up_shared": 1, "down_shared": 1, "gate_up": 1, "down": 1, "combine": 1, "bias_update": 1,
            "down_combine": 2, "ffn": 1}


def launches_of(name, cfg):
    """Kernel launches of one stage (the fused routed + shared GEMM stages run
    as two launches for E4M3 layers)."""
    if name in ("gate_up", "down") and cfg.dtype == "e4m3":
        return 2
    return LAUNCHES[name]


def stage_model(cfg):
    """Algorithmic FLOPs and bytes of each stage (no padding, no re-reads)."""
    T, H, E, I, Is, k = cfg.T, cfg.H, cfg.E, cfg.I, cfg.I_s, cfg.k
    R = T * k
    ab = 1 if cfg.dtype == "e4m3" else 2
    m = {
        "route": {"flops": 2.0 * T * H * E, "bytes": T * H * 2 + E * H * 2 + T * E * 4 + R * 8},
        # E4M3 layers read x in bf16 and write codes + 1x128 scales (also the
        # shared expert's unpermuted codes)
        "permute": {"flops": 0.0, "bytes": (T * H * 2 + R * (H + H // 32) + T * (H + H // 32) + R * 20)
                    if ab == 1 else (T * H * 2 + R * H * 2 + R * 20)},
        "gate_up_routed": {"flops": 2.0 * R * H * 2 * I, "bytes": E * 2 * I * H * ab + R * H * ab + R * I * ab},
        "down_routed": {"flops": 2.0 * R * I * H, "bytes": E * H * I * ab + R * I * ab + R * H * 2},
        "gate_up_shared": {"flops": 2.0 * T * H * 2 * Is, "bytes": 2 * Is * H * ab + T * H * ab + T * Is * ab},
        "down_shared": {"flops": 2.0 * T * Is * H, "bytes": H * Is * ab + T * Is * ab + T * H * 2},
        "combine": {"flops": 0.0, "bytes": R * H * 2 + T * H * 2 + T * H * 2 + R * 4},
        "bias_update": {"flops": 0.0, "bytes": E * 12},
    }
    # routed + shared expert in one launch per GEMM
    for fused, parts in (("gate_up", ("gate_up_routed", "gate_up_shared")), ("down", ("down_routed", "down_shared"))):
        m[fused] = {key: sum(m[p][key] for p in parts) for key in ("flops", "bytes")}
    # both GEMMs, routed + shared expert, in one launch (h still makes its round trip)
    m["ffn"] = {key: m["gate_up"][key] + m["down"][key] for key in ("flops", "bytes")}
    # down GEMMs with the combine in the epilogue: weights and h in, y out
    m["down_combine"] = {"flops": m["down"]["flops"],
                         "bytes": E * H * I * ab + R * I * ab + H * Is * ab + T * Is * ab + T * H * 2}
    return m


def run_ours(args):
    import numpy as np
    import torch
    import torch.distributed as dist
    from datetime import timedelta
    from moe_inputs import get_config, make_inputs
    from mixture_experts_layer_limited_b200 import MoELayer, LayerSpec, HostPipeline, load_library
    from mixture_experts_layer_limited_b200 import dist as mdist

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    if world > 1:
        dist.init_process_group("nccl", timeout=timedelta(seconds=300),
                                device_id=torch.device("cuda", local))
    load_library()
    cfg = get_config(args.config)
    inp = make_inputs(cfg, device="cuda")
    if rank > 0:   # same weights, this replica's own tokens
        g = torch.Generator(device="cuda")
        g.manual_seed(cfg.seed + 100003 * rank)
        inp.x = torch.randn(cfg.T, cfg.H, generator=g, device="cuda").to(torch.bfloat16)
    layer = MoELayer(LayerSpec.from_config(cfg), inp.gate, inp.w13, inp.w2, inp.sw13, inp.sw2,
                     inp.bias, cfg.T, fuse_combine=args.fuse_combine, fuse_ffn=False if args.split_ffn else (True if args.fuse_ffn else None))
    T_global = cfg.T * world
    stream = torch.cuda.current_stream()
    stages = layer.stages(inp.x)
    names = [n for n, _ in stages] + (["bias_update"] if layer.bias is not None else [])

    def step(marks=None):
        for i, (_, run) in enumerate(stages):
            run()
            if marks is not None:
                marks[i].record(stream)
        if layer.bias is not None:
            mdist.allreduce_counts_(layer.counts)
            layer.bias_step(T_global, cfg.gamma, load_cv=False)
            if marks is not None:
                marks[len(stages)].record(stream)

    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize()
    assert layer.device_status() == 0, "device status flagged during warm-up"

    K = args.steps
    marks = [[torch.cuda.Event(enable_timing=True) for _ in names] for _ in range(K)]
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(local)
    mdist.barrier()
    torch.cuda.synchronize()
    clocks.start()
    time.sleep(0.3)                                   # sampler up before the clock starts
    start.record(stream)
    for i in range(K):
        step(marks[i])
    end.record(stream)
    torch.cuda.synchronize()
    mdist.barrier()
    clk = clocks.stop()
    ms_local = start.elapsed_time(end)
    ms = mdist.max_over_ranks(ms_local, device="cuda")
    status = layer.device_status()

    # per-stage device time from consecutive events on the launching stream
    per = {n: [] for n in names}
    for i in range(K):
        prev = start if i == 0 else marks[i - 1][-1]
        for j, n in enumerate(names):
            per[n].append(prev.elapsed_time(marks[i][j]))
            prev = marks[i][j]
    avg = {n: sum(v) / len(v) for n, v in per.items()}
    model = stage_model(cfg)
    peaks = load_peaks()
    kernels = {}
    for n in names:
        m = model[n]
        d = {"ms": round(avg[n], 4), "launches": launches_of(n, cfg)}
        if m["flops"]:
            d["tflops"] = round(m["flops"] / (avg[n] * 1e-3) / 1e12, 1)
        if m["bytes"] and avg[n] > 0:
            d["gbs"] = round(m["bytes"] / (avg[n] * 1e-3) / 1e9, 1)
        kernels[n] = d

    tokens = cfg.T * world * K
    value = tokens / (ms * 1e-3)
    flops_step = cfg.flops()
    dom = "ffn" if "ffn" in avg else "gate_up" if "gate_up" in avg else "gate_up_routed"
    achieved = model[dom]["flops"] / (avg[dom] * 1e-3) / 1e12
    # the timed region is well under a second, at the clock the sampler saw:
    # the peak is the burst figure (a GEMM timed alone); the sustained one
    # (seconds under the power cap, at a lower clock) only as a second number
    peak = peaks["bf16_tflops"]
    what = "routed experts + shared expert, one launch" if dom in ("gate_up", "ffn") else "routed experts"
    kname = ("grouped_ffn_bf16 (gate/up + SwiGLU and down + routing weight, " if dom == "ffn"
             else "grouped_gemm_bf16 (gate/up + SwiGLU, ") + what + ")"
    roofline = {"kernel": kname, "bound": "tensor",
                "achieved": round(achieved, 1), "peak": peak, "unit": "TFLOP/s",
                "frac": round(achieved / peak, 4), "traffic": profiled_traffic(dom, cfg.name),
                "sm_mhz": clk.get("sm_mhz"),
                "peak_note": f"bf16 burst, {peaks['source']} (MEASURED_PEAKS.json)" if peaks["source"] == "measured"
                             else "bf16 burst, fallback figure of this pool (no MEASURED_PEAKS.json)",
                "frac_of_sustained": round(achieved / peaks["bf16_tflops_sustained"], 4),
                "algorithmic_flops_per_launch": model[dom]["flops"],
                "algorithmic_bytes_per_launch": model[dom]["bytes"]}
    if cfg.dtype == "e4m3":
        # E4M3 decode: every expert's weights stream once for a few tokens each
        gbs = model[dom]["bytes"] / (avg[dom] * 1e-3) / 1e9
        roofline = {"kernel": f"grouped_gemm_e4m3 (gate/up + SwiGLU, {what})", "bound": "hbm",
                    "achieved": round(gbs, 1), "peak": peaks["hbm_gbs"], "unit": "GB/s",
                    "frac": round(gbs / peaks["hbm_gbs"], 4), "traffic": profiled_traffic(dom, cfg.name),
                    "sm_mhz": clk.get("sm_mhz"),
                    "peak_note": f"HBM copy, {peaks['source']}",
                    "algorithmic_flops_per_launch": model[dom]["flops"],
                    "algorithmic_bytes_per_launch": model[dom]["bytes"]}

    # ---- the same step replayed as one CUDA graph (launch overhead gone)
    replay = layer.capture(inp.x, cfg.gamma if layer.bias is not None else None) if world == 1 else None
    graph_ms = None
    if replay is not None:
        for _ in range(3):
            replay()
        torch.cuda.synchronize()
        g0, g1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        g0.record(stream)
        for _ in range(K):
            replay()
        g1.record(stream)
        torch.cuda.synchronize()
        graph_ms = g0.elapsed_time(g1) / K

    # ---- end to end: host x -> device, forward + bias step, y -> host. Each
    # step copies its batch in from pinned host memory and its output back out;
    # HostPipeline overlaps those copies with the neighbouring steps' compute.
    g = torch.Generator(device="cuda")
    g.manual_seed(cfg.seed + 4242 + rank)
    x_hosts = [inp.x.cpu().pin_memory(),
               torch.randn(cfg.T, cfg.H, generator=g, device="cuda").to(torch.bfloat16).cpu().pin_memory()]
    y_hosts = [torch.empty(cfg.T, cfg.H, dtype=torch.bfloat16).pin_memory() for _ in range(2)]
    pipe = HostPipeline(layer, cfg.T)

    def bias_after(_i):
        if layer.bias is not None:
            mdist.allreduce_counts_(layer.counts)
            layer.bias_step(T_global, cfg.gamma, load_cv=False)

    def run_e2e(n):
        pipe.run([x_hosts[i % 2] for i in range(n)], [y_hosts[i % 2] for i in range(n)], bias_after)

    run_e2e(3)
    torch.cuda.synchronize()
    mdist.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    run_e2e(K)
    e1.record(stream)
    torch.cuda.synchronize()
    mdist.barrier()
    ms_e2e = mdist.max_over_ranks(e0.elapsed_time(e1), device="cuda")
    e2e = {"value": cfg.T * world * K / (ms_e2e * 1e-3), "unit": "tokens/s",
           "h2d_bytes_per_step": cfg.T * cfg.H * 2, "d2h_bytes_per_step": cfg.T * cfg.H * 2,
           "path": "HostPipeline over MoELayer (C ABI): per step pinned host x in and y out, "
                   "copies on two streams overlapped with the neighbouring steps"}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        layer.forward(inp.x)                          # the bench's own batch: its routing picks the sample
        toks, hot, n_hot, cold, n_cold = cpu_sample_tokens(layer, cfg, min(args.cpu_sample_tokens, cfg.T))
        rate, dt = oracle_tokens_per_s(cfg, inp, toks, host_threads())
        cpu = {"value": rate, "unit": "tokens/s", "cores": host_threads(), "kind": "oracle",
               "sample": f"{len(toks)} of the {cfg.T} tokens of the timed batch ({dt:.1f} s of fp64 logits, "
                         f"routing, their experts, shared expert, combine; weights fetched per expert, "
                         f"fetch time excluded): every token of the hottest expert ({hot}, {n_hot} tokens) "
                         f"and of the coldest ({cold}, {n_cold}), the rest random. Per-token rate; "
                         f"extrapolated to the whole batch: {cfg.T / rate:.0f} s per step"}
        if cfg.name == "v3":
            secs, scfg = oracle_bias_loop_s()
            cpu["bias_loop"] = {"workload": f"skewed V3 layer, T={scfg.T}, {scfg.bias_steps} bias steps",
                                "seconds": round(secs, 2),
                                "what": f"fp64 logits of all tokens once, then {scfg.bias_steps + 1} routing "
                                        f"passes of every token and {scfg.bias_steps} bias updates"}

    if rank == 0:
        line = {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": K,
                "warmup": args.warmup, "ms_per_step": ms / K, "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": "bf16" if cfg.dtype == "bf16" else "e4m3",
                "data": f"synthetic (seeded random inputs and weights, {cfg.name} shapes)",
                "config": dict(config_block(cfg, world),
                               **({"combine": "inside the down GEMM (atomic fp32 adds)"} if args.fuse_combine else {})),
                "tflops": round(flops_step * world * K / (ms * 1e-3) / 1e12, 1),
                "tflops_frac_of_burst": round(flops_step * K / (ms * 1e-3) / 1e12 / peaks["bf16_tflops"], 4),
                "tflops_frac_of_sustained": round(flops_step * K / (ms * 1e-3) / 1e12
                                                  / peaks["bf16_tflops_sustained"], 4),
                "roofline": roofline, "kernels": kernels, "cpu_baseline": cpu, "e2e": e2e,
                "gpu_launches": K * sum(launches_of(n, cfg) for n in names), "clocks": clk,
                "graph_ms_per_step": round(graph_ms, 4) if graph_ms is not None else None,
                "device_status": status}
        print(json.dumps(line))
    if world > 1:
        dist.destroy_process_group()
    return 0


def run_routing_sweep(args):
    """The group-limit experiment of the V3 teardown page (§4: lowering
    topk_group from 4 to 2 concentrates load, 8 removes the limit): for each
    topk_group, one routing pass of the V3 and of the skewed inputs through
    moe_route, then the load CV (moe_bias_update with gamma 0 leaves the bias
    as it is) and the sequence-level aux loss, and the router's device time."""
    import torch
    from moe_inputs import get_config, make_inputs
    from mixture_experts_layer_limited_b200 import native as N
    N.load_library()
    dev = "cuda"
    for name in ("v3", "v3_skewed"):
        cfg = get_config(name)
        inp = make_inputs(cfg, device=dev, experts=False, shared=False)
        T, E, k = cfg.T, cfg.E, cfg.k
        f32, i32 = torch.float32, torch.int32
        logits = torch.empty(T, E, dtype=f32, device=dev)
        ids = torch.empty(T, k, dtype=i32, device=dev)
        w = torch.empty(T, k, dtype=f32, device=dev)
        counts = torch.empty(E, dtype=i32, device=dev)
        cv = torch.empty(1, dtype=f32, device=dev)
        aux = torch.empty(1, dtype=f32, device=dev)
        bias = inp.bias.clone()
        ws = torch.empty(N.moe_aux_loss_workspace_size(T, E, T), dtype=torch.uint8, device=dev)
        for g in (8, 4, 2, 1):
            def route():
                N.moe_route(T, cfg.H, E, k, cfg.n_group, g, N.MOE_SIGMOID, cfg.norm_topk_prob, cfg.scale,
                            inp.x, inp.gate, bias, logits, ids, w, counts)
            for _ in range(3):
                route()
            reps = 20
            t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            t0.record()
            for _ in range(reps):
                route()
            t1.record()
            N.moe_bias_update(E, T, k, counts, bias, 0.0, cv)
            N.moe_aux_loss(T, E, k, T, N.MOE_SIGMOID, logits, ids, 0.001, aux, ws)
            torch.cuda.synchronize()
            c = counts.cpu()
            print(json.dumps({"sweep": "topk_group", "workload": name, "T": T, "E": E, "k": k,
                              "n_group": cfg.n_group, "topk_group": g, "load_cv": round(cv.item(), 5),
                              "max_load_over_mean": round(int(c.max()) * E / (T * k), 3),
                              "hot_0_15_share": round(int(c[:16].sum()) / (T * k), 4),
                              "aux_loss": float(f"{aux.item():.6g}"),
                              "route_ms": round(t0.elapsed_time(t1) / reps, 4)}))
    return 0


def main():
    args = parse_args()
    if args.routing_sweep:
        return run_routing_sweep(args)
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
