#!/usr/bin/env python
"""Benchmark of the fused COAT FP8-state AdamW step on B200.

One step = one coat_adamw_fp8_step over the whole OLMo-7B-shaped parameter
set (6,888,095,744 FP32 parameters, BF16 gradients, FP8 m/v with per-group
k and scale, G = 128) resident in HBM.  Prints ONE JSON line (rank 0).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--v-fmt e4m3|e5m2]
  python bench.py --impl reference ...    # the CPU oracle on a bounded sample

Multi-GPU (torchrun): every rank owns its own full parameter set (the step
has no cross-rank exchange), so per-GPU work is fixed: weak scaling, value =
parameters stepped by all ranks / max-over-ranks time.
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
sys.path.insert(0, ROOT)

METRIC = "params/s for fused FP8-state AdamW step (OLMo-7B set); % of B200 HBM peak"
FALLBACK_HBM_GBS = 6650.0
KERNEL_SOURCES = ["quantized_optimizer_states_b200/csrc/step_kernels.cuh",
                  "quantized_optimizer_states_b200/csrc/state_codec.cuh",
                  "quantized_optimizer_states_b200/csrc/fp8_device.cuh"]


def bytes_per_param(G: int) -> float:
    """Algorithmic HBM bytes per parameter of one fused step: theta read +
    write (8), BF16 gradient read (2), m and v codes read + write (4), and
    per group (k, s) x 2 states x 4 B x (read + write) = 32 B over G."""
    return 14.0 + 32.0 / G


# sources of the activation quantizers (the traffic record of the 1xG
# kernel is valid while these are unchanged)
ACT_KERNEL_SOURCES = ["quantized_optimizer_states_b200/csrc/act_kernels.cuh",
                      "quantized_optimizer_states_b200/csrc/bulk_pipe.cuh",
                      "quantized_optimizer_states_b200/csrc/fp8_device.cuh"]


def kernel_source_hash(sources=None) -> str:
    h = hashlib.sha256()
    for rel in (KERNEL_SOURCES if sources is None else sources):
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return json.load(f), "measured"
    except OSError:
        return {"hbm_gbs": FALLBACK_HBM_GBS}, "fallback"


def recorded_traffic(n: int, G: int):
    """DRAM bytes per launch from the committed ncu summary, scaled to n
    parameters; None if the kernel source changed since the capture."""
    path = os.path.join(ROOT, "profiles", "adamw_fp8_step_traffic.json")
    try:
        with open(path) as f:
            rec = json.load(f)
    except OSError:
        return None
    if rec.get("kernel_source_hash") != kernel_source_hash() or rec.get("group_size") != G:
        return None
    return rec["dram_bytes_per_param"] * n


def recorded_act_traffic(n: int):
    """DRAM bytes of one 1xG quantizer launch on the activation workload, from
    the committed ncu summary; None if its sources changed since the capture
    or the size differs."""
    path = os.path.join(ROOT, "profiles", "group_quant_1xG_traffic.json")
    try:
        with open(path) as f:
            rec = json.load(f)
    except OSError:
        return None
    if (rec.get("kernel_source_hash") != kernel_source_hash(ACT_KERNEL_SOURCES)
            or rec.get("elements") != n):
        return None
    return rec["dram_bytes_read"] + rec["dram_bytes_write"]


class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons during timing."""
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, uuid: str | None):
        self.proc = None
        # the raw samples (the JSON line carries their summary)
        log_dir = os.environ.get("COAT_BENCH_LOG_DIR") or os.path.join(ROOT, "bench_logs")
        self.path = os.path.join(log_dir, f"clocks_{os.getpid()}.csv")
        self.uuid = uuid

    def start(self):
        try:
            os.makedirs(os.path.dirname(self.path), exist_ok=True)
            cmd = ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                   "-lms", "100"]
            if self.uuid:
                cmd[1:1] = ["-i", self.uuid]
            self.out = open(self.path, "w")
            self.proc = subprocess.Popen(cmd, stdout=self.out, stderr=subprocess.DEVNULL)
        except (OSError, ValueError):
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.out.close()
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 8:
                    continue
                try:
                    sm.append(float(parts[0]))
                    mx.append(float(parts[1]))
                except ValueError:
                    continue
                for nm, val in zip(names, parts[4:8]):
                    if val.lower() == "active":
                        reasons.add(nm)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "samples": len(sm),
                "reasons": sorted(reasons)}


def cpu_baseline(workload, G: int, sample: int, v_fmt: int):
    """The oracle (single-threaded C) on the first `sample` parameters."""
    import oracle
    from quantized_optimizer_states_b200 import inputs
    x = inputs.host_step_inputs(workload, sample)
    st = oracle.quantize_state(x["m0"], G, 0) + oracle.quantize_state(x["v0"], G, v_fmt)
    t0 = time.perf_counter()
    oracle.adamw_fp8_step(x["theta"], x["grad"], *st, step=10, group_size=G, v_fmt=v_fmt,
                          **inputs.HYPER)
    dt = time.perf_counter() - t0
    return {"value": sample / dt, "unit": "params/s", "cores": oracle.threads_used(),
            "kind": "oracle",
            "sample": f"first {sample} parameters of the {workload.name} set, one step"}


def run_reference(args):
    """--impl reference: the CPU oracle timed on bounded samples."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    from quantized_optimizer_states_b200 import inputs
    import oracle
    v_fmt = 0 if args.v_fmt == "e4m3" else 1
    w = inputs.olmo_7b(v_fmt=args.v_fmt)
    G = w.group_size
    sample = args.ref_sample
    x = inputs.host_step_inputs(w, sample)
    st = oracle.quantize_state(x["m0"], G, 0) + oracle.quantize_state(x["v0"], G, v_fmt)
    th = x["theta"]
    times = []
    for i in range(args.warmup + args.steps):
        t0 = time.perf_counter()
        out = oracle.adamw_fp8_step(th, x["grad"], *st, step=10 + i, group_size=G, v_fmt=v_fmt,
                                    **inputs.HYPER)
        dt = time.perf_counter() - t0
        th, st = out[0], out[1:7]
        if i >= args.warmup:
            times.append(dt)
    total = sum(times)
    value = sample * len(times) / total
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "params/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * total / len(times), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": {"workload": f"olmo-7b set (bounded sample of {sample} parameters per step)",
                   "group_size": G, "m_fmt": "e4m3", "v_fmt": args.v_fmt},
        "cpu_baseline": {"value": value, "unit": "params/s", "cores": oracle.threads_used(),
                         "kind": "oracle",
                         "sample": f"first {sample} parameters of the olmo-7b set per step"},
        "e2e": {"value": value, "unit": "params/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


ACT_RING = 8  # distinct activation tensors cycled by the activation bench


def run_activations(args):
    """The activation-side kernels on the activation workload (BF16 [16384,
    2048], G = 128, E4M3): 1xG quantization, Group Scaling (standalone: steps
    (i)-(iii)), the SwiGLU and LayerNorm producers with fused maxima, Group
    Scaling's steps (ii)-(iii) after a producer, and dequantization.

    Steady state: each kernel is launched back to back over a ring of
    ACT_RING distinct input (and output) sets -- 8 x 64 MiB of BF16 input
    alone, four times the 126 MB L2 -- so every launch reads its input from
    HBM, and one pair of CUDA events brackets the K timed launches (the
    event timer ticks in ~2 us steps on this part, too coarse for a single
    20 us launch).  One JSON line: elements/s of the 1xG quantizer as the
    headline; every kernel's time per launch, achieved GB/s and fraction of
    the measured HBM copy bandwidth in `kernels`."""
    import torch
    import quantized_optimizer_states_b200 as coat
    from quantized_optimizer_states_b200 import build as coat_build
    from quantized_optimizer_states_b200 import inputs
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    coat_build.build()
    coat.load()
    w0 = inputs.activations()
    G = w0.group_size
    n = w0.rows * w0.cols
    ng = n // G
    wsn = coat.coat_group_scaling_workspace_bytes(n, G) // 4
    ring = []
    for r in range(ACT_RING):
        w = inputs.activations(seed=w0.seed + 101 * r)
        gate, up = inputs.device_swiglu_inputs(w, dev)
        ring.append({
            "x": inputs.device_activations(w, dev), "gate": gate.reshape(-1), "up": up.reshape(-1),
            "q": torch.empty(n, dtype=torch.uint8, device=dev),
            "sc": torch.empty(ng, dtype=torch.float32, device=dev),
            "ws": torch.empty(wsn, dtype=torch.float32, device=dev),
            "ws_h": torch.empty(wsn, dtype=torch.float32, device=dev),
            "s1": torch.empty(1, dtype=torch.float32, device=dev),
            "h": torch.empty(n, dtype=torch.bfloat16, device=dev),
            "ln": torch.empty(w.rows, w.cols, dtype=torch.bfloat16, device=dev),
            "out": torch.empty(n, dtype=torch.float32, device=dev)})
    for b in ring:  # the producer's outputs that the after-producer case reads
        coat.coat_swiglu_group_amax(b["gate"], b["up"], b["h"], b["ws_h"], group_size=G,
                                    tensor_amax=b["ws_h"][ng:])
    cases = {
        # name: (callable on one ring slot, algorithmic bytes per element)
        "group_quant_1xG": (lambda b: coat.coat_group_quant_1xG(b["x"], b["q"], b["sc"],
                                                                group_size=G),
                            2 + 1 + 4.0 / G),
        "group_scaling_standalone": (
            lambda b: coat.coat_group_scaling_quant_pertensor(b["x"].reshape(-1), b["ws"], b["q"],
                                                              b["s1"], group_size=G),
            2 + 2 + 1 + 8.0 / G),
        "swiglu_fused_amax": (
            lambda b: coat.coat_swiglu_group_amax(b["gate"], b["up"], b["h"], b["ws_h"],
                                                  group_size=G, tensor_amax=b["ws_h"][ng:]),
            2 + 2 + 2 + 4.0 / G),
        "layernorm_fused_amax": (
            lambda b: coat.coat_norm_group_amax(b["x"], b["ln"], b["ws"], group_size=G),
            2 + 2 + 4.0 / G),
        "group_scaling_after_producer": (
            lambda b: coat.coat_group_scaling_quant_pertensor(b["h"], b["ws_h"], b["q"], b["s1"],
                                                              group_size=G,
                                                              amax_precomputed=1),
            2 + 1 + 4.0 / G),
        "group_scaling_after_producer_with_tensor_max": (
            lambda b: coat.coat_group_scaling_quant_pertensor(b["h"], b["ws_h"], b["q"], b["s1"],
                                                              group_size=G,
                                                              amax_precomputed=2),
            2 + 1),
        "dequant_pertensor": (
            lambda b: coat.coat_dequant(b["q"], None, b["s1"], b["out"], group_size=n), 1 + 4),
    }
    peaks, peak_kind = measured_peaks()
    peak = float(peaks["hbm_gbs"])
    res = {}
    stream = torch.cuda.current_stream(dev)
    sampler = ClockSampler(None)
    sampler.start()
    time.sleep(0.3)
    for name, (fn, bpe) in cases.items():
        for i in range(max(args.warmup, ACT_RING)):
            fn(ring[i % ACT_RING])
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for i in range(args.steps):
            fn(ring[i % ACT_RING])
        e1.record(stream)
        torch.cuda.synchronize()
        ms = e0.elapsed_time(e1) / args.steps
        gbs = bpe * n / (ms / 1e3) / 1e9
        res[name] = {"ms": ms, "elements_per_s": n / (ms / 1e3), "GB/s": gbs,
                     "frac_of_hbm": gbs / peak, "algorithmic_bytes_per_element": bpe}
    clocks = sampler.stop()
    head = res["group_quant_1xG"]
    line = {"metric": "elements/s for 1xG FP8 activation quantization (BF16 [16384, 2048], G=128)",
            "value": head["elements_per_s"], "unit": "elements/s", "n_gpus": 1,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": head["ms"],
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic",
            "config": {"workload": "activations [16384, 2048] BF16 with GLU spike channels",
                       "group_size": G, "fmt": "e4m3",
                       "l2": f"inputs larger than L2: a ring of {ACT_RING} distinct input sets "
                             "(512 MiB of BF16 activations) launched back to back"},
            "roofline": {"bound": "hbm", "achieved": head["GB/s"], "peak": peak, "unit": "GB/s",
                         "frac": head["frac_of_hbm"], "traffic": recorded_act_traffic(n),
                         "peak_source": f"{peak_kind} copy bandwidth"},
            "kernels": res, "clocks": clocks,
            # 1xG 1; GS standalone 2; SwiGLU 2 (zeroing the tensor-max slot, the
            # producer); LayerNorm 1; GS after the producer 2 (step (ii), cast);
            # the cast alone 1; dequant 1
            "gpu_launches": args.steps * (1 + 2 + 2 + 1 + 2 + 1 + 1)}
    print(json.dumps(line), flush=True)
    return 0


def run_optimizer(args):
    """`CoatAdamW.step()` -- the call a training loop makes -- on the OLMo-7B
    set as 226 FP32 parameters.  Headline: flat_grads=True, the gradients
    living in one flat FP32 buffer that the parameters' .grad view, read by
    the step directly (coat_adamw_fp8_step_fp32grad; algorithmic 16 + 32/G
    B/param).  Beside it: the same optimizer with per-parameter gradient
    tensors, packed to BF16 first (coat_pack_bf16; 6 + 14 + 32/G B/param),
    and the pack alone."""
    import torch
    import quantized_optimizer_states_b200 as coat
    from quantized_optimizer_states_b200 import build as coat_build
    from quantized_optimizer_states_b200 import inputs
    from quantized_optimizer_states_b200.optim import CoatAdamW
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    coat_build.build()
    coat.load()
    w = inputs.olmo_7b()
    G = w.group_size
    gen = torch.Generator(device=dev)
    gen.manual_seed(w.seed)
    stds = inputs._tensor_grad_stds(w, len(w.sizes))
    params = [torch.nn.Parameter(torch.empty(shape, device=dev).normal_(0.0, w.theta_std,
                                                                          generator=gen))
              for _, shape in inputs.OLMO_7B]
    n = sum(p.numel() for p in params)
    h = w.hyper
    opt = CoatAdamW(params, lr=h["lr"], betas=(h["beta1"], h["beta2"]), eps=h["eps"],
                    weight_decay=h["weight_decay"], group_size=G, flat_grads=True)
    with torch.no_grad():
        for p, sd in zip(params, stds):
            p.grad.normal_(0.0, float(sd), generator=gen)   # into the flat buffer
    stream = torch.cuda.current_stream(dev)

    def timed(fn):
        for _ in range(args.warmup):
            fn()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(args.steps):
            fn()
        e1.record(stream)
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / args.steps

    sampler = ClockSampler(None)
    sampler.start()
    time.sleep(0.3)
    assert opt._grads_are_views(opt._flat[0])
    ms = timed(opt.step)
    clocks = sampler.stop()
    # per-parameter gradient tensors instead: the optimizer packs them first
    with torch.no_grad():
        for p in params:
            p.grad = p.grad.clone()
    assert not opt._grads_are_views(opt._flat[0])
    packed_ms = timed(opt.step)
    pack_ms = timed(lambda: opt._gather_grads(opt._flat[0]))
    peaks, peak_kind = measured_peaks()
    peak = float(peaks["hbm_gbs"])
    bpp = 2.0 + bytes_per_param(G)
    achieved = bpp * n / (ms / 1e3) / 1e9
    line = {"metric": "params/s for CoatAdamW.step() (OLMo-7B set, FP32 parameters and gradients)",
            "value": n / (ms / 1e3), "unit": "params/s", "n_gpus": 1, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "config": {"workload": f"olmo-7b set as {len(params)} FP32 parameters, "
                                   "CoatAdamW(group_size=128, flat_grads=True)",
                       "group_size": G, "params": n,
                       "l2": "no flush needed: 112 GB moved per step"},
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                         "frac": achieved / peak, "traffic": None,
                         "peak_source": f"{peak_kind} copy bandwidth",
                         "algorithmic_bytes_per_param": bpp},
            "kernels": {"flat_grads_step_ms": ms, "packed_step_ms": packed_ms,
                        "pack_bf16_ms": pack_ms,
                        "packed_params_per_s": n / (packed_ms / 1e3)},
            "clocks": clocks, "gpu_launches": args.steps}
    print(json.dumps(line), flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="coat", choices=["coat", "reference"])
    ap.add_argument("--v-fmt", default=None, choices=["e4m3", "e5m2"],
                    help="second-moment format (default: e5m2 for the OLMo-1B set, as that "
                         "workload specifies; e4m3 otherwise)")
    ap.add_argument("--e2e-steps", type=int, default=3)
    ap.add_argument("--cpu-sample", type=int, default=1 << 25)
    ap.add_argument("--ref-sample", type=int, default=1 << 22)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--workload", default="olmo-7b",
                    choices=["olmo-7b", "olmo-1b", "sweep", "activations", "optimizer"])
    ap.add_argument("--group-size", type=int, default=128, help="sweep workload only")
    ap.add_argument("--regime", default="late", choices=["early", "late", "typical"],
                    help="sweep workload only")
    args = ap.parse_args()
    if args.warmup < 3 and args.impl == "coat":
        print("warning: fewer than 3 warm-up steps", file=sys.stderr)
    if args.v_fmt is None:
        args.v_fmt = "e5m2" if args.workload == "olmo-1b" else "e4m3"
    if args.impl == "reference":
        return run_reference(args)
    if args.workload == "activations":
        return run_activations(args)
    if args.workload == "optimizer":
        return run_optimizer(args)

    import torch
    import torch.distributed as dist
    import quantized_optimizer_states_b200 as coat
    from quantized_optimizer_states_b200 import inputs
    from quantized_optimizer_states_b200 import build as coat_build

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        from datetime import timedelta
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=timedelta(seconds=300),
                                device_id=torch.device("cuda", local))
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    coat_build.build()
    coat.load()

    v_fmt = coat.COAT_E4M3 if args.v_fmt == "e4m3" else coat.COAT_E5M2
    if args.workload == "olmo-7b":
        w = inputs.olmo_7b(seed=1237 + rank, v_fmt=args.v_fmt)
    elif args.workload == "olmo-1b":
        w = inputs.olmo_1b(seed=1235 + rank)
        w.v_fmt = args.v_fmt
    else:
        w = inputs.sweep(args.group_size, args.v_fmt, args.regime, seed=1238 + rank)
    n, G = w.n, w.group_size
    ng = -(-n // G)
    hyper = dict(w.hyper)

    # ---- inputs resident in HBM --------------------------------------------------
    theta, grad, chunks = inputs.device_step_inputs(w, dev)
    m_code = torch.empty(n, dtype=torch.uint8, device=dev)
    v_code = torch.empty(n, dtype=torch.uint8, device=dev)
    m_k = torch.empty(ng, dtype=torch.float32, device=dev)
    m_s = torch.empty_like(m_k)
    v_k = torch.empty_like(m_k)
    v_s = torch.empty_like(m_k)
    for off, m0, v0 in chunks():
        c = m0.numel()
        g0, g1 = off // G, -(-(off + c) // G)
        coat.coat_quantize_state(m0, m_code[off:off + c], m_k[g0:g1], m_s[g0:g1], group_size=G,
                                 fmt=coat.COAT_E4M3)
        coat.coat_quantize_state(v0, v_code[off:off + c], v_k[g0:g1], v_s[g0:g1], group_size=G,
                                 fmt=v_fmt)
    torch.cuda.synchronize()

    stream = torch.cuda.current_stream(dev)
    step_no = [w.step]

    def step():
        coat.coat_adamw_fp8_step(theta, grad, m_code, m_k, m_s, v_code, v_k, v_s,
                                 step=step_no[0], group_size=G, v_fmt=v_fmt, **hyper)
        step_no[0] += 1

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()

    uuid = None
    try:
        uuid = "GPU-" + str(torch.cuda.get_device_properties(dev).uuid)
    except Exception:
        uuid = None
    sampler = ClockSampler(uuid)
    sampler.start()
    time.sleep(0.3)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    evs = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps + 1)]
    # the timed region is an NVTX range, so a profiler can list exactly its launches
    torch.cuda.nvtx.range_push("timed")
    evs[0].record(stream)
    for i in range(args.steps):
        step()
        evs[i + 1].record(stream)
    torch.cuda.synchronize()
    torch.cuda.nvtx.range_pop()
    if world > 1:
        dist.barrier()
    clocks = sampler.stop()
    per = [evs[i].elapsed_time(evs[i + 1]) for i in range(args.steps)]
    total_ms = evs[0].elapsed_time(evs[-1])
    if world > 1:
        t = torch.tensor([total_ms], device=dev)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        total_ms = float(t.item())
    value = world * n * args.steps / (total_ms / 1e3)
    kernel_ms = sum(per) / len(per)

    peaks, peak_kind = measured_peaks()
    peak = float(peaks["hbm_gbs"])
    achieved = bytes_per_param(G) * n / (kernel_ms / 1e3) / 1e9
    roofline = {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                "frac": achieved / peak, "traffic": recorded_traffic(n, G),
                "peak_source": f"{peak_kind} copy bandwidth (MEASURED_PEAKS.json hbm_gbs)"
                if peak_kind == "measured" else "fallback 6650 GB/s",
                "algorithmic_bytes_per_param": bytes_per_param(G),
                "frac_of_8TBs_spec": achieved / 8000.0}

    # ---- end to end: gradients from pinned host memory each step ----------------
    e2e = None
    if args.e2e_steps > 0:
        # The step's input (the BF16 gradients) streams in from pinned host
        # memory in group-aligned chunks on a copy stream; the step runs chunk
        # by chunk (the same public call on buffer slices) as soon as its
        # gradients have arrived, so the transfer overlaps the kernel.  Every
        # chunk crosses PCIe from one pinned staging buffer of chunk size
        # (2n bytes per step, as with a full host copy, without pinning the
        # whole gradient on every rank of a multi-GPU run).
        copy_stream = torch.cuda.Stream(device=dev)
        nchunks = 16
        per = -(-n // nchunks)
        per = -(-per // 4096) * 4096
        bounds = [(a, min(n, a + per)) for a in range(0, n, per)]
        host_grad = torch.empty(per, dtype=torch.bfloat16, pin_memory=True)
        host_grad.copy_(grad[:per])
        result = torch.empty(4, dtype=torch.float32, pin_memory=True)
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()

        def e2e_step():
            t = step_no[0]
            done = []
            for a, b in bounds:
                with torch.cuda.stream(copy_stream):
                    grad[a:b].copy_(host_grad[:b - a], non_blocking=True)
                    ev = torch.cuda.Event()
                    ev.record(copy_stream)
                done.append(ev)
            for (a, b), ev in zip(bounds, done):
                stream.wait_event(ev)
                g0, g1 = a // G, -(-b // G)
                coat.coat_adamw_fp8_step(theta[a:b], grad[a:b], m_code[a:b], m_k[g0:g1],
                                         m_s[g0:g1], v_code[a:b], v_k[g0:g1], v_s[g0:g1],
                                         step=t, group_size=G, v_fmt=v_fmt, **hyper)
            # the next step's copies must not overwrite gradients still in use
            copy_stream.wait_stream(stream)
            step_no[0] += 1
            result[0:1].copy_(m_k[-1:], non_blocking=True)
            result[1:2].copy_(m_s[-1:], non_blocking=True)
            result[2:3].copy_(v_k[-1:], non_blocking=True)
            result[3:4].copy_(v_s[-1:], non_blocking=True)

        e2e_step()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(args.e2e_steps):
            e2e_step()
        e1.record(stream)
        torch.cuda.synchronize()
        e2e_ms = e0.elapsed_time(e1)
        if world > 1:
            t = torch.tensor([e2e_ms], device=dev)
            dist.all_reduce(t, op=dist.ReduceOp.MAX)
            e2e_ms = float(t.item())
        e2e = {"value": world * n * args.e2e_steps / (e2e_ms / 1e3), "unit": "params/s",
               "h2d_bytes_per_step": 2 * n, "d2h_bytes_per_step": 16,
               "what": "BF16 gradients copied from pinned host memory every step in 16 chunks "
                       "(from one chunk-sized pinned staging buffer) on a copy stream, each "
                       "chunk stepped as soon as it has arrived (coat_adamw_fp8_step on the "
                       "slices), then a 16-byte read-back of the last group's (k, s) pairs"}
        del host_grad

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(w, G, args.cpu_sample, v_fmt)

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "params/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": total_ms / args.steps, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "config": {"workload": f"{w.name} set: {n} FP32 params, BF16 grads, FP8 m (e4m3) / "
                                   f"v ({args.v_fmt}) + per-group k, scale",
                       "group_size": G, "m_fmt": "e4m3", "v_fmt": args.v_fmt,
                       "params_per_gpu": n, "parallelism": f"{world} independent shards",
                       "l2": f"no flush needed: {bytes_per_param(G) * n / 1e9:.1f} GB moved "
                             "per step, far above the 126 MB L2"},
            "roofline": roofline,
            "cpu_baseline": cpu,
            "e2e": e2e,
            "gpu_launches": args.steps,
            "clocks": clocks,
            "kernel_ms": kernel_ms,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
