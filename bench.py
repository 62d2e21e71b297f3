#!/usr/bin/env python
"""Benchmark of the fused COAT FP8-state AdamW step on B200.

One step = one coat_adamw_fp8_step over the whole OLMo-7B-shaped parameter
set (6,888,095,744 FP32 parameters, BF16 gradients, FP8 m/v with per-group
k and scale, G = 128) resident in HBM.  Prints ONE JSON line (rank 0).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--v-fmt e4m3|e5m2]
  python bench.py --impl reference ...    # the CPU oracle on a bounded sample

Multi-GPU (`--gpus N`, N > 1; started through torchrun by this script when
it is not already running under it): the ZeRO-1 data-parallel step over one
parameter set split at group boundaries -- BF16 reduce-scatter of every
rank's full gradient, the fused step on each rank's 1/N shard, BF16
all-gather of the updated parameters (quantized_optimizer_states_b200.zero).
Total work is fixed as N grows: strong scaling, value = parameters of the
set / max-over-ranks time.  `--workload ranks` only checks that all N ranks
join the process group.
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


# sources of the 1xG quantizer (its traffic record is valid while these are
# unchanged): the activation header up to the end of the 1xG section (the
# shared helpers and the 1xG kernels; the producers and the other kernels
# below it do not enter the 1xG launch), and the headers it includes
ACT_KERNEL_SOURCES = [("quantized_optimizer_states_b200/csrc/act_kernels.cuh",
                       "// ---- Group Scaling per-tensor quantization"),
                      "quantized_optimizer_states_b200/csrc/step_kernels.cuh",
                      "quantized_optimizer_states_b200/csrc/state_codec.cuh",
                      "quantized_optimizer_states_b200/csrc/fp8_device.cuh"]


def kernel_source_hash(sources=None) -> str:
    """Hash of the kernel sources a traffic record was captured from; an
    entry (path, marker) takes the file up to the line that starts with the
    marker."""
    h = hashlib.sha256()
    for ent in (KERNEL_SOURCES if sources is None else sources):
        rel, marker = ent if isinstance(ent, tuple) else (ent, None)
        with open(os.path.join(ROOT, rel), "rb") as f:
            data = f.read()
        if marker is not None:
            cut = data.find(b"\n" + marker.encode())
            if cut < 0:
                raise ValueError(f"{rel}: no line starts with {marker!r}")
            data = data[:cut + 1]
        h.update(data)
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


def host_cores() -> int:
    """Host cores this process may run on (nproc)."""
    try:
        return len(os.sched_getaffinity(0))
    except (AttributeError, OSError):
        return os.cpu_count() or 1


def oracle_step_threads(x, st, G: int, v_fmt: int, threads: int, step: int = 10) -> float:
    """One oracle step over a host sample split into `threads` group-aligned
    slices, each stepped by its own thread (the oracle is a plain C call
    through ctypes, which releases the GIL while it runs); returns seconds."""
    from concurrent.futures import ThreadPoolExecutor
    import oracle
    from quantized_optimizer_states_b200 import inputs
    n = x["theta"].size
    ng = -(-n // G)
    per = -(-ng // threads) * G
    cuts = [(a, min(n, a + per)) for a in range(0, n, per)]

    def run(ab):
        a, b = ab
        g0, g1 = a // G, -(-b // G)
        oracle.adamw_fp8_step(x["theta"][a:b], x["grad"][a:b], st[0][a:b], st[1][g0:g1],
                              st[2][g0:g1], st[3][a:b], st[4][g0:g1], st[5][g0:g1], step=step,
                              group_size=G, v_fmt=v_fmt, **inputs.HYPER)

    with ThreadPoolExecutor(max_workers=len(cuts)) as ex:
        t0 = time.perf_counter()
        list(ex.map(run, cuts))
        return time.perf_counter() - t0


def cpu_baseline(workload, G: int, sample: int, v_fmt: int):
    """The oracle (plain single-threaded C, run as it stands) on the first
    `sample` parameters: once on one thread, once split at group boundaries
    over every host core."""
    import oracle
    from quantized_optimizer_states_b200 import inputs
    x = inputs.host_step_inputs(workload, sample)
    st = oracle.quantize_state(x["m0"], G, 0) + oracle.quantize_state(x["v0"], G, v_fmt)
    one = oracle_step_threads(x, st, G, v_fmt, 1)
    cores = host_cores()
    allc = oracle_step_threads(x, st, G, v_fmt, cores)
    return {"value": sample / allc, "unit": "params/s", "cores": cores, "kind": "oracle",
            "sample": f"first {sample} parameters of the {workload.name} set, one step, split "
                      f"at group boundaries over {cores} threads",
            "single_thread": {"value": sample / one, "cores": 1}}


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
    cores = host_cores()
    times = []
    for i in range(args.warmup + args.steps):
        # the oracle on every host core (group-aligned slices, one per thread);
        # each step starts from the same state, as the steps of one sample
        dt = oracle_step_threads(x, st, G, v_fmt, cores, step=10 + i)
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
        "cpu_baseline": {"value": value, "unit": "params/s", "cores": cores,
                         "kind": "oracle",
                         "sample": f"first {sample} parameters of the olmo-7b set per step, "
                                   f"split at group boundaries over {cores} threads"},
        "e2e": {"value": value, "unit": "params/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


ACT_RING = 8  # distinct activation tensors cycled by the activation bench


def measure_activations(dev, steps: int, warmup: int):
    """Time the activation-side kernels on the activation workload (see
    run_activations); returns (per-kernel results, clock summary, n, G,
    peak, peak kind)."""
    import torch
    import quantized_optimizer_states_b200 as coat
    from quantized_optimizer_states_b200 import inputs
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
        # name: (callable on one ring slot, algorithmic bytes per element,
        #        kernel launches per call)
        "group_quant_1xG": (lambda b: coat.coat_group_quant_1xG(b["x"], b["q"], b["sc"],
                                                                group_size=G),
                            2 + 1 + 4.0 / G, 1),
        # zeroing the tensor maximum, step (i), the cast
        "group_scaling_standalone": (
            lambda b: coat.coat_group_scaling_quant_pertensor(b["x"].reshape(-1), b["ws"], b["q"],
                                                              b["s1"], group_size=G),
            2 + 2 + 1 + 8.0 / G, 3),
        # zeroing its tensor-maximum slot, the producer
        "swiglu_fused_amax": (
            lambda b: coat.coat_swiglu_group_amax(b["gate"], b["up"], b["h"], b["ws_h"],
                                                  group_size=G, tensor_amax=b["ws_h"][ng:]),
            2 + 2 + 2 + 4.0 / G, 2),
        # the same two: handed a whole workspace, the producer also writes
        # the tensor maximum into its last slot
        "layernorm_fused_amax": (
            lambda b: coat.coat_norm_group_amax(b["x"], b["ln"], b["ws"], group_size=G),
            2 + 2 + 4.0 / G, 2),
        # zeroing, step (ii), the cast
        "group_scaling_after_producer": (
            lambda b: coat.coat_group_scaling_quant_pertensor(b["h"], b["ws_h"], b["q"], b["s1"],
                                                              group_size=G,
                                                              amax_precomputed=1),
            2 + 1 + 4.0 / G, 3),
        # the cast alone
        "group_scaling_after_producer_with_tensor_max": (
            lambda b: coat.coat_group_scaling_quant_pertensor(b["h"], b["ws_h"], b["q"], b["s1"],
                                                              group_size=G,
                                                              amax_precomputed=2),
            2 + 1, 1),
        "dequant_pertensor": (
            lambda b: coat.coat_dequant(b["q"], None, b["s1"], b["out"], group_size=n), 1 + 4, 1),
    }
    peaks, peak_kind = measured_peaks()
    peak = float(peaks["hbm_gbs"])
    res = {}
    stream = torch.cuda.current_stream(dev)
    sampler = ClockSampler(None)
    sampler.start()
    time.sleep(0.3)
    for name, (fn, bpe, launches) in cases.items():
        for i in range(max(warmup, ACT_RING)):
            fn(ring[i % ACT_RING])
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for i in range(steps):
            fn(ring[i % ACT_RING])
        e1.record(stream)
        torch.cuda.synchronize()
        ms = e0.elapsed_time(e1) / steps
        gbs = bpe * n / (ms / 1e3) / 1e9
        res[name] = {"ms": ms, "elements_per_s": n / (ms / 1e3), "GB/s": gbs,
                     "frac_of_hbm": gbs / peak, "algorithmic_bytes_per_element": bpe,
                     "launches_per_call": launches}
    clocks = sampler.stop()
    return res, clocks, n, G, peak, peak_kind


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
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    coat_build.build()
    coat.load()
    res, clocks, n, G, peak, peak_kind = measure_activations(dev, args.steps, args.warmup)
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
            "gpu_launches": args.steps * sum(r["launches_per_call"] for r in res.values())}
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


def main(argv=None):
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
    ap.add_argument("--ref-sample", type=int, default=1 << 24)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extra", action="store_true",
                    help="skip the records beside the headline (the other v format, the "
                         "activation kernels, the OLMo-1B set and the 2^28 sweep)")
    ap.add_argument("--variant-steps", type=int, default=10)
    ap.add_argument("--workload", default="olmo-7b",
                    choices=["olmo-7b", "olmo-1b", "sweep", "activations", "optimizer",
                             "ranks"])
    ap.add_argument("--group-size", type=int, default=128, help="sweep workload only")
    ap.add_argument("--regime", default="late", choices=["early", "late", "typical"],
                    help="sweep workload only")
    ap.add_argument("--zero1-path", default="peers", choices=["peers", "nccl"],
                    help="ZeRO-1 step: one kernel over peer memory (peers) or NCCL "
                         "reduce-scatter, step, NCCL all-gather (nccl)")
    ap.add_argument("--zero1", action="store_true",
                    help="time the ZeRO-1 data-parallel step even on one GPU (a one-rank "
                         "process group: the collectives reduce to copies)")
    ap.add_argument("--launch-timeout", type=int, default=3600,
                    help="seconds before the ranks started by --gpus N are stopped")
    args = ap.parse_args(argv)
    if args.warmup < 3 and args.impl == "coat":
        print("warning: fewer than 3 warm-up steps", file=sys.stderr)
    if args.v_fmt is None:
        args.v_fmt = "e5m2" if args.workload == "olmo-1b" else "e4m3"
    if args.impl == "reference":
        return run_reference(args)
    world = int(os.environ.get("WORLD_SIZE", "0"))
    if args.gpus > 1 and world == 0:
        # not started by torchrun: start the N ranks (one process per GPU) here
        return launch_ranks(args.gpus, sys.argv[1:] if argv is None else list(argv),
                            args.launch_timeout)
    if args.workload == "ranks":
        return run_ranks(args)
    if args.workload == "activations":
        return run_activations(args)
    if args.workload == "optimizer":
        return run_optimizer(args)
    if world > 1 or args.zero1:
        return run_zero1(args)
    return run_step(args)


def free_port() -> int:
    import socket
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def launch_command(n: int, argv: list[str], timeout_s: int, port: int) -> list[str]:
    """torchrun over n local ranks running this script with the same
    arguments, bounded by `timeout -k 60` (a last resort above the process
    group's own timeout)."""
    return ["timeout", "-k", "60", str(timeout_s), sys.executable, "-m",
            "torch.distributed.run", "--nnodes=1", f"--nproc-per-node={n}",
            "--master-addr", "127.0.0.1", "--master-port", str(port),
            os.path.abspath(__file__), *argv]


def launch_ranks(n: int, argv: list[str], timeout_s: int) -> int:
    """`bench.py --gpus N` run without torchrun: start N ranks through
    torchrun (rendezvous on 127.0.0.1) and return their exit status; rank 0
    prints the JSON line.  NCCL's communicator set-up lines stay on
    (NCCL_DEBUG=INFO, subsystem INIT) so the ranks can be counted in the log."""
    env = dict(os.environ)
    env.setdefault("NCCL_DEBUG", "INFO")
    env.setdefault("NCCL_DEBUG_SUBSYS", "INIT")
    return subprocess.run(launch_command(n, argv, timeout_s, free_port()), env=env).returncode


def init_ranks(timeout_s: int = 300, single: bool = False):
    """Join the process group torchrun set up: NCCL with one GPU per rank, or
    gloo where there is no GPU; returns (world, rank, local rank).  With
    `single`, a process not started by torchrun forms a one-rank group."""
    import torch
    import torch.distributed as dist
    from datetime import timedelta
    if single and "WORLD_SIZE" not in os.environ:
        os.environ.update(WORLD_SIZE="1", RANK="0", LOCAL_RANK="0", MASTER_ADDR="127.0.0.1",
                          MASTER_PORT=str(free_port()))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if (world > 1 or single) and not dist.is_initialized():
        # NCCL's communicator set-up lines, so the log shows every rank joining
        os.environ.setdefault("NCCL_DEBUG", "INFO")
        os.environ.setdefault("NCCL_DEBUG_SUBSYS", "INIT")
        if torch.cuda.is_available():
            torch.cuda.set_device(local)
            dist.init_process_group("nccl", timeout=timedelta(seconds=timeout_s),
                                    device_id=torch.device("cuda", local))
        else:
            dist.init_process_group("gloo", timeout=timedelta(seconds=timeout_s))
    return world, rank, local


def run_ranks(args):
    """--workload ranks: every rank joins the process group and adds one to
    an all-reduce; rank 0 prints how many ranks took part (no kernels)."""
    import torch
    import torch.distributed as dist
    world, rank, local = init_ranks()
    dev = torch.device("cuda", local) if torch.cuda.is_available() else torch.device("cpu")
    joined = world
    if world > 1:
        t = torch.ones(1, dtype=torch.float32, device=dev)
        dist.all_reduce(t)
        joined = int(t.item())
    if rank == 0:
        print(json.dumps({"workload": "ranks", "n_gpus": world, "ranks_joined": joined,
                          "backend": dist.get_backend() if world > 1 else None}), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def step_workload(args, seed_offset: int = 0):
    from quantized_optimizer_states_b200 import inputs
    if args.workload == "olmo-7b":
        return inputs.olmo_7b(seed=1237 + seed_offset, v_fmt=args.v_fmt)
    if args.workload == "olmo-1b":
        w = inputs.olmo_1b(seed=1235 + seed_offset)
        w.v_fmt = args.v_fmt
        return w
    return inputs.sweep(args.group_size, args.v_fmt, args.regime, seed=1238 + seed_offset)


def run_zero1(args):
    """N > 1 ranks (one GPU each): the ZeRO-1 data-parallel step over ONE
    parameter set split at group boundaries (zero.Zero1Shard): BF16
    reduce-scatter of every rank's full gradient, coat_adamw_fp8_step on the
    rank's 1/N shard, BF16 all-gather of the updated parameters.  Total work
    is fixed as N grows (strong scaling); value = parameters of the set per
    second of the slowest rank.  The three phases are timed with CUDA events
    on the launching stream (the collectives are ordered on it)."""
    import torch
    import torch.distributed as dist
    import quantized_optimizer_states_b200 as coat
    from quantized_optimizer_states_b200 import inputs, zero
    from quantized_optimizer_states_b200 import build as coat_build

    world, rank, local = init_ranks(single=True)
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    if rank == 0:
        coat_build.build()
    dist.barrier()
    coat.load()
    v_fmt = coat.COAT_E4M3 if args.v_fmt == "e4m3" else coat.COAT_E5M2
    # every rank: the same parameters, its own gradient
    w = step_workload(args)
    n, G = w.n, w.group_size
    hyper = dict(w.hyper)
    theta, grad_unused, chunks = inputs.device_step_inputs(w, dev)
    del grad_unused
    shard = zero.Zero1Shard(theta, group_size=G, v_fmt=v_fmt)
    del theta
    L, lo = shard.L, rank * shard.L
    for off, m0, v0 in chunks():          # initial states of this rank's shard
        a, b = max(off, lo), min(off + m0.numel(), lo + L, n)
        if a >= b:
            continue
        g0, g1 = (a - lo) // G, -(-(b - lo) // G)
        coat.coat_quantize_state(m0[a - off:b - off], shard.m_code[a - lo:b - lo],
                                 shard.m_k[g0:g1], shard.m_s[g0:g1], group_size=G,
                                 fmt=coat.COAT_E4M3)
        coat.coat_quantize_state(v0[a - off:b - off], shard.v_code[a - lo:b - lo],
                                 shard.v_k[g0:g1], shard.v_s[g0:g1], group_size=G, fmt=v_fmt)
    wg = step_workload(args, seed_offset=1000 * (rank + 1))
    th_unused, g_rank, _ = inputs.device_step_inputs(wg, dev)
    del th_unused
    peers = args.zero1_path == "peers"
    peer_fallback = None
    if peers:
        # every rank's gradient and parameter buffers, mapped into every rank;
        # if the mapping fails on any rank, every rank takes the NCCL path
        try:
            bufs = zero.PeerBuffers(shard, torch.bfloat16)
            ok = 1
        except Exception as e:  # noqa: BLE001 -- reported in the JSON line
            bufs, ok, peer_fallback = None, 0, f"{type(e).__name__}: {e}"[:300]
        flag = torch.tensor([ok], dtype=torch.int32, device=dev)
        dist.all_reduce(flag, op=dist.ReduceOp.MIN)
        if int(flag.item()) == 0:
            peers = False
            peer_fallback = peer_fallback or "the peer-buffer mapping failed on another rank"
            del bufs
    if peers:
        grad = bufs.grad
    else:
        grad = torch.zeros(shard.padded_numel, dtype=torch.bfloat16, device=dev)
    grad[:n].copy_(g_rank)             # the flat gradient, padded: no copy per step
    del g_rank
    torch.cuda.empty_cache()
    torch.cuda.synchronize()

    stream = torch.cuda.current_stream(dev)
    step_no = [w.step]
    marks = []

    def step(record=False):
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(4)] if record else None
        if peers:
            # phases: barrier + kernel + barrier, the kernel alone in ev[1..2]
            if record:
                ev[0].record(stream)
            shard.step_peers(bufs, step_no[0], hyper,
                             kernel_events=(ev[1], ev[2]) if record else None)
            if record:
                ev[3].record(stream)
                marks.append(ev)
            step_no[0] += 1
            return
        if record:
            ev[0].record(stream)
        g = shard.reduce_gradient_bf16(grad)
        if record:
            ev[1].record(stream)
        zero._coat_step(shard, g, step_no[0], hyper)
        if record:
            ev[2].record(stream)
        shard.gather_params(torch.bfloat16)
        if record:
            ev[3].record(stream)
            marks.append(ev)
        step_no[0] += 1

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    sampler = ClockSampler(None) if rank == 0 else None
    if sampler:
        sampler.start()
        time.sleep(0.3)
    dist.barrier()
    torch.cuda.synchronize()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    torch.cuda.nvtx.range_push("timed")
    t0.record(stream)
    for _ in range(args.steps):
        step(record=True)
    t1.record(stream)
    torch.cuda.synchronize()
    torch.cuda.nvtx.range_pop()
    dist.barrier()
    clocks = sampler.stop() if sampler else None
    total_ms = t0.elapsed_time(t1)
    rs_ms = sum(e[0].elapsed_time(e[1]) for e in marks) / args.steps
    st_ms = sum(e[1].elapsed_time(e[2]) for e in marks) / args.steps
    ag_ms = sum(e[2].elapsed_time(e[3]) for e in marks) / args.steps
    t = torch.tensor([total_ms, rs_ms, st_ms, ag_ms], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    total_ms, rs_ms, st_ms, ag_ms = (float(x) for x in t.tolist())

    # ---- end to end: each rank's gradient from pinned host memory every step ----
    e2e = None
    if args.e2e_steps > 0:
        nchunks = 16
        per = -(-n // nchunks)
        host = torch.empty(per, dtype=torch.bfloat16, pin_memory=True)
        host.copy_(grad[:per])
        result = torch.empty(4, dtype=torch.float32, pin_memory=True)
        torch.cuda.synchronize()

        def e2e_step():
            for a in range(0, n, per):
                b = min(n, a + per)
                grad[a:b].copy_(host[:b - a], non_blocking=True)
            step()
            result[0:1].copy_(shard.m_k[-1:], non_blocking=True)
            result[1:2].copy_(shard.m_s[-1:], non_blocking=True)
            result[2:3].copy_(shard.v_k[-1:], non_blocking=True)
            result[3:4].copy_(shard.v_s[-1:], non_blocking=True)

        e2e_step()
        torch.cuda.synchronize()
        dist.barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(args.e2e_steps):
            e2e_step()
        e1.record(stream)
        torch.cuda.synchronize()
        t = torch.tensor([e0.elapsed_time(e1)], dtype=torch.float64, device=dev)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        e2e = {"value": n * args.e2e_steps / (float(t.item()) / 1e3), "unit": "params/s",
               "h2d_bytes_per_step": 2 * n * world, "d2h_bytes_per_step": 16 * world,
               "what": "every rank's BF16 gradient copied from pinned host memory every step "
                       "(16 chunks through one chunk-sized pinned staging buffer), then the "
                       "ZeRO-1 step, then a 16-byte read-back of the last group's (k, s) pairs "
                       "on every rank"}
        del host

    if rank == 0 and peers:
        print(json.dumps(zero1_peers_line(args, w, shard, world, total_ms, rs_ms, st_ms, ag_ms,
                                          e2e, clocks)), flush=True)
    elif rank == 0:
        peaks, peak_kind = measured_peaks()
        peak = float(peaks["hbm_gbs"])
        achieved = bytes_per_param(G) * L / (st_ms / 1e3) / 1e9
        # ring collectives: (N - 1)/N of the buffer leaves (and enters) each rank
        frac = (world - 1) / world
        rs_bytes, ag_bytes = frac * 2 * shard.padded_numel, frac * 2 * shard.padded_numel
        line = {
            "metric": METRIC, "value": n * args.steps / (total_ms / 1e3), "unit": "params/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": total_ms / args.steps, "higher_is_better": True,
            "scaling": "strong", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "config": {"workload": f"{w.name} set: {n} FP32 params, BF16 grads, FP8 m (e4m3) / "
                                   f"v ({args.v_fmt}) + per-group k, scale",
                       "group_size": G, "m_fmt": "e4m3", "v_fmt": args.v_fmt,
                       "params_per_gpu": L,
                       "parallelism": f"zero1 dp{world}: BF16 reduce-scatter of each rank's "
                                      "full gradient, coat_adamw_fp8_step on the rank's "
                                      f"1/{world} shard, BF16 all-gather of the parameters",
                       "l2": "no flush needed: every phase moves far more than the 126 MB L2"},
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                         "frac": achieved / peak, "traffic": None,
                         "peak_source": f"{peak_kind} copy bandwidth",
                         "kernel": "coat_adamw_fp8_step on the shard",
                         "algorithmic_bytes_per_param": bytes_per_param(G)},
            "collectives": {"reduce_scatter_ms": rs_ms, "step_ms": st_ms,
                            "all_gather_ms": ag_ms,
                            "reduce_scatter_GBps_per_rank": rs_bytes / (rs_ms / 1e3) / 1e9
                            if rs_bytes else None,
                            "all_gather_GBps_per_rank": ag_bytes / (ag_ms / 1e3) / 1e9
                            if ag_bytes else None,
                            "link_peak_GBps": 770.0,
                            "link_peak_source": "measured peer copy per direction on this pool",
                            "bytes_per_rank_per_step": rs_bytes + ag_bytes},
            "cpu_baseline": None,
            "e2e": e2e,
            # the step kernel, plus a tail launch when the shard is not a whole
            # number of 1024-parameter blocks (the division after the
            # reduce-scatter and the BF16 rounding before the all-gather are
            # torch's)
            "gpu_launches": args.steps * (1 + (L % 1024 != 0)),
            "clocks": clocks,
        }
        if peer_fallback:
            line["peer_path_unavailable"] = peer_fallback
        print(json.dumps(line), flush=True)
    if peers:
        del bufs, grad              # unmap the other ranks' buffers before any rank exits
        torch.cuda.synchronize()
    dist.barrier()
    dist.destroy_process_group()
    return 0


LINK_GBPS = 770.0   # measured peer copy per direction on this machine


def zero1_peers_bytes(L: int, world: int, G: int) -> dict:
    """Algorithmic bytes of one rank's one-kernel ZeRO-1 step on a shard of L
    parameters: HBM of the rank's own GPU (the step's 14 + 32/G B, the
    BF16 copy of its updated shard into its own buffer, and its gradient
    read by the other ranks: 2 (W - 1) B per shard parameter) and NVLink
    per direction (in: the other ranks' gradients of its shard and their
    updated shards written into its buffer; out: the same amounts in the
    other direction), 2 (W - 1) + 2 (W - 1) B per shard parameter."""
    hbm = (bytes_per_param(G) + 2 + 2 * (world - 1) + 2 * (world - 1)) * L
    link = 4 * (world - 1) * L
    return {"hbm": hbm, "link_per_direction": link}


def zero1_peers_line(args, w, shard, world, total_ms, bar0_ms, kern_ms, bar1_ms, e2e, clocks):
    """The JSON line of the one-kernel ZeRO-1 path: value = parameters of the
    set per second of the slowest rank; the kernel's roofline is the slower
    of its HBM bytes at the measured copy bandwidth and its NVLink bytes at
    the measured peer-copy bandwidth."""
    peaks, peak_kind = measured_peaks()
    hbm_peak = float(peaks["hbm_gbs"])
    n, G, L = w.n, w.group_size, shard.L
    b = zero1_peers_bytes(L, world, G)
    t_hbm = b["hbm"] / (hbm_peak * 1e9)
    t_link = b["link_per_direction"] / (LINK_GBPS * 1e9)
    bound = "hbm" if t_hbm >= t_link else "nvlink"
    target_s = max(t_hbm, t_link)
    kern_s = kern_ms / 1e3
    if bound == "hbm":
        roof = {"bound": "hbm", "achieved": b["hbm"] / kern_s / 1e9, "peak": hbm_peak,
                "unit": "GB/s", "peak_source": f"{peak_kind} copy bandwidth"}
    else:
        roof = {"bound": "nvlink", "achieved": b["link_per_direction"] / kern_s / 1e9,
                "peak": LINK_GBPS, "unit": "GB/s",
                "peak_source": "measured peer copy per direction on this pool"}
    roof.update(frac=target_s / kern_s, traffic=None,
                kernel="coat_adamw_fp8_step_peers on the shard (gradient mean, step, "
                       "parameter copies into every rank)",
                algorithmic_bytes=b)
    return {
        "metric": METRIC, "value": n * args.steps / (total_ms / 1e3), "unit": "params/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": total_ms / args.steps, "higher_is_better": True, "scaling": "strong",
        "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": {"workload": f"{w.name} set: {n} FP32 params, BF16 grads, FP8 m (e4m3) / "
                               f"v ({args.v_fmt}) + per-group k, scale",
                   "group_size": G, "m_fmt": "e4m3", "v_fmt": args.v_fmt,
                   "params_per_gpu": L,
                   "parallelism": f"zero1 dp{world}: one kernel per rank reads every rank's "
                                  "BF16 gradient of its 1/N shard over peer memory, steps "
                                  "the shard and writes the BF16 parameters into every "
                                  "rank's buffer, between two barriers of the ranks",
                   "l2": "no flush needed: every step moves far more than the 126 MB L2"},
        "roofline": roof,
        "phases": {"barrier_ms": bar0_ms + bar1_ms, "kernel_ms": kern_ms},
        "cpu_baseline": None,
        "e2e": e2e,
        # the fused kernel, plus a tail launch when the shard is not a whole
        # number of 1024-parameter blocks (the barriers are NCCL's)
        "gpu_launches": args.steps * (1 + (L % 1024 != 0)),
        "clocks": clocks,
    }


def time_step_set(w, v_fmt: int, steps: int, warmup: int, dev) -> dict:
    """The public step on workload w (inputs built on the device, states
    quantized with coat_quantize_state), `steps` timed steps after `warmup`,
    CUDA events on the launching stream; returns its record."""
    import torch
    import quantized_optimizer_states_b200 as coat
    from quantized_optimizer_states_b200 import inputs
    n, G = w.n, w.group_size
    ng = -(-n // G)
    theta, grad, chunks = inputs.device_step_inputs(w, dev)
    mc = torch.empty(n, dtype=torch.uint8, device=dev)
    vc = torch.empty(n, dtype=torch.uint8, device=dev)
    mk, ms, vk, vs = (torch.empty(ng, dtype=torch.float32, device=dev) for _ in range(4))
    for off, m0, v0 in chunks():
        c = m0.numel()
        g0, g1 = off // G, -(-(off + c) // G)
        coat.coat_quantize_state(m0, mc[off:off + c], mk[g0:g1], ms[g0:g1], group_size=G,
                                 fmt=coat.COAT_E4M3)
        coat.coat_quantize_state(v0, vc[off:off + c], vk[g0:g1], vs[g0:g1], group_size=G,
                                 fmt=v_fmt)
    t = [w.step]

    def step():
        coat.coat_adamw_fp8_step(theta, grad, mc, mk, ms, vc, vk, vs, step=t[0], group_size=G,
                                 v_fmt=v_fmt, **w.hyper)
        t[0] += 1

    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize()
    ms_ = e0.elapsed_time(e1) / steps
    peak = float(measured_peaks()[0]["hbm_gbs"])
    gbs = bytes_per_param(G) * n / (ms_ / 1e3) / 1e9
    del theta, grad, mc, vc, mk, ms, vk, vs
    torch.cuda.empty_cache()
    return {"params": n, "group_size": G,
            "v_fmt": "e4m3" if v_fmt == coat.COAT_E4M3 else "e5m2", "steps": steps,
            "ms_per_step": ms_, "params_per_s": n / (ms_ / 1e3), "GB/s": gbs,
            "frac_of_hbm": gbs / peak}


def clock_normalised(value, clocks):
    """value x (max SM clock / median SM clock under load), or None when the
    clocks were not sampled."""
    med, top = (clocks or {}).get("sm_mhz"), (clocks or {}).get("sm_max_mhz")
    if not med or not top:
        return None
    return {"params_per_s_at_max_clock": value * top / med, "sm_mhz": med, "sm_max_mhz": top}


def run_step(args):
    """One GPU: coat_adamw_fp8_step over the whole resident parameter set."""
    import torch
    import quantized_optimizer_states_b200 as coat
    from quantized_optimizer_states_b200 import inputs
    from quantized_optimizer_states_b200 import build as coat_build

    world, rank, local = 1, 0, int(os.environ.get("LOCAL_RANK", "0"))
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    coat_build.build()
    coat.load()

    v_fmt = coat.COAT_E4M3 if args.v_fmt == "e4m3" else coat.COAT_E5M2
    w = step_workload(args)
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
    clocks = sampler.stop()
    per = [evs[i].elapsed_time(evs[i + 1]) for i in range(args.steps)]
    total_ms = evs[0].elapsed_time(evs[-1])
    value = n * args.steps / (total_ms / 1e3)
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
        e2e = {"value": n * args.e2e_steps / (e2e_ms / 1e3), "unit": "params/s",
               "h2d_bytes_per_step": 2 * n, "d2h_bytes_per_step": 16,
               "what": "BF16 gradients copied from pinned host memory every step in 16 chunks "
                       "(from one chunk-sized pinned staging buffer) on a copy stream, each "
                       "chunk stepped as soon as it has arrived (coat_adamw_fp8_step on the "
                       "slices), then a 16-byte read-back of the last group's (k, s) pairs"}
        del host_grad

    cpu = None
    if not args.no_cpu_baseline:
        cpu = cpu_baseline(w, G, args.cpu_sample, v_fmt)

    # ---- the rest of the path, recorded beside the headline -------------------------
    variant = acts = sets = None
    if not args.no_extra:
        # the other second-moment format of the same set: v re-quantized, timed alone
        other = coat.COAT_E5M2 if v_fmt == coat.COAT_E4M3 else coat.COAT_E4M3
        for off, m0, v0 in chunks():
            c = m0.numel()
            g0, g1 = off // G, -(-(off + c) // G)
            coat.coat_quantize_state(v0, v_code[off:off + c], v_k[g0:g1], v_s[g0:g1],
                                     group_size=G, fmt=other)
        torch.cuda.synchronize()

        def step_other():
            coat.coat_adamw_fp8_step(theta, grad, m_code, m_k, m_s, v_code, v_k, v_s,
                                     step=step_no[0], group_size=G, v_fmt=other, **hyper)
            step_no[0] += 1

        for _ in range(3):
            step_other()
        sampler = ClockSampler(uuid)
        sampler.start()
        time.sleep(0.2)
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(args.variant_steps):
            step_other()
        e1.record(stream)
        torch.cuda.synchronize()
        vclocks = sampler.stop()
        vms = e0.elapsed_time(e1) / args.variant_steps
        vgbs = bytes_per_param(G) * n / (vms / 1e3) / 1e9
        variant = {"v_fmt": "e5m2" if other == coat.COAT_E5M2 else "e4m3", "steps": args.variant_steps,
                   "ms_per_step": vms, "params_per_s": n / (vms / 1e3), "GB/s": vgbs,
                   "frac_of_hbm": vgbs / peak, "clocks": vclocks}
        # the activation-side kernels on the activation workload
        res, aclocks, an, aG, _, _ = measure_activations(dev, 40, 8)
        acts = {"workload": "activations [16384, 2048] BF16 with GLU spike channels, G = 128, "
                            "E4M3; 40 launches over a ring of 8 input sets",
                "kernels": res, "clocks": aclocks,
                "roofline_1xG_traffic": recorded_act_traffic(an)}
        # the other parameter sets: OLMo-1B (v E5M2) and the 2^28 group-size /
        # format sweep (late regime), with the big set's buffers released first
        del theta, grad, m_code, v_code, m_k, m_s, v_k, v_s
        torch.cuda.empty_cache()
        sampler = ClockSampler(uuid)
        sampler.start()
        sets = {"olmo_1b_v_e5m2": time_step_set(inputs.olmo_1b(), coat.COAT_E5M2, 10, 3, dev),
                "sweep_2p28_late": [time_step_set(inputs.sweep(gs, vf, "late"),
                                                  coat.COAT_E4M3 if vf == "e4m3"
                                                  else coat.COAT_E5M2, 10, 3, dev)
                                    for gs in (32, 64, 128, 256, 1024)
                                    for vf in ("e4m3", "e5m2")],
                "sweep_2p28_early_G128": [time_step_set(inputs.sweep(128, vf, "early"),
                                                        coat.COAT_E4M3 if vf == "e4m3"
                                                        else coat.COAT_E5M2, 10, 3, dev)
                                          for vf in ("e4m3", "e5m2")]}
        sets["clocks"] = sampler.stop()

    line = {
        "metric": METRIC, "value": value, "unit": "params/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": total_ms / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": {"workload": f"{w.name} set: {n} FP32 params, BF16 grads, FP8 m (e4m3) / "
                               f"v ({args.v_fmt}) + per-group k, scale",
                   "group_size": G, "m_fmt": "e4m3", "v_fmt": args.v_fmt,
                   "params_per_gpu": n, "parallelism": "one GPU",
                   "l2": f"no flush needed: {bytes_per_param(G) * n / 1e9:.1f} GB moved "
                         "per step, far above the 126 MB L2"},
        "roofline": roofline,
        "cpu_baseline": cpu,
        "e2e": e2e,
        "gpu_launches": args.steps,
        "clocks": clocks,
        # the headline scaled by max / median SM clock of the timed region:
        # what the same kernel gives where the power cap does not lower the
        # clock (an estimate beside the measured value, not a measurement)
        "clock_normalised": clock_normalised(value, clocks),
        "kernel_ms": kernel_ms,
        # beside the headline, outside its timed region
        "variant_other_v_fmt": variant,
        "activation_kernels": acts,
        "other_parameter_sets": sets,
    }
    print(json.dumps(line), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
