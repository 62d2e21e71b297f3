"""Seeded synthetic inputs for the COAT step and the activation quantizers.

This module only draws random numbers with the shapes and distributions of
the workloads; it holds none of the method's arithmetic (no quantization,
no optimizer math).  The tests feed its host arrays to both the oracle and
the CUDA library; the benchmark and the full-size tests draw the same
distributions directly on the device.

Workloads (shapes from the OLMo models the COAT summary page trains on, its
section "结果和边界"; distributions are synthetic stand-ins for real
checkpoints and data, which are not used):
  tiny        one flat tensor of 2^20 parameters
  olmo-1b     d=2048, 16 layers, MLP 8192, vocab 50304, tied embedding
  olmo-7b     d=4096, 32 layers, MLP 11008, vocab 50304, untied head
  sweep       one flat tensor of 2^28 parameters
  activations BF16 [16384, 2048] with GLU-style spike channels
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np

# AdamW hyper-parameters of the workloads (beta1, beta2, lr, eps, lambda).
HYPER = dict(beta1=0.9, beta2=0.999, lr=1e-4, eps=1e-8, weight_decay=0.1)


def olmo_shapes(d_model: int, n_layers: int, d_mlp: int, vocab: int, tied: bool):
    """Parameter tensors of an OLMo-style decoder in storage order.

    OLMo's LayerNorm is non-parametric, so there are no norm weights.
    """
    shapes = [("embed", (vocab, d_model))]
    for layer in range(n_layers):
        for nm in ("q", "k", "v", "o"):
            shapes.append((f"l{layer}.{nm}", (d_model, d_model)))
        shapes.append((f"l{layer}.up", (d_mlp, d_model)))
        shapes.append((f"l{layer}.gate", (d_mlp, d_model)))
        shapes.append((f"l{layer}.down", (d_model, d_mlp)))
    if not tied:
        shapes.append(("lm_head", (vocab, d_model)))
    return shapes


OLMO_1B = olmo_shapes(2048, 16, 8192, 50304, tied=True)
OLMO_7B = olmo_shapes(4096, 32, 11008, 50304, tied=False)


def tensor_sizes(shapes) -> list[int]:
    return [int(np.prod(s)) for _, s in shapes]


@dataclass
class StepWorkload:
    """Distribution recipe of one optimizer-step workload."""
    name: str
    n: int
    seed: int
    sizes: list[int] | None = None     # per-tensor sizes (None: one tensor)
    theta_std: float = 0.02
    grad_std: float = 1e-3             # used when grad_std_lognormal is None
    grad_std_lognormal: tuple[float, float] | None = None  # (mu, sigma) per tensor
    zero_frac: float = 0.0             # fraction of gradients set to exactly 0
    spike_frac: float = 0.0            # fraction of gradients multiplied by spike_mult
    spike_mult: float = 100.0
    m_std: float = 1e-4
    v_mu: float = -18.0
    v_sigma: float = 1.0
    group_size: int = 128
    v_fmt: str = "e4m3"
    step: int = 10
    hyper: dict = field(default_factory=lambda: dict(HYPER))


def tiny(seed: int = 1234) -> StepWorkload:
    return StepWorkload("tiny", 1 << 20, seed)


def olmo_1b(seed: int = 1235) -> StepWorkload:
    sizes = tensor_sizes(OLMO_1B)
    return StepWorkload("olmo-1b", sum(sizes), seed, sizes=sizes, grad_std_lognormal=(-7.0, 1.0),
                        zero_frac=0.01, spike_frac=0.001, v_fmt="e5m2")


def olmo_7b(seed: int = 1237, v_fmt: str = "e4m3") -> StepWorkload:
    sizes = tensor_sizes(OLMO_7B)
    return StepWorkload("olmo-7b", sum(sizes), seed, sizes=sizes, grad_std_lognormal=(-7.0, 1.0),
                        zero_frac=0.01, spike_frac=0.001, v_fmt=v_fmt)


def sweep(G: int, v_fmt: str, regime: str, seed: int = 1238, n: int = 1 << 28) -> StepWorkload:
    """Group-size / format sweep; regime 'early' (v ~ logN(-25, 2)),
    'late' (v ~ logN(-14, 2)) or 'typical' (v ~ logN(-18, 0.25))."""
    mu, sigma = {"early": (-25.0, 2.0), "late": (-14.0, 2.0), "typical": (-18.0, 0.25)}[regime]
    return StepWorkload(f"sweep-G{G}-{v_fmt}-{regime}", n, seed, v_mu=mu, v_sigma=sigma,
                        group_size=G, v_fmt=v_fmt)


def _bf16_bits(x: np.ndarray) -> np.ndarray:
    """float32 -> BF16 bit patterns (uint16) via torch's nearest-even cast."""
    import torch
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16).copy()


def _tensor_grad_stds(w: StepWorkload, count: int) -> np.ndarray:
    """Per-tensor gradient standard deviations (same on host and device)."""
    if w.grad_std_lognormal is None:
        return np.full(count, w.grad_std)
    mu, sg = w.grad_std_lognormal
    return np.random.default_rng(w.seed + 1).lognormal(mu, sg, count)


def host_step_inputs(w: StepWorkload, n: int | None = None) -> dict:
    """Host arrays for a step workload (first n elements when n is given).

    Returns theta f32[n], grad uint16[n] (BF16 bits), m0 f32[n], v0 f32[n]:
    theta ~ N(0, theta_std^2); grad ~ N(0, sigma_T^2) per tensor (sigma_T
    lognormal, or grad_std), then zero_frac exact zeros and spike_frac
    spikes (disjoint); m0 ~ N(0, m_std^2); v0 ~ logN(v_mu, v_sigma^2).
    """
    n = w.n if n is None else n
    rng = np.random.default_rng(w.seed)
    theta = rng.normal(0.0, w.theta_std, n).astype(np.float32)
    sizes = w.sizes or [w.n]
    stds = _tensor_grad_stds(w, len(sizes))
    per_elem_std = np.empty(n, dtype=np.float64)
    off = 0
    for sz, sd in zip(sizes, stds):
        if off >= n:
            break
        per_elem_std[off:min(n, off + sz)] = sd
        off += sz
    grad = rng.standard_normal(n) * per_elem_std
    if w.zero_frac or w.spike_frac:
        u = rng.random(n)
        grad[u < w.zero_frac] = 0.0
        sp = (u >= w.zero_frac) & (u < w.zero_frac + w.spike_frac)
        grad[sp] *= w.spike_mult
    m0 = rng.normal(0.0, w.m_std, n).astype(np.float32)
    v0 = rng.lognormal(w.v_mu, w.v_sigma, n).astype(np.float32)
    return dict(theta=theta, grad=_bf16_bits(grad.astype(np.float32)), m0=m0, v0=v0)


# ---- device-side draws (same distributions, torch's CUDA generator) -------

def device_step_inputs(w: StepWorkload, device, chunk: int = 1 << 28):
    """Allocate and fill theta (f32) and grad (bf16) on `device`.

    Returns (theta, grad, state_chunks) where state_chunks() yields
    (offset, m0_chunk, v0_chunk) float32 device tensors of at most `chunk`
    elements, so the FP32 initial moments are never all resident at once.
    """
    import torch
    gen = torch.Generator(device=device)
    gen.manual_seed(w.seed)
    n = w.n
    theta = torch.empty(n, dtype=torch.float32, device=device)
    grad = torch.empty(n, dtype=torch.bfloat16, device=device)
    sizes = w.sizes or [n]
    stds = _tensor_grad_stds(w, len(sizes))
    for off in range(0, n, chunk):
        c = min(chunk, n - off)
        theta[off:off + c].normal_(0.0, w.theta_std, generator=gen)
    tmp = torch.empty(min(chunk, n), dtype=torch.float32, device=device)
    toff = 0
    for sz, sd in zip(sizes, stds):
        for off in range(0, sz, chunk):
            c = min(chunk, sz - off)
            t = tmp[:c]
            t.normal_(0.0, float(sd), generator=gen)
            if w.zero_frac or w.spike_frac:
                u = torch.rand(c, device=device, generator=gen)
                t.masked_fill_(u < w.zero_frac, 0.0)
                sp = (u >= w.zero_frac) & (u < w.zero_frac + w.spike_frac)
                t.mul_(torch.where(sp, w.spike_mult, 1.0))
                del u, sp
            grad[toff + off:toff + off + c].copy_(t)
        toff += sz
    del tmp

    def state_chunks():
        g2 = torch.Generator(device=device)
        g2.manual_seed(w.seed + 7919)
        for off in range(0, n, chunk):
            c = min(chunk, n - off)
            m0 = torch.empty(c, dtype=torch.float32, device=device).normal_(
                0.0, w.m_std, generator=g2)
            v0 = torch.empty(c, dtype=torch.float32, device=device).log_normal_(
                w.v_mu, w.v_sigma, generator=g2)
            yield off, m0, v0

    return theta, grad, state_chunks


# ---- activations -----------------------------------------------------------

@dataclass
class ActWorkload:
    name: str
    rows: int
    cols: int
    seed: int
    spike_frac: float = 0.0005      # fraction of channels carrying spikes
    spike_lo: float = 50.0
    spike_hi: float = 500.0
    group_size: int = 128


def activations(seed: int = 1236) -> ActWorkload:
    """BF16 RMSNorm/SwiGLU-input-like activations: 8 x 2048 tokens by 2048
    channels, N(0, 1), with GLU-style spike channels (COAT summary page,
    section "激活为什么难压": outliers one to two orders of magnitude above
    typical values)."""
    return ActWorkload("activations", 16384, 2048, seed)


def _spike_channels(w: ActWorkload, rng: np.random.Generator) -> np.ndarray:
    count = max(1, int(round(w.spike_frac * w.cols)))
    return rng.choice(w.cols, size=count, replace=False)


def host_activations(w: ActWorkload, rows: int | None = None) -> np.ndarray:
    """uint16 BF16 bits [rows, cols]."""
    rows = w.rows if rows is None else rows
    rng = np.random.default_rng(w.seed)
    x = rng.standard_normal((rows, w.cols)).astype(np.float32)
    ch = _spike_channels(w, rng)
    mult = rng.uniform(w.spike_lo, w.spike_hi, (rows, ch.size)).astype(np.float32)
    x[:, ch] *= mult
    return _bf16_bits(x).reshape(rows, w.cols)


def device_activations(w: ActWorkload, device):
    import torch
    gen = torch.Generator(device=device)
    gen.manual_seed(w.seed)
    x = torch.randn(w.rows, w.cols, device=device, generator=gen)
    ch = torch.from_numpy(_spike_channels(w, np.random.default_rng(w.seed))).to(device)
    mult = torch.empty(w.rows, ch.numel(), device=device).uniform_(w.spike_lo, w.spike_hi,
                                                                   generator=gen)
    x[:, ch] *= mult
    return x.to(torch.bfloat16)


def host_swiglu_inputs(w: ActWorkload, rows: int | None = None):
    """(gate, up) uint16 BF16 bits [rows, cols] for the SwiGLU producer:
    gate ~ N(0, 1.5^2), up ~ N(0, 1) with the workload's GLU-style spike
    channels scaled by U[spike_lo, spike_hi] per token."""
    rows = w.rows if rows is None else rows
    rng = np.random.default_rng(w.seed + 17)
    gate = (rng.standard_normal((rows, w.cols)) * 1.5).astype(np.float32)
    up = rng.standard_normal((rows, w.cols)).astype(np.float32)
    ch = _spike_channels(w, rng)
    up[:, ch] *= rng.uniform(w.spike_lo, w.spike_hi, (rows, ch.size)).astype(np.float32)
    return _bf16_bits(gate).reshape(rows, w.cols), _bf16_bits(up).reshape(rows, w.cols)


def device_swiglu_inputs(w: ActWorkload, device):
    import torch
    gen = torch.Generator(device=device)
    gen.manual_seed(w.seed + 17)
    gate = torch.randn(w.rows, w.cols, device=device, generator=gen) * 1.5
    up = torch.randn(w.rows, w.cols, device=device, generator=gen)
    ch = torch.from_numpy(_spike_channels(w, np.random.default_rng(w.seed + 17))).to(device)
    up[:, ch] *= torch.empty(w.rows, ch.numel(), device=device).uniform_(
        w.spike_lo, w.spike_hi, generator=gen)
    return gate.to(torch.bfloat16), up.to(torch.bfloat16)
