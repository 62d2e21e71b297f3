"""`CoatAdamW`: a torch.optim.Optimizer over COAT FP8 optimizer states.

AdamW with decoupled weight decay (LLM Atlas "systems/numerics", section 08
"Adam -> AdamW") whose first and second moments are stored as FP8 codes with
a per-1xG-group expansion exponent k and scale s (COAT summary page, section
"扩展函数：把窄分布拉宽"), on FP32 master weights with BF16 gradients.  The
whole update of a parameter group is one `coat_adamw_fp8_step` call.

Layout.  The tensors of a parameter group are laid end to end in one flat
buffer, each padded to a multiple of the group size G (so that no 1xG group
straddles two tensors and every slice starts 16-byte aligned).  The flat
buffers are: FP32 master weights, BF16 gradients, m and v codes (uint8), and
per group m_k, m_s, v_k, v_s (float32).  Padding elements hold zeros and stay
zero (a zero moment with a zero gradient on a zero weight is a fixed point of
the rule).

* FP32 parameters become views into the master buffer (the step updates them
  in place); their FP32 gradients are cast to BF16 (round to nearest even)
  into the flat gradient buffer before each step.
* BF16 parameters keep a separate FP32 master copy; their BF16 gradients are
  copied into the flat buffer, and after the step the master values are
  rounded back into the parameters.
Both moves are one multi-tensor launch per 128 parameters
(coat_pack_bf16 / coat_unpack_bf16), not one copy per parameter.

With flat_grads=True, FP32 parameter groups also get a flat FP32 gradient
buffer and every parameter's .grad becomes a view into it; backward then
accumulates in place into the buffer, and the step reads it directly
(coat_adamw_fp8_step_fp32grad rounds each gradient to BF16 as it loads it),
so no separate pack pass runs.  zero_grad() zeroes the buffer and keeps the
views (a .grad replaced by another tensor is noticed and packed instead).

Fresh states are all-zero groups (codes 0, k = 1, s = 0).  `state_dict()`
holds the flat buffers themselves, so saving and loading reproduces the run
bit for bit.
"""
from __future__ import annotations

import operator
from dataclasses import dataclass

import torch

from . import _lib


def padded_layout(numels: list[int], group_size: int) -> tuple[list[int], int]:
    """Offsets of tensors laid end to end, each padded to a multiple of
    max(G, 16) elements, and the total padded length."""
    if group_size < 1:
        raise ValueError("group_size must be >= 1")
    unit = max(group_size, 16)
    offsets, off = [], 0
    for n in numels:
        if n < 0:
            raise ValueError("negative tensor size")
        offsets.append(off)
        off += -(-n // unit) * unit
    return offsets, off


def _check_group_size(G) -> None:
    """The 1xG group sizes the step kernels are built for: powers of two
    from 16 to 4096."""
    try:
        g = operator.index(G)          # Python or NumPy integers, not floats
    except TypeError:
        g = None
    if g is None or g < 16 or g > 4096 or g & (g - 1):
        raise ValueError(f"group_size must be a power of two in [16, 4096], got {G!r}")


@dataclass
class _FlatGroup:
    params: list
    offsets: list[int]
    n: int
    master: torch.Tensor
    grad: torch.Tensor | None   # flat BF16 gradients (allocated on first use)
    m_code: torch.Tensor
    v_code: torch.Tensor
    m_k: torch.Tensor
    m_s: torch.Tensor
    v_k: torch.Tensor
    v_s: torch.Tensor
    bf16_params: bool
    table: _lib.PackTable
    grad32: torch.Tensor | None = None   # flat FP32 gradients (flat_grads)
    step: int = 0


_FMT = {"e4m3": _lib.COAT_E4M3, "e5m2": _lib.COAT_E5M2,
        _lib.COAT_E4M3: _lib.COAT_E4M3, _lib.COAT_E5M2: _lib.COAT_E5M2}


class CoatAdamW(torch.optim.Optimizer):
    """AdamW with FP8 (COAT) moments.

    Args:
      params: CUDA tensors (all FP32 or all BF16 within a parameter group).
      lr, betas, eps, weight_decay: the AdamW hyper-parameters.
      group_size: G of the 1xG quantization groups (power of two, 16..4096).
      v_fmt: "e4m3" (default) or "e5m2" for the second moment; the first
        moment is always E4M3.
      k_range: 0 = k fills E4M3's range for both moments, 1 = the storage
        format's own range.
      k_max: clamp of the expansion exponent (0 = none).
      skip_nonfinite: count inf/NaN gradients first (on the device) and skip
        the whole step of a parameter group that has any; the group's step
        counter then does not advance (one host read of the count per step).
      flat_grads: give FP32 parameter groups a flat FP32 gradient buffer that
        the parameters' .grad view (see the module docstring).
    """

    def __init__(self, params, lr: float = 1e-3, betas=(0.9, 0.999), eps: float = 1e-8,
                 weight_decay: float = 1e-2, *, group_size: int = 128, v_fmt="e4m3",
                 k_range: int = 0, k_max: float = 64.0, skip_nonfinite: bool = False,
                 flat_grads: bool = False):
        if not 0.0 <= betas[0] < 1.0 or not 0.0 <= betas[1] < 1.0:
            raise ValueError("betas must be in [0, 1)")
        if lr < 0.0 or eps < 0.0 or weight_decay < 0.0:
            raise ValueError("lr, eps and weight_decay must be non-negative")
        if v_fmt not in _FMT:
            raise ValueError("v_fmt must be 'e4m3' or 'e5m2'")
        _check_group_size(group_size)
        if k_range not in (0, 1):
            raise ValueError("k_range must be 0 (E4M3's range) or 1 (the storage format's)")
        if not k_max >= 0.0:
            raise ValueError("k_max must be >= 0 (0: no clamp)")
        defaults = dict(lr=lr, betas=tuple(betas), eps=eps, weight_decay=weight_decay,
                        group_size=group_size, v_fmt=_FMT[v_fmt], k_range=k_range,
                        k_max=k_max)
        super().__init__(params, defaults)
        self.skip_nonfinite = skip_nonfinite
        self.skipped_steps = 0
        self._flat_grads = flat_grads
        self._flat: list[_FlatGroup] = [self._build(g) for g in self.param_groups]

    def add_param_group(self, param_group):
        """torch.optim's add_param_group, with the group's COAT settings
        checked first (v_fmt may be given by name); a group added after
        construction gets its flat buffers at once -- step() walks one
        _FlatGroup per parameter group, in the same order -- or, if they
        cannot be built, is not added."""
        param_group = dict(param_group)
        if "v_fmt" in param_group:
            if param_group["v_fmt"] not in _FMT:
                raise ValueError("v_fmt must be 'e4m3' or 'e5m2'")
            param_group["v_fmt"] = _FMT[param_group["v_fmt"]]
        if "group_size" in param_group:
            _check_group_size(param_group["group_size"])
        if param_group.get("k_range", 0) not in (0, 1):
            raise ValueError("k_range must be 0 (E4M3's range) or 1 (the storage format's)")
        if not param_group.get("k_max", 0.0) >= 0.0:
            raise ValueError("k_max must be >= 0 (0: no clamp)")
        super().add_param_group(param_group)
        if hasattr(self, "_flat"):
            try:
                self._flat.append(self._build(self.param_groups[-1]))
            except Exception:
                self.param_groups.pop()
                raise

    # ---- flat buffers --------------------------------------------------------

    def _build(self, group) -> _FlatGroup:
        ps = list(group["params"])
        if not ps:
            raise ValueError("empty parameter group")
        dev = ps[0].device
        if dev.type != "cuda":
            raise ValueError("CoatAdamW needs CUDA parameters")
        if any(p.device != dev for p in ps):
            raise ValueError("the parameters of a group must be on one device")
        _check_group_size(group["group_size"])
        dtypes = {p.dtype for p in ps}
        if dtypes not in ({torch.float32}, {torch.bfloat16}):
            raise ValueError("a parameter group must be all float32 or all bfloat16")
        bf16 = dtypes == {torch.bfloat16}
        G = group["group_size"]
        offsets, n = padded_layout([p.numel() for p in ps], G)
        ng = -(-n // G)
        master = torch.zeros(n, dtype=torch.float32, device=dev)
        with torch.no_grad():
            for p, off in zip(ps, offsets):
                master[off:off + p.numel()].copy_(p.detach().reshape(-1))
                if not bf16:
                    # the parameter becomes a view of the master buffer
                    p.data = master[off:off + p.numel()].view_as(p)
        z8 = lambda: torch.zeros(n, dtype=torch.uint8, device=dev)  # noqa: E731
        fg = _FlatGroup(
            params=ps, offsets=offsets, n=n, master=master,
            grad=None,
            m_code=z8(), v_code=z8(),
            m_k=torch.ones(ng, dtype=torch.float32, device=dev),
            m_s=torch.zeros(ng, dtype=torch.float32, device=dev),
            v_k=torch.ones(ng, dtype=torch.float32, device=dev),
            v_s=torch.zeros(ng, dtype=torch.float32, device=dev),
            bf16_params=bf16, table=_lib.PackTable([p.numel() for p in ps], offsets))
        if self._flat_grads and not bf16:
            fg.grad32 = torch.zeros(n, dtype=torch.float32, device=dev)
            self._attach_grad_views(fg)
        return fg

    def _attach_grad_views(self, fg: _FlatGroup):
        for p, off in zip(fg.params, fg.offsets):
            p.grad = fg.grad32[off:off + p.numel()].view_as(p)

    def _grads_are_views(self, fg: _FlatGroup) -> bool:
        base, size = fg.grad32.data_ptr(), fg.grad32.element_size()
        return all(p.grad is not None and p.grad.data_ptr() == base + off * size
                   and p.grad.is_contiguous() for p, off in zip(fg.params, fg.offsets))

    def zero_grad(self, set_to_none: bool = True):
        super().zero_grad(set_to_none=set_to_none)
        for fg in self._flat:
            if fg.grad32 is not None:
                fg.grad32.zero_()
                self._attach_grad_views(fg)

    @torch.no_grad()
    def _gather_grads(self, fg: _FlatGroup):
        if fg.grad is None:
            fg.grad = torch.zeros(fg.n, dtype=torch.bfloat16, device=fg.master.device)
        want = torch.bfloat16 if fg.bf16_params else torch.float32
        grads = []
        for p in fg.params:
            g = p.grad
            if g is not None:
                g = g.detach()
                if g.dtype != want:
                    g = g.to(want)
                if not g.is_contiguous():
                    g = g.contiguous()
            grads.append(g)  # None: the slice is zero-filled
        _lib.coat_pack_bf16(grads, fg.table, fg.grad)

    @torch.no_grad()
    def _write_back_bf16(self, fg: _FlatGroup):
        if all(p.is_contiguous() for p in fg.params):
            _lib.coat_unpack_bf16(fg.master, fg.table, [p.data for p in fg.params])
        else:
            for p, off in zip(fg.params, fg.offsets):
                p.copy_(fg.master[off:off + p.numel()].view_as(p))

    # ---- the step --------------------------------------------------------------

    @torch.no_grad()
    def step(self, closure=None):
        loss = None
        if closure is not None:
            with torch.enable_grad():
                loss = closure()
        for group, fg in zip(self.param_groups, self._flat):
            # each group's launches go to its own device (and that device's
            # current stream), whatever device is current
            with torch.cuda.device(fg.master.device):
                self._step_group(group, fg)
        return loss

    def _step_group(self, group, fg: _FlatGroup):
        direct = (fg.grad32 is not None and not self.skip_nonfinite
                  and self._grads_are_views(fg))
        if not direct:
            self._gather_grads(fg)
        if self.skip_nonfinite:
            count = torch.zeros(1, dtype=torch.int32, device=fg.grad.device)
            _lib.coat_count_nonfinite_bf16(fg.grad, count)
            if int(count.item()) != 0:
                self.skipped_steps += 1
                return
        fg.step += 1
        b1, b2 = group["betas"]
        _lib.coat_adamw_fp8_step(
            fg.master, fg.grad32 if direct else fg.grad, fg.m_code, fg.m_k, fg.m_s,
            fg.v_code, fg.v_k, fg.v_s,
            beta1=b1, beta2=b2, lr=group["lr"], eps=group["eps"],
            weight_decay=group["weight_decay"], step=fg.step,
            group_size=group["group_size"], v_fmt=group["v_fmt"],
            k_range=group["k_range"], k_max=group["k_max"])
        if fg.bf16_params:
            self._write_back_bf16(fg)

    # ---- inspection ------------------------------------------------------------

    @torch.no_grad()
    def dequantized_moments(self, group_index: int = 0):
        """(m, v) of a parameter group as FP32 flat tensors (padded layout),
        decoded by coat_dequant."""
        fg = self._flat[group_index]
        G = self.param_groups[group_index]["group_size"]
        vf = self.param_groups[group_index]["v_fmt"]
        m = torch.empty(fg.n, dtype=torch.float32, device=fg.master.device)
        v = torch.empty_like(m)
        with torch.cuda.device(fg.master.device):
            _lib.coat_dequant(fg.m_code, fg.m_k, fg.m_s, m, group_size=G, fmt=_lib.COAT_E4M3)
            _lib.coat_dequant(fg.v_code, fg.v_k, fg.v_s, v, group_size=G, fmt=vf)
        return m, v

    def state_stats(self, group_index: int = 0) -> dict:
        """Monitoring counts of a parameter group's two compressed moments
        (coat_state_stats): {"m": {...}, "v": {...}}."""
        fg = self._flat[group_index]
        G = self.param_groups[group_index]["group_size"]
        vf = self.param_groups[group_index]["v_fmt"]
        with torch.cuda.device(fg.master.device):
            return {"m": _lib.coat_state_stats(fg.m_code, fg.m_k, fg.m_s, group_size=G,
                                               fmt=_lib.COAT_E4M3),
                    "v": _lib.coat_state_stats(fg.v_code, fg.v_k, fg.v_s, group_size=G,
                                               fmt=vf)}

    def flat_master(self, group_index: int = 0) -> torch.Tensor:
        return self._flat[group_index].master

    # ---- checkpoints -----------------------------------------------------------

    _KEYS = ("master", "m_code", "v_code", "m_k", "m_s", "v_k", "v_s")

    def state_dict(self):
        sd = super().state_dict()
        sd["coat"] = [{"step": fg.step, "n": fg.n, "offsets": list(fg.offsets),
                       **{k: getattr(fg, k).detach().clone() for k in self._KEYS}}
                      for fg in self._flat]
        return sd

    def load_state_dict(self, state_dict):
        coat = state_dict.get("coat")
        if coat is None or len(coat) != len(self._flat):
            raise ValueError("not a CoatAdamW state dict for this parameter layout")
        rest = {k: v for k, v in state_dict.items() if k != "coat"}
        super().load_state_dict(rest)
        with torch.no_grad():
            for fg, saved in zip(self._flat, coat):
                if saved["n"] != fg.n or list(saved["offsets"]) != list(fg.offsets):
                    raise ValueError("parameter layout differs from the checkpoint")
                for k in self._KEYS:
                    getattr(fg, k).copy_(saved[k].to(getattr(fg, k).device))
                fg.step = int(saved["step"])
                if fg.bf16_params:
                    with torch.cuda.device(fg.master.device):
                        self._write_back_bf16(fg)
