"""ZeRO-1 style data-parallel COAT step over torch.distributed.

In data-parallel training every rank computes a full BF16 gradient of the
same parameters.  The optimizer state -- FP32 master weights and the FP8
moments with their per-group k and s (COAT summary page, section
"扩展函数：把窄分布拉宽") -- is partitioned across the ranks at 1xG group
boundaries, so each rank keeps 1/world of it.  One step:

  1. reduce-scatter of the gradients: each rank receives, over its shard,
     the mean of all ranks' gradients.  By default the collective sums the
     BF16 gradients themselves (2 bytes per parameter on the wire; the
     collective rounds its partial sums to BF16) and the sum is divided by
     the rank count in BF16.  With reduce_dtype=torch.float32 the BF16
     values are widened and summed in binary32 instead (4 bytes per
     parameter on the wire), one shard-sized chunk at a time so the binary32
     staging buffer stays bounded, and the mean is rounded to BF16 as the
     step loads it;
  2. the COAT step on the shard (one `coat_adamw_fp8_step` call);
  3. all-gather of the updated master weights (FP32, or each shard rounded
     to BF16 first: half the bytes).

`Zero1Shard.step_peers` does all three in one kernel per rank over peer
memory (`PeerBuffers` maps every rank's gradient and parameter buffers into
every process): the rank's kernel reads the ranks' gradients over its shard
from their buffers, averages them in binary32 in rank order, steps the
shard and writes the updated parameters into every rank's buffer; two
barriers of the ranks frame it.

No 1xG group straddles two shards, so the sharded step computes exactly
what a single-rank step over the whole buffer computes on the reduced
gradient.  The collectives go through the default (or given) process group:
NCCL over NVLink/NVSwitch on B200 nodes, gloo on CPU for the tests.

Costs per parameter of the flat buffer, per rank and step, with W ranks and
a ring collective: the reduce-scatter moves (W - 1)/W x 2 bytes each way
(BF16) or (W - 1)/W x 4 bytes (binary32); the all-gather (W - 1)/W x 4
bytes (FP32 parameters) or x 2 (BF16).  A gradient whose length is not
W x L (L = shard length) is first copied into a padded buffer (2 bytes read,
2 written); callers that allocate their flat gradient with
`padded_numel` elements skip that copy.
"""
from __future__ import annotations

import torch
import torch.distributed as dist

from . import _lib


def shard_length(n: int, group_size: int, world: int) -> int:
    """Per-rank length: ceil(n / world) rounded up to a multiple of
    max(G, 16), so every shard is whole groups and 16-byte aligned for all
    element sizes."""
    if n < 0 or group_size < 1 or world < 1:
        raise ValueError("bad shard arguments")
    unit = max(group_size, 16)
    per = -(-n // world)
    return -(-per // unit) * unit


def _coat_step(shard: "Zero1Shard", grad_shard: torch.Tensor, t: int, hyper: dict):
    with torch.cuda.device(shard.master.device):      # the shard's own device
        _lib.coat_adamw_fp8_step(
            shard.master, grad_shard, shard.m_code, shard.m_k, shard.m_s, shard.v_code,
            shard.v_k, shard.v_s, step=t, group_size=shard.group_size, v_fmt=shard.v_fmt,
            k_range=shard.k_range, k_max=shard.k_max, **hyper)


class Zero1Shard:
    """This rank's share of the COAT optimizer state for one flat parameter
    buffer of n elements.

    `theta` is the full FP32 parameter buffer (the same on every rank); the
    rank keeps a copy of its shard as master weights.  Fresh moments are
    all-zero groups (codes 0, k = 1, s = 0).  `reduce_dtype` selects the
    gradient reduce-scatter: BF16 (default) or binary32.
    """

    def __init__(self, theta: torch.Tensor, *, group_size: int = 128, v_fmt: int = 0,
                 k_range: int = 0, k_max: float = 64.0, group=None,
                 reduce_dtype: torch.dtype = torch.bfloat16):
        if reduce_dtype not in (torch.bfloat16, torch.float32):
            raise ValueError("gradients are reduced as bfloat16 or float32")
        self.reduce_dtype = reduce_dtype
        self.pg = group
        self.world = dist.get_world_size(group) if dist.is_initialized() else 1
        self.rank = dist.get_rank(group) if dist.is_initialized() else 0
        self.n = theta.numel()
        self.group_size, self.v_fmt, self.k_range, self.k_max = group_size, v_fmt, k_range, k_max
        self.L = shard_length(self.n, group_size, self.world)
        dev = theta.device
        lo = self.rank * self.L
        self.master = torch.zeros(self.L, dtype=torch.float32, device=dev)
        hi = min(self.n, lo + self.L)
        if hi > lo:
            self.master[:hi - lo].copy_(theta.reshape(-1)[lo:hi])
        ng = self.L // group_size
        self.m_code = torch.zeros(self.L, dtype=torch.uint8, device=dev)
        self.v_code = torch.zeros(self.L, dtype=torch.uint8, device=dev)
        self.m_k = torch.ones(ng, dtype=torch.float32, device=dev)
        self.v_k = torch.ones(ng, dtype=torch.float32, device=dev)
        self.m_s = torch.zeros(ng, dtype=torch.float32, device=dev)
        self.v_s = torch.zeros(ng, dtype=torch.float32, device=dev)

    _STATE = ("master", "m_code", "m_k", "m_s", "v_code", "v_k", "v_s")
    _LAYOUT = ("n", "world", "rank", "L", "group_size", "v_fmt", "k_range", "k_max")

    def state_dict(self) -> dict:
        """This rank's share of the optimizer state (copies) and the layout it
        belongs to.  Every rank saves its own; loading them back into shards
        made for the same buffer length, group size, formats and rank count
        resumes the run bit for bit (the caller keeps the step count t)."""
        return {**{k: getattr(self, k) for k in self._LAYOUT},
                **{k: getattr(self, k).detach().clone() for k in self._STATE}}

    def load_state_dict(self, sd: dict) -> None:
        """Restore a shard saved by state_dict(); the layout must match."""
        for k in self._LAYOUT:
            if sd.get(k) != getattr(self, k):
                raise ValueError(f"checkpoint {k} = {sd.get(k)!r} differs from this shard's "
                                 f"{getattr(self, k)!r}")
        with torch.no_grad():
            for k in self._STATE:
                dst = getattr(self, k)
                if tuple(sd[k].shape) != tuple(dst.shape) or sd[k].dtype != dst.dtype:
                    raise ValueError(f"checkpoint tensor {k} has the wrong shape or type")
                dst.copy_(sd[k].to(dst.device))

    @property
    def padded_numel(self) -> int:
        """Length of a flat gradient the reduce-scatter takes without a copy:
        world x L (the first n elements are the parameters', the rest zero)."""
        return self.world * self.L

    def _padded(self, grad: torch.Tensor) -> torch.Tensor:
        g = grad.reshape(-1)
        if g.numel() == self.padded_numel:
            return g
        if g.numel() != self.n:
            raise ValueError(f"gradient has {g.numel()} elements, expected {self.n} "
                             f"or {self.padded_numel}")
        buf = getattr(self, "_gpad", None)
        if buf is None or buf.dtype != g.dtype or buf.device != g.device:
            buf = torch.zeros(self.padded_numel, dtype=g.dtype, device=g.device)
            self._gpad = buf
        buf[:self.n].copy_(g)
        return buf

    # binary32 reduce-scatter: elements per chunk of a rank's shard
    F32_CHUNK = 1 << 24

    def reduce_gradient_f32(self, grad: torch.Tensor) -> torch.Tensor:
        """Mean over ranks of the full BF16 gradients, this rank's shard, in
        binary32: the values are widened and summed in binary32 by the
        collective, chunk by chunk (a staging buffer of world x F32_CHUNK
        floats), and divided by the rank count."""
        g = self._padded(grad).view(self.world, self.L)
        part = torch.empty(self.L, dtype=torch.float32, device=grad.device)
        if self.world == 1:
            part.copy_(g[0])
            return part
        C = min(self.F32_CHUNK, self.L)
        stage = torch.empty(self.world * C, dtype=torch.float32, device=grad.device)
        for off in range(0, self.L, C):
            c = min(C, self.L - off)
            st = stage[:self.world * c].view(self.world, c)
            st.copy_(g[:, off:off + c])
            dist.reduce_scatter_tensor(part[off:off + c], stage[:self.world * c],
                                       op=dist.ReduceOp.SUM, group=self.pg)
        part.div_(float(self.world))
        return part

    def reduce_gradient_bf16(self, grad: torch.Tensor) -> torch.Tensor:
        """Mean over ranks of the full BF16 gradients, this rank's shard, with
        the reduce-scatter on the BF16 values themselves (the collective's
        partial sums are BF16) and the division by the rank count in BF16."""
        g = self._padded(grad)
        if g.dtype != torch.bfloat16:
            raise ValueError("the BF16 reduce-scatter takes a BF16 gradient")
        part = torch.empty(self.L, dtype=torch.bfloat16, device=grad.device)
        if self.world == 1:
            part.copy_(g)
            return part
        dist.reduce_scatter_tensor(part, g, op=dist.ReduceOp.SUM, group=self.pg)
        part.div_(float(self.world))
        return part

    def reduce_gradient(self, grad: torch.Tensor) -> torch.Tensor:
        """The reduced gradient the step uses, as BF16: the BF16 reduce-scatter
        (reduce_dtype torch.bfloat16) or the binary32 mean rounded to BF16
        nearest-even (reduce_dtype torch.float32)."""
        if self.reduce_dtype == torch.bfloat16:
            return self.reduce_gradient_bf16(grad)
        return self.reduce_gradient_f32(grad).to(torch.bfloat16)

    def gather_params(self, dtype: torch.dtype = torch.float32) -> torch.Tensor:
        """The full updated parameter buffer (first n elements): the FP32
        master weights, or, with dtype=torch.bfloat16, each rank's shard
        rounded to BF16 (nearest even) before the all-gather, which moves
        half the bytes -- what a model that holds BF16 weights needs."""
        if dtype not in (torch.float32, torch.bfloat16):
            raise ValueError("parameters are gathered as float32 or bfloat16")
        src = self.master if dtype == torch.float32 else self.master.to(torch.bfloat16)
        full = torch.empty(self.world * self.L, dtype=dtype, device=self.master.device)
        if self.world > 1:
            # BF16 moves as pairs of 16-bit patterns in 32-bit words (a shard
            # is a whole number of 16-element units), which every backend carries
            view = torch.int32 if dtype == torch.bfloat16 else dtype
            dist.all_gather_into_tensor(full.view(view), src.view(view), group=self.pg)
        else:
            full.copy_(src)
        return full[:self.n]

    def step(self, grad: torch.Tensor, t: int, hyper: dict, step_fn=None,
             gather_dtype: torch.dtype = torch.float32) -> torch.Tensor:
        """One data-parallel step with this rank's full BF16 gradient `grad`;
        returns the full updated parameters (FP32, or BF16 with
        gather_dtype=torch.bfloat16).  `step_fn(shard, grad_shard, t, hyper)`
        replaces the CUDA step (the CPU tests pass the oracle)."""
        if step_fn is not None:
            step_fn(self, self.reduce_gradient(grad), t, hyper)
        elif self.reduce_dtype == torch.bfloat16:
            _coat_step(self, self.reduce_gradient_bf16(grad), t, hyper)
        else:
            _coat_step(self, self.reduce_gradient_f32(grad), t, hyper)  # rounded on load
        return self.gather_params(gather_dtype)

    def step_peers(self, bufs: "PeerBuffers", t: int, hyper: dict,
                   kernel_events=None) -> torch.Tensor:
        """One data-parallel step in one kernel per rank: after a barrier (every
        rank's gradient in `bufs.grad` is complete), this rank's kernel reads the
        ranks' gradients over its shard from their buffers, averages them
        (binary32 sum in rank order, divided by the rank count, rounded to
        BF16), steps its shard and writes the updated parameters into every
        rank's `bufs.param`; a second barrier follows, so every rank's
        `bufs.param` holds the whole updated set when this returns (in stream
        order).  Per parameter of the buffer and per rank: (W - 1)/W x 2 bytes of
        gradient read from other ranks and (W - 1)/W x 2 (BF16) or x 4 (FP32)
        bytes of parameters written to them, no staging buffer, one launch.
        Returns the first n elements of this rank's `bufs.param`.
        kernel_events: an optional pair of CUDA events recorded on the current
        stream around the kernel alone (for timing)."""
        dev = self.master.device
        off = self.rank * self.L
        with torch.cuda.device(dev):
            _barrier(self, dev)
            if kernel_events is not None:
                kernel_events[0].record()
            _lib.coat_adamw_fp8_step_peers(
                bufs.grads, self.master, self.m_code, self.m_k, self.m_s, self.v_code, self.v_k,
                self.v_s, grad_offset=off, params_out=bufs.params, params_out_offset=off, step=t,
                group_size=self.group_size, v_fmt=self.v_fmt, k_range=self.k_range,
                k_max=self.k_max, **hyper)
            if kernel_events is not None:
                kernel_events[1].record()
            _barrier(self, dev)
        return bufs.param[:self.n]


# ---- the step over peer memory ----------------------------------------------------

def _share(t: torch.Tensor):
    """A picklable description of a CUDA tensor that another process can map
    (CUDA IPC, as torch.multiprocessing shares CUDA tensors)."""
    from torch.multiprocessing.reductions import reduce_tensor
    return reduce_tensor(t)


def _open(shared) -> torch.Tensor:
    fn, args = shared
    return fn(*args)


class PeerBuffers:
    """Every rank's flat gradient and parameter buffers, mapped into every
    rank's process, for `Zero1Shard.step_peers`.

    `grad` (BF16, `shard.padded_numel` elements: the first n are the
    parameters', the rest stay zero) is where this rank's backward pass
    leaves its full gradient; `param` (BF16 or FP32, the same length) is where
    every rank's step writes its updated shard, so after a step it holds the
    whole updated parameter set.  `grads[r]` and `params[r]` are rank r's
    buffers as seen from this process (its own are the local tensors).  The
    buffers are exchanged once, here, through the process group (CUDA IPC
    handles; on a node with NVLink a peer's buffer is read and written over
    it).  Every rank keeps its PeerBuffers alive as long as any rank uses
    them."""

    def __init__(self, shard: "Zero1Shard", param_dtype: torch.dtype = torch.bfloat16):
        if param_dtype not in (torch.bfloat16, torch.float32):
            raise ValueError("parameters are replicated as bfloat16 or float32")
        if shard.world > _lib.COAT_MAX_PEERS:
            raise ValueError(f"at most {_lib.COAT_MAX_PEERS} ranks")
        dev = shard.master.device
        total = shard.padded_numel
        if shard.world == 1:
            self.grad = torch.zeros(total, dtype=torch.bfloat16, device=dev)
            self.param = torch.zeros(total, dtype=param_dtype, device=dev)
            self.grads, self.params = [self.grad], [self.param]
            return
        # every rank reaches the exchange, also when its own part failed, so
        # that no rank is left waiting in it
        err = None
        try:
            self.grad = torch.zeros(total, dtype=torch.bfloat16, device=dev)
            self.param = torch.zeros(total, dtype=param_dtype, device=dev)
            mine = (_share(self.grad), _share(self.param))
        except Exception as e:  # noqa: BLE001 -- re-raised after the exchange
            mine, err = None, e
        every = [None] * shard.world
        dist.all_gather_object(every, mine, group=shard.pg)
        if err is not None:
            raise err
        if any(x is None for x in every):
            raise RuntimeError("another rank could not share its buffers")
        self.grads = [self.grad if r == shard.rank else _open(every[r][0])
                      for r in range(shard.world)]
        self.params = [self.param if r == shard.rank else _open(every[r][1])
                       for r in range(shard.world)]
        # the step kernel runs on this rank's device and reads and writes the
        # other ranks' buffers where they live: enable access to every other
        # GPU among them (raises where two GPUs cannot reach each other)
        with torch.cuda.device(dev):
            for d in sorted({t.get_device() for t in self.grads + self.params} - {dev.index}):
                _lib.coat_enable_peer_access(d)


def _barrier(shard: "Zero1Shard", device: torch.device):
    """Every rank's work issued so far on its current stream is complete
    before any rank's later work runs: an all-reduce of one word on the
    stream (NCCL), or a device synchronisation and a host barrier (other
    backends)."""
    if shard.world == 1:
        return
    if dist.get_backend(shard.pg) == "nccl":
        flag = getattr(shard, "_flag", None)
        if flag is None:
            flag = shard._flag = torch.zeros(1, dtype=torch.int32, device=device)
        dist.all_reduce(flag, group=shard.pg)
    else:
        torch.cuda.synchronize(device)
        dist.barrier(group=shard.pg)
