"""ctypes binding of libcoat.so (declared in include/coat.h).

Argument marshalling only: torch tensors are passed as device pointers and
the current CUDA stream as the stream handle; every step of the computation
runs in the library's kernels.  If the library is missing or cannot be
loaded the functions raise -- there is no fallback path.
"""
from __future__ import annotations

import ctypes
import os

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "libcoat.so")

COAT_E4M3 = 0
COAT_E5M2 = 1
COAT_FORCE_K1 = 0x1

STATUS = {0: "ok", 1: "invalid argument", 2: "misaligned", 3: "unsupported", 4: "CUDA error",
          5: "non-finite", 6: "timeout"}


class CoatError(RuntimeError):
    def __init__(self, fn: str, status: int, cuda_err: int = 0):
        msg = f"{fn} failed: {STATUS.get(status, status)} (status {status})"
        if status == 4:
            msg += f", cudaError {cuda_err}"
        super().__init__(msg)
        self.status = status


class CoatAdamwCfg(ctypes.Structure):
    """Mirror of coat_adamw_cfg_t."""
    _fields_ = [
        ("beta1", ctypes.c_float),
        ("beta2", ctypes.c_float),
        ("lr", ctypes.c_float),
        ("eps", ctypes.c_float),
        ("weight_decay", ctypes.c_float),
        ("step", ctypes.c_int64),
        ("group_size", ctypes.c_int32),
        ("m_fmt", ctypes.c_int32),
        ("v_fmt", ctypes.c_int32),
        ("k_range", ctypes.c_int32),
        ("k_max", ctypes.c_float),
        ("flags", ctypes.c_int32),
    ]


_lib = None

# name -> (restype, argtypes)
_P = ctypes.c_void_p
_I64 = ctypes.c_int64
_I32 = ctypes.c_int32
_F = ctypes.c_float
SIGNATURES = {
    "coat_adamw_fp8_step": (_I32, [_P, _P, _P, _P, _P, _P, _P, _P, _I64,
                                   ctypes.POINTER(CoatAdamwCfg), _P]),
    "coat_quantize_state": (_I32, [_P, _I64, _I32, _I32, _I32, _F, _I32, _P, _P, _P, _P]),
    "coat_dequant": (_I32, [_P, _P, _P, _I64, _I64, _I32, _I32, _P, _P]),
    "coat_group_quant_1xG": (_I32, [_P, _I64, _I64, _I64, _I32, _I32, _P, _P, _P]),
    "coat_group_scaling_workspace_bytes": (_I64, [_I64, _I32]),
    "coat_group_scaling_quant_pertensor": (_I32, [_P, _I64, _I32, _I32, _P, _I32, _P, _P, _P]),
    "coat_group_scaling_quant_pertensor_noalloc": (_I32, [_P, _I64, _I32, _I32, _P, _P, _P]),
    "coat_swiglu_group_amax": (_I32, [_P, _P, _I64, _I32, _P, _P, _P, _P]),
    "coat_fp8_encode": (_I32, [_P, _I64, _I32, _P, _P]),
    "coat_norm_group_amax": (_I32, [_P, _I64, _I64, _I32, _F, _P, _P, _I32, _P, _P, _P, _P]),
    "coat_count_nonfinite_bf16": (_I32, [_P, _I64, _P, _P]),
    "coat_adamw_fp8_step_peers": (_I32, [ctypes.POINTER(_P), _I32, _I64, _P, ctypes.POINTER(_P),
                                         _I32, _I64, _P, _P, _P, _P, _P, _P, _I64,
                                         ctypes.POINTER(CoatAdamwCfg), _P]),
    "coat_enable_peer_access": (_I32, [_I32]),
    "coat_adamw_fp8_step_guarded": (_I32, [_P, _P, _P, _P, _P, _P, _P, _P, _I64,
                                           ctypes.POINTER(CoatAdamwCfg), _P, _P]),
    "coat_adamw_fp8_step_fp32grad": (_I32, [_P, _P, _P, _P, _P, _P, _P, _P, _I64,
                                            ctypes.POINTER(CoatAdamwCfg), _P]),
    "coat_pack_bf16": (_I32, [ctypes.POINTER(_P), ctypes.POINTER(_I64), ctypes.POINTER(_I64),
                              _I32, _I32, _P, _I64, _P]),
    "coat_unpack_bf16": (_I32, [_P, ctypes.POINTER(_I64), ctypes.POINTER(_I64), _I32,
                                ctypes.POINTER(_P), _I64, _P]),
    "coat_state_stats": (_I32, [_P, _P, _P, _I64, _I32, _I32, _P, _P]),
    "coat_last_cuda_error": (_I32, []),
    "coat_status_string": (ctypes.c_char_p, [_I32]),
    "coat_version": (_I32, []),
}


def load(path: str = LIB_PATH):
    """Load libcoat.so once; raise if it is not there."""
    global _lib
    if _lib is None:
        if not os.path.exists(path):
            raise RuntimeError(
                f"libcoat.so not found at {path}: build it with "
                "`python -m quantized_optimizer_states_b200.build` (nvcc, sm_100a)")
        lib = ctypes.CDLL(path)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _lib = lib
    return _lib


def _check(name: str, status: int):
    if status != 0:
        raise CoatError(name, status, load().coat_last_cuda_error())


def _current_device() -> int:
    """Index of the current CUDA device (torch's own cheap query where it
    has one: the binding runs on every call of every entry point)."""
    import torch
    get = getattr(torch._C, "_cuda_getDevice", None)
    return int(get()) if get is not None else torch.cuda.current_device()


def _stream(stream):
    """The stream handle: the given one, else torch's current stream on the
    current device (its raw handle, without building a Stream object)."""
    if stream is not None:
        return ctypes.c_void_p(int(stream))
    import torch
    raw = getattr(torch._C, "_cuda_getCurrentRawStream", None)
    if raw is not None:
        return raw(_current_device())
    return torch.cuda.current_stream().cuda_stream


def _on_current_device(t, what):
    """The kernels run on the current CUDA device; a tensor of another device
    would be an illegal address there, so it is refused on the host."""
    cur = _current_device()
    if t.get_device() != cur:
        raise ValueError(f"{what} is on {t.device} but the current device is cuda:{cur} "
                         f"(call under torch.cuda.device({t.device}))")


def _ptr(t, dtype=None, what="tensor"):
    """The device address of a contiguous CUDA tensor on the current device
    (an int, which ctypes passes as a pointer)."""
    if t is None:
        return None
    dev = t.get_device()
    if dev < 0:
        raise ValueError(f"{what} must be a CUDA tensor")
    if dev != _current_device():
        _on_current_device(t, what)
    if not t.is_contiguous():
        raise ValueError(f"{what} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{what} must be {dtype}, got {t.dtype}")
    return t.data_ptr()


def _slot(t):
    """An optional float32 device slot (e.g. a one-element view of a workspace)."""
    if t is None:
        return None
    import torch
    if t.dtype != torch.float32 or not t.is_cuda or t.numel() < 1:
        raise ValueError("tensor_amax must be a float32 CUDA tensor of at least one element")
    _on_current_device(t, "tensor_amax")
    return ctypes.c_void_p(t.data_ptr())


def _u16(t, what):
    """BF16 or int16/uint16 tensors are all passed as their bit patterns."""
    import torch
    if t.dtype not in (torch.bfloat16, torch.int16, torch.uint16):
        raise ValueError(f"{what} must hold BF16 bit patterns, got {t.dtype}")
    return _ptr(t, None, what)


def coat_adamw_fp8_step(param, grad, m_code, m_k, m_scale, v_code, v_k, v_scale, *, beta1: float,
                        beta2: float, lr: float, eps: float, weight_decay: float, step: int,
                        group_size: int = 128, m_fmt: int = COAT_E4M3, v_fmt: int = COAT_E4M3,
                        k_range: int = 0, k_max: float = 64.0, flags: int = 0,
                        skip_if_nonzero=None, stream=None):
    """One fused COAT AdamW step, in place (see include/coat.h).  grad holds
    BF16 gradients (bfloat16 / int16 / uint16 bit patterns) or float32
    gradients, which the kernel rounds to BF16 as it loads them
    (coat_adamw_fp8_step_fp32grad).  With skip_if_nonzero (a CUDA
    int32/uint32 tensor of one element) the guarded form runs: the step is a
    no-op when that word is nonzero (BF16 gradients only)."""
    import torch
    cfg = CoatAdamwCfg(beta1, beta2, lr, eps, weight_decay, step, group_size, m_fmt, v_fmt,
                       k_range, k_max, flags)
    f32 = grad.dtype == torch.float32
    if f32 and skip_if_nonzero is not None:
        raise ValueError("the guarded step takes BF16 gradients")
    n = param.numel()
    if grad.numel() != n or m_code.numel() != n or v_code.numel() != n:
        raise ValueError("grad, m_code and v_code must have as many elements as param")
    if 16 <= group_size <= 4096 and group_size & (group_size - 1) == 0:
        # (an unsupported G is reported by the library itself)
        ng = -(-n // group_size)
        if min(m_k.numel(), m_scale.numel(), v_k.numel(), v_scale.numel()) < ng:
            raise ValueError(f"k and scale arrays need ceil(n / G) = {ng} elements")
    args = [_ptr(param, torch.float32, "param"),
            _ptr(grad, None, "grad") if f32 else _u16(grad, "grad"),
            _ptr(m_code, torch.uint8, "m_code"), _ptr(m_k, torch.float32, "m_k"),
            _ptr(m_scale, torch.float32, "m_scale"), _ptr(v_code, torch.uint8, "v_code"),
            _ptr(v_k, torch.float32, "v_k"), _ptr(v_scale, torch.float32, "v_scale"),
            param.numel(), ctypes.byref(cfg)]
    if f32:
        st = load().coat_adamw_fp8_step_fp32grad(*args, _stream(stream))
        _check("coat_adamw_fp8_step_fp32grad", st)
    elif skip_if_nonzero is None:
        st = load().coat_adamw_fp8_step(*args, _stream(stream))
        _check("coat_adamw_fp8_step", st)
    else:
        if skip_if_nonzero.dtype not in (torch.int32, torch.uint32):
            raise ValueError("skip_if_nonzero must be an int32/uint32 tensor")
        st = load().coat_adamw_fp8_step_guarded(*args, _ptr(skip_if_nonzero, None, "skip"),
                                                _stream(stream))
        _check("coat_adamw_fp8_step_guarded", st)


COAT_MAX_PEERS = 8  # mirrors include/coat.h


def _peer_ptr(t, dtype, what):
    """Address of a contiguous CUDA tensor that may live on another GPU (a
    rank's buffer mapped into this process); None stays None."""
    if t is None:
        return None
    if t.get_device() < 0:
        raise ValueError(f"{what} must be a CUDA tensor")
    if not t.is_contiguous() or t.dtype != dtype:
        raise ValueError(f"{what} must be a contiguous {dtype} tensor")
    return t.data_ptr()


def coat_enable_peer_access(peer_device: int):
    """Let the current device's kernels access GPU `peer_device`'s memory
    (see include/coat.h); raises CoatError where the two cannot reach each
    other."""
    _check("coat_enable_peer_access", load().coat_enable_peer_access(int(peer_device)))


def coat_adamw_fp8_step_peers(grads, param, m_code, m_k, m_scale, v_code, v_k, v_scale, *,
                              grad_offset: int, params_out=None, params_out_offset: int = 0,
                              beta1: float, beta2: float, lr: float, eps: float,
                              weight_decay: float, step: int, group_size: int = 128,
                              m_fmt: int = COAT_E4M3, v_fmt: int = COAT_E4M3, k_range: int = 0,
                              k_max: float = 64.0, flags: int = 0, stream=None):
    """The ZeRO-1 step of this rank's shard in one kernel (see include/coat.h):
    grads = every rank's full BF16 gradient buffer (rank order; tensors that
    may live on other GPUs), the shard starting at grad_offset; params_out =
    every rank's full parameter buffer (float32 or bfloat16, one dtype for
    all; None entries or None: no copy), the shard at params_out_offset;
    param and the states are this rank's shard."""
    import torch
    world = len(grads)
    if not 1 <= world <= COAT_MAX_PEERS:
        raise ValueError(f"1 to {COAT_MAX_PEERS} ranks")
    n = param.numel()
    if m_code.numel() != n or v_code.numel() != n:
        raise ValueError("m_code and v_code must have as many elements as param")
    for g in grads:
        if g.numel() < grad_offset + n:
            raise ValueError("a gradient buffer ends before the shard does")
    out_bf16 = 0
    outs = [None] * world
    if params_out is not None:
        if len(params_out) != world:
            raise ValueError("params_out needs one entry per rank")
        dts = {t.dtype for t in params_out if t is not None}
        if len(dts) > 1 or not dts <= {torch.float32, torch.bfloat16}:
            raise ValueError("params_out tensors must all be float32 or all bfloat16")
        out_bf16 = int(dts == {torch.bfloat16})
        for r, t in enumerate(params_out):
            if t is not None and t.numel() < params_out_offset + n:
                raise ValueError("a parameter buffer ends before the shard does")
            outs[r] = _peer_ptr(t, torch.bfloat16 if out_bf16 else torch.float32,
                                f"params_out[{r}]")
    gptr = (_P * world)(*[_peer_ptr(g.view(torch.int16) if g.dtype != torch.int16 else g,
                                    torch.int16, f"grads[{r}]") for r, g in enumerate(grads)])
    optr = (_P * world)(*outs) if params_out is not None else None
    cfg = CoatAdamwCfg(beta1, beta2, lr, eps, weight_decay, step, group_size, m_fmt, v_fmt,
                       k_range, k_max, flags)
    st = load().coat_adamw_fp8_step_peers(
        gptr, world, grad_offset, _ptr(param, torch.float32, "param"), optr, out_bf16,
        params_out_offset, _ptr(m_code, torch.uint8, "m_code"), _ptr(m_k, torch.float32, "m_k"),
        _ptr(m_scale, torch.float32, "m_scale"), _ptr(v_code, torch.uint8, "v_code"),
        _ptr(v_k, torch.float32, "v_k"), _ptr(v_scale, torch.float32, "v_scale"), n,
        ctypes.byref(cfg), _stream(stream))
    _check("coat_adamw_fp8_step_peers", st)


def coat_count_nonfinite_bf16(x, count, *, stream=None):
    """count[0] += number of inf/NaN values in the BF16 tensor x."""
    import torch
    if count.dtype not in (torch.int32, torch.uint32):
        raise ValueError("count must be an int32/uint32 tensor")
    st = load().coat_count_nonfinite_bf16(_u16(x, "x"), x.numel(), _ptr(count, None, "count"),
                                          _stream(stream))
    _check("coat_count_nonfinite_bf16", st)


def coat_quantize_state(x, code, k, scale, *, group_size: int = 128, fmt: int = COAT_E4M3,
                        k_range: int = 0, k_max: float = 64.0, flags: int = 0, stream=None):
    import torch
    st = load().coat_quantize_state(
        _ptr(x, torch.float32, "x"), x.numel(), group_size, fmt, k_range, k_max, flags,
        _ptr(code, torch.uint8, "code"), _ptr(k, torch.float32, "k"),
        _ptr(scale, torch.float32, "scale"), _stream(stream))
    _check("coat_quantize_state", st)


def coat_dequant(q, k, scale, out, *, group_size: int, fmt: int = COAT_E4M3, stream=None):
    """out: float32 tensor (FP32 output) or bfloat16 tensor (BF16 output)."""
    import torch
    out_bf16 = out.dtype == torch.bfloat16
    if not out_bf16 and out.dtype != torch.float32:
        raise ValueError("out must be float32 or bfloat16")
    st = load().coat_dequant(
        _ptr(q, torch.uint8, "q"), _ptr(k, torch.float32, "k") if k is not None else None,
        _ptr(scale, torch.float32, "scale"), q.numel(), group_size, fmt, int(out_bf16),
        _ptr(out, None, "out"), _stream(stream))
    _check("coat_dequant", st)


def coat_group_quant_1xG(x, q, scale, *, group_size: int = 128, fmt: int = COAT_E4M3,
                         stream=None):
    """x: [rows, cols] BF16 (row stride x.stride(0)), q: uint8 [rows, cols],
    scale: float32 [rows, cols // group_size]."""
    import torch
    if x.dim() != 2 or x.stride(1) != 1:
        raise ValueError("x must be 2-D with unit column stride")
    rows, cols = x.shape
    dev = x.get_device()
    if dev < 0:
        raise ValueError("x must be a CUDA tensor")
    if dev != _current_device():
        _on_current_device(x, "x")
    if x.dtype not in (torch.bfloat16, torch.int16, torch.uint16):
        raise ValueError("x must hold BF16 bit patterns")
    st = load().coat_group_quant_1xG(
        x.data_ptr(), rows, cols, x.stride(0), group_size, fmt,
        _ptr(q, torch.uint8, "q"), _ptr(scale, torch.float32, "scale"), _stream(stream))
    _check("coat_group_quant_1xG", st)


def coat_group_scaling_workspace_bytes(n: int, group_size: int) -> int:
    return int(load().coat_group_scaling_workspace_bytes(n, group_size))


def coat_group_scaling_quant_pertensor(x, workspace, q, scale, *, group_size: int = 128,
                                       fmt: int = COAT_E4M3, amax_precomputed: int = 0,
                                       stream=None):
    """x: BF16 [n]; workspace: float32 [ceil(n/G) + 1]; q: uint8 [n]; scale:
    float32 [1].  amax_precomputed: 0 (steps (i)-(iii)), 1 (the producer
    wrote the group maxima) or 2 (it also wrote the tensor maximum into the
    last workspace slot: the cast alone); True counts as 1."""
    import torch
    n = x.numel()
    need = (-(-n // group_size) + 1) * 4 if group_size >= 1 else 0  # as the library sizes it
    if workspace.numel() * workspace.element_size() < need:
        raise ValueError(f"workspace needs {need} bytes")
    st = load().coat_group_scaling_quant_pertensor(
        _u16(x, "x"), n, group_size, fmt, _ptr(workspace, torch.float32, "workspace"),
        int(amax_precomputed), _ptr(q, torch.uint8, "q"),
        _ptr(scale, torch.float32, "scale"), _stream(stream))
    _check("coat_group_scaling_quant_pertensor", st)


COAT_NOALLOC_MAX_GROUPS = 1 << 20  # mirrors include/coat.h


def coat_group_scaling_quant_pertensor_noalloc(x, q, scale, *, group_size: int = 128,
                                               fmt: int = COAT_E4M3, stream=None):
    """Group Scaling quantization with the library's own fixed scratch: no
    workspace argument and no allocation (see include/coat.h)."""
    import torch
    st = load().coat_group_scaling_quant_pertensor_noalloc(
        _u16(x, "x"), x.numel(), group_size, fmt, _ptr(q, torch.uint8, "q"),
        _ptr(scale, torch.float32, "scale"), _stream(stream))
    _check("coat_group_scaling_quant_pertensor_noalloc", st)


def _tensor_amax_slot(tensor_amax, group_amax, ng):
    """The producers' tensor-maximum slot: "auto" takes the slot after the
    group maxima when group_amax is a whole Group Scaling workspace
    (ceil(n/G) + 1 floats), so that Group Scaling can run as the cast alone
    (amax_precomputed=2); None writes no tensor maximum."""
    if isinstance(tensor_amax, str):
        if tensor_amax != "auto":
            raise ValueError('tensor_amax must be a tensor, None or "auto"')
        return _slot(group_amax[ng:ng + 1]) if group_amax.numel() > ng else None
    return _slot(tensor_amax)


def coat_swiglu_group_amax(gate, up, out, group_amax, *, group_size: int = 128,
                           tensor_amax="auto", stream=None):
    """out = RN_bf16(silu(gate) * up) and the per-1xG maxima of out, ready
    for coat_group_scaling_quant_pertensor(..., amax_precomputed=1); with a
    tensor_amax slot (a float32 tensor; by default the slot after the group
    maxima when group_amax is a whole Group Scaling workspace) also the
    maximum of all of out, for amax_precomputed=2."""
    import torch
    if gate.numel() != up.numel() or out.numel() != gate.numel():
        raise ValueError("gate, up and out must have the same number of elements")
    ng = -(-gate.numel() // group_size)
    if group_amax.numel() < ng:
        raise ValueError(f"group_amax needs {ng} float32 slots")
    st = load().coat_swiglu_group_amax(
        _u16(gate, "gate"), _u16(up, "up"), gate.numel(), group_size, _u16(out, "out"),
        _ptr(group_amax, torch.float32, "group_amax"),
        _tensor_amax_slot(tensor_amax, group_amax, ng), _stream(stream))
    _check("coat_swiglu_group_amax", st)


def coat_norm_group_amax(x, out, group_amax, *, rms: bool = False, eps: float = 1e-5,
                         weight=None, bias=None, group_size: int = 128, tensor_amax="auto",
                         stream=None):
    """LayerNorm (or RMSNorm) of BF16 rows x [rows, cols] into BF16 `out` with
    the maxima of every 1xG run of the output in `group_amax` (see
    include/coat.h); tensor_amax as for coat_swiglu_group_amax."""
    import torch
    if x.dim() != 2 or out.shape != x.shape:
        raise ValueError("x and out must be [rows, cols] tensors of the same shape")
    rows, cols = x.shape
    ng = rows * (cols // max(group_size, 1))
    if group_amax.numel() < ng:
        raise ValueError("group_amax needs rows * cols / G elements")
    for t, what in ((weight, "weight"), (bias, "bias")):
        if t is not None and t.numel() != cols:
            raise ValueError(f"{what} needs cols elements")
    _check("coat_norm_group_amax", load().coat_norm_group_amax(
        _u16(x, "x"), rows, cols, int(rms), float(eps), _ptr(weight, torch.float32, "weight"),
        _ptr(bias, torch.float32, "bias"), group_size, _u16(out, "out"),
        _ptr(group_amax, torch.float32, "group_amax"),
        _tensor_amax_slot(tensor_amax, group_amax, ng), _stream(stream)))


def coat_fp8_encode(y, q, *, fmt: int = COAT_E4M3, stream=None):
    """q = RNE_satfinite FP8 codes of the float32 tensor y."""
    import torch
    if q.numel() != y.numel():
        raise ValueError("y and q must have the same number of elements")
    st = load().coat_fp8_encode(_ptr(y, torch.float32, "y"), y.numel(), fmt,
                                _ptr(q, torch.uint8, "q"), _stream(stream))
    _check("coat_fp8_encode", st)


class PackTable:
    """Host tables (sizes, flat offsets) of a fixed list of tensors, built
    once, for coat_pack_bf16 / coat_unpack_bf16."""

    def __init__(self, numels, offsets):
        if len(numels) != len(offsets):
            raise ValueError("numels and offsets differ in length")
        self.count = len(numels)
        self.numel = (_I64 * self.count)(*[int(x) for x in numels])
        self.offset = (_I64 * self.count)(*[int(x) for x in offsets])

    def pointers(self, tensors):
        if len(tensors) != self.count:
            raise ValueError("wrong number of tensors")
        return (_P * self.count)(*[None if t is None else t.data_ptr() for t in tensors])


def coat_pack_bf16(srcs, table: PackTable, dst, *, stream=None):
    """dst[offset[i] + j] = bf16(srcs[i][j]) for CUDA tensors srcs (all FP32, or
    all BF16 / int16 / uint16 bit patterns; None = zeros) into the flat BF16
    tensor dst."""
    import torch
    dtypes = {t.dtype for t in srcs if t is not None}
    bits16 = {torch.bfloat16, torch.int16, torch.uint16}
    if not dtypes <= {torch.float32} and not dtypes <= bits16:
        raise ValueError("sources must be all float32 or all BF16 (bit patterns)")
    for t in srcs:
        if t is not None and (not t.is_cuda or not t.is_contiguous()):
            raise ValueError("sources must be contiguous CUDA tensors")
        if t is not None:
            _on_current_device(t, "source")
    src_f32 = int(dtypes == {torch.float32})
    _check("coat_pack_bf16", load().coat_pack_bf16(
        table.pointers(srcs), table.numel, table.offset, table.count, src_f32,
        _u16(dst, "dst"), dst.numel(), _stream(stream)))


def coat_unpack_bf16(src, table: PackTable, dsts, *, stream=None):
    """dsts[i][j] = bf16(src[offset[i] + j]) from the flat FP32 tensor src into
    contiguous BF16 CUDA tensors dsts."""
    for t in dsts:
        if t is None or not t.is_cuda or not t.is_contiguous():
            raise ValueError("destinations must be contiguous CUDA tensors")
        _u16(t, "destination")     # (checks the device too)
    import torch
    _check("coat_unpack_bf16", load().coat_unpack_bf16(
        _ptr(src, torch.float32, "src"), table.numel, table.offset, table.count,
        table.pointers(dsts), src.numel(), _stream(stream)))


class CoatStateStats(ctypes.Structure):
    _fields_ = [("groups", ctypes.c_uint64), ("zero_groups", ctypes.c_uint64),
                ("k1_groups", ctypes.c_uint64), ("max_codes", ctypes.c_uint64),
                ("zero_codes", ctypes.c_uint64), ("nonfinite_codes", ctypes.c_uint64),
                ("k_sum", ctypes.c_double), ("k_min", ctypes.c_float), ("k_max", ctypes.c_float)]


def coat_state_stats(code, k, scale, *, group_size: int, fmt: int = COAT_E4M3, out=None,
                     stream=None) -> dict:
    """Monitoring counts of one compressed state (see include/coat.h).  With
    `out` (a CUDA uint8 tensor of sizeof(coat_state_stats_t) bytes) the call
    stays asynchronous and returns None; otherwise it synchronises and returns
    the counts as a dict."""
    import torch
    size = ctypes.sizeof(CoatStateStats)
    buf = out if out is not None else torch.empty(size, dtype=torch.uint8, device=code.device)
    if buf.numel() < size:
        raise ValueError(f"out needs {size} bytes")
    _check("coat_state_stats", load().coat_state_stats(
        _ptr(code, torch.uint8, "code"), _ptr(k, torch.float32, "k"),
        _ptr(scale, torch.float32, "scale"), code.numel(), group_size, fmt,
        _ptr(buf, torch.uint8, "out"), _stream(stream)))
    if out is not None:
        return None
    raw = bytes(buf.cpu().numpy().tobytes())
    st = CoatStateStats.from_buffer_copy(raw)
    return {name: getattr(st, name) for name, _ in CoatStateStats._fields_}


def coat_version() -> int:
    return int(load().coat_version())


def coat_status_string(status: int) -> str:
    return load().coat_status_string(status).decode()
