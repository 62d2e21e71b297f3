"""COAT oracle -- TEST INFRASTRUCTURE ONLY.

Python face of the plain C oracle (``coat_oracle.c``) plus an unquantized
binary64 AdamW.  Only the test suite, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package; the CUDA library
and its binding never do.

Pages cited (by title and section):
  COAT summary, "COAT: 压缩优化器状态和激活以实现内存高效的 FP8 训练"
  (blog.daoxuan.cc/posts/57954): sections on the AdamW rule and why v is
  sensitive, the expansion function f(x) = sign(x)|x|^k with
  k = log(R_E4M3)/log(R_X), mixed granularity (1xG groups and Group Scaling),
  and the results section (training on several GPUs: the data-parallel
  gradient mean of grad_mean_bf16).
  LLM Atlas "systems/numerics" (llm-atlas.k1412.top): section 03 "FP8"
  (format limits) and section 08 "Adam -> AdamW" (the update rule).

Parity status: pinned by tests/test_oracle_*.py; the magnitude of the error
reduction from the expansion function is "parity unpinned" (direction only).
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

from . import build as _build

E4M3 = 0
E5M2 = 1

_lib = None


class AdamWCfg(ctypes.Structure):
    _fields_ = [
        ("beta1", ctypes.c_float),
        ("beta2", ctypes.c_float),
        ("lr", ctypes.c_float),
        ("eps", ctypes.c_float),
        ("weight_decay", ctypes.c_float),
        ("step", ctypes.c_int64),
        ("group_size", ctypes.c_int64),
        ("m_fmt", ctypes.c_int32),
        ("v_fmt", ctypes.c_int32),
        ("k_range", ctypes.c_int32),
        ("k_max", ctypes.c_float),
        ("force_k1", ctypes.c_int32),
    ]


def lib():
    """The compiled C oracle: oracle/liborc.so, built on first use, or the
    build named by the COAT_ORACLE_LIB environment variable (the mutation
    tests point it at copies of the oracle with a planted mistake)."""
    global _lib
    if _lib is None:
        path = os.environ.get("COAT_ORACLE_LIB") or _build.build()
        L = ctypes.CDLL(path)
        P = ctypes.c_void_p
        i64 = ctypes.c_int64
        L.orc_exmy_value.restype = ctypes.c_double
        L.orc_exmy_value.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_uint32,
                                     ctypes.c_uint32]
        L.orc_fp8_decode.restype = ctypes.c_double
        L.orc_fp8_decode.argtypes = [ctypes.c_uint8, ctypes.c_int]
        L.orc_fp8_encode.restype = ctypes.c_uint8
        L.orc_fp8_encode.argtypes = [ctypes.c_float, ctypes.c_int]
        for name in ("orc_fp8_max", "orc_fp8_min_subnormal", "orc_fp8_range"):
            getattr(L, name).restype = ctypes.c_double
            getattr(L, name).argtypes = [ctypes.c_int]
        L.orc_bf16_to_f32.restype = ctypes.c_float
        L.orc_bf16_to_f32.argtypes = [ctypes.c_uint16]
        L.orc_f32_to_bf16.restype = ctypes.c_uint16
        L.orc_f32_to_bf16.argtypes = [ctypes.c_float]
        L.orc_fp8_encode_array.restype = None
        L.orc_fp8_encode_array.argtypes = [P, i64, ctypes.c_int, P]
        L.orc_f32_to_bf16_array.restype = None
        L.orc_f32_to_bf16_array.argtypes = [P, i64, P]
        L.orc_state_dequant_one.restype = ctypes.c_float
        L.orc_state_dequant_one.argtypes = [ctypes.c_uint8, ctypes.c_float, ctypes.c_float,
                                            ctypes.c_int]
        L.orc_quantize_state.restype = ctypes.c_int
        L.orc_quantize_state.argtypes = [P, i64, i64, ctypes.c_int, ctypes.c_int, ctypes.c_float,
                                         ctypes.c_int, P, P, P]
        L.orc_dequant.restype = ctypes.c_int
        L.orc_dequant.argtypes = [P, P, P, i64, i64, ctypes.c_int, P]
        L.orc_adamw_fp8_step.restype = ctypes.c_int
        L.orc_adamw_fp8_step.argtypes = [P, P, P, P, P, P, P, P, i64,
                                         ctypes.POINTER(AdamWCfg), P, P]
        L.orc_group_quant_1xG.restype = ctypes.c_int
        L.orc_group_quant_1xG.argtypes = [P, i64, i64, i64, i64, ctypes.c_int, P, P]
        L.orc_group_scaling_pertensor.restype = ctypes.c_int
        L.orc_group_scaling_pertensor.argtypes = [P, i64, i64, ctypes.c_int, P, ctypes.c_int,
                                                  P, P]
        _lib = L
    return _lib


def _ptr(a: np.ndarray | None):
    if a is None:
        return None
    assert a.flags["C_CONTIGUOUS"], "oracle buffers must be contiguous"
    return a.ctypes.data


def _check(rc: int, what: str):
    if rc != 0:
        raise ValueError(f"oracle {what} rejected its arguments (rc={rc})")


# ---- formats ---------------------------------------------------------------

def exmy_value(ebits: int, mbits: int, bias: int, e: int, m: int) -> float:
    return lib().orc_exmy_value(ebits, mbits, bias, e, m)


def fp8_decode(code: int, fmt: int) -> float:
    return lib().orc_fp8_decode(code, fmt)


def fp8_encode(y: float, fmt: int) -> int:
    return lib().orc_fp8_encode(y, fmt)


def fp8_encode_array(y: np.ndarray, fmt: int) -> np.ndarray:
    """fp8_encode applied to every element (the loop runs in C)."""
    y = np.ascontiguousarray(y, dtype=np.float32)
    out = np.empty(y.shape, dtype=np.uint8)
    lib().orc_fp8_encode_array(_ptr(y), y.size, fmt, _ptr(out))
    return out


def fp8_max(fmt: int) -> float:
    return lib().orc_fp8_max(fmt)


def fp8_min_subnormal(fmt: int) -> float:
    return lib().orc_fp8_min_subnormal(fmt)


def fp8_range(fmt: int) -> float:
    return lib().orc_fp8_range(fmt)


def bf16_to_f32(b: int) -> float:
    return lib().orc_bf16_to_f32(b)


def f32_to_bf16(f: float) -> int:
    return lib().orc_f32_to_bf16(f)


# ---- optimizer states ------------------------------------------------------

def n_groups(n: int, G: int) -> int:
    return (n + G - 1) // G


def quantize_state(x: np.ndarray, G: int, fmt: int, k_range: int = 0, k_max: float = 64.0,
                   force_k1: bool = False):
    """FP32 state -> (codes u8[n], k f32[ngroups], s f32[ngroups])."""
    x = np.ascontiguousarray(x, dtype=np.float32).reshape(-1)
    n = x.size
    code = np.empty(n, dtype=np.uint8)
    k = np.empty(n_groups(n, G), dtype=np.float32)
    s = np.empty(n_groups(n, G), dtype=np.float32)
    _check(lib().orc_quantize_state(_ptr(x), n, G, fmt, k_range, k_max, int(force_k1),
                                    _ptr(code), _ptr(k), _ptr(s)), "quantize_state")
    return code, k, s


def dequant(q: np.ndarray, k: np.ndarray | None, s: np.ndarray, G: int, fmt: int) -> np.ndarray:
    q = np.ascontiguousarray(q, dtype=np.uint8).reshape(-1)
    s = np.ascontiguousarray(s, dtype=np.float32).reshape(-1)
    kk = None if k is None else np.ascontiguousarray(k, dtype=np.float32).reshape(-1)
    out = np.empty(q.size, dtype=np.float32)
    _check(lib().orc_dequant(_ptr(q), _ptr(kk), _ptr(s), q.size, G, fmt, _ptr(out)), "dequant")
    return out


def to_bf16_array(x: np.ndarray) -> np.ndarray:
    """binary32 -> BF16 bits, nearest-even, for every element (loop in C)."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    out = np.empty(x.shape, dtype=np.uint16)
    lib().orc_f32_to_bf16_array(_ptr(x), x.size, _ptr(out))
    return out


def grad_mean_bf16(grads) -> np.ndarray:
    """The data-parallel gradient of one step (COAT summary, section
    "结果和边界": multi-GPU training, every rank computing a full BF16
    gradient): the mean of the ranks' BF16 gradients, summed in binary32 in
    rank order (one rounding per addition), divided by the rank count in
    binary32 and rounded to BF16 (nearest even).  grads: a sequence of BF16
    bit arrays of one shape; one rank gives its gradient unchanged."""
    grads = [np.asarray(g, dtype=np.uint16) for g in grads]
    acc = bf16_bits_to_f64(grads[0]).astype(np.float32)
    for g in grads[1:]:
        acc = np.add(acc, bf16_bits_to_f64(g).astype(np.float32), dtype=np.float32)
    if len(grads) > 1:
        acc = np.divide(acc, np.float32(len(grads)), dtype=np.float32)
    return to_bf16_array(acc)


def adamw_fp8_step(theta, grad_bf16, m_code, m_k, m_s, v_code, v_k, v_s, *, beta1, beta2, lr,
                   eps, weight_decay, step, group_size, m_fmt=E4M3, v_fmt=E4M3, k_range=0,
                   k_max=64.0, force_k1=False, return_moments=False):
    """One COAT step; returns new copies (inputs untouched).

    Returns (theta, m_code, m_k, m_s, v_code, v_k, v_s) and, with
    return_moments, the FP32 m_t and v_t before re-quantization.
    """
    th = np.array(theta, dtype=np.float32, copy=True).reshape(-1)
    g = np.ascontiguousarray(grad_bf16, dtype=np.uint16).reshape(-1)
    mc = np.array(m_code, dtype=np.uint8, copy=True).reshape(-1)
    vc = np.array(v_code, dtype=np.uint8, copy=True).reshape(-1)
    mk = np.array(m_k, dtype=np.float32, copy=True).reshape(-1)
    ms = np.array(m_s, dtype=np.float32, copy=True).reshape(-1)
    vk = np.array(v_k, dtype=np.float32, copy=True).reshape(-1)
    vs = np.array(v_s, dtype=np.float32, copy=True).reshape(-1)
    n = th.size
    assert g.size == n and mc.size == n and vc.size == n
    assert mk.size == n_groups(n, group_size) == vk.size
    cfg = AdamWCfg(beta1, beta2, lr, eps, weight_decay, step, group_size, m_fmt, v_fmt,
                   k_range, k_max, int(force_k1))
    mt = np.empty(n, dtype=np.float32) if return_moments else None
    vt = np.empty(n, dtype=np.float32) if return_moments else None
    _check(lib().orc_adamw_fp8_step(_ptr(th), _ptr(g), _ptr(mc), _ptr(mk), _ptr(ms), _ptr(vc),
                                    _ptr(vk), _ptr(vs), n, ctypes.byref(cfg), _ptr(mt),
                                    _ptr(vt)), "adamw_fp8_step")
    out = (th, mc, mk, ms, vc, vk, vs)
    return out + (mt, vt) if return_moments else out


def adamw_fp64(theta, grad, m, v, *, step, beta1, beta2, lr, eps, weight_decay):
    """Unquantized AdamW in binary64 (LLM Atlas, section 08 "Adam -> AdamW").

    m_t = b1 m + (1-b1) g ; v_t = b2 v + (1-b2) g^2 ;
    theta_t = (1 - lr*wd) theta - lr * m_hat / (sqrt(v_hat) + eps).
    Returns (theta_t, m_t, v_t) as float64 arrays.
    """
    theta = np.asarray(theta, dtype=np.float64)
    g = np.asarray(grad, dtype=np.float64)
    m = np.asarray(m, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    b1, b2 = float(np.float32(beta1)), float(np.float32(beta2))
    m_t = b1 * m + (1.0 - b1) * g
    v_t = b2 * v + (1.0 - b2) * g * g
    m_hat = m_t / (1.0 - b1 ** step)
    v_hat = v_t / (1.0 - b2 ** step)
    th = theta * (1.0 - float(np.float32(lr)) * float(np.float32(weight_decay)))
    th = th - float(np.float32(lr)) * m_hat / (np.sqrt(v_hat) + float(np.float32(eps)))
    return th, m_t, v_t


# ---- activations -----------------------------------------------------------

def group_quant_1xG(x_bf16: np.ndarray, G: int, fmt: int = E4M3, cols: int | None = None):
    """x_bf16: uint16 [rows, ld] -> (q u8 [rows, cols], scale f32 [rows, cols/G]) for the
    first `cols` columns of each row (all of them by default): rows of a
    larger buffer, row stride ld."""
    x = np.ascontiguousarray(x_bf16, dtype=np.uint16)
    rows, ld = x.shape
    cols = ld if cols is None else cols
    q = np.empty((rows, cols), dtype=np.uint8)
    sc = np.empty((rows, cols // G), dtype=np.float32)
    _check(lib().orc_group_quant_1xG(_ptr(x), rows, cols, ld, G, fmt, _ptr(q), _ptr(sc)),
           "group_quant_1xG")
    return q, sc


def group_scaling_pertensor(x_bf16: np.ndarray, G: int, fmt: int = E4M3,
                            group_amax: np.ndarray | None = None):
    """Flat BF16 -> (q u8[n], scale float, group_amax f32[ceil(n/G)])."""
    x = np.ascontiguousarray(x_bf16, dtype=np.uint16).reshape(-1)
    n = x.size
    pre = group_amax is not None
    ga = (np.array(group_amax, dtype=np.float32, copy=True) if pre
          else np.empty(n_groups(n, G), dtype=np.float32))
    q = np.empty(n, dtype=np.uint8)
    sc = np.empty(1, dtype=np.float32)
    _check(lib().orc_group_scaling_pertensor(_ptr(x), n, G, fmt, _ptr(ga), int(pre), _ptr(q),
                                             _ptr(sc)), "group_scaling_pertensor")
    return q, float(sc[0]), ga


BF16_MAX = float.fromhex("0x1.fep+127")


def round_to_bf16(x) -> np.ndarray:
    """binary64 values -> BF16 bit patterns, round to nearest even, with BF16
    subnormals and overflow to infinity (QA page on BF16: 8 exponent bits, 7
    explicit mantissa bits).  x = m 2^e with 0.5 <= |m| < 1 keeps 8
    significant bits: rint(x 2^(8-e)) 2^(e-8); below 2^-126 the quantum is
    the subnormal spacing 2^-133."""
    x = np.asarray(x, dtype=np.float64)
    with np.errstate(invalid="ignore", over="ignore"):
        _, e = np.frexp(x)
        e = np.maximum(e, -125)
        q = np.ldexp(np.rint(np.ldexp(x, 8 - e)), e - 8)
        q = np.where(np.abs(q) > BF16_MAX, np.copysign(np.inf, x), q)
    return (q.astype(np.float32).view(np.uint32) >> 16).astype(np.uint16)


def bf16_bits_to_f64(b) -> np.ndarray:
    b = np.asarray(b, dtype=np.uint16).astype(np.uint32) << 16
    return b.view(np.float32).astype(np.float64)


def swiglu_bf16(gate_bf16: np.ndarray, up_bf16: np.ndarray) -> np.ndarray:
    """SwiGLU of BF16 inputs, the producer of a GLU MLP's down-projection
    input (COAT summary page, sections "激活为什么难压" and "混合粒度"):
    RN_bf16(silu(g) u) with silu(g) = g / (1 + e^-g), evaluated in binary64
    and rounded once to BF16."""
    g = bf16_bits_to_f64(gate_bf16)
    u = bf16_bits_to_f64(up_bf16)
    with np.errstate(over="ignore"):
        h = g / (1.0 + np.exp(-g)) * u
    return round_to_bf16(h)


def norm_f64(x_bf16: np.ndarray, *, rms: bool, eps: float, weight=None,
             bias=None) -> np.ndarray:
    """Row-wise LayerNorm (rms=False: (x - mean) / sqrt(var + eps), var the
    mean squared deviation) or RMSNorm (rms=True: x / sqrt(mean(x^2) + eps))
    of BF16 rows, times an optional per-column weight plus an optional
    per-column bias, all in binary64 (eps as the binary32 value the library
    receives).  The norm is one of the nonlinear layers of the COAT summary
    page (section "激活为什么难压") and produces a linear layer's input."""
    x = bf16_bits_to_f64(x_bf16)
    e = float(np.float32(eps))
    if rms:
        y = x / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + e)
    else:
        d = x - np.mean(x, axis=-1, keepdims=True)
        y = d / np.sqrt(np.mean(d * d, axis=-1, keepdims=True) + e)
    if weight is not None:
        y = y * np.asarray(weight, dtype=np.float32).astype(np.float64)
    if bias is not None:
        y = y + np.asarray(bias, dtype=np.float32).astype(np.float64)
    return y


def norm_bf16(x_bf16: np.ndarray, **kw) -> np.ndarray:
    """norm_f64 rounded once to BF16 (bit patterns)."""
    return round_to_bf16(norm_f64(x_bf16, **kw))


def group_amax_of(x_bf16: np.ndarray, G: int) -> np.ndarray:
    """Per-1xG max |x| of a flat BF16 tensor (a shorter last group allowed)."""
    x = np.abs(bf16_bits_to_f64(np.ascontiguousarray(x_bf16).reshape(-1)))
    ng = n_groups(x.size, G)
    pad = np.zeros(ng * G)
    pad[:x.size] = x
    return pad.reshape(ng, G).max(axis=1).astype(np.float32)


def state_stats(code: np.ndarray, k: np.ndarray, s: np.ndarray, G: int, fmt: int) -> dict:
    """Monitoring counts of one compressed state, written from their
    definitions (nothing here is on the pages beyond the format maxima of the
    LLM Atlas "systems/numerics" page, section 03 "FP8"): groups, all-zero
    groups (scale 0), other groups stored with k == 1, codes at the largest
    finite magnitude / at +-0 / on inf-NaN patterns, and the sum, min and max
    of k over the nonzero groups."""
    code = np.ascontiguousarray(code, dtype=np.uint8).reshape(-1)
    k = np.asarray(k, dtype=np.float32).reshape(-1)
    s = np.asarray(s, dtype=np.float32).reshape(-1)
    ng = n_groups(code.size, G)
    k, s = k[:ng], s[:ng]
    top = 0x7E if fmt == E4M3 else 0x7B      # 448 = 0x7E (E4M3), 57344 = 0x7B (E5M2)
    mag = code & 0x7F
    nz = s != 0
    kn = k[nz].astype(np.float64)
    return {"groups": ng, "zero_groups": int((~nz).sum()),
            "k1_groups": int((k[nz] == 1.0).sum()),
            "max_codes": int((mag == top).sum()), "zero_codes": int((mag == 0).sum()),
            "nonfinite_codes": int((mag > top).sum()),
            "k_sum": float(kn.sum()) if kn.size else 0.0,
            "k_min": float(kn.min()) if kn.size else float("inf"),
            "k_max": float(kn.max()) if kn.size else float("-inf")}


def threads_used() -> int:
    return 1


__all__ = [n for n in dir() if not n.startswith("_")]
