"""Shared helpers of the GPU parity tests: move host arrays through the CUDA
library and compare with the oracle under the stated tolerances.

Tolerances (GPU vs oracle, same inputs, one step):
  - FP8 state codes identical except at most 1e-4 of the elements of each
    state, each off by one code, and only next to a rounding tie;
  - per-group k and s: relative error <= 1e-5;
  - FP32 parameters: |d theta| <= 1e-6 * max(|theta_ref|, lr);
  - activation codes and scales: bit-exact.
"""
from __future__ import annotations

import numpy as np

CODE_FLIP_FRACTION = 1e-4
KS_RTOL = 1e-5
THETA_RTOL = 1e-6
FMAX = {0: 448.0, 1: 57344.0}


def to_dev(a, dtype=None):
    import torch
    t = torch.from_numpy(np.ascontiguousarray(a))
    if dtype is not None:
        t = t.view(dtype)
    return t.cuda()


def to_host(t):
    import torch
    t = t.detach()
    if t.dtype == torch.bfloat16:
        t = t.view(torch.int16)
    return t.cpu().numpy()


def gpu_step(lib, th, g, mc, mk, ms, vc, vk, vs, **cfg):
    """Run coat_adamw_fp8_step on copies of host arrays; return host arrays."""
    import torch
    d = [to_dev(th), to_dev(g.view(np.int16)), to_dev(mc), to_dev(mk), to_dev(ms), to_dev(vc),
         to_dev(vk), to_dev(vs)]
    lib.coat_adamw_fp8_step(*d, **cfg)
    torch.cuda.synchronize()
    return tuple(to_host(t) for t in (d[0], d[2], d[3], d[4], d[5], d[6], d[7]))


def code_index(c: np.ndarray) -> np.ndarray:
    """Signed position of an FP8 code on the number line (sign-magnitude)."""
    c = c.astype(np.int32)
    mag = c & 0x7F
    return np.where(c & 0x80, -mag, mag)


def compare_codes(name, got, ref, near_tie=None):
    """Return (n_flips); assert the flip budget and the one-code rule."""
    diff = code_index(got) - code_index(ref)
    bad = np.nonzero(diff)[0]
    budget = CODE_FLIP_FRACTION * got.size
    assert bad.size <= budget, f"{name}: {bad.size} codes differ (budget {budget:.1f})"
    if bad.size:
        assert np.all(np.abs(diff[bad]) == 1), \
            f"{name}: codes differ by more than one step at {bad[:8]}"
        if near_tie is not None:
            assert np.all(near_tie(bad)), f"{name}: a flipped code is not next to a tie"
    return int(bad.size)


def compare_rel(name, got, ref, rtol):
    got = got.astype(np.float64)
    ref = ref.astype(np.float64)
    err = np.abs(got - ref) / np.maximum(np.abs(ref), np.finfo(np.float32).tiny)
    both_zero = (got == 0) & (ref == 0)
    err[both_zero] = 0.0
    worst = float(err.max()) if err.size else 0.0
    assert worst <= rtol, f"{name}: max relative error {worst:.3g} > {rtol}"
    return worst


def compare_theta(got, ref, lr):
    err = np.abs(got.astype(np.float64) - ref) / np.maximum(np.abs(ref.astype(np.float64)), lr)
    worst = float(err.max()) if err.size else 0.0
    assert worst <= THETA_RTOL, f"theta: max scaled error {worst:.3g} > {THETA_RTOL}"
    return worst


def tie_checker(x, k, G, fmt):
    """Predicate over element indices: is the expanded value of x next to a
    rounding midpoint of the FP8 grid (relative distance <= 1e-4)?  The
    group maximum M and k come from the oracle's outputs."""
    x = np.asarray(x, dtype=np.float64)

    def check(idx):
        import oracle
        ok = []
        for i in idx:
            gi = i // G
            xs = np.abs(x[gi * G:(gi + 1) * G])
            M = xs.max()
            y = FMAX[fmt] * (abs(x[i]) / M) ** float(k[gi])
            lo = oracle.fp8_encode(float(np.float32(y)), fmt)
            vlo = abs(oracle.fp8_decode(lo, fmt))
            other = lo + 1 if vlo <= y else lo - 1
            vo = abs(oracle.fp8_decode(max(other, 0), fmt))
            mid = 0.5 * (vlo + vo)
            ok.append(abs(y - mid) <= 1e-4 * max(mid, 1e-30))
        return np.array(ok, dtype=bool)

    return check


def assert_step_parity(gpu, orc, lr, G, v_fmt, moments=None):
    """gpu / orc: (theta, mc, mk, ms, vc, vk, vs).  Returns a stats dict."""
    th_g, mc_g, mk_g, ms_g, vc_g, vk_g, vs_g = gpu
    th_o, mc_o, mk_o, ms_o, vc_o, vk_o, vs_o = orc[:7]
    st = {}
    st["theta_err"] = compare_theta(th_g, th_o, lr)
    st["m_k_err"] = compare_rel("m_k", mk_g, mk_o, KS_RTOL)
    st["v_k_err"] = compare_rel("v_k", vk_g, vk_o, KS_RTOL)
    st["m_s_err"] = compare_rel("m_scale", ms_g, ms_o, KS_RTOL)
    st["v_s_err"] = compare_rel("v_scale", vs_g, vs_o, KS_RTOL)
    mt = vt = None
    if moments is not None:
        mt, vt = moments
    st["m_flips"] = compare_codes("m_code", mc_g, mc_o,
                                  tie_checker(mt, mk_o, G, 0) if mt is not None else None)
    st["v_flips"] = compare_codes("v_code", vc_g, vc_o,
                                  tie_checker(vt, vk_o, G, v_fmt) if vt is not None else None)
    return st
