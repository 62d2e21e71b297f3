"""The C ABI library builds, loads without a GPU, and exports every entry
point that include/*.h declares; host-side argument checks reject bad calls
before any launch (CPU only: no kernel runs here)."""
import ctypes
import glob
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    from quantized_optimizer_states_b200 import build
    build.build()
    import quantized_optimizer_states_b200 as q
    return q.load()


def declared_functions():
    names = set()
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        src = open(h).read()
        src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
        for m in re.finditer(r"^\s*[A-Za-z_][\w\s\*]*?\b(coat_\w+)\s*\(", src, flags=re.M):
            names.add(m.group(1))
    return sorted(names)


def test_header_declares_the_boundary():
    names = declared_functions()
    for want in ("coat_adamw_fp8_step", "coat_group_quant_1xG",
                 "coat_group_scaling_quant_pertensor", "coat_dequant", "coat_quantize_state"):
        assert want in names


def test_every_declared_symbol_is_exported(lib):
    so = os.path.join(ROOT, "quantized_optimizer_states_b200", "libcoat.so")
    out = subprocess.run(["nm", "-D", "--defined-only", so], capture_output=True, text=True,
                         check=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if line.strip()}
    for name in declared_functions():
        assert name in exported, name
        assert hasattr(lib, name)


def test_host_functions_without_gpu(lib):
    assert lib.coat_version() == 0x000100
    assert lib.coat_status_string(2) == b"buffer not 16-byte aligned"
    assert lib.coat_group_scaling_workspace_bytes(1000, 128) == (8 + 1) * 4
    assert lib.coat_group_scaling_workspace_bytes(-1, 128) == -1


def test_argument_checks_return_before_any_launch(lib):
    """Invalid calls are rejected on the host: status codes only, no CUDA."""
    from quantized_optimizer_states_b200._lib import CoatAdamwCfg
    P = ctypes.c_void_p
    fake = P(0x10000)      # never dereferenced: every call below fails a host check
    odd = P(0x10004)
    cfg = CoatAdamwCfg(0.9, 0.999, 1e-4, 1e-8, 0.1, 10, 128, 0, 0, 0, 64.0, 0)
    args = [fake] * 8
    step = lib.coat_adamw_fp8_step
    assert step(*args, -1, ctypes.byref(cfg), None) == 1               # n < 0
    assert step(*args, 0, ctypes.byref(cfg), None) == 0                # empty: no launch
    assert step(None, *args[1:], 16, ctypes.byref(cfg), None) == 1     # null pointer
    assert step(odd, *args[1:], 16, ctypes.byref(cfg), None) == 2      # misaligned
    for field, val, want in (("group_size", 96, 3), ("group_size", 8, 3), ("group_size", 8192, 3),
                             ("m_fmt", 1, 3), ("v_fmt", 2, 3), ("k_range", 2, 3),
                             ("flags", 0x40, 3), ("step", 0, 1), ("beta1", 1.0, 1),
                             ("beta2", -0.1, 1), ("k_max", -1.0, 1)):
        bad = CoatAdamwCfg.from_buffer_copy(cfg)
        setattr(bad, field, val)
        assert step(*args, 16, ctypes.byref(bad), None) == want, field
    assert step(*args, 16, None, None) == 1
    q = lib.coat_quantize_state
    assert q(fake, 16, 100, 0, 0, 64.0, 0, fake, fake, fake, None) == 3
    assert q(odd, 16, 128, 0, 0, 64.0, 0, fake, fake, fake, None) == 2
    d = lib.coat_dequant
    assert d(fake, None, fake, 100, 48, 0, 0, fake, None) == 3            # G not a power of 2
    assert d(fake, None, fake, 100, 0, 0, 0, fake, None) == 1
    assert d(odd, None, fake, 100, 100, 0, 0, fake, None) == 2
    g = lib.coat_group_quant_1xG
    assert g(fake, 4, 200, 200, 128, 0, fake, fake, None) == 1           # cols % G != 0
    assert g(fake, 4, 256, 100, 128, 0, fake, fake, None) == 1           # ld < cols
    assert g(fake, 4, 256, 260, 128, 0, fake, fake, None) == 2           # ld not 16-byte rows
    gs = lib.coat_group_scaling_quant_pertensor
    assert gs(fake, 100, 128, 5, fake, 0, fake, fake, None) == 3
    assert gs(odd, 100, 128, 0, fake, 0, fake, fake, None) == 2
    assert gs(fake, 0, 128, 0, fake, 0, fake, fake, None) == 0


def test_peer_step_argument_checks(lib):
    """coat_adamw_fp8_step_peers validates its rank tables on the host (these
    calls never reach the device)."""
    from quantized_optimizer_states_b200._lib import CoatAdamwCfg
    P = ctypes.c_void_p
    fake = P(0x10000)
    cfg = ctypes.byref(CoatAdamwCfg(0.9, 0.999, 1e-4, 1e-8, 0.1, 10, 128, 0, 0, 0, 64.0, 0))
    grads = (P * 9)(*([0x10000] * 9))
    outs = (P * 2)(0x20000, 0x30000)
    st = [fake] * 6
    pe = lib.coat_adamw_fp8_step_peers
    assert pe(grads, 0, 0, fake, None, 0, 0, *st, 16, cfg, None) == 1        # no rank
    assert pe(grads, 9, 0, fake, None, 0, 0, *st, 16, cfg, None) == 1        # above the maximum
    assert pe(None, 2, 0, fake, None, 0, 0, *st, 16, cfg, None) == 1         # no gradient table
    assert pe(grads, 2, -16, fake, None, 0, 0, *st, 16, cfg, None) == 1      # negative offset
    assert pe(grads, 2, 0, fake, outs, 2, 0, *st, 16, cfg, None) == 1        # bf16 flag not 0/1
    assert pe((P * 2)(0x10000, None), 2, 0, fake, None, 0, 0, *st, 16, cfg, None) == 1
    assert pe(grads, 2, 4, fake, None, 0, 0, *st, 16, cfg, None) == 2        # 8-byte offset
    assert pe(grads, 2, 0, fake, outs, 0, 2, *st, 16, cfg, None) == 2        # FP32 copy at 8 bytes
    assert pe(grads, 2, 0, fake, outs, 1, 4, *st, 16, cfg, None) == 2        # BF16 copy at 8 bytes
    assert pe(grads, 2, 0, P(0x10004), outs, 1, 8, *st, 16, cfg, None) == 2  # shard misaligned
    assert pe(grads, 2, 0, fake, outs, 1, 8, *st, 0, cfg, None) == 0         # empty: no launch


def test_pack_argument_checks(lib):
    """coat_pack_bf16 / coat_unpack_bf16 validate their host tables before any
    launch (these calls never reach the device)."""
    P, I64 = ctypes.c_void_p, ctypes.c_int64
    fake = P(1 << 20)
    ptrs = (P * 2)(1 << 20, 1 << 21)

    def tab(*v):
        return (I64 * len(v))(*v)

    pk, up = lib.coat_pack_bf16, lib.coat_unpack_bf16
    assert pk(ptrs, tab(8, 8), tab(0, 16), -1, 1, fake, 64, None) == 1    # count < 0
    assert pk(None, tab(8, 8), tab(0, 16), 2, 1, fake, 64, None) == 1     # no pointer table
    assert pk(ptrs, tab(8, -1), tab(0, 16), 2, 1, fake, 64, None) == 1    # negative size
    assert pk(ptrs, tab(8, 8), tab(0, 60), 2, 1, fake, 64, None) == 1     # slice beyond n
    assert pk(ptrs, tab(8, 8), tab(0, 12), 2, 1, fake, 64, None) == 2     # offset not a multiple of 8
    assert pk(ptrs, tab(8, 8), tab(0, 16), 2, 1, None, 64, None) == 1     # no destination
    assert pk(ptrs, tab(8, 8), tab(0, 16), 2, 1, P((1 << 20) + 4), 64, None) == 2
    assert pk(ptrs, tab(0, 0), tab(0, 16), 2, 1, None, 64, None) == 0     # nothing to move
    assert pk(None, None, None, 0, 1, None, 0, None) == 0
    nulls = (P * 2)(None, 1 << 21)
    assert up(fake, tab(8, 8), tab(0, 16), 2, nulls, 64, None) == 1       # unpack into NULL
    assert pk(nulls, tab(0, 8), tab(0, 16), 2, 1, P((1 << 20) + 8), 64, None) == 2


def test_state_stats_argument_checks(lib):
    P = ctypes.c_void_p
    fake, odd = P(1 << 20), P((1 << 20) + 4)
    st = lib.coat_state_stats
    assert st(fake, fake, fake, 64, 128, 0, None, None) == 1      # no output
    assert st(None, fake, fake, 64, 128, 0, fake, None) == 1      # no codes
    assert st(fake, fake, fake, 64, 100, 0, fake, None) == 3      # G not a power of 2
    assert st(fake, fake, fake, 64, 128, 4, fake, None) == 3      # no such format
    assert st(odd, fake, fake, 64, 128, 0, fake, None) == 2       # codes not 16-byte aligned
    assert st(fake, fake, fake, 64, 128, 0, odd, None) == 2       # output not 8-byte aligned


def test_product_path_fails_loudly_without_library(tmp_path):
    from quantized_optimizer_states_b200 import _lib
    saved = _lib._lib
    try:
        _lib._lib = None
        with pytest.raises(RuntimeError, match="libcoat.so not found"):
            _lib.load(str(tmp_path / "missing" / "libcoat.so"))
    finally:
        _lib._lib = saved


def test_product_package_never_imports_the_oracle():
    pkg = os.path.join(ROOT, "quantized_optimizer_states_b200")
    for path in glob.glob(os.path.join(pkg, "**", "*"), recursive=True):
        if path.endswith((".py", ".cu", ".cuh", ".h")):
            src = open(path).read()
            assert "import oracle" not in src and "from oracle" not in src, path
            assert "coat_oracle" not in src and "liborc" not in src, path


def test_more_argument_checks_and_metadata_alignment(lib):
    """The entry points not covered above, and the 4-byte alignment of float
    metadata (k, s, scales) and the element alignment of pack pointers: all
    rejected on the host (these calls never reach the device)."""
    from quantized_optimizer_states_b200._lib import CoatAdamwCfg
    P, I64 = ctypes.c_void_p, ctypes.c_int64
    fake, odd4, odd2 = P(1 << 20), P((1 << 20) + 2), P((1 << 20) + 1)
    cfg = CoatAdamwCfg(0.9, 0.999, 1e-4, 1e-8, 0.1, 10, 128, 0, 0, 0, 64.0, 0)
    a8 = [fake] * 8
    # metadata of the step (m_k, m_s, v_k, v_s are arguments 3, 4, 6, 7)
    for i in (3, 4, 6, 7):
        args = list(a8)
        args[i] = odd4
        assert lib.coat_adamw_fp8_step(*args, 16, ctypes.byref(cfg), None) == 2, i
        assert lib.coat_adamw_fp8_step_fp32grad(*args, 16, ctypes.byref(cfg), None) == 2, i
    f32 = lib.coat_adamw_fp8_step_fp32grad
    assert f32(*a8, -1, ctypes.byref(cfg), None) == 1
    assert f32(P((1 << 20) + 4), *a8[1:], 16, ctypes.byref(cfg), None) == 2
    gd = lib.coat_adamw_fp8_step_guarded
    assert gd(*a8, 16, ctypes.byref(cfg), None, None) == 1          # no skip word
    assert gd(*a8, 16, ctypes.byref(cfg), odd4, None) == 2          # skip word misaligned
    assert gd(*a8, -1, ctypes.byref(cfg), fake, None) == 1
    q = lib.coat_quantize_state
    assert q(fake, 16, 128, 0, 0, 64.0, 0, fake, odd4, fake, None) == 2
    assert q(fake, 16, 128, 0, 0, 64.0, 0, fake, fake, odd4, None) == 2
    d = lib.coat_dequant
    assert d(fake, odd4, fake, 256, 128, 0, 0, fake, None) == 2
    assert d(fake, None, odd4, 256, 128, 0, 0, fake, None) == 2
    assert lib.coat_group_quant_1xG(fake, 4, 256, 256, 128, 0, fake, odd4, None) == 2
    gs = lib.coat_group_scaling_quant_pertensor
    assert gs(fake, 100, 128, 0, fake, 0, fake, odd4, None) == 2    # scale
    assert gs(fake, 100, 128, 0, odd4, 0, fake, fake, None) == 2    # workspace
    assert gs(fake, 100, 128, 0, fake, 3, fake, fake, None) == 1    # amax_precomputed
    na = lib.coat_group_scaling_quant_pertensor_noalloc
    assert na(fake, -1, 128, 0, fake, fake, None) == 1
    assert na(None, 100, 128, 0, fake, fake, None) == 1
    assert na(fake, 100, 96, 0, fake, fake, None) == 3
    assert na(fake, 100, 128, 2, fake, fake, None) == 3
    assert na(odd4, 100, 128, 0, fake, fake, None) == 2
    assert na(fake, 100, 128, 0, fake, odd4, None) == 2
    assert na(fake, 0, 128, 0, None, None, None) == 0
    sw = lib.coat_swiglu_group_amax
    assert sw(fake, fake, -1, 128, fake, fake, None, None) == 1
    assert sw(fake, None, 64, 128, fake, fake, None, None) == 1
    assert sw(fake, fake, 64, 100, fake, fake, None, None) == 3
    assert sw(fake, odd4, 64, 128, fake, fake, None, None) == 2
    assert sw(fake, fake, 64, 128, fake, odd4, None, None) == 2
    assert sw(fake, fake, 64, 128, fake, fake, odd4, None) == 2
    assert sw(None, None, 0, 128, None, None, None, None) == 0
    enc = lib.coat_fp8_encode
    assert enc(fake, -1, 0, fake, None) == 1
    assert enc(fake, 16, 0, None, None) == 1
    assert enc(fake, 16, 7, fake, None) == 3
    assert enc(odd4, 16, 0, fake, None) == 2
    cnt = lib.coat_count_nonfinite_bf16
    assert cnt(fake, 16, None, None) == 1
    assert cnt(None, 16, fake, None) == 1
    assert cnt(odd4, 16, fake, None) == 2
    assert cnt(fake, 16, odd2, None) == 2
    nm = lib.coat_norm_group_amax
    #      x     rows cols rms eps   weight bias  G    out   ga    tmax
    assert nm(fake, -1, 256, 0, 1e-5, None, None, 128, fake, fake, None, None) == 1
    assert nm(fake, 4, 256, 2, 1e-5, None, None, 128, fake, fake, None, None) == 1
    assert nm(fake, 4, 256, 1, 1e-5, None, fake, 128, fake, fake, None, None) == 1  # RMS + bias
    assert nm(fake, 4, 256, 0, -1.0, None, None, 128, fake, fake, None, None) == 1
    assert nm(fake, 4, 200, 0, 1e-5, None, None, 128, fake, fake, None, None) == 1  # G | cols
    assert nm(fake, 4, 256, 0, 1e-5, None, None, 96, fake, fake, None, None) == 3
    assert nm(fake, 4, 32768, 0, 1e-5, None, None, 128, fake, fake, None, None) == 3
    assert nm(odd4, 4, 256, 0, 1e-5, None, None, 128, fake, fake, None, None) == 2
    assert nm(fake, 4, 256, 0, 1e-5, odd2, None, 128, fake, fake, None, None) == 2
    assert nm(fake, 4, 256, 0, 1e-5, None, None, 128, fake, fake, odd2, None) == 2
    assert nm(fake, 0, 256, 0, 1e-5, None, None, 128, None, None, None, None) == 0
    st = lib.coat_state_stats
    assert st(fake, odd4, fake, 64, 128, 0, fake, None) == 2       # k
    assert st(fake, fake, odd4, 64, 128, 0, fake, None) == 2       # s

    def tab(*v):
        return (I64 * len(v))(*v)

    pk, up = lib.coat_pack_bf16, lib.coat_unpack_bf16
    f32src = (P * 2)(1 << 20, (1 << 21) + 2)          # second float32 source 2 bytes off
    assert pk(f32src, tab(8, 8), tab(0, 16), 2, 1, fake, 64, None) == 2
    bsrc = (P * 2)(1 << 20, (1 << 21) + 1)            # a BF16 source on an odd byte
    assert pk(bsrc, tab(8, 8), tab(0, 16), 2, 0, fake, 64, None) == 2
    assert up(fake, tab(8, 8), tab(0, 16), 2, bsrc, 64, None) == 2


def test_tensors_of_another_device_are_refused(monkeypatch):
    """The binding refuses a tensor that is not on the current CUDA device
    (the kernel would run on the current device and fault on its address).
    Checked with a stand-in tensor: this machine needs no GPU for it."""
    import torch
    from quantized_optimizer_states_b200 import _lib
    monkeypatch.setattr(_lib, "_current_device", lambda: 0)

    class OnDevice1:
        device = "cuda:1"

        def get_device(self):
            return 1

    class OnDevice0(OnDevice1):
        device = "cuda:0"

        def get_device(self):
            return 0

    with pytest.raises(ValueError, match="current device is cuda:0"):
        _lib._on_current_device(OnDevice1(), "x")
    _lib._on_current_device(OnDevice0(), "x")
    with pytest.raises(ValueError, match="must be a CUDA tensor"):
        _lib._ptr(torch.empty(4), torch.float32, "x")


def test_ctypes_structures_match_the_header(tmp_path):
    """The binding's ctypes mirrors of coat_adamw_cfg_t and
    coat_state_stats_t have the C structs' size and field offsets (a C
    program built against include/coat.h with gcc prints them)."""
    import subprocess
    from quantized_optimizer_states_b200._lib import CoatAdamwCfg, CoatStateStats
    structs = {"coat_adamw_cfg_t": CoatAdamwCfg, "coat_state_stats_t": CoatStateStats}
    lines = ["#include <stddef.h>", "#include <stdio.h>", '#include "coat.h"', "int main(void) {"]
    for cname, cls in structs.items():
        lines.append(f'  printf("{cname} size %zu\\n", sizeof({cname}));')
        for field, _ in cls._fields_:
            lines.append(f'  printf("{cname} {field} %zu\\n", offsetof({cname}, {field}));')
    lines += ["  return 0;", "}"]
    src = tmp_path / "layout.c"
    src.write_text("\n".join(lines) + "\n")
    exe = tmp_path / "layout"
    subprocess.run(["gcc", "-std=c99", "-Wall", "-I", os.path.join(ROOT, "include"), "-o",
                    str(exe), str(src)], check=True)
    out = subprocess.run([str(exe)], check=True, capture_output=True, text=True).stdout
    got = {tuple(ln.split()[:2]): int(ln.split()[2]) for ln in out.splitlines()}
    for cname, cls in structs.items():
        assert got[(cname, "size")] == ctypes.sizeof(cls), cname
        for field, _ in cls._fields_:
            assert got[(cname, field)] == getattr(cls, field).offset, (cname, field)


def _c_kind(decl: str) -> str:
    decl = decl.strip()
    if "*" in decl:
        return "ptr"
    base = decl.replace("const ", "").split()[0]
    return {"int64_t": "i64", "int32_t": "i32", "coat_status_t": "i32", "float": "f32",
            "uint32_t": "u32", "size_t": "u64"}[base]


def _ctypes_kind(t) -> str:
    if t in (ctypes.c_void_p, ctypes.c_char_p) or hasattr(t, "_type_") and t.__name__.startswith("LP_"):
        return "ptr"
    return {ctypes.c_int64: "i64", ctypes.c_int32: "i32", ctypes.c_float: "f32",
            ctypes.c_uint32: "u32", ctypes.c_uint64: "u64"}[t]


def test_binding_signatures_match_the_header():
    """Every prototype of include/coat.h has a SIGNATURES entry in the binding
    with the same number of arguments and the same kind of each (pointer,
    32/64-bit integer, float) and of the result, and the other way round: a
    stale entry would pass its arguments in the wrong registers."""
    from quantized_optimizer_states_b200._lib import SIGNATURES
    with open(os.path.join(ROOT, "include", "coat.h")) as f:
        text = re.sub(r"/\*.*?\*/", " ", f.read(), flags=re.S)
    protos = {}
    for m in re.finditer(r"(coat_status_t|int64_t|int32_t|const\s+char\s*\*)\s*(coat_\w+)\s*"
                         r"\(([^)]*)\)\s*;", text):
        res, name, params = m.group(1), m.group(2), m.group(3).strip()
        args = [] if params in ("", "void") else [p for p in params.split(",")]
        protos[name] = ("ptr" if "*" in res else _c_kind(res), [_c_kind(a) for a in args])
    assert set(protos) == set(SIGNATURES), set(protos) ^ set(SIGNATURES)
    for name, (res, args) in SIGNATURES.items():
        want_res, want_args = protos[name]
        assert _ctypes_kind(res) == want_res, name
        assert [_ctypes_kind(a) for a in args] == want_args, name


def test_peer_step_binding_checks_before_any_call():
    """The binding of coat_adamw_fp8_step_peers refuses bad rank lists on the
    host, before it touches a device pointer (CPU tensors stand in)."""
    import torch
    from quantized_optimizer_states_b200 import _lib
    n = 256
    th = torch.zeros(n)
    st = [torch.zeros(n, dtype=torch.uint8), torch.ones(2), torch.zeros(2),
          torch.zeros(n, dtype=torch.uint8), torch.ones(2), torch.zeros(2)]
    g = torch.zeros(2 * n, dtype=torch.bfloat16)
    kw = dict(step=1, beta1=0.9, beta2=0.999, lr=1e-4, eps=1e-8, weight_decay=0.0)
    for grads, extra, what in (
            ([], {}, "1 to 8 ranks"),
            ([g] * 9, {}, "1 to 8 ranks"),
            ([g, g], {"grad_offset": 384}, "ends before the shard"),
            ([g, g], {"params_out": [g]}, "one entry per rank"),
            ([g, g], {"params_out": [g, torch.zeros(2 * n)]}, "must all be float32 or all bfloat16"),
            ([g, g], {"params_out": [torch.zeros(n, dtype=torch.bfloat16), g],
                      "params_out_offset": 128}, "ends before the shard")):
        args = {"grad_offset": 0, **extra}
        with pytest.raises(ValueError, match=what):
            _lib.coat_adamw_fp8_step_peers(grads, th, *st, **args, **kw)
