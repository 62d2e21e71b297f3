"""Guard canaries around the outputs of every activation-side, producer,
pack and monitoring kernel, a check that needs no memory-checking tool: each
output is a slice of a larger buffer whose 256 bytes before and after hold
a sentinel, sizes are ragged (partial blocks and tiles, tail
vectors, tail groups), and after the calls the sentinels must be intact
(the outputs' values are the parity tests' business)."""
import numpy as np
import pytest

import parity
from quantized_optimizer_states_b200 import inputs

pytestmark = pytest.mark.gpu

PAD = 256           # bytes of sentinel on each side
SENT = 0xA5


@pytest.fixture(scope="module")
def lib():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from quantized_optimizer_states_b200 import build
    build.build()
    import quantized_optimizer_states_b200 as q
    q.load()
    return q


class Guarded:
    """A tensor of `numel` elements of `dtype` inside a byte buffer with PAD
    sentinel bytes on both sides (the slice stays 256-byte aligned)."""

    def __init__(self, numel, dtype):
        import torch
        self.size = torch.empty(0, dtype=dtype).element_size() * numel
        self.buf = torch.full((PAD + self.size + PAD,), SENT, dtype=torch.uint8, device="cuda")
        self.t = self.buf[PAD:PAD + self.size].view(dtype)

    def check(self, what):
        import torch
        torch.cuda.synchronize()
        b = self.buf.cpu().numpy()
        assert np.all(b[:PAD] == SENT) and np.all(b[PAD + self.size:] == SENT), what


@pytest.mark.parametrize("rows", [3, 9])
def test_activation_kernels_stay_inside(lib, rows):
    import torch
    G = 128
    cols = 2048
    x = inputs.host_activations(inputs.activations(seed=rows), rows=rows)
    n = x.size - 48                                  # ragged flat length
    xf = parity.to_dev(x.reshape(-1)[:n].view(np.int16))
    # 1xG on contiguous rows (the flat kernel, a partial last block)
    q = Guarded(rows * cols, torch.uint8)
    sc = Guarded(rows * cols // G, torch.float32)
    lib.coat_group_quant_1xG(parity.to_dev(x.view(np.int16)), q.t.view(rows, cols),
                             sc.t.view(rows, cols // G), group_size=G)
    q.check("1xG codes"), sc.check("1xG scales")
    # Group Scaling on a ragged length (a tail vector), both workspace modes
    ng = -(-n // G)
    ws = Guarded(ng + 1, torch.float32)
    qg = Guarded(n, torch.uint8)
    s1 = Guarded(1, torch.float32)
    lib.coat_group_scaling_quant_pertensor(xf, ws.t, qg.t, s1.t, group_size=G)
    lib.coat_group_scaling_quant_pertensor(xf, ws.t, qg.t, s1.t, group_size=G,
                                           amax_precomputed=1)
    ws.check("GS workspace"), qg.check("GS codes"), s1.check("GS scale")
    # producers with their maxima and tensor maximum
    gate, up = inputs.host_swiglu_inputs(inputs.activations(seed=5), rows=rows)
    out = Guarded(n, torch.int16)
    ga = Guarded(ng + 1, torch.float32)
    lib.coat_swiglu_group_amax(parity.to_dev(gate.reshape(-1)[:n].view(np.int16)),
                               parity.to_dev(up.reshape(-1)[:n].view(np.int16)), out.t,
                               ga.t[:ng], group_size=G, tensor_amax=ga.t[ng:])
    out.check("SwiGLU out"), ga.check("SwiGLU maxima")
    ln = Guarded(rows * cols, torch.int16)
    gl = Guarded(rows * cols // G + 1, torch.float32)
    lib.coat_norm_group_amax(parity.to_dev(x.view(np.int16)), ln.t.view(rows, cols),
                             gl.t[:rows * cols // G], group_size=G,
                             tensor_amax=gl.t[rows * cols // G:])
    ln.check("norm out"), gl.check("norm maxima")
    # dequant (FP32 and BF16 out), the FP8 cast alone
    for dt in (torch.float32, torch.bfloat16):
        dq = Guarded(n, dt)
        lib.coat_dequant(qg.t, None, s1.t, dq.t, group_size=n)
        dq.check(f"dequant {dt}")
    y = parity.to_dev((np.random.default_rng(rows).standard_normal(n) * 100).astype(np.float32))
    qe = Guarded(n, torch.uint8)
    lib.coat_fp8_encode(y, qe.t)
    qe.check("fp8 encode")


def test_state_kernels_stay_inside(lib):
    import torch
    G, n = 128, 5 * 1024 + 77
    rng = np.random.default_rng(4)
    xs = parity.to_dev((rng.standard_normal(n) * 1e-4).astype(np.float32))
    ng = -(-n // G)
    code = Guarded(n, torch.uint8)
    k = Guarded(ng, torch.float32)
    s = Guarded(ng, torch.float32)
    lib.coat_quantize_state(xs, code.t, k.t, s.t, group_size=G)
    code.check("codes"), k.check("k"), s.check("s")
    st = Guarded(64, torch.uint8)
    lib.coat_state_stats(code.t, k.t, s.t, group_size=G, out=st.t)
    st.check("stats")
    dq = Guarded(n, torch.float32)
    lib.coat_dequant(code.t, k.t, s.t, dq.t, group_size=G)
    dq.check("state dequant")
    cnt = Guarded(1, torch.int32)
    g = parity.to_dev((rng.standard_normal(n) * 1e-3).astype(np.float32)).to(torch.bfloat16)
    lib.coat_count_nonfinite_bf16(g, cnt.t)
    cnt.check("non-finite count")


def test_pack_kernels_stay_inside(lib):
    import torch
    sizes = [7, 2049, 0, 300, 16]
    offs, off = [], 0
    for m in sizes:
        offs.append(off)
        off += -(-m // 16) * 16
    table = lib.PackTable(sizes, offs)
    rng = np.random.default_rng(6)
    srcs = [parity.to_dev(rng.standard_normal(m).astype(np.float32)) for m in sizes]
    flat = Guarded(off, torch.int16)
    lib.coat_pack_bf16(srcs, table, flat.t)
    flat.check("pack")
    outs = [Guarded(m, torch.int16) for m in sizes]
    master = parity.to_dev(rng.standard_normal(off).astype(np.float32))
    lib.coat_unpack_bf16(master, table, [o.t for o in outs])
    for o in outs:
        o.check("unpack")
