"""The library's calls inside CUDA graphs: a chain of activation-side calls
(SwiGLU producer with its maxima and tensor maximum, Group Scaling as the
cast alone, 1xG quantization, dequantization) and the fused step, each
captured once with torch.cuda.graph and replayed on new inputs copied into
the captured buffers; every replay gives the same bits as the same calls
run eagerly.  The activation kernels are launched with programmatic
dependent launch, which a capture turns into programmatic graph edges."""
import numpy as np
import pytest

import parity
from quantized_optimizer_states_b200 import inputs

pytestmark = pytest.mark.gpu
H = inputs.HYPER


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


def _act_chain(lib, b, G):
    ng = b["gate"].numel() // G
    lib.coat_swiglu_group_amax(b["gate"], b["up"], b["h"], b["ws"], group_size=G)
    lib.coat_group_scaling_quant_pertensor(b["h"], b["ws"], b["q"], b["s1"], group_size=G,
                                           amax_precomputed=2)
    lib.coat_group_quant_1xG(b["h"].view(b["rows"], -1), b["q1"], b["sc"], group_size=G)
    lib.coat_dequant(b["q1"].reshape(-1), None, b["sc"].reshape(-1), b["deq"], group_size=G)
    assert ng == b["sc"].numel()


def _act_buffers(torch, rows, cols, G):
    n = rows * cols
    return {"rows": rows,
            "gate": torch.empty(n, dtype=torch.bfloat16, device="cuda"),
            "up": torch.empty(n, dtype=torch.bfloat16, device="cuda"),
            "h": torch.empty(n, dtype=torch.bfloat16, device="cuda"),
            "ws": torch.empty(n // G + 1, dtype=torch.float32, device="cuda"),
            "q": torch.empty(n, dtype=torch.uint8, device="cuda"),
            "s1": torch.empty(1, dtype=torch.float32, device="cuda"),
            "q1": torch.empty(rows, cols, dtype=torch.uint8, device="cuda"),
            "sc": torch.empty(rows, cols // G, dtype=torch.float32, device="cuda"),
            "deq": torch.empty(n, dtype=torch.float32, device="cuda")}


def _fill(torch, b, seed):
    w = inputs.activations(seed=seed)
    gate, up = inputs.host_swiglu_inputs(w, rows=b["rows"])
    b["gate"].copy_(torch.from_numpy(gate[:, :b["q1"].shape[1]].reshape(-1).view(np.int16))
                    .view(torch.bfloat16))
    b["up"].copy_(torch.from_numpy(up[:, :b["q1"].shape[1]].reshape(-1).view(np.int16))
                  .view(torch.bfloat16))


def test_activation_chain_replays_bit_for_bit(lib):
    import torch
    rows, cols, G = 96, 2048, 128
    b = _act_buffers(torch, rows, cols, G)
    _fill(torch, b, 1)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        _act_chain(lib, b, G)                # first calls outside the capture
    torch.cuda.current_stream().wait_stream(s)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        _act_chain(lib, b, G)
    for seed in (2, 3):
        _fill(torch, b, seed)
        g.replay()
        torch.cuda.synchronize()
        got = {k: b[k].clone() for k in ("h", "ws", "q", "s1", "q1", "sc", "deq")}
        _act_chain(lib, b, G)                # the same calls, eager
        torch.cuda.synchronize()
        for k, v in got.items():
            assert torch.equal(v.view(torch.uint8), b[k].view(torch.uint8)), (seed, k)


def test_step_replays_bit_for_bit(lib, orc):
    import torch
    G, n = 128, 9 * 4096 + 3 * 128 + 5
    x = inputs.host_step_inputs(inputs.olmo_1b(), n)
    st0 = [*orc.quantize_state(x["m0"], G, 0), *orc.quantize_state(x["v0"], G, 0)]
    cfg = dict(step=10, group_size=G, **H)
    bufs = [parity.to_dev(x["theta"]), parity.to_dev(x["grad"].view(np.int16))] + \
        [parity.to_dev(a) for a in st0]
    start = [t.clone() for t in bufs]

    def step():
        lib.coat_adamw_fp8_step(bufs[0], bufs[1], *bufs[2:], **cfg)

    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        step()
    torch.cuda.current_stream().wait_stream(s)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        step()
    for a, b0 in zip(bufs, start):
        a.copy_(b0)
    g.replay()
    torch.cuda.synchronize()
    got = [t.clone() for t in bufs]
    for a, b0 in zip(bufs, start):
        a.copy_(b0)
    step()
    torch.cuda.synchronize()
    for a, b1 in zip(got, bufs):
        assert torch.equal(a, b1)
