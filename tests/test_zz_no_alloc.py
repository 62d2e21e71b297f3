"""The no-allocation Group Scaling entry point (GPU).

Some callers cannot allocate device memory once they are running -- a
serving process with a budget fixed at start-up, or a plug-in whose host
framework owns every allocation.  coat_group_scaling_quant_pertensor_noalloc
serves them: it uses scratch compiled into the library instead of a
caller-supplied workspace.  These tests call it through the C ABI and check
it, bit for bit, against the oracle's Group Scaling and against the
workspace entry point, on consecutive calls (the shared scratch keeps the
previous call's contents, so the second call checks that nothing leaks from
the first).  This file is collected last.
"""
import ctypes

import pytest

from quantized_optimizer_states_b200 import inputs

pytestmark = pytest.mark.gpu


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


def _with_workspace(lib, x, G, fmt):
    import torch
    n = x.numel()
    ws = torch.empty(lib.coat_group_scaling_workspace_bytes(n, G) // 4, dtype=torch.float32,
                     device="cuda")
    q = torch.empty(n, dtype=torch.uint8, device="cuda")
    s = torch.empty(1, dtype=torch.float32, device="cuda")
    lib.coat_group_scaling_quant_pertensor(x, ws, q, s, group_size=G, fmt=fmt)
    return q, s


def _without_workspace(lib, x, G, fmt):
    import torch
    n = x.numel()
    q = torch.empty(n, dtype=torch.uint8, device="cuda")
    s = torch.empty(1, dtype=torch.float32, device="cuda")
    raw = lib.load()
    st = raw.coat_group_scaling_quant_pertensor_noalloc(
        ctypes.c_void_p(x.data_ptr()), n, G, fmt, ctypes.c_void_p(q.data_ptr()),
        ctypes.c_void_p(s.data_ptr()), ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == 0, lib.coat_status_string(st)
    return q, s


def test_noalloc_matches_the_oracle_and_the_workspace_variant_on_consecutive_calls(lib, orc):
    import numpy as np
    import torch
    # a large tensor first, then a smaller one whose maximum is far below the
    # first call's: stale scratch from call one would change call two
    big = inputs.device_activations(inputs.activations(), torch.device("cuda")).reshape(-1)
    small = (torch.randn(300_007, device="cuda") * 0.01).to(torch.bfloat16)
    for x, G, fmt in ((big, 128, 0), (small, 128, 0), (small, 1024, 1)):
        q_ref, s_ref = _with_workspace(lib, x, G, fmt)
        q, s = _without_workspace(lib, x, G, fmt)
        torch.cuda.synchronize()
        q_orc, s_orc, _ = orc.group_scaling_pertensor(
            x.view(torch.int16).cpu().numpy().view(np.uint16), G, fmt)
        assert s.item() == s_orc
        assert np.array_equal(q.cpu().numpy(), q_orc)
        assert torch.equal(s, s_ref)
        assert torch.equal(q, q_ref)


def test_noalloc_rejects_sizes_beyond_its_scratch(lib):
    import torch
    raw = lib.load()
    G = 16
    n = (lib.COAT_NOALLOC_MAX_GROUPS + 1) * G       # one group too many
    x = torch.empty(16, dtype=torch.bfloat16, device="cuda")
    q = torch.empty(16, dtype=torch.uint8, device="cuda")
    s = torch.empty(1, dtype=torch.float32, device="cuda")
    # rejected on the host before anything touches the (too small) buffers
    st = raw.coat_group_scaling_quant_pertensor_noalloc(
        ctypes.c_void_p(x.data_ptr()), n, G, 0, ctypes.c_void_p(q.data_ptr()),
        ctypes.c_void_p(s.data_ptr()), None)
    assert st == 3
