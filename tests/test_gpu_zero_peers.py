"""GPU parity of the ZeRO-1 step in one kernel (coat_adamw_fp8_step_peers):
the mean of the ranks' BF16 gradients read from their buffers, the COAT
step on this rank's shard, and the updated parameters written into every
rank's parameter buffer.  The ranks' buffers are emulated by separate
buffers on one GPU (the kernel does not know whether a pointer is local or
a peer's); the result is checked against the oracle's step on the oracle's
gradient mean, and the replicas against the updated shard."""
import numpy as np
import pytest

import parity
from quantized_optimizer_states_b200 import inputs

pytestmark = pytest.mark.gpu

E4M3, E5M2 = 0, 1
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


def _case(orc, world, G, v_fmt, n, stride, seed):
    x = inputs.host_step_inputs(inputs.olmo_1b(), n)
    mc, mk, ms = orc.quantize_state(x["m0"], G, E4M3)
    vc, vk, vs = orc.quantize_state(x["v0"], G, v_fmt)
    rng = np.random.default_rng(seed)
    grads = [orc.to_bf16_array((rng.standard_normal(world * stride) * 10.0 ** -rng.integers(2, 5))
                               .astype(np.float32)) for _ in range(world)]
    return x["theta"], (mc, mk, ms, vc, vk, vs), grads


@pytest.mark.parametrize("world,rank,G,v_fmt,out", [
    (1, 0, 128, E4M3, "f32"), (2, 1, 128, E4M3, "bf16"), (3, 1, 256, E5M2, "f32"),
    (4, 3, 128, E4M3, "bf16"), (8, 5, 64, E4M3, "bf16"), (5, 2, 1024, E5M2, "f32")])
def test_peer_step_matches_the_oracle_on_the_mean_gradient(lib, orc, world, rank, G, v_fmt,
                                                           out):
    import torch
    stride = 3 * 4096 + 4 * max(G, 16)               # a rank's shard stride (whole groups)
    n = stride - 2 * G + 7 if rank == world - 1 else stride   # the last shard is ragged
    off = rank * stride
    th, st, grads = _case(orc, world, G, v_fmt, n, stride, seed=world * 100 + rank)
    cfg = dict(step=10, group_size=G, v_fmt=v_fmt, **H)
    g_mean = orc.grad_mean_bf16([g[off:off + n] for g in grads])
    ref = orc.adamw_fp8_step(th, g_mean, *st, return_moments=True, **cfg)

    gd = [parity.to_dev(g.view(np.int16)) for g in grads]
    pdt = torch.bfloat16 if out == "bf16" else torch.float32
    sentinel = 7.0
    outs = [torch.full((world * stride,), sentinel, dtype=pdt, device="cuda")
            for _ in range(world)]
    d = [parity.to_dev(th)] + [parity.to_dev(a) for a in st]
    lib.coat_adamw_fp8_step_peers(gd, *d, grad_offset=off, params_out=outs,
                                  params_out_offset=off, **cfg)
    torch.cuda.synchronize()
    got = tuple(parity.to_host(t) for t in d)
    parity.assert_step_parity(got, ref, H["lr"], G, v_fmt, moments=(ref[7], ref[8]))
    want = torch.from_numpy(got[0]).to(pdt)          # the replicas: the updated shard
    for r, o in enumerate(outs):
        oc = o.cpu()
        assert torch.equal(oc[off:off + n].view(torch.int16 if out == "bf16" else torch.int32),
                           want.view(torch.int16 if out == "bf16" else torch.int32)), r
        rest = torch.cat([oc[:off], oc[off + n:]])
        assert torch.all(rest == sentinel), r


def test_one_rank_without_copies_is_the_plain_step(lib, orc):
    """world = 1 with no parameter copies: bit-identical to
    coat_adamw_fp8_step on the same gradient."""
    import torch
    G, n = 128, 5 * 4096 + 3 * 128 + 5
    th, st, grads = _case(orc, 1, G, E4M3, n, n, seed=3)
    cfg = dict(step=7, group_size=G, v_fmt=E4M3, **H)
    a = [parity.to_dev(th)] + [parity.to_dev(x) for x in st]
    b = [parity.to_dev(th)] + [parity.to_dev(x) for x in st]
    g = parity.to_dev(grads[0][:n].view(np.int16))
    lib.coat_adamw_fp8_step_peers([g], *a, grad_offset=0, **cfg)
    lib.coat_adamw_fp8_step(b[0], g, *b[1:], **cfg)
    torch.cuda.synchronize()
    for x, y in zip(a, b):
        assert torch.equal(x, y)


def test_peer_step_argument_errors(lib):
    import torch
    th = torch.zeros(256, device="cuda")
    st = [torch.zeros(256, dtype=torch.uint8, device="cuda"), torch.ones(2, device="cuda"),
          torch.zeros(2, device="cuda"), torch.zeros(256, dtype=torch.uint8, device="cuda"),
          torch.ones(2, device="cuda"), torch.zeros(2, device="cuda")]
    g = torch.zeros(512, dtype=torch.bfloat16, device="cuda")
    cfg = dict(step=1, group_size=128, **H)
    with pytest.raises(ValueError):
        lib.coat_adamw_fp8_step_peers([], th, *st, grad_offset=0, **cfg)
    with pytest.raises(ValueError):
        lib.coat_adamw_fp8_step_peers([g] * 9, th, *st, grad_offset=0, **cfg)
    with pytest.raises(ValueError):                      # gradient shorter than the shard
        lib.coat_adamw_fp8_step_peers([g, g], th, *st, grad_offset=384, **cfg)
    with pytest.raises(lib.CoatError) as e:              # 8-byte gradient offset
        lib.coat_adamw_fp8_step_peers([g, g], th, *st, grad_offset=4, **cfg)
    assert e.value.status == 2


def test_enable_peer_access_argument_handling(lib):
    """The current device needs no enabling; a device index the machine does
    not have is refused before any CUDA call that could change state."""
    import torch
    cur = torch.cuda.current_device()
    lib.coat_enable_peer_access(cur)                    # a no-op
    with pytest.raises(lib.CoatError) as e:
        lib.coat_enable_peer_access(torch.cuda.device_count() + 3)
    assert e.value.status == 1
