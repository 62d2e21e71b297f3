"""The synthetic input recipe (CPU only): the OLMo-shaped parameter sets, the
activation workload and the step workloads carry the sizes and
distributions they are described with -- OLMo-1B / OLMo-7B tensor shapes
(tied / untied embedding, non-parametric LayerNorm), hyper-parameters of
the COAT summary page's AdamW setting, GLU-style spike channels (COAT
summary page, section "激活为什么难压"), and the gradient zeros and spikes of
the step sets."""
import numpy as np

from quantized_optimizer_states_b200 import inputs


def test_olmo_parameter_sets():
    s1 = inputs.tensor_sizes(inputs.OLMO_1B)
    s7 = inputs.tensor_sizes(inputs.OLMO_7B)
    assert sum(s1) == 1_176_764_416 and len(s1) == 1 + 16 * 7          # tied embedding
    assert sum(s7) == 6_888_095_744 and len(s7) == 1 + 32 * 7 + 1      # untied head
    assert sum(s7) // 128 == 53_813_248 and sum(s7) % 128 == 0
    # every tensor is whole 1xG groups for every supported G up to 1024, so
    # no group straddles two tensors of the flat buffer
    assert all(n % 1024 == 0 for n in s1 + s7)
    # resident OLMo-7B step state: theta 4 B, BF16 grad 2 B, two codes 2 B,
    # and (k, s) for two states per 128-element group
    gb = (sum(s7) * 8 + (sum(s7) // 128) * 16) / 1e9
    assert 55.0 < gb < 57.0
    w = inputs.olmo_7b()
    assert w.n == sum(s7) and w.group_size == 128 and w.v_fmt == "e4m3"
    assert inputs.olmo_7b(v_fmt="e5m2").v_fmt == "e5m2" and inputs.olmo_1b().v_fmt == "e5m2"


def test_hyper_parameters_and_sweep_regimes():
    assert inputs.HYPER == dict(beta1=0.9, beta2=0.999, lr=1e-4, eps=1e-8, weight_decay=0.1)
    for regime, (mu, sg) in {"early": (-25.0, 2.0), "late": (-14.0, 2.0),
                             "typical": (-18.0, 0.25)}.items():
        w = inputs.sweep(128, "e4m3", regime)
        assert (w.v_mu, w.v_sigma, w.n) == (mu, sg, 1 << 28)
    assert inputs.tiny().n == 1 << 20 and inputs.tiny().step == 10


def test_step_gradients_have_the_stated_zeros_and_spikes():
    w = inputs.olmo_1b()
    n = 1 << 20                               # inside the first (embedding) tensor
    a = inputs.host_step_inputs(w, n)
    b = inputs.host_step_inputs(w, n)
    assert all(np.array_equal(a[k], b[k]) for k in a)                # seeded
    g = a["grad"].view(np.int16).astype(np.int32) << 16
    gf = g.astype(np.uint32).view(np.float32).astype(np.float64)
    zeros = np.mean(gf == 0.0)
    assert 0.009 < zeros < 0.011                                      # 1% exact zeros
    sd = np.median(np.abs(gf[gf != 0])) / 0.6745                      # robust sigma_T
    spikes = np.mean(np.abs(gf) > 20 * sd)
    assert 0.0007 < spikes < 0.0013                                   # 0.1% x 100
    assert abs(float(np.std(a["theta"])) - 0.02) < 2e-4
    assert abs(float(np.std(a["m0"])) - 1e-4) < 1e-6
    lv = np.log(a["v0"].astype(np.float64))
    assert abs(lv.mean() + 18.0) < 0.01 and abs(lv.std() - 1.0) < 0.01


def test_activation_workload():
    w = inputs.activations()
    assert (w.rows, w.cols, w.group_size) == (16384, 2048, 128)
    x = inputs.host_activations(w, rows=256)
    assert x.shape == (256, 2048) and x.dtype == np.uint16
    assert np.array_equal(x, inputs.host_activations(w, rows=256))   # seeded
    xf = (x.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    col_max = np.abs(xf).max(axis=0)
    spiky = np.nonzero(col_max > 20.0)[0]
    assert spiky.size == max(1, round(0.0005 * 2048)) == 1           # one spike channel
    mult = np.abs(xf[:, spiky[0]])
    assert mult.max() < 500 * 6 and np.median(mult) > 10             # N(0,1) x U[50, 500]
    rest = np.delete(xf, spiky, axis=1)
    assert abs(rest.std() - 1.0) < 0.01 and np.abs(rest).max() < 7.0
