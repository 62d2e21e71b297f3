"""Mutation tests of the oracle's pins (CPU only).

Each case plants one plausible mistake in a copy of the C oracle -- a wrong
bias or exponent in the FP8 codec, a broken tie rule, a dropped term, sign
or bias correction in the AdamW rule, a transposed operand, a wrong range or
exponent in COAT's expansion, a wrong scale in the activation quantizers --
compiles the copy with the oracle's own flags, and runs the oracle's pin
tests (tests/test_oracle_codec.py, test_oracle_state.py, test_oracle_act.py)
against it.  The oracle's Python half (BF16 rounding, SwiGLU, LayerNorm /
RMSNorm, the unquantized binary64 AdamW, the state statistics, the array
wrappers) is mutated the same way: a copy of oracle/__init__.py with the
mistake is executed into the imported module before pytest starts in that
process, and every pin file runs against it.  Every mutant must make at
least one pin fail: a mutant that passes would be a mistake the pins cannot
see.  The pins themselves are unchanged; only the oracle under them is
swapped."""
import os
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

import pytest

from oracle import build as orc_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PIN_FILES = ["tests/test_oracle_codec.py", "tests/test_oracle_state.py",
             "tests/test_oracle_act.py"]
PY_PIN_FILES = PIN_FILES + ["tests/test_oracle_norm.py", "tests/test_oracle_swiglu.py",
                            "tests/test_oracle_grad_mean.py"]
PY_SRC = os.path.join(ROOT, "oracle", "__init__.py")

# (name, text in oracle/__init__.py, replacement)
PY_MUTANTS = [
    ("bf16_ties_away", "q = np.ldexp(np.rint(np.ldexp(x, 8 - e)), e - 8)",
     "q = np.ldexp(np.floor(np.ldexp(x, 8 - e) + 0.5), e - 8)"),
    ("bf16_no_subnormal_quantum", "e = np.maximum(e, -125)", "e = e"),
    ("bf16_bits_shift", "b = np.asarray(b, dtype=np.uint16).astype(np.uint32) << 16",
     "b = np.asarray(b, dtype=np.uint16).astype(np.uint32) << 15"),
    ("silu_sign", "h = g / (1.0 + np.exp(-g)) * u", "h = g / (1.0 + np.exp(g)) * u"),
    ("sigmoid_for_silu", "h = g / (1.0 + np.exp(-g)) * u", "h = 1.0 / (1.0 + np.exp(-g)) * u"),
    ("layernorm_not_centred", "d = x - np.mean(x, axis=-1, keepdims=True)", "d = x"),
    ("layernorm_eps_outside_root",
     "y = d / np.sqrt(np.mean(d * d, axis=-1, keepdims=True) + e)",
     "y = d / (np.sqrt(np.mean(d * d, axis=-1, keepdims=True)) + e)"),
    ("rmsnorm_square_of_mean", "y = x / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + e)",
     "y = x / np.sqrt(np.mean(x, axis=-1, keepdims=True) ** 2 + e)"),
    ("norm_weight_reversed", "y = y * np.asarray(weight, dtype=np.float32).astype(np.float64)",
     "y = y * np.asarray(weight, dtype=np.float32)[::-1].astype(np.float64)"),
    ("norm_bias_dropped", "y = y + np.asarray(bias, dtype=np.float32).astype(np.float64)",
     "y = y"),
    ("fp64_adamw_v_not_squared", "v_t = b2 * v + (1.0 - b2) * g * g", "v_t = b2 * v + (1.0 - b2) * g"),
    ("fp64_adamw_no_bias_correction", "m_hat = m_t / (1.0 - b1 ** step)", "m_hat = m_t"),
    ("fp64_adamw_decay_without_lr",
     "th = theta * (1.0 - float(np.float32(lr)) * float(np.float32(weight_decay)))",
     "th = theta * (1.0 - float(np.float32(weight_decay)))"),
    ("fp64_adamw_eps_inside_root",
     "m_hat / (np.sqrt(v_hat) + float(np.float32(eps)))",
     "m_hat / np.sqrt(v_hat + float(np.float32(eps)))"),
    ("group_amax_signed",
     "x = np.abs(bf16_bits_to_f64(np.ascontiguousarray(x_bf16).reshape(-1)))",
     "x = bf16_bits_to_f64(np.ascontiguousarray(x_bf16).reshape(-1))"),
    ("stats_top_code_e4m3_only", "top = 0x7E if fmt == E4M3 else 0x7B", "top = 0x7E"),
    ("stats_k1_counts_zero_groups", '"k1_groups": int((k[nz] == 1.0).sum())',
     '"k1_groups": int((k == 1.0).sum())'),
    ("stats_nonfinite_includes_max", '"nonfinite_codes": int((mag > top).sum())',
     '"nonfinite_codes": int((mag >= top).sum())'),
    ("stats_k_sum_over_all_groups", "kn = k[nz].astype(np.float64)", "kn = k.astype(np.float64)"),
    ("grad_mean_not_divided", "        acc = np.divide(acc, np.float32(len(grads)), dtype=np.float32)",
     "        acc = acc"),
    ("grad_mean_divides_by_world_minus_one",
     "acc = np.divide(acc, np.float32(len(grads)), dtype=np.float32)",
     "acc = np.divide(acc, np.float32(len(grads) - 1), dtype=np.float32)"),
    ("grad_mean_drops_the_last_rank", "    for g in grads[1:]:", "    for g in grads[1:-1]:"),
    ("grad_mean_first_rank_only", "    for g in grads[1:]:\n        acc = np.add(",
     "    for g in []:\n        acc = np.add("),
    ("step_wrapper_swaps_k_and_s",
     "_ptr(th), _ptr(g), _ptr(mc), _ptr(mk), _ptr(ms), _ptr(vc),",
     "_ptr(th), _ptr(g), _ptr(mc), _ptr(ms), _ptr(mk), _ptr(vc),"),
]

# executes a mutated copy of oracle/__init__.py into the imported oracle
# module, then runs pytest in the same process
PY_RUNNER = (
    "import sys, oracle, pytest\n"
    "src = open(sys.argv[1]).read()\n"
    "exec(compile(src, oracle.__file__, 'exec'), oracle.__dict__)\n"
    "sys.exit(pytest.main(sys.argv[2:]))\n")

# (name, text in coat_oracle.c, replacement): each text occurs exactly once
MUTANTS = [
    # FP8 codec
    ("e4m3_bias_8", "v = orc_exmy_value(4, 3, 7, e, m);", "v = orc_exmy_value(4, 3, 8, e, m);"),
    ("subnormal_exponent", "return frac * ldexp(1.0, 1 - bias);",
     "return frac * ldexp(1.0, -bias);"),
    ("e4m3_top_binade_all_nan", "if (e == 15u && m == 7u)", "if (e == 15u)"),
    ("e5m2_no_infinity", "return m == 0u ? (neg ? -INFINITY : INFINITY) : NAN;", "return NAN;"),
    ("fp8_ties_down", "c = (lo & 1) ? lo + 1 : lo;", "c = lo;"),
    ("fp8_nan_to_zero", "    if (isnan(y))\n        return 0x7F;",
     "    if (isnan(y))\n        return 0x00;"),
    ("bf16_ties_away", "r = ((lo_bits >> 16) & 1u) ? hi_bits : lo_bits;", "r = hi_bits;"),
    ("bf16_decode_low_half", "uint32_t u = (uint32_t)b << 16;", "uint32_t u = (uint32_t)b << 15;"),
    # COAT expansion and state codec
    ("k_from_storage_range", "return k_range == 1 ? orc_fp8_range(store_fmt) : "
     "orc_fp8_range(ORC_E4M3);", "return orc_fp8_range(store_fmt);"),
    ("k_ratio_inverted", "log((double)M / (double)mn)", "log((double)mn / (double)M) * -0.5"),
    ("range_min_counts_zeros", "if (a > 0.0f && a < mn)", "if (a < mn)"),
    ("no_k_clamp", "if (k_max > 0.0f && kd > (double)k_max)", "if (0)"),
    ("scale_ignores_k", "float s = (float)((double)M * pow(fmax, -1.0 / (double)kf));",
     "float s = (float)((double)M / fmax);"),
    ("expansion_inverse_power", "pow((double)fabsf(xi) / (double)M, (double)kf)",
     "pow((double)fabsf(xi) / (double)M, 1.0 / (double)kf)"),
    ("decode_power_not_inverted", "pow(fabs(d), 1.0 / (double)k)", "pow(fabs(d), (double)k)"),
    ("code_sign_dropped", "code[i] = (uint8_t)(xi < 0.0f ? (c | 0x80) : c);", "code[i] = c;"),
    ("zero_group_scale_one", "        *k_out = 1.0f;\n        *s_out = 0.0f;",
     "        *k_out = 1.0f;\n        *s_out = 1.0f;"),
    # AdamW rule
    ("v_uses_beta1", "float v_new = b2 * v + c2 * (g * g);", "float v_new = b1 * v + c1 * (g * g);"),
    ("v_gradient_not_squared", "float v_new = b2 * v + c2 * (g * g);",
     "float v_new = b2 * v + c2 * fabsf(g);"),
    ("no_bias_correction_m", "float m_hat = m_new / bc1;", "float m_hat = m_new;"),
    ("no_bias_correction_v", "float v_hat = v_new / bc2;", "float v_hat = v_new;"),
    ("bias_correction_off_by_one", "pow((double)b1, (double)cfg->step)",
     "pow((double)b1, (double)(cfg->step + 1))"),
    ("eps_inside_root", "float u = m_hat / (sqrtf(v_hat) + eps);",
     "float u = m_hat / sqrtf(v_hat + eps);"),
    ("decay_without_lr", "const float decay = 1.0f - cfg->lr * cfg->weight_decay;",
     "const float decay = 1.0f - cfg->weight_decay;"),
    ("update_sign", "theta[i] = theta[i] * decay - lr * u;", "theta[i] = theta[i] * decay + lr * u;"),
    ("stores_bias_corrected_m", "mt[j] = m_new;", "mt[j] = m_hat;"),
    ("m_decoded_with_v_params",
     "float m = orc_state_dequant_one(m_code[i], m_k[gi], m_s[gi], cfg->m_fmt);",
     "float m = orc_state_dequant_one(m_code[i], v_k[gi], v_s[gi], cfg->m_fmt);"),
    ("v_stored_in_m_format",
     "orc_quant_group(vt, len, cfg->v_fmt, cfg->k_range,",
     "orc_quant_group(vt, len, cfg->m_fmt, cfg->k_range,"),
    # activation quantizers
    ("act_scale_inverted", "*s = amax / fmax;", "*s = fmax / amax;"),
    ("act_zero_scale", "        *s = 1.0f;\n        *inv = 1.0f;",
     "        *s = 0.0f;\n        *inv = 1.0f;"),
    ("1xG_ignores_row_stride", "const uint16_t *xg = x + r * ld + gi * G;",
     "const uint16_t *xg = x + r * cols + gi * G;"),
    ("group_scaling_skips_last_group", "    for (int64_t gi = 0; gi < ng; ++gi)\n        if (group_amax[gi] > amax)",
     "    for (int64_t gi = 0; gi + 1 < ng; ++gi)\n        if (group_amax[gi] > amax)"),
    ("group_scaling_recomputes_given_maxima", "    if (!amax_precomputed) {", "    if (1) {"),
]


def _build_mutant(src: str, name: str, old: str, new: str, out_dir: str) -> str:
    assert src.count(old) == 1, f"{name}: the text to mutate must occur exactly once"
    path = os.path.join(out_dir, f"coat_oracle_{name}.c")
    with open(path, "w") as f:
        f.write(src.replace(old, new))
    lib = os.path.join(out_dir, f"liborc_{name}.so")
    subprocess.run(["gcc", *orc_build.CFLAGS, "-w", "-o", lib, path, "-lm"], check=True)
    return lib


def _pins_fail(lib: str) -> tuple[int, str]:
    env = dict(os.environ, COAT_ORACLE_LIB=lib)
    r = subprocess.run([sys.executable, "-m", "pytest", *PIN_FILES, "-x", "-q",
                        "-p", "no:cacheprovider", "-m", "not gpu",
                        "-k", "not torch_adamw"],          # that pin is Python-only
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    tail = (r.stdout + r.stderr).strip().splitlines()
    return r.returncode, tail[-1] if tail else ""


def _py_pins_fail(src_path: str) -> tuple[int, str]:
    r = subprocess.run([sys.executable, "-c", PY_RUNNER, src_path, *PY_PIN_FILES, "-x", "-q",
                        "-p", "no:cacheprovider", "-m", "not gpu"],
                       cwd=ROOT, capture_output=True, text=True, timeout=600)
    tail = (r.stdout + r.stderr).strip().splitlines()
    return r.returncode, tail[-1] if tail else ""


def test_mutant_texts_are_unique():
    with open(orc_build.SRC) as f:
        src = f.read()
    for name, old, _ in MUTANTS:
        assert src.count(old) == 1, name
    with open(PY_SRC) as f:
        py = f.read()
    for name, old, _ in PY_MUTANTS:
        assert py.count(old) == 1, name


def test_unmutated_copy_passes_the_pins(tmp_path):
    """Control: the same machinery with no mistake planted passes."""
    with open(orc_build.SRC) as f:
        src = f.read()
    anchor = MUTANTS[0][1]
    lib = _build_mutant(src, "control", anchor, anchor, str(tmp_path))
    rc, tail = _pins_fail(lib)
    assert rc == 0, tail
    path = os.path.join(str(tmp_path), "oracle_init_control.py")
    with open(PY_SRC) as f, open(path, "w") as g:
        g.write(f.read())
    rc, tail = _py_pins_fail(path)
    assert rc == 0, tail


def test_every_planted_mistake_fails_a_pin(tmp_path):
    with open(orc_build.SRC) as f:
        src = f.read()
    libs = [(name, _build_mutant(src, name, old, new, str(tmp_path)))
            for name, old, new in MUTANTS]
    with ThreadPoolExecutor(max_workers=max(1, min(8, os.cpu_count() or 1))) as ex:
        results = list(ex.map(lambda nl: (nl[0], *_pins_fail(nl[1])), libs))
    survivors = [(name, tail) for name, rc, tail in results if rc != 1]
    assert not survivors, f"mistakes no pin catches (or runs that did not fail cleanly): {survivors}"


def test_every_planted_mistake_in_the_python_half_fails_a_pin(tmp_path):
    with open(PY_SRC) as f:
        src = f.read()
    paths = []
    for name, old, new in PY_MUTANTS:
        assert src.count(old) == 1, name
        path = os.path.join(str(tmp_path), f"oracle_init_{name}.py")
        with open(path, "w") as f:
            f.write(src.replace(old, new))
        paths.append((name, path))
    with ThreadPoolExecutor(max_workers=max(1, min(8, os.cpu_count() or 1))) as ex:
        results = list(ex.map(lambda np_: (np_[0], *_py_pins_fail(np_[1])), paths))
    survivors = [(name, tail) for name, rc, tail in results if rc != 1]
    assert not survivors, f"mistakes no pin catches (or runs that did not fail cleanly): {survivors}"
