"""Mutation check of the oracle's pins: a copy of the oracle with one
plausible mistake planted (a dropped weight, a wrong rounding or tie rule, an
off-by-one in a grid, a wrong bit order, ...) must fail at least one pin.
Mistakes are planted only in temporary copies of the oracle, on the CPU."""
import importlib.util
import inspect
import os
import subprocess

import pytest

import test_oracle_pins as pins

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "tq_oracle.c")

MUTANTS = {
    "imatrix_weight_dropped": ("L += (double)m[j] * (e * e);\n        if (v_out) v_out[j] = (int8_t)v;",
                               "L += (e * e);\n        if (v_out) v_out[j] = (int8_t)v;"),
    "round_half_away": ("double q = nearbyint((double)y); /* current rounding mode", "double q = round((double)y); /* current rounding mode"),
    "stage2_narrow": ("return (float)((center - delta) + (2.0 * delta", "return (float)((center - 0.5 * delta) + (1.0 * delta"),
    "int3_offset": ("int u = (j < I ? v[r * I + j] : 0) + 4;", "int u = (j < I ? v[r * I + j] : 0) + 3;"),
    "int3_high_bit_order": ("rec[16 + i / 8] |= (uint8_t)(((u >> 2) & 1) << (i % 8));", "rec[16 + i / 8] |= (uint8_t)(((u >> 2) & 1) << (7 - i % 8));"),
    "zero_grid_16": ("return (int)nearbyint((15.0 * (double)i) / (double)(nz - 1));", "return (int)nearbyint((16.0 * (double)i) / (double)(nz - 1));"),
    "asym_clamp_14": ("if (q > 15.0) q = 15.0;\n        }\n        double e = (double)w[j] - (double)s * (q - (double)z);",
                      "if (q > 14.0) q = 14.0;\n        }\n        double e = (double)w[j] - (double)s * (q - (double)z);"),
    "no_sign_flip": ("return negative ? -a : a;", "return a;"),
    "window_ties_high": ("if (d < bd) { bd = d; best = c; }   /* strict: ties keep the lower code */",
                         "if (d <= bd) { bd = d; best = c; }   /* strict: ties keep the lower code */"),
    "e2m1_ties_odd": ("if (d < best_d || (d == best_d && (i % 2) == 0))", "if (d < best_d || (d == best_d && (i % 2) == 1))"),
    "imatrix_bessel": ("m[j] = T > 0 ? s / (double)T : 0.0;", "m[j] = T > 1 ? s / (double)(T - 1) : 0.0;"),
    "proxy_den_error": ("b += (double)m[j] * (w * w);", "b += (double)m[j] * (e * e) + (double)m[j] * (w * w) * 0.0 + (double)m[j] * (w * w);"),
    "argmin_last_tie": ("if (L < bestL) { bestL = L; best = 2 * k + sg; bestS = s; }", "if (L <= bestL) { bestL = L; best = 2 * k + sg; bestS = s; }"),
    "nvfp4_global_448": ("return (float)((double)amax / 2688.0);", "return (float)((double)amax / 448.0);"),
    "hessian_transposed_operand": ("for (int64_t t = 0; t < T; ++t) s += (double)X[t * ld + i] * (double)X[t * ld + j];\n            H[i * I + j] = s;",
                                   "for (int64_t t = 0; t < T; ++t) s += (double)X[t * ld + i] * (double)X[j * ld + (t % I)];\n            H[i * I + j] = s;"),
    "hessian_last_token_dropped": ("for (int64_t t = 0; t < T; ++t) s += (double)X[t * ld + i] * (double)X[t * ld + j];\n            H[i * I + j] = s;",
                                   "for (int64_t t = 0; t + 1 < T; ++t) s += (double)X[t * ld + i] * (double)X[t * ld + j];\n            H[i * I + j] = s;"),
    "proxy_full_diagonal_only": ("hn += H[i * I + j] * ((double)w[j] - (double)wh[j]);",
                                 "hn += (i == j) * H[i * I + j] * ((double)w[j] - (double)wh[j]);"),
    "e4m3_ties_away": ("v = nearbyint(a / step) * step;                       /* a / step is exact */",
                       "v = round(a / step) * step;                       /* a / step is exact */"),
    "e4m3_subnormal_step": ("double step = a < ldexp(1.0, -6) ? ldexp(1.0, -9) : ldexp(1.0, ilogb(a) - 3);",
                            "double step = a < ldexp(1.0, -7) ? ldexp(1.0, -9) : ldexp(1.0, ilogb(a) - 3);"),
    "fp8_scale_240": ("return (float)((double)r * (double)amax / 448.0);", "return (float)((double)r * (double)amax / 240.0);"),
    "fp8_loss_unweighted": ("L += (double)me[j] * (d * d);", "L += (d * d);"),
    "lloyd_ties_up": ("if (u > ((double)c[i] + (double)c[i + 1]) / 2.0) a = i + 1;", "if (u >= ((double)c[i] + (double)c[i + 1]) / 2.0) a = i + 1;"),
    "lloyd_scale_not_squared": ("double om = (double)m[e * m_stride + j] * (double)s * (double)s;", "double om = (double)m[e * m_stride + j] * (double)s;"),
    "gptq_update_sign": ("for (int64_t j = i + 1; j < I; ++j) w[j] = fmaf(-e, U[i * ldu + j], w[j]);",
                         "for (int64_t j = i + 1; j < I; ++j) w[j] = fmaf(e, U[i * ldu + j], w[j]);"),
    "gptq_transposed_factor": ("for (int64_t j = i + 1; j < I; ++j) w[j] = fmaf(-e, U[i * ldu + j], w[j]);",
                               "for (int64_t j = i + 1; j < I; ++j) w[j] = fmaf(-e, U[j * ldu + i], w[j]);"),
    "gptq_no_diagonal_division": ("const float e = (w[i] - what) / U[i * ldu + i];", "const float e = (w[i] - what);"),
    "gptq_skips_next_column": ("for (int64_t j = i + 1; j < I; ++j) w[j] = fmaf(-e, U[i * ldu + j], w[j]);",
                               "for (int64_t j = i + 2; j < I; ++j) w[j] = fmaf(-e, U[i * ldu + j], w[j]);"),
    "act_block_amax_first_element": ("float a = fabsf(X[r * I + j]);\n                if (a > b) b = a;",
                                     "float a = fabsf(X[r * I + j]);\n                if (j == 16 * k) b = a;"),
    "w4a4_drops_activation_global": ("y[b * O + o] = (double)gw * (double)gx * acc;", "y[b * O + o] = (double)gw * acc;"),
    "w4a4_first_block_scale": ("acc += orc_e4m3_decode(ew[o * G + k]) * orc_e4m3_decode(ex[b * G + k]) * p;",
                               "acc += orc_e4m3_decode(ew[o * G + k]) * orc_e4m3_decode(ex[b * G]) * p;"),
    "proxy_full_den_uses_error": ("hd += H[i * I + j] * (double)w[j];",
                                  "hd += H[i * I + j] * ((double)w[j] - (double)wh[j]);"),
    "proxy_full_drops_last_column": ("for (int64_t j = 0; j < I; ++j) {\n                hn += H[i * I + j]",
                                     "for (int64_t j = 0; j + 1 < I; ++j) {\n                hn += H[i * I + j]"),
    "dequant_int4_no_zero": ("out[r * I + j] = (float)((double)scales[gi] * ((double)q[r * I + j] - (double)zeros[gi]));",
                             "out[r * I + j] = (float)((double)scales[gi] * ((double)q[r * I + j]));"),
}


def _mutant_module(tmp_path, name, a, b):
    src = open(SRC).read()
    assert a in src, f"mutation site of {name} not found"
    d = tmp_path / name
    d.mkdir()
    (d / "tq_oracle.c").write_text(src.replace(a, b, 1))
    so = d / "liboracle.so"
    subprocess.run(["gcc", "-O1", "-std=c11", "-fPIC", "-shared", "-fopenmp", "-ffp-contract=off", "-o", str(so),
                    str(d / "tq_oracle.c"), "-lm"], check=True)
    spec = importlib.util.spec_from_file_location(f"oracle_mut_{name}", os.path.join(ROOT, "oracle", "__init__.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    mod._LIB_PATH = str(so)
    mod.build = lambda force=False: str(so)
    return mod


def _pin_calls():
    """Every pin of test_oracle_pins, with its parametrisations, as callables of orc."""
    calls = []
    for name, fn in inspect.getmembers(pins, inspect.isfunction):
        if not name.startswith("test_"):
            continue
        marks = getattr(fn, "pytestmark", [])
        params = [m for m in marks if m.name == "parametrize"]
        if not params:
            calls.append((name, lambda orc, fn=fn: fn(orc)))
            continue
        argnames, values = params[0].args
        argnames = [s.strip() for s in argnames.split(",")] if isinstance(argnames, str) else list(argnames)
        for v in values:
            v = v if isinstance(v, (tuple, list)) and len(argnames) > 1 else (v,)
            calls.append((f"{name}{v}", lambda orc, fn=fn, v=v: fn(orc, *v)))
    return calls


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_every_planted_mistake_fails_a_pin(tmp_path, name):
    a, b = MUTANTS[name]
    orc = _mutant_module(tmp_path, name, a, b)
    caught = []
    for pin, call in _pin_calls():
        try:
            call(orc)
        except (AssertionError, ValueError, IndexError):
            caught.append(pin)
            break
    assert caught, f"no pin catches the planted mistake {name}"
