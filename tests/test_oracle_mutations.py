"""Planted mistakes: each mutation below is a plausible bug in the oracle's arithmetic,
applied to a temporary copy of its C source and built on the CPU. The pins of
``test_oracle_pins.py`` are then run against the mutant; at least one must fail. This
shows the pins constrain every part of the oracle (hash, resolution, axis pairing,
weights, corner count, accumulation), not just the parts they were written for.
"""
import ctypes
import os
import shutil
import subprocess

import pytest

import oracle
import tests.test_oracle_pins as pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "hashgrid_oracle.c")

MUTATIONS = {
    # x fraction paired with the z offset, as in the pages' own snippets
    "axis_swap": ("w *= d ? frac[i] : 1.0 - frac[i];", "w *= d ? frac[2 - i] : 1.0 - frac[2 - i];"),
    "weight_sign": ("w *= d ? frac[i] : 1.0 - frac[i];", "w *= d ? 1.0 - frac[i] : frac[i];"),
    "dropped_corner": ("double w = corner(v, frac, c, vc);\n                uint32_t h = oracle_hash3(vc[0], vc[1], vc[2]) & mask;\n                for (int f = 0; f < F; ++f)\n                    acc[f]",
                       "double w = (c == 7) ? 0.0 : corner(v, frac, c, vc);\n                uint32_t h = oracle_hash3(vc[0], vc[1], vc[2]) & mask;\n                for (int f = 0; f < F; ++f)\n                    acc[f]"),
    "wrong_prime": ("#define ORACLE_PRIME_Z 805459861u", "#define ORACLE_PRIME_Z 805459867u"),
    "scale_by_N_minus_1": ("float xs = xp[i] * (float)res_l;", "float xs = xp[i] * (float)(res_l - 1);"),
    "literal_double_floor": ("if (fabs(v - r) <= 1e-9 * v)", "if (0)"),
    "overwrite_not_add": ("dtable[((size_t)l * T + h) * F + f] +=", "dtable[((size_t)l * T + h) * F + f] ="),
    "dx_weight_sign": ("double dw = (double)res[l] * (((c >> i) & 1) ? 1.0 : -1.0);",
                       "double dw = (double)res[l] * (((c >> i) & 1) ? -1.0 : 1.0);"),
    "dx_missing_resolution": ("double dw = (double)res[l] * (((c >> i) & 1) ? 1.0 : -1.0);",
                              "double dw = 1.0 * (((c >> i) & 1) ? 1.0 : -1.0);"),
    "adam_no_bias_correction": ("double mhat = m[i] / c1;", "double mhat = m[i];"),
    "adam_not_sparse": ("        if (g == 0.0)\n            continue;\n        m[i]", "        m[i]"),
    "nd_fourth_prime": ("2654435761u, 805459861u, 3674653429u,", "2654435761u, 805459861u, 3674653427u,"),
    "int64_hash_low_bits_lost": ("return (u0 * ORACLE_PRIME_X) ^ (u1 * ORACLE_PRIME_Y) ^ (u2 * ORACLE_PRIME_Z);",
                                 "return ((u0 * ORACLE_PRIME_X) ^ (u1 * ORACLE_PRIME_Y) ^ (u2 * ORACLE_PRIME_Z)) & 0x7fffffffu;"),
    # the MLP and its bf16 weights
    "mlp_missing_relu": ("            a1[o] = s > 0.0 ? s : 0.0;", "            a1[o] = s;"),
    "mlp_bias_dropped": ("            double s = (double)b2[o];", "            double s = 0.0;"),
    "mlp_w1_transposed": ("oracle_bf16_to_double(w1[o * in + k])", "oracle_bf16_to_double(w1[k * hid + o])"),
    "bf16_half_ulp": ("uint32_t u = (uint32_t)b << 16;", "uint32_t u = ((uint32_t)b << 16) | 0x8000u;"),
    "mlp_second_relu_dropped": ("            a2[o] = s > 0.0 ? s : 0.0;", "            a2[o] = s;"),
    "mlp_w2_transposed": ("oracle_bf16_to_double(w2[o * hid + k])", "oracle_bf16_to_double(w2[k * hid + o])"),
    "mlp_w3_row_shift": ("oracle_bf16_to_double(w3[o * hid + k])", "oracle_bf16_to_double(w3[((o + 1) % nout) * hid + k])"),
    # D-dimensional inputs (strings that occur only in the N-d functions)
    "nd_weight_axis_swap": ("int64_t *vc)\n{\n    double w = 1.0;\n    for (int i = 0; i < D; ++i) {\n        int d = (c >> i) & 1;\n"
                            "        vc[i] = v[i] + d;\n        w *= d ? frac[i] : 1.0 - frac[i];",
                            "int64_t *vc)\n{\n    double w = 1.0;\n    for (int i = 0; i < D; ++i) {\n        int d = (c >> i) & 1;\n"
                            "        vc[i] = v[i] + d;\n        w *= d ? frac[D - 1 - i] : 1.0 - frac[D - 1 - i];"),
    # the index export laid out [point][corner][level] (a wrong stride; same size, in bounds)
    "nd_index_stride": ("idx[((size_t)p * L + l) * nc + c] = oracle_hash_nd(D, vc) & mask;",
                        "idx[((size_t)p * nc + c) * L + l] = oracle_hash_nd(D, vc) & mask;"),
    "nd_scale_by_N_minus_1": ("double *frac)\n{\n    for (int i = 0; i < D; ++i) {\n        float xs = xp[i] * (float)res_l;",
                              "double *frac)\n{\n    for (int i = 0; i < D; ++i) {\n        float xs = xp[i] * (float)(res_l - 1);"),
}

def _pin_calls():
    """Every pin as (name, function, kwargs), parametrized pins expanded."""
    calls = []
    for name in dir(pins):
        if not name.startswith("test_"):
            continue
        fn = getattr(pins, name)
        marks = [m for m in getattr(fn, "pytestmark", []) if m.name == "parametrize"]
        if not marks:
            calls.append((name, fn, {}))
            continue
        argname, values = marks[0].args[0], marks[0].args[1]
        for v in values:
            calls.append((name, fn, {argname: v}))
    return calls


PIN_TESTS = _pin_calls()


def build_mutant(tmp_path, name):
    src = open(SRC).read()
    old, new = MUTATIONS[name]
    assert src.count(old) >= 1, f"mutation {name} does not apply"
    path = tmp_path / f"{name}.c"
    path.write_text(src.replace(old, new, 1))   # first occurrence: the 3-D function
    lib = tmp_path / f"lib_{name}.so"
    subprocess.run(["gcc", "-std=c11", "-O2", "-ffp-contract=off", "-fopenmp", "-fPIC", "-shared",
                    "-o", str(lib), str(path), "-lm"], check=True)
    return str(lib)


@pytest.mark.skipif(shutil.which("gcc") is None, reason="gcc missing")
@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_pins_catch_mutation(tmp_path, name, monkeypatch):
    path = build_mutant(tmp_path, name)
    good = oracle._lib()                      # typed prototypes of the real library
    mut = ctypes.CDLL(path)
    for fn in ("oracle_resolutions", "oracle_hash3", "oracle_half_to_double", "oracle_indices",
               "oracle_forward", "oracle_backward", "oracle_backward_x", "oracle_adam_step",
               "oracle_hash_nd", "oracle_indices_nd", "oracle_forward_nd", "oracle_backward_nd", "oracle_backward_x_nd",
               "oracle_bf16_to_double", "oracle_mlp_forward"):
        getattr(mut, fn).argtypes = getattr(good, fn).argtypes
        getattr(mut, fn).restype = getattr(good, fn).restype
    monkeypatch.setattr(oracle, "_LIB", mut)
    failed = []
    for name, fn, kwargs in PIN_TESTS:
        try:
            fn(**kwargs)
        except (AssertionError, ValueError):
            failed.append(name)
    assert failed, f"mutation {name} passed every pin"
