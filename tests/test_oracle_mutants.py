"""The oracle's pins catch plausible mistakes.

Each case plants one mistake in a copy of the oracle's C source (on the CPU,
in a temporary directory), builds it, swaps it in for the real oracle, and
checks that at least one pin in test_oracle_pins.py or test_oracle_ex2.py
fails.  The real oracle is
restored afterwards.
"""
import ctypes
import os
import subprocess
import tempfile

import numpy as np
import pytest

import oracle
from tests import test_oracle_ex2 as ex2
from tests import test_oracle_gptq as gptq
from tests import test_oracle_pins as pins
from tests import test_oracle_presets as presets

SRC = os.path.join(os.path.dirname(oracle.__file__), "rqo.c")

MUTANTS = {
    # rounding half away from zero instead of half to even
    "round_half_away": ("float r = rintf(t);", "float r = roundf(t);"),
    # codes against the fp32 scale instead of the stored fp16 scale
    "divide_by_s32": ("volatile float t = w[i] / sf;", "volatile float t = w[i] / s32;"),
    # even k in the high nibble
    "nibble_order": ("if (k % 2 == 0) *b = (uint8_t)((*b & 0xF0u) | nib);",
                     "if (k % 2 == 1) *b = (uint8_t)((*b & 0xF0u) | nib);"),
    # fp16 conversion truncates instead of rounding to nearest
    "fp16_truncate": ("if (rem > half || (rem == half && (q & 1u))) q += 1u;", ";"),
    # fp16 ties away from zero
    "fp16_ties_away": ("if (rem > half || (rem == half && (q & 1u))) q += 1u;",
                       "if (rem >= half) q += 1u;"),
    # amax taken over signed values
    "amax_signed": ("float a = fabsf(w[i]);", "float a = w[i];"),
    # wrong group index for the scale in products
    "scale_index": ("scales[n * (K / RQO_GROUP) + k / RQO_GROUP]",
                    "scales[n * (K / RQO_GROUP) + (k / RQO_GROUP + 1) % (K / RQO_GROUP)]"),
    # transposed x index in products
    "x_transposed": ("double xv = rqo_f16_to_f64(x[m * K + k]);",
                     "double xv = rqo_f16_to_f64(x[k * (K > 0 ? 1 : 0) + m * 0 + (k % K)]);"),
    # qmax of int8 taken as 128
    "qmax_int8": ("return bits == 4 ? 7 : 127;", "return bits == 4 ? 7 : 128;"),
    # scale from amax / (qmax + 1)
    "qmax_plus_one": ("volatile float s32 = amax / (float)qmax;",
                      "volatile float s32 = amax / (float)(qmax + 1);"),
    # E[x^2] search: a tie goes to the later candidate
    "ex2_ties_last": ("if (best < 0 || err < best_err) {", "if (best < 0 || err <= best_err) {"),
    # E[x^2] search: the error is not weighted by E[x^2]
    "ex2_unweighted": ("volatile float pr = e2[i] * q;", "volatile float pr = q;"),
    # E[x^2] search: the candidate factor is ignored
    "ex2_no_factor": ("volatile float a32 = amax * f[j];", "volatile float a32 = amax;"),
    # E[x^2] search: absolute instead of squared error
    "ex2_abs_error": ("volatile float q = d * d;", "volatile float q = fabsf(d);"),
    # E[x^2] search: every group weighted by the first group's channels
    "ex2_channel_index": ("&e2[g * RQO_GROUP]", "&e2[0]"),
    # GPTQ: the rounding error is not spread (RTN)
    "gptq_no_spread": ("w[k] = fmaf(-e, U[j * K + k], w[k]);", "w[k] = w[k];"),
    # GPTQ: the error spread along a column of U instead of its row
    "gptq_u_transposed": ("w[k] = fmaf(-e, U[j * K + k], w[k]);", "w[k] = fmaf(-e, U[k * K + j], w[k]);"),
    # GPTQ: the error is not divided by the diagonal of U
    "gptq_no_diag_divide": ("volatile float ev = d / U[j * K + j];", "volatile float ev = d;"),
    # GPTQ: the error spread with the wrong sign
    "gptq_sign": ("w[k] = fmaf(-e, U[j * K + k], w[k]);", "w[k] = fmaf(e, U[j * K + k], w[k]);"),
    # presets, asymmetric: the group range not widened to include 0
    "p4a_range_unclamped": ("    float lo = 0.0f, hi = 0.0f;\n    for (i = 0; i < 32; i++) {",
                            "    float lo = w[0], hi = w[0];\n    for (i = 0; i < 32; i++) {"),
    # presets, asymmetric: sub-codes truncated instead of rounded
    "p4a_subcode_floor": ("                    a = rint_clamp(t, 0, 63);",
                          "                    a = rint_clamp(floorf(t), 0, 63);"),
    # presets, asymmetric: the offset's sign lost
    "p4a_offset_sign": ("                volatile float O = -(dmf * (float)b);",
                        "                volatile float O = (dmf * (float)b);"),
    # presets, asymmetric: the offset super-scale over 64 steps
    "p4a_dm_steps": ("            volatile float dm32 = omax / 63.0f;", "            volatile float dm32 = omax / 64.0f;"),
    # presets, symmetric: every group searched with the first group's E[x^2]
    "sym_e2_index": ("e2 ? &e2[g * G] : 0", "e2 ? &e2[0] : 0"),
    # GPTQ: every group keeps the first group's scale
    "gptq_scale_once": ("if (j % RQO_GROUP == 0) {\n            /* the group's scale", "if (j == 0) {\n            /* the group's scale"),
}

PIN_TESTS = [
    lambda: pins.test_hand_examples(4),
    lambda: pins.test_hand_examples(8),
    pins.test_hand_int4_exact_reconstruction_row,
    pins.test_fp16_conversion_edges,
    lambda: pins.test_quantizer_matches_numpy_restatement(4, (37, 192), 0.02),
    lambda: pins.test_quantizer_matches_numpy_restatement(8, (5, 768), 1.0),
    lambda: pins.test_quantizer_invariants(8),
    lambda: pins.test_exact_reconstruction_on_grid(8),
    lambda: pins.test_products_match_numpy_fp64(4),
    pins.test_unit_vector_picks_column,
    ex2.test_hand_worked_group,
    lambda: ex2.test_zero_weights_tie_first_wins(4),
    lambda: ex2.test_single_factor_one_is_rtn(4),
    lambda: ex2.test_matches_numpy_restatement(4, (3, 192)),
    lambda: ex2.test_matches_numpy_restatement(8, (2, 256)),
    lambda: gptq.test_diagonal_hessian_is_rtn(4),
    lambda: gptq.test_matches_sequential_obs(4),
    gptq.test_hand_worked_rows,
    lambda: presets.test_sym_g16_matches_restatement(True),
    lambda: presets.test_p4a_matches_restatement(False),
    lambda: presets.test_p4a_matches_restatement(True),
    presets.test_p4a_hand_built_superblock_reproduced,
    lambda: presets.test_preset_products_match_numpy(4),
    lambda: gptq.test_layer_error_below_rtn(8),
]


def _build_mutant(name, old, new, tmp):
    src = open(SRC).read()
    assert old in src, f"mutation site for {name} not found"
    path_c = os.path.join(tmp, f"{name}.c")
    with open(path_c, "w") as f:
        f.write(src.replace(old, new))
    path_so = os.path.join(tmp, f"{name}.so")
    subprocess.run(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp",
                    "-ffp-contract=off", path_c, "-o", path_so, "-lm"], check=True)
    return path_so


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_mutant(name):
    real = oracle._load()
    old, new = MUTANTS[name]
    with tempfile.TemporaryDirectory() as tmp:
        so = _build_mutant(name, old, new, tmp)
        lib = ctypes.CDLL(so)
        for fn in ("rqo_f32_to_f16", "rqo_f16_to_f64", "rqo_quantize_g64", "rqo_quantize_g64_ex2",
                   "rqo_matmul", "rqo_matmul_sampled", "rqo_get_code", "rqo_gptq_g64",
                   "rqo_quantize_sym", "rqo_quantize_p4a", "rqo_get_ucode4", "rqo_matmul_fmt"):
            getattr(lib, fn).argtypes = getattr(real, fn).argtypes
            getattr(lib, fn).restype = getattr(real, fn).restype
        caught = False
        oracle._lib = lib
        try:
            for t in PIN_TESTS:
                try:
                    with np.errstate(all="ignore"):
                        t()
                except AssertionError:
                    caught = True
                    break
        finally:
            oracle._lib = real
    assert caught, f"no pin fails for mutant {name}"
