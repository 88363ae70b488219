"""Planted mistakes: every plausible slip in the oracle must fail a pin.

Each case copies ``oracle/gq_oracle.c``, plants one mistake (a dropped term, a
wrong rounding rule, a wrong index or bit order, a transposed operand...),
compiles the copy on the CPU and runs the pin checks of
``test_oracle_pins.py`` against it.  The mutant passes this test only if at
least one pin rejects it.  Nothing here touches a GPU.
"""
from __future__ import annotations

import os
import subprocess
import tempfile

import pytest

import oracle
from oracle import build as obuild
from tests import test_oracle_pins as pins

MUTANTS = {
    "round_half_away": ("float r = nearbyintf(t);", "float r = roundf(t);"),
    "select_wrong_end": ("return scratch[k - 1];", "return scratch[n - k];"),
    "pack_bit_order": ("v |= u << (6 * j);", "v |= u << (6 * (3 - j));"),
    "pack_5bit_field": ("u = (uint32_t)q[col] & 0x3Fu;", "u = (uint32_t)q[col] & 0x1Fu;"),
    "unpack_no_sign_ext": ("q[col] = (int8_t)(u >= 32 ? u - 64 : u);", "q[col] = (int8_t)u;"),
    "drop_clip": ("if (wc > c) wc = c;", ""),
    "scale_off_by_one": ("float s32 = c / (float)qmax;", "float s32 = c / (float)(qmax + 1);"),
    "reciprocal_multiply": ("float t = wc / s;", "float t = wc * (1.0f / s);"),
    "transposed_divide": ("float t = wc / s;", "float t = s / wc;"),
    "k_floor": ("double up = ceil(prod);", "double up = floor(prod);"),
    "export_uses_fp32_scale": ("s = or_f16_to_f32(h);", "(void)0;"),
    "f16_ties_away": ("if (rem > 0x1000u || (rem == 0x1000u && (n & 1u)))",
                      "if (rem >= 0x1000u)"),
    "f16_subnormal_shift": ("int shift = -E - 1;", "int shift = -E - 2;"),
    "bf16_ties_away": ("if (lower > 0x8000u || (lower == 0x8000u && (upper & 1u)))",
                       "if (lower >= 0x8000u)"),
    "int6_allows_minus_32": ("if (r < (float)-qmax) r = (float)-qmax;",
                             "if (r < (float)(-qmax - 1)) r = (float)(-qmax - 1);"),
    "ste_accumulate_drops_term": ("store_elem(g_w, dtype, i, a + b);",
                                  "store_elem(g_w, dtype, i, b);"),
    "mean_weight_off_by_one": ("float t = 1.0f / (float)(count + 1);",
                               "float t = 1.0f / (float)(count + 2);"),
    "mean_first_blended": ("if (count == 0) {", "if (count < 0) {"),
    "mean_drops_average": ("a[i] = a[i] + u;", "a[i] = u;"),
    "ema_wrong_factor": ("float added = c * xi;", "float added = decay * xi;"),
    "ema_sign": ("float c = 1.0f - decay;", "float c = decay - 1.0f;"),
    "colscale_divides": ("float y = x * t[c];", "float y = x / t[c];"),
    "colscale_first_entry": ("float y = x * t[c];", "float y = x * t[0];"),
    "colscale_dense_read": ("float x = load_elem(w, dtype, r * ld + c);",
                            "float x = load_elem(w, dtype, r * cols + c);"),
    "colscale_drops_last": ("for (int64_t c = 0; c < cols; ++c) {\n            float x = load_elem(w, dtype, r * ld + c);",
                            "for (int64_t c = 0; c + 1 < cols; ++c) {\n            float x = load_elem(w, dtype, r * ld + c);"),
}

CHECKS = [   # cheapest first: a mutant stops at the first pin that rejects it
    lambda o: [pins.check_worked_example(o, n) for n in pins.WORKED],
    pins.check_k_from_p,
    lambda o: pins.check_brute_force(o, trials=120),
    lambda o: pins.check_near_ties(o, n_scales=4),
    lambda o: pins.test_ste_identity_and_accumulate(o),
    pins.check_f16,
    pins.check_bf16,
    pins.check_kthvalue,
    pins.check_torch_round,
    pins.check_invariants,
    pins.check_pack_roundtrip_exhaustive,
    pins.check_average,
    pins.check_col_scale,
]


def _build_mutant(tmpdir, old, new):
    src = open(obuild.SRC).read()
    assert src.count(old) == 1, f"mutation anchor not unique: {old!r}"
    path_c = os.path.join(tmpdir, "mutant.c")
    with open(path_c, "w") as f:
        f.write(src.replace(old, new))
    path_so = os.path.join(tmpdir, "mutant.so")
    subprocess.run(["gcc", *obuild.CFLAGS, "-w", path_c, "-o", path_so, "-lm"], check=True)
    return oracle.Oracle(path_so)


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name):
    old, new = MUTANTS[name]
    with tempfile.TemporaryDirectory() as d:
        mut = _build_mutant(d, old, new)
        caught = None
        for i, check in enumerate(CHECKS):
            try:
                check(mut)
            except (AssertionError, ValueError):
                caught = i
                break
        assert caught is not None, f"planted mistake {name!r} passed every pin"
