"""Pin strength: plausible mistakes planted in copies of the oracle each fail a pin.

The mistakes are planted on the CPU, in temporary copies of the oracle's C
source; the real oracle and the CUDA library are never touched.  Every mutation
keeps all memory accesses in bounds.
"""
import os

import pytest

import oracle
from oracle_pins import ALL_PINS

SRC = os.path.join(os.path.dirname(oracle.__file__), "spear_oracle.c")

MUTATIONS = {
    "nibble_order_swapped": ("out[2 * b] = ((double)(v & 0xF) - z) * s;",
                             "out[2 * b] = ((double)(v >> 4) - z) * s;"),
    "dequant_zero_sign": ("out[2 * b + 1] = ((double)(v >> 4) - z) * s;",
                          "out[2 * b + 1] = ((double)(v >> 4) + z) * s;"),
    "gate_dropped": ("acc += g[m] * e;", "acc += e;"),
    "gate_sign": ("return 1.0 / (1.0 + exp(-p));", "return 1.0 / (1.0 + exp(p));"),
    "gate_bias_dropped": ("acc += (double)b_g;", "acc += 0.0;"),
    "B_transposed": ("e += t[m * r + j] * oracle_bf16_to_f64(B[(int64_t)j * N + n]);",
                     "e += t[m * r + j] * oracle_bf16_to_f64(B[(int64_t)n * r + j]);"),
    "A_transposed": ("oracle_bf16_to_f64(A[k * r + j]);", "oracle_bf16_to_f64(A[j * K + k]);"),
    "truncate_not_round": ("float r = rintf(w[k] / s);", "float r = truncf(w[k] / s);"),
    "range_excludes_zero": ("float lo = 0.0f, hi = 0.0f;", "float lo = w[0], hi = w[0];"),
    "levels_16": ("float s32 = range / 15.0f;\n    uint16_t sb", "float s32 = range / 16.0f;\n    uint16_t sb"),
    "zero_point_sign": ("rintf(negl / s)", "rintf(lo / s)"),
    "f16_ties_away": ("if (rem > half || (rem == half && (kept & 1u))) q += 1;",
                      "if (rem >= half) q += 1;"),
    "mlp_relu_dropped": ("h[i] = pre > 0.0 ? pre : 0.0;", "h[i] = pre;"),
    "mlp_alpha_inside_sigmoid": ("u[m * r + j] = (double)alpha * (1.0 / (1.0 + exp(-pre))) * tm[j];",
                                 "u[m * r + j] = (1.0 / (1.0 + exp(-(double)alpha * pre))) * tm[j];"),
    "mlp_W1_transposed": ("(double)W1[(int64_t)i * r + j] * tm[j]", "(double)W1[(int64_t)j * H + i] * tm[j]"),
    "mlp_W2_transposed": ("(double)W2[(int64_t)j * H + i] * h[i]", "(double)W2[(int64_t)i * r + j] * h[i]"),
    "grouped_index_modulo": ("int64_t grp = k / G;", "int64_t grp = k % ng;"),
    "grouped_zero_of_first_group": ("(q - oracle_f16_to_f64(z_bits[n * ng + grp]))", "(q - oracle_f16_to_f64(z_bits[n * ng]))"),
    "grouped_scale_of_next_row": ("* oracle_f16_to_f64(s_bits[n * ng + grp]);", "* oracle_f16_to_f64(s_bits[((n + 1) % N) * ng + grp]);"),
    "main_term_dropped_last_k": ("for (int64_t k = 0; k < K; ++k) acc += xr[k] * wrow[k];",
                                 "for (int64_t k = 0; k < K - 1; ++k) acc += xr[k] * wrow[k];"),
}


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_mutant_fails_a_pin(name, tmp_path):
    old, new = MUTATIONS[name]
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation anchor for {name} not unique/present"
    mpath = tmp_path / f"mut_{name}.c"
    mpath.write_text(src.replace(old, new))
    lib = oracle.build(force=True, src=str(mpath), out=str(tmp_path / f"lib_{name}.so"))
    mut = oracle.Oracle(lib)
    failed = []
    for pin in ALL_PINS:
        try:
            pin(mut)
        except AssertionError:
            failed.append(pin.__name__)
    assert failed, f"mutation {name} passed every pin"
