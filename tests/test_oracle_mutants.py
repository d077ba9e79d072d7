"""The pins catch plausible mistakes in the oracle (no GPU).

Each case plants one mistake in a private copy of ``oracle/oracle.c``,
compiles it, and requires that at least one pin fails on the broken copy.
The real oracle source is never modified.
"""
import os
import shutil
import tempfile

import pytest

import oracle as oracle_pkg
from oracle import build as oracle_build

import pins

SRC = os.path.join(os.path.dirname(oracle_pkg.__file__), "oracle.c")

# (name, text in the oracle, replacement) -- each a mistake a reader might make
MUTANTS = [
    ("sign_of_zero_is_plus", "return v > 0.0 ? 1 : -1;", "return v >= 0.0 ? 1 : -1;"),
    ("msb_first_bits", "(k % 32)", "(31 - k % 32)"),
    ("row_stride_floor", "return (K + 31) / 32;", "return K / 32 > 0 ? K / 32 : 1;"),
    ("fbi_alpha_signed_mean", "abs_sum += fabs(w);", "abs_sum += w;"),
    ("fbi_alpha_divides_by_n", "alpha[j] = (float)(abs_sum / (double)K);",
     "alpha[j] = (float)(abs_sum / (double)N);"),
    ("bitnet_no_shift", "sign_pm1((double)W[j * K + k] - alpha)", "sign_pm1((double)W[j * K + k])"),
    ("bitnet_beta_from_signed_sum", "*beta_out = abs_sum / count;", "*beta_out = sum / count;"),
    ("bitnet_alpha_per_row_count", "double alpha = sum / count;", "double alpha = sum / (double)K;"),
    ("dropped_last_term", "for (int64_t k = 0; k < K; ++k)\n        dot +=",
     "for (int64_t k = 0; k < K - 1; ++k)\n        dot +="),
    ("alpha_indexed_by_token", "return (double)alpha[j] * dot;", "return (double)alpha[m] * dot;"),
    ("sample_index_swapped", "y[i] = w1a16_one(x, packed, alpha, K, ms[i], js[i]);",
     "y[i] = w1a16_one(x, packed, alpha, K, js[i] % 1, js[i]);"),
    ("variance_unbiased", "double var = sq / (double)K;", "double var = sq / (double)(K - 1);"),
    ("eps_outside_sqrt", "double root = sqrt(var + eps);", "double root = sqrt(var) + eps;"),
    ("no_mean_subtraction",
     "double ln = (bf16_value(row[k]) - mu) / root;\n            if (fabs(ln) > gamma)",
     "double ln = bf16_value(row[k]) / root;\n            if (fabs(ln) > gamma)"),
    ("round_half_away", "double r = nearbyint(v);", "double r = round(v);"),
    ("truncate_not_round", "double r = nearbyint(v);", "double r = trunc(v);"),
    ("no_clamp", "if (r > 127.0) r = 127.0;", ""),
    ("clamp_to_128", "if (r < -127.0) r = -127.0;", "if (r < -128.0) r = -128.0;"),
    ("qb_127", "const double Qb = 128.0;\n    for (int64_t m = 0; m < M; ++m) {\n        const uint16_t",
     "const double Qb = 127.0;\n    for (int64_t m = 0; m < M; ++m) {\n        const uint16_t"),
    ("rescale_without_qb", "* beta * gamma[m] / Qb;", "* beta * gamma[m];"),
    ("rescale_without_gamma", "* beta * gamma[m] / Qb;", "* beta / Qb;"),
    ("acc_sign_ignored", "acc += (int64_t)packed_sign(packed, K, j, k) * (int64_t)xq[m * K + k];",
     "acc += (int64_t)xq[m * K + k];"),
    ("w1a1_and_not_xnor", "s += (int64_t)packed_sign(a, K, m, k) * (int64_t)packed_sign(b, K, j, k);",
     "s += (packed_sign(a, K, m, k) == 1 && packed_sign(b, K, j, k) == 1) ? 1 : -1;"),
    ("bf16_decode_wrong_half", "uint32_t u = (uint32_t)h << 16;", "uint32_t u = (uint32_t)h << 15;"),
    # per-tensor Eq.(5) and non-negative Eq.(6) quantisers
    ("tensor_gamma_per_token", "            if (fabs(ln[i]) > gamma) gamma = fabs(ln[i]);",
     "            if (fabs(ln[i]) > gamma && i < K) gamma = fabs(ln[i]);"),
    ("nonneg_no_eta_shift", "v = (mode == 1 ? ln[i] - eta : ln[i]) * Qb / gamma;", "v = ln[i] * Qb / gamma;"),
    ("nonneg_gamma_absmax", "            if (ln[i] - eta > gamma) gamma = ln[i] - eta;",
     "            if (fabs(ln[i]) > gamma) gamma = fabs(ln[i]);"),
    # (a symmetric lower clamp is not observable in mode 1: LN - eta >= 0)
    ("nonneg_eta_first_token", "            if (ln[i] < eta) eta = ln[i];",
     "            if (ln[i] < eta && i < K) eta = ln[i];"),
    # b1.58 ternary weights
    ("ternary_round_half_away", "double r = nearbyint((double)W[j * K + k] / (gamma + eps));",
     "double r = round((double)W[j * K + k] / (gamma + eps));"),
    # (dropping the clip altogether is not observable: a +-2 sets the same plane
    # bit as +-1, so the two-plane layout itself clips)
    ("ternary_clip_low_to_zero", "if (r < -1.0) r = -1.0;\n            if (r == 0.0) continue;",
     "if (r < -1.0) r = 0.0;\n            if (r == 0.0) continue;"),
    ("ternary_gamma_signed_mean", "for (int64_t k = 0; k < K; ++k) abs_sum += fabs((double)W[j * K + k]);",
     "for (int64_t k = 0; k < K; ++k) abs_sum += (double)W[j * K + k];"),
    ("ternary_eps_ignored", "/ (gamma + eps));", "/ gamma);"),
    ("ternary_planes_swapped", "blk[(r > 0.0 ? 0 : 4) + o / 32]", "blk[(r > 0.0 ? 4 : 0) + o / 32]"),
    ("ternary_block_stride", "(k / 128) * 8;\n    int64_t o = k % 128;\n    uint32_t plus",
     "(k / 128) * 4;\n    int64_t o = k % 128;\n    uint32_t plus"),
    ("ternary_acc_sign_ignored",
     "acc += (int64_t)ternary_value(packed, K, j, k) * (int64_t)xq[m * K + k];",
     "acc += (int64_t)(ternary_value(packed, K, j, k) != 0) * (int64_t)xq[m * K + k];"),
    ("ternary_sample_index_swapped", "acc[i] = w158a8_acc_one(xq, packed, K, ms[i], js[i]);",
     "acc[i] = w158a8_acc_one(xq, packed, K, js[i] % 5, ms[i]);"),
    # straight-through backward
    ("backward_dx_without_alpha", "s += bf16_value(dy[m * N + j]) * (double)alpha[j] * (double)packed_sign(packed, K, j, k);",
     "s += bf16_value(dy[m * N + j]) * (double)packed_sign(packed, K, j, k);"),
    ("backward_dx_sign_dropped", "s += bf16_value(dy[m * N + j]) * (double)alpha[j] * (double)packed_sign(packed, K, j, k);",
     "s += bf16_value(dy[m * N + j]) * (double)alpha[j];"),
    ("backward_dw_without_alpha", "dw[j * K + k] = (double)alpha[j] * s;", "dw[j * K + k] = s;"),
    ("backward_dw_gated_by_sign", "dw[j * K + k] = (double)alpha[j] * s;",
     "dw[j * K + k] = (double)alpha[j] * s * (packed_sign(packed, K, j, k) > 0 ? 1.0 : 0.0);"),
    ("backward_dw_token_row_swapped", "s += bf16_value(dy[m * N + j]) * bf16_value(x[m * K + k]);",
     "s += bf16_value(dy[m * N + j]) * bf16_value(x[(M - 1 - m) * K + k]);"),
    ("backward_dalpha_scaled", "        dalpha[j] = s;", "        dalpha[j] = (double)alpha[j] * s;"),
    ("backward_dalpha_last_input_dropped",
     "            for (int64_t k = 0; k < K; ++k)\n                z +=",
     "            for (int64_t k = 0; k < K - 1; ++k)\n                z +="),
]


@pytest.fixture(scope="module")
def workdir():
    d = tempfile.mkdtemp(prefix="oracle_mutants_")
    yield d
    shutil.rmtree(d, ignore_errors=True)


def test_real_oracle_passes_every_pin(oracle):
    assert pins.run_pins(oracle) == []


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_pins_catch_planted_mistake(workdir, name, old, new):
    text = open(SRC).read()
    assert text.count(old) >= 1, f"pattern for {name} not found in oracle.c"
    src = os.path.join(workdir, f"{name}.c")
    with open(src, "w") as f:
        f.write(text.replace(old, new))
    lib = oracle_build.build(src, os.path.join(workdir, f"{name}.so"), strict=False)
    failures = pins.run_pins(oracle_pkg.Oracle(lib))
    assert failures, f"no pin caught the planted mistake {name}"
