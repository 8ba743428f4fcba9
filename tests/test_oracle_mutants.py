"""Plants plausible mistakes in copies of the CPU oracle and checks that the pins catch
each one (no GPU).  A mutant that passes every pin would mean a hole in the pins."""
import os
import subprocess

import pytest

import oracle
import oracle_pins
from oracle import build as oracle_build

# (name, original text, mutated text): each original must occur exactly once.
# Not listed: widening the activation clip to -128.  It is an equivalent mutant: with
# s = max|x| (or the 1e-5 floor above it) |127 x / s| <= 127 always holds, so the clip
# never binds.
MUTANTS = [
    ("tie_higher_index_wins", "(mag[j] == mag[i] && j < i)", "(mag[j] == mag[i] && j > i)"),
    ("keeps_n_plus_one", "(uint8_t)(rank < N)", "(uint8_t)(rank <= N)"),
    ("mask_not_applied", "ws_out[idx] = keep ? t : 0;", "ws_out[idx] = t;"),
    ("mask_from_codes", "mag[i] = fabsf(bf16_bits_to_float(W[r * K + base + i]));",
     "mag[i] = fabsf((float)ternary_code(bf16_bits_to_float(W[r * K + base + i]), g));"),
    ("code_signs_swapped", "(v == 1 ? 1u : 3u)", "(v == 1 ? 3u : 1u)"),
    ("code_bit_order", "int shift = 6 - 2 * (int)((e % 16) / 4);",
     "int shift = 2 * (int)((e % 16) / 4);"),
    ("code_byte_order", "int64_t byte = 4 * (e / 16) + e % 4;",
     "int64_t byte = 4 * (e / 16) + 3 - e % 4;"),
    ("pruned_not_zeroed_dense", "int8_t v = kept ? t[r * K + k] : 0;", "int8_t v = t[r * K + k];"),
    ("meta_nibble_order", "<< (4 * (gi % 2)));", "<< (4 * (1 - gi % 2)));"),
    ("index_order_swapped", "idx |= (unsigned)i << (2 * kept);",
     "idx |= (unsigned)i << (2 - 2 * kept);"),
    ("gamma_wrong_count", "((double)n * 16777216.0)", "((double)(n + 1) * 16777216.0)"),
    ("gamma_drops_eps", "float g = gamma + eps;", "float g = gamma;"),
    ("round_half_away", "float r = rintf(q);", "float r = roundf(q);"),
    ("act_qb_128", "rintf((127.0f * x) / s)", "rintf((128.0f * x) / s)"),
    ("act_round_half_away", "rintf((127.0f * x) / s)", "roundf((127.0f * x) / s)"),
    ("act_scale_floor_missing", "(a < 1e-5f) ? 1e-5f : a", "a"),
    ("acc_transposed", "acc[t * O + o] = (int32_t)sum;", "acc[o * T + t] = (int32_t)sum;"),
    ("rescale_qb_128", "(double)s[t] / 127.0", "(double)s[t] / 128.0"),
    ("rescale_drops_g", "(double)acc[t * O + o] * (double)g * (double)s[t]",
     "(double)acc[t * O + o] * (double)s[t]"),
    ("zero_count_counts_nonzeros", "if (t[i] == 0) ++c;", "if (t[i] != 0) ++c;"),
    ("flips_one_direction", "if ((keep_a[i] != 0) != (keep_b[i] != 0)) ++c;",
     "if (keep_a[i] && !keep_b[i]) ++c;"),
    ("backward_dw_masked",
     "acc += (double)dY[t * O + o] * (((double)s[t]) / 127.0 * (double)Xq[t * K + k]);",
     "acc += (double)dY[t * O + o] * (((double)s[t]) / 127.0 * (double)Xq[t * K + k]) *"
     " (Ws[o * K + k] != 0);"),
    ("backward_dx_drops_g", "acc += (double)dY[t * O + o] * ((double)g * (double)Ws[o * K + k]);",
     "acc += (double)dY[t * O + o] * ((double)Ws[o * K + k]);"),
    ("backward_dw_unscaled_acts", "(((double)s[t]) / 127.0 * (double)Xq[t * K + k])",
     "((double)Xq[t * K + k])"),
    ("backward_dw_ungated",
     "dW[o * K + k] = oracle_ste_pass(bf16_bits_to_float(W[o * K + k]), g) ? acc : 0.0;",
     "dW[o * K + k] = acc;"),
    ("backward_gate_round_range", "return fabsf(w) / g <= 1.0f;", "return fabsf(w) / g < 1.5f;"),
    ("backward_gate_strict", "return fabsf(w) / g <= 1.0f;", "return fabsf(w) / g < 1.0f;"),
    ("group_codes_one_scale", "const float q = wi / g[(base + i) / kg];", "const float q = wi / g[0];"),
    ("group_gamma_whole_row_count", "((double)O * (double)kg * 16777216.0)",
     "((double)O * (double)K * 16777216.0)"),
    ("group_rescale_first_scale", "(double)g[j] * (double)s[t * G + j] / 127.0",
     "(double)g[j] * (double)s[t * G] / 127.0"),
    ("group_acts_row_absmax", "for (int64_t k = j * kg; k < (j + 1) * kg; ++k) {\n        float v = fabsf",
     "for (int64_t k = 0; k < K; ++k) {\n        float v = fabsf"),
    ("backward_gate_by_mask",
     "dW[o * K + k] = oracle_ste_pass(bf16_bits_to_float(W[o * K + k]), g) ? acc : 0.0;",
     "dW[o * K + k] = Ws[o * K + k] != 0 ? acc : 0.0;"),
]


@pytest.fixture(scope="module")
def source():
    with open(oracle_build.SRC) as f:
        return f.read()


@pytest.mark.parametrize("name,orig,mut", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_mutant_is_caught(tmp_path, source, name, orig, mut):
    assert source.count(orig) == 1, f"mutation site for {name} not unique/present"
    src = tmp_path / f"{name}.c"
    src.write_text(source.replace(orig, mut))
    lib_path = str(tmp_path / f"lib{name}.so")
    subprocess.check_call(["gcc", *oracle_build.CFLAGS, str(src), "-o", lib_path, "-lm"])
    lib = oracle.load_library(lib_path)
    oracle.use_library(lib)
    failed = []
    try:
        for check in oracle_pins.ALL:
            try:
                check(oracle)
            except (AssertionError, OverflowError, IndexError, ValueError):
                failed.append(check.__name__)
    finally:
        oracle.use_library(None)
    assert failed, f"mutant {name} passed every pin"
    os.environ.setdefault("SBN_LAST_MUTANT_CAUGHT_BY", ",".join(failed))
