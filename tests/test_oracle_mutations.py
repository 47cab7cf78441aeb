"""The oracle's pins catch planted mistakes (CPU only).

Each case below plants one plausible mistake in a copy of the oracle source
(a flipped tie rule, a swapped nibble, a scale off by one, a transposed
operand, a dropped rounding, ...), compiles the copy with the oracle's own
flags and runs the whole pin suite (tests/test_oracle_pins.py) against it in
a subprocess.  The pins must fail for every mutant, and must all pass for an
unmodified copy built the same way (so a failure is the mistake's doing, not
the harness's).  The mutants are built and run in parallel, once per session.
"""
import concurrent.futures
import os
import subprocess
import sys

import pytest

import oracle
from oracle import build as oracle_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PINS = os.path.join(ROOT, "tests", "test_oracle_pins.py")

# name -> (text in oracle/mxq_oracle.c, replacement, which occurrence (0-based)).
# Left out as equivalent (no input can tell them apart from the oracle):
# dropping the clamp of the NVFP4 block-scale quotient at 448 (the quotient is
# at most 448 (1 + 2^-22) and the E4M3 cast saturates at 448); dropping the
# +0 fix-up of unpacked fp4 zeros (table entry 8 is already +0.0); dropping the
# zero-weight shortcut of the mse element cast (0 / d, even 0 / 0, casts to
# code 0, and -0.0 < 0 is false).
MUTATIONS = {
    # E2M1 element cast
    "tie_rule_flipped": ("(a == E2M1_MIDPOINTS[i]) && (i % 2 == 1)",
                         "(a == E2M1_MIDPOINTS[i]) && (i % 2 == 0)", 0),
    "table_entries_swapped": ("0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0,",
                              "0.0, 0.5, 1.0, 1.5, 2.0, 4.0, 3.0, 6.0,", 0),
    "last_midpoint_wrong": ("{0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0}",
                            "{0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 4.5}", 0),
    "sign_bit_from_negative_zero": ("return mag | (v < 0.0 ? 8 : 0);",
                                    "return mag | (signbit(v) ? 8 : 0);", 0),
    # binary rounding
    "ties_away_from_zero": ("if (rem > 0.5 || (rem == 0.5 && fmod(f, 2.0) != 0.0)) f += 1.0;",
                            "if (rem >= 0.5) f += 1.0;", 0),
    "f16_min_exponent": ("round_to_precision(v, 11, -14)", "round_to_precision(v, 11, -15)", 0),
    "e4m3_not_saturating_at_448": ("if (fabs(r) > 448.0) r = copysign(448.0, v);",
                                   "if (fabs(r) > 480.0) r = copysign(480.0, v);", 0),
    "e4m3_encode_bias": ("return s | (uint8_t)((e + 7) << 3) | m;",
                         "return s | (uint8_t)((e + 8) << 3) | m;", 0),
    # MXFP4 pack / unpack
    "mx_scale_floor_minus_1": ("int e = ilogb(amax) - 2;", "int e = ilogb(amax) - 1;", 0),
    "mx_pack_nibbles_swapped": ("packed[r * (K / 2) + b * 16 + j] = (uint8_t)(lo | (hi << 4));",
                                "packed[r * (K / 2) + b * 16 + j] = (uint8_t)(hi | (lo << 4));", 0),
    "mx_unpack_nibbles_swapped": ("int nib = (k % 2 == 0) ? (byte & 15) : (byte >> 4);",
                                  "int nib = (k % 2 == 0) ? (byte >> 4) : (byte & 15);", 0),
    "e8m0_bias_off_by_one": ("return E2M1_TABLE[nib] * ldexp(1.0, (int)s - 127);",
                             "return E2M1_TABLE[nib] * ldexp(1.0, (int)s - 126);", 0),
    "e8m0_nan_byte_ignored": ("if (s == 0xFF) return NAN;", "if (s == 0xFF) s = 0xFE;", 0),
    # cache fake quantization
    "cache_ceiling_strict": ("while (ldexp(qmax, k) < amax) ++k;",
                             "while (ldexp(qmax, k) <= amax) ++k;", 0),
    "cache_fp8_qmax": ("return fmt == ORC_FP8 ? 448.0 : 6.0;",
                       "return fmt == ORC_FP8 ? 240.0 : 6.0;", 0),
    "cache_nvfp4_upper_clamp": ("return fmt == ORC_NVFP4 ? 8 : 127;",
                                "return fmt == ORC_NVFP4 ? 9 : 127;", 0),
    "cache_nvfp4_lower_clamp": ("return fmt == ORC_NVFP4 ? -9 : -126;",
                                "return fmt == ORC_NVFP4 ? -10 : -126;", 0),
    # grouped GEMM
    "gemm_forward_transposed_weight": ("acc += decode_bf16(at[k]) * w[n * K + k];",
                                       "acc += decode_bf16(at[k]) * w[k * N + n];", 0),
    "gemm_dgrad_transposed_weight": ("o[k] += g * w[n * K + k];", "o[k] += g * w[k * N + n];", 0),
    "gemm_expert_rows_off_by_one": ("int64_t lo = e == 0 ? 0 : offs[e - 1], hi = offs[e];",
                                    "int64_t lo = e == 0 ? 0 : offs[e - 1] + 1, hi = offs[e];", 0),
    "offs_not_checked_for_order": ("if (offs[e] < prev) return ORC_EOFFS;",
                                   "if (offs[e] < prev && 0) return ORC_EOFFS;", 0),
    "offs_total_not_checked": ("return prev == T ? ORC_OK : ORC_EOFFS;", "return ORC_OK;", 0),
    # NVFP4 two-level
    "nvfp4_dequant_rounding_order": ("double v = f32_mul(E2M1_TABLE[nib] * s, (double)global_scale);",
                                     "double v = E2M1_TABLE[nib] * f32_mul(s, (double)global_scale);", 0),
    "nvfp4_global_scale_without_6": ("f32_div(amax, 6.0 * 448.0)", "f32_div(amax, 448.0)", 0),
    "nvfp4_zero_block_scale_not_one": ("if (q == 0.0) q = 1.0;", "if (q == 0.0) q = 0.0;", 0),
    "nvfp4_scale_lower_clamp_dropped": ("if (q < ldexp(1.0, -9)) q = ldexp(1.0, -9);",
                                        "if (q < ldexp(1.0, -9)) q = q;", 0),
    "nvfp4_dequant_scale_byte_bias": ("double s = orc_decode_e4m3(block_scales[r * (K / 16) + k / 16]);",
                                      "double s = 2.0 * orc_decode_e4m3(block_scales[r * (K / 16) + k / 16]);", 0),
    # packed cache storage
    "packed_cache_e8m0_bias": ("return (uint8_t)(k + 127);", "return (uint8_t)(k + 128);", 0),
    "packed_cache_nibbles_swapped": ("if (c % 2 == 0) *byte = (uint8_t)code;\n"
                                     "          else *byte = (uint8_t)(*byte | (code << 4));",
                                     "if (c % 2 == 1) *byte = (uint8_t)code;\n"
                                     "          else *byte = (uint8_t)(*byte | (code << 4));", 0),
    # NVFP4 mse sweep
    "mse_last_minimum": ("if (err < best_err) {", "if (err <= best_err) {", 0),
    "mse_error_sign": ("double e = fma(q, d, -w[i]);", "double e = fma(q, d, w[i]);", 0),
    "mse_drops_code_126": ("for (int c = 1; c <= 126; ++c) {", "for (int c = 1; c < 126; ++c) {", 0),
    # element codecs
    "f16_decode_subnormal_scale": ("v = ldexp((double)m, -24);", "v = ldexp((double)m, -25);", 0),
    "f16_encode_bias": ("return s | (uint16_t)((e + 15) << 10) | m;",
                        "return s | (uint16_t)((e + 16) << 10) | m;", 0),
    "f32_overflow_threshold": ("if (fabs(r) > ldexp(16777215.0, 104)) r = copysign(INFINITY, v);",
                               "if (fabs(r) > ldexp(16777215.0, 103)) r = copysign(INFINITY, v);", 0),
    "bf16_overflow_threshold": ("if (fabs(r) > ldexp(255.0, 120)) r = copysign(INFINITY, v);",
                                "if (fabs(r) > ldexp(255.0, 119)) r = copysign(INFINITY, v);", 0),
    # cache tail group and zero signs
    "cache_tail_group_reads_past_the_row": ("int64_t c1 = c0 + B < C ? c0 + B : C;",
                                            "int64_t c1 = c0 + B;", 0),
    "cache_fp8_loses_negative_zero": ("if (fmt == ORC_FP8) return ldexp(orc_round_e4m3(v), k);",
                                      "if (fmt == ORC_FP8) return ldexp(orc_round_e4m3(v), k) + 0.0;", 0),
    "packed_cache_e8m0_nan_byte": (": sb == 0xFF       ? NAN /* the E8M0 NaN */",
                                   ": sb == 0xFF       ? 0.0 /* the E8M0 NaN */", 0),
    "cache_zero_block_scale": ("if (amax == 0.0) return lo;", "if (amax == 0.0) return 0;", 0),
    # mse degenerate cases
    "mse_zero_tensor_scale": ("int code = g == 0.0 ? 0x38 : orc_nvfp4_mse_code(w, g);",
                              "int code = g == 0.0 ? 0x01 : orc_nvfp4_mse_code(w, g);", 0),
    "mse_sign_from_the_quotient": ("nib[h] = (orc_e2m1_code(fabs(f32_div(xi, d))) & 7) | (xi < 0.0 ? 8 : 0);",
                                   "nib[h] = orc_e2m1_code(f32_div(xi, d));", 0),
    "nvfp4_sign_from_the_quotient": ("lo = (orc_e2m1_code(fabs(f32_div(x0, d))) & 7) | (x0 < 0.0 ? 8 : 0);",
                                     "lo = orc_e2m1_code(f32_div(x0, d));", 0),
    # W4A4
    "w4a4_activations_not_quantized": ("for (int64_t k = 0; k < K; ++k) xa[k] = mx_element(qp, qs, K, 0, k);",
                                       "for (int64_t k = 0; k < K; ++k) xa[k] = decode_bf16(x[t * K + k]);", 0),
    "nvfp4_w4a4_activation_global_scale_dropped": ("xa[k] = nv_element(qp, qs, k, gx);",
                                                   "xa[k] = nv_element(qp, qs, k, 1.0);", 0),
    "nvfp4_w4a4_first_expert_global_scale": ("k, (double)w_global[e]);", "k, (double)w_global[0]);", 0),
}


def plant(src, old, new, occurrence):
    start = -1
    for _ in range(occurrence + 1):
        start = src.find(old, start + 1)
        assert start >= 0, "mutation site not found: %r" % old
    return src[:start] + new + src[start + len(old):]


def run_pins(lib_path):
    env = dict(os.environ, **{oracle.LIB_ENV: lib_path})
    p = subprocess.run([sys.executable, "-m", "pytest", PINS, "-x", "-q", "-p", "no:cacheprovider"],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    tail = (p.stdout.strip().splitlines() or [""])[-1]
    return p.returncode, tail


@pytest.fixture(scope="session")
def mutant_results(tmp_path_factory):
    """name -> (pytest return code, last line), for every mutant and for an
    unmodified copy ("identity")."""
    src = open(oracle_build.SRC).read()
    work = tmp_path_factory.mktemp("oracle_mutants")
    cases = dict(MUTATIONS, identity=("", "", None))

    def one(name):
        old, new, occ = cases[name]
        text = src if occ is None else plant(src, old, new, occ)
        c_path = os.path.join(str(work), name + ".c")
        with open(c_path, "w") as f:
            f.write(text)
        lib_path = oracle_build.compile_to(c_path, os.path.join(str(work), "lib" + name + ".so"))
        return name, run_pins(lib_path)

    with concurrent.futures.ThreadPoolExecutor(max_workers=min(8, os.cpu_count() or 1)) as ex:
        return dict(ex.map(one, cases))


def test_unmodified_copy_passes_every_pin(mutant_results):
    rc, tail = mutant_results["identity"]
    assert rc == 0, tail


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_pins_catch_the_planted_mistake(mutant_results, name):
    rc, tail = mutant_results[name]
    # 1: some pin failed (a crash or a collection error would be another code)
    assert rc == 1, "pins did not catch %s (pytest exit %d: %s)" % (name, rc, tail)
