"""The oracle's pins must catch plausible mistakes (no GPU).

Each case copies the oracle source, plants one mistake of the kind a careful
reader could still make (a rounding mode, a dropped term, a wrong sign,
index or operand order), builds the copy with the same flags, and runs the
oracle pin tests against it.  Every mutant must make at least one pin fail;
the unmutated copy must pass.
"""
import os
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "dsqref.c")
PINS = ["tests/test_oracle_formats.py", "tests/test_oracle_gemv.py", "tests/test_oracle_prefill.py"]

MUTANTS = {
    "round_half_even": ("float v = roundf(x[i] / d32);", "float v = rintf(x[i] / d32);"),
    "q8_scale_from_amax": ("wr16(ob, dsqref_f32_to_f16(d32));", "wr16(ob, dsqref_f32_to_f16(d32 * 127.0f));"),
    "act_sum_of_magnitudes": ("for (int i = 0; i < DSQREF_QK8_0; ++i) s += q[i];",
                              "for (int i = 0; i < DSQREF_QK8_0; ++i) s += q[i] < 0 ? -q[i] : q[i];"),
    "f16_ties_away": ("if (rem > 0x1000u || (rem == 0x1000u && (h & 1u)))",
                      "if (rem >= 0x1000u)"),
    "nibble_halves_swapped": ("return (j & 1) ? (byte >> 4) : (byte & 15);",
                              "return (j & 1) ? (byte & 15) : (byte >> 4);"),
    "scale_high_bits_wrong_byte": ("*sc = (s[j + 4] & 15) | ((s[j - 4] >> 6) << 4);",
                                   "*sc = (s[j + 4] & 15) | ((s[j] >> 6) << 4);"),
    "q4k_dequant_min_sign": ("out[r * K + sb * DSQREF_QK_K + 32 * j + l] = aq - b;",
                             "out[r * K + sb * DSQREF_QK_K + 32 * j + l] = aq + b;"),
    "gemv_min_term_dropped": ("acc += t1 - t2;", "acc += t1;"),
    "gemv_min_term_sign": ("acc += t1 - t2;", "acc += t1 + t2;"),
    "gemv_wrong_act_scale_index": ("double t = ((double)dsqref_f16_to_f32(rd16(blk)) * (double)xd[b]) * (double)isum[b];",
                                   "double t = ((double)dsqref_f16_to_f32(rd16(blk)) * (double)xd[0]) * (double)isum[b];"),
    "block_sum_wrong_superblock": ("const uint8_t *blk = w + (n * (K / DSQREF_QK_K) + b / 8) * DSQREF_Q4_K_BYTES;",
                                   "const uint8_t *blk = w + (n * (K / DSQREF_QK_K)) * DSQREF_Q4_K_BYTES;"),
    "prefill_transposed_output": ("            y[m * N + n] = acc;\n", "            y[n * M + m] = acc;\n"),
    "prefill_shift_not_undone": ("y[m * N + n] = ldexp(acc, -shift[m]);", "y[m * N + n] = acc;"),
    "q4k_quantizer_no_zero_in_range": ("float lo = 0.0f, hi = xs[32 * j];", "float lo = xs[32 * j], hi = xs[32 * j];"),
    # the condition scale behind the GEMV tolerance's denominator floor
    "absum_min_term_dropped": ("mag += fabs(t1) + fabs(t2);", "mag += fabs(t1);"),
    "absum_of_difference": ("mag += fabs(t1) + fabs(t2);", "mag += fabs(t1 - t2);"),
    "absum_doubled": ("                mag += fabs(t);\n", "                mag += 2.0 * fabs(t);\n"),
    "absum_is_abs_of_sum": ("if (absum) absum[n] = mag;", "if (absum) absum[n] = fabs(acc);"),
    "row_shift_narrow_clamp": ("if (s < -113) s = -113;", "if (s < -64) s = -64;"),
}


def _build(tmp_path, name, patch):
    src = open(SRC).read()
    if patch is not None:
        old, new = patch
        assert src.count(old) == 1, f"mutant {name}: pattern must occur exactly once"
        src = src.replace(old, new)
    d = tmp_path / name
    d.mkdir()
    (d / "dsqref.c").write_text(src)
    (d / "dsqref.h").write_text(open(os.path.join(ROOT, "oracle", "dsqref.h")).read())
    lib = d / "libdsqref.so"
    subprocess.check_call(["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math",
                           "-fPIC", "-shared", "-w", "-o", str(lib), str(d / "dsqref.c"), "-lm"])
    return str(lib)


def _run_pins(lib):
    env = dict(os.environ, DSQREF_LIB=lib)
    return subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider", *PINS],
                          cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)


@pytest.fixture(scope="module")
def outcomes(tmp_path_factory):
    """Build and run every copy concurrently (one pytest process each)."""
    tmp = tmp_path_factory.mktemp("mutants")
    cases = {"clean": None, **MUTANTS}
    libs = {name: _build(tmp, name, patch) for name, patch in cases.items()}
    with ThreadPoolExecutor(max_workers=max(2, min(8, os.cpu_count() or 2))) as ex:
        futs = {name: ex.submit(_run_pins, lib) for name, lib in libs.items()}
        return {name: f.result() for name, f in futs.items()}


def test_unmutated_copy_passes(outcomes):
    r = outcomes["clean"]
    assert r.returncode == 0, r.stdout[-2000:]


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(outcomes, name):
    assert outcomes[name].returncode != 0, f"planted mistake '{name}' passed every pin"
