"""The pins must be able to fail: each plausible mistake planted in a copy of the
oracle's C source (a dropped term, a wrong index, sign or layer, a missing block
function, a lost accumulation) is compiled on the CPU and must break at least one
pin.  The planted copies live in a temporary directory; the oracle itself is
untouched."""
import ctypes
import subprocess
from pathlib import Path

import pytest

import oracle
from tests import test_oracle_pins as P
from tests import test_schedule as S

SRC = (Path(oracle.__file__).parent / "oracle.c").read_text()

MUTANTS = {
    "lazy_drops_current_term": ("for (int64_t s = 0; s <= t; ++s) acc += h[t - s] * y[s];",
                                "for (int64_t s = 0; s < t; ++s) acc += h[t - s] * y[s];"),
    "stack_wrong_tap_index": ("acc += (double)hl[t - s] * prev[s];",
                              "acc += (double)hl[t - s + 1] * prev[s];"),
    "stack_missing_block": ("a[(int64_t)l * T + t] = tanh(acc);",
                            "a[(int64_t)l * T + t] = acc;"),
    "stack_closed_loop_wrong_layer": ("else in = fp32 ? (double)af[(int64_t)M * T + t - 1] : a[(int64_t)M * T + t - 1];",
                                      "else in = fp32 ? (double)af[(int64_t)M * T + t - 1] : a[(int64_t)(M - 1) * T + t - 1];"),
    "tau_off_by_one_lag": ("acc += (double)b[j] * (double)rho[U + r - j];",
                           "acc += (double)b[j] * (double)rho[U + r - j - 1];"),
    "schedule_wrong_block_end": ("int64_t hi = n + U - 1;", "int64_t hi = n + U;"),
    "schedule_wrong_power": ("while ((n % (2 * U)) == 0) U *= 2;\n        int64_t hi",
                             "while ((n % (2 * U)) == 0 && U < 4) U *= 2;\n        int64_t hi"),
    "relaxed_overwrites": ("out[n + r] += acc;", "out[n + r] = acc;"),
    "fft_sign_flipped": ("double ang = sign * two_pi", "double ang = -sign * two_pi"),
    "spectrum_shifted_taps": ("for (int64_t m = 0; m < N; ++m) re[m] = (double)taps[i * ldt + m];",
                              "for (int64_t m = 0; m < N; ++m) re[m] = (double)taps[i * ldt + m + 1];"),
}

PINS = [
    lambda: P.test_causal_conv_equals_numpy_convolve(64),
    lambda: P.test_own_fft_equals_numpy_fft(64),
    lambda: P.test_fft_conv_equals_lazy_and_numpy(33),
    lambda: P.test_stack_equals_numpy_restatement(False),
    lambda: P.test_stack_equals_numpy_restatement(True),
    lambda: P.test_stack_delta_filters_closed_form(),
    lambda: P.test_relaxed_tiling_equals_lazy(False),
    lambda: P.test_tau_is_the_window_of_a_2U_circular_convolution(8),
    lambda: P.test_filter_spectrum_equals_numpy_rfft(16),
    lambda: S.test_tile_histogram_proposition_1(6),
    lambda: S.test_every_pair_covered_exactly_once(32),
]


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_planted_mistake_breaks_a_pin(name, tmp_path, monkeypatch):
    old, new = MUTANTS[name]
    assert SRC.count(old) == 1, "mutation anchor not found uniquely: " + name
    src = tmp_path / "mutant.c"
    src.write_text(SRC.replace(old, new))
    so = tmp_path / "libmutant.so"
    subprocess.run(["gcc", "-O1", "-std=c11", "-fopenmp", "-fPIC", "-shared", str(src),
                    "-o", str(so), "-lm"], check=True)
    monkeypatch.setattr(oracle, "_lib", oracle.load(so))
    failed = 0
    for pin in PINS:
        try:
            pin()
        except (AssertionError, RuntimeError, ValueError):
            failed += 1
    assert failed >= 1, "planted mistake %s passed every pin" % name
