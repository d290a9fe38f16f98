"""Mutation check of the oracle's pins (CPU only).

Each case plants one plausible mistake in a copy of the oracle's source: a dropped term, a flipped sign, a wrong
index or operand, an unmasked padded key or query, a wrong tail normalisation, a reversed order or tie-break, or an
off-by-one in the prefix cut. The copy is built the same way as the oracle, and at least one pin in
tests/test_oracle_pins.py must fail against it. The unmodified source, built the same way, must pass every pin.
The oracle on disk is never modified.
"""
import concurrent.futures
import inspect
import os
import subprocess

import numpy as np
import pytest

import oracle
from tests import test_oracle_pins as pins

SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "oracle", "losa_oracle.cpp")

_SEL_SORT = ("std::sort(ord.begin(), ord.end(), [&](int a, int b) { return m[a] > m[b] || (m[a] == m[b] && a < b); });\n"
             "    // Integer units")
_TOPK_SORT = ("std::sort(ord.begin(), ord.end(), [&](int a, int b) { return m[a] > m[b] || (m[a] == m[b] && a < b); });\n"
              "        std::vector<int> kept")
_ALL_KEYS_LSE = ("{ std::vector<int> all(N); std::iota(all.begin(), all.end(), 0); std::vector<double> sa; "
                 "logits(q + head + (size_t)qi * d, k + head, d, scale, all, sa); lse[row] = log_sum_exp(sa); }")

MUTATIONS = {
    "logit scale dropped": ("s[t] = scale * acc;", "s[t] = acc;"),
    "log-sum-exp loses its shift": ("return m + std::log(sum);", "return std::log(sum);"),
    "softmax weight with the sign flipped": ("std::exp(s[t] - lse)", "std::exp(lse - s[t])"),
    "restricted logits read key row t": ("const float* kr = kh + (size_t)keys[t] * d;",
                                         "const float* kr = kh + (size_t)t * d;"),
    "restricted values read value row t": ("const float* vr = vh + (size_t)keys[t] * d;",
                                           "const float* vr = vh + (size_t)t * d;"),
    "padded keys take part in dense attention": ("std::vector<int> keys(N);\n    std::iota(keys.begin(), keys.end(), 0);  // R1",
                                                 "std::vector<int> keys(Np);\n    std::iota(keys.begin(), keys.end(), 0);  // R1"),
    "mass divided by R instead of the real rows": ("row[j] /= (double)rows;", "row[j] /= (double)R;"),
    "mass summed into the wrong block": ("row[kk / C] += ", "row[kk % nk] += "),
    "mass with the exponent's sign flipped": ("std::exp(s[kk] - l)", "std::exp(l - s[kk])"),
    "mass over padded query rows": ("const int rows = std::min(R, N - i * R);", "const int rows = R;"),
    "selection in ascending mass": (_SEL_SORT, _SEL_SORT.replace("m[a] > m[b]", "m[a] < m[b]")),
    "selection ties to the higher index": (_SEL_SORT, _SEL_SORT.replace("a < b", "a > b")),
    "selection units rounded down": ("u[j] = (uint64_t)std::ceil(std::ldexp((double)m[j], 52));",
                                     "u[j] = (uint64_t)std::floor(std::ldexp((double)m[j], 52));"),
    "selection cut one block late": ("if (prefix >= target) { s = r + 1; break; }",
                                     "if (prefix > target) { s = r + 1; break; }"),
    "selection cut one block early": ("if (prefix >= target) { s = r + 1; break; }",
                                      "if (prefix >= target) { s = r > 0 ? r : 1; break; }"),
    "selected blocks left in mass order": ("std::sort(kept.begin(), kept.end());  // R5", ""),
    "top-k ties to the higher index": (_TOPK_SORT, _TOPK_SORT.replace("a < b", "a > b")),
    "work order ties by descending id": ("std::iota(ids.begin(), ids.end(), 0);\n    std::stable_sort",
                                         "std::iota(ids.rbegin(), ids.rend(), 0);\n    std::stable_sort"),
    "work order shortest first": ("return counts[a] > counts[b];", "return counts[a] < counts[b];"),
    "restricted softmax normalised over all keys": ("lse[row] = log_sum_exp(s);", _ALL_KEYS_LSE),
    "restricted attention reads padded keys": ("kk < (j + 1) * C && kk < N; ++kk", "kk < (j + 1) * C; ++kk"),
    "recall ignores the row mapping": ("const int r = rows[t];", "const int r = t;"),
}


def _pin_calls():
    """Every pin of tests/test_oracle_pins.py as (name, zero-argument callable)."""
    calls = []
    for name, fn in vars(pins).items():
        if not (name.startswith("test_") and inspect.isfunction(fn)):
            continue
        params = list(inspect.signature(fn).parameters)
        if not params:
            calls.append((name, fn))
        elif params == ["dtype"]:
            for dt in (np.float64, np.float32):
                calls.append((f"{name}[{dt.__name__}]", lambda fn=fn, dt=dt: fn(dt)))
        else:
            raise AssertionError(f"pin {name} takes arguments this check does not know: {params}")
    return calls


def _failing_pin(monkeypatch, lib_path):
    """Name of the first pin that fails against the library at lib_path, or None if all pass."""
    monkeypatch.setattr(oracle, "_lib", oracle.bind(lib_path))
    for name, call in _pin_calls():
        try:
            call()
        except Exception:  # an assertion, or the oracle rejecting its own output
            return name
    return None


@pytest.fixture(scope="module")
def builds(tmp_path_factory):
    """The unmodified source and every mutant, built in parallel; maps case name -> library path."""
    src = open(SRC).read()
    out = tmp_path_factory.mktemp("oracle_mutants")
    jobs = {"(unmodified)": src}
    for case, (old, new) in MUTATIONS.items():
        assert src.count(old) == 1, f"{case}: the planted site is no longer unique in the oracle source"
        jobs[case] = src.replace(old, new)

    def build(item):
        i, (case, text) = item
        path = out / f"m{i}.cpp"
        path.write_text(text)
        lib = str(out / f"libm{i}.so")
        subprocess.run(oracle.compile_command(str(path), lib), check=True, capture_output=True)
        return case, lib

    with concurrent.futures.ThreadPoolExecutor(max_workers=min(8, os.cpu_count() or 1)) as ex:
        return dict(ex.map(build, enumerate(jobs.items())))


def test_unmodified_source_passes_every_pin(builds, monkeypatch):
    assert _failing_pin(monkeypatch, builds["(unmodified)"]) is None


@pytest.mark.parametrize("case", list(MUTATIONS))
def test_planted_mistake_fails_a_pin(case, builds, monkeypatch):
    assert _failing_pin(monkeypatch, builds[case]) is not None, f"no pin catches: {case}"
