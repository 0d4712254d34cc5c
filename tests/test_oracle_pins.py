"""CPU tests: the fp64 oracle against its pins, and the pins against planted
mistakes in copies of the oracle source (each mutant must fail at least one pin)."""
import os

import pytest

import oracle
import pins


@pytest.mark.parametrize("pin", pins.ALL_PINS, ids=lambda f: f.__name__)
def test_pin(pin):
    pin(oracle)


# (description, text in the oracle source, replacement)
MUTATIONS = [
    ("drop the D skip term", "double yp = acc + d->D[h] * x[p];", "double yp = acc;"),
    ("wrong decay sign", "const double a = exp(dt * d->A[h]);", "const double a = exp(-dt * d->A[h]);"),
    ("drop dt on the input term", "row[n] = a * row[n] + dt * x[p] * Bt[n];", "row[n] = a * row[n] + x[p] * Bt[n];"),
    ("output reads B instead of C", "acc += Ct[n] * row[n];", "acc += Bt[n] * row[n];"),
    ("output before the state update",
     "row[n] = a * row[n] + dt * x[p] * Bt[n];\n            acc += Ct[n] * row[n];",
     "acc += Ct[n] * row[n];\n            row[n] = a * row[n] + dt * x[p] * Bt[n];"),
    ("wrong head-to-group map", "const int64_t g = h / (H / G);", "const int64_t g = h % G;"),
    ("boundary state off by one", "if (states && (t + 1) % T == 0) {", "if (states && t % T == 0 && t > 0) {"),
    ("reverse keeps the previous block's state",
     "    memset(hs, 0, sizeof(double) * P * N);\n    for (int64_t t = t1 - 1;",
     "    for (int64_t t = t1 - 1;"),
    ("reverse runs left to right", "for (int64_t t = t1 - 1; t >= t0; --t) {", "for (int64_t t = t0; t < t1; ++t) {"),
    ("noisy block starts from its own end state",
     "memcpy(hs, states + ((b * K + k - 1) * H + h) * PN, sizeof(double) * PN);",
     "memcpy(hs, states + ((b * K + k) * H + h) * PN, sizeof(double) * PN);"),
    ("h0 ignored", "        memcpy(hs, src + (b * H + h) * PN, sizeof(double) * PN);",
     "        memset(hs, 0, sizeof(double) * PN);"),
    ("transposed x B^T", "row[n] = a * row[n] + dt * x[p] * Bt[n];",
     "row[n] = a * row[n] + dt * x[n % P] * Bt[p % N];"),
    ("gate on the wrong tensor", "if (d->z) yp *= silu(d->z[((b * L + t) * H + h) * P + p]);",
     "if (d->z) yp *= silu(d->x[((b * L + t) * H + h) * P + p]);"),
]


@pytest.mark.parametrize("desc,old,new", MUTATIONS, ids=[m[0] for m in MUTATIONS])
def test_planted_mistake_is_caught(desc, old, new, tmp_path):
    src = oracle.source_text()
    assert src.count(old) == 1, f"mutation anchor not found for: {desc}"
    lib = oracle.compile_variant(src.replace(old, new), str(tmp_path / "mutant.so"))
    variant = oracle.Variant(lib)
    failed = []
    for pin in pins.ALL_PINS:
        try:
            pin(variant)
        except (AssertionError, ValueError):
            failed.append(pin.__name__)
    assert failed, f"no pin caught the planted mistake: {desc}"
