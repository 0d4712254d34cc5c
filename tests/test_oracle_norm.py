"""CPU tests: the oracle's gated RMSNorm against its pins (unit RMS, scale
invariance, closed form of constant groups, group independence, gate placement,
weight linearity), and the pins against planted mistakes in copies of the
oracle source."""
import pytest

import oracle
import pins_norm as pn


@pytest.mark.parametrize("pin", pn.ALL_NORM_PINS, ids=lambda f: f.__name__)
def test_norm_pin(pin):
    pin(oracle)


# (description, text in the oracle source, replacement)
MUTATIONS = [
    ("sum of squares instead of the mean", "const double rstd = 1.0 / sqrt(ss / (double)gs + eps);",
     "const double rstd = 1.0 / sqrt(ss + eps);"),
    ("eps outside the square root", "const double rstd = 1.0 / sqrt(ss / (double)gs + eps);",
     "const double rstd = 1.0 / (sqrt(ss / (double)gs) + eps);"),
    ("gate applied after the norm (RMS of the ungated values)",
     "const double v = y[r * channels + c] * (z ? silu(z[r * channels + c]) : 1.0);\n                ss += v * v;",
     "const double v = y[r * channels + c];\n                ss += v * v;"),
    ("squares summed over the whole row",
     "for (int64_t c = g * gs; c < (g + 1) * gs; ++c) {\n                const double v = y[r * channels + c] * (z ? silu(z[r * channels + c]) : 1.0);\n                ss += v * v;",
     "for (int64_t c = 0; c < channels; ++c) {\n                const double v = y[r * channels + c] * (z ? silu(z[r * channels + c]) : 1.0);\n                ss += v * v;"),
    ("weight indexed per group", "out[r * channels + c] = v * rstd * w[c];", "out[r * channels + c] = v * rstd * w[g];"),
    ("gate without the sigmoid",
     "const double v = y[r * channels + c] * (z ? silu(z[r * channels + c]) : 1.0);\n                ss += v * v;",
     "const double v = y[r * channels + c] * (z ? z[r * channels + c] : 1.0);\n                ss += v * v;"),
]


@pytest.mark.parametrize("desc,old,new", MUTATIONS, ids=[m[0] for m in MUTATIONS])
def test_planted_norm_mistake_is_caught(desc, old, new, tmp_path):
    src = oracle.source_text()
    assert src.count(old) == 1, f"mutation anchor not found for: {desc}"
    lib = oracle.compile_variant(src.replace(old, new), str(tmp_path / "mutant.so"))
    variant = oracle.Variant(lib)
    failed = []
    for pin in pn.ALL_NORM_PINS:
        try:
            pin(variant)
        except (AssertionError, ValueError):
            failed.append(pin.__name__)
    assert failed, f"no pin caught the planted mistake: {desc}"
