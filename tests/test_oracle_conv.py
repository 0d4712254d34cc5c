"""CPU tests: the oracle's short convolution against its pins (numpy's
correlate, impulse responses, closed forms of the activation, the conv state,
the all-block halo), and the pins against planted mistakes in copies of the
oracle source."""
import pytest

import oracle
import pins_conv as pc


@pytest.mark.parametrize("pin", pc.ALL_CONV_PINS, ids=lambda f: f.__name__)
def test_conv_pin(pin):
    pin(oracle)


# (description, text in the oracle source, replacement)
MUTATIONS = [
    ("taps reversed in the causal convolution",
     "acc += d->w[c * W + j] * conv_input(s, d->u, own_from, halo, state, b, t - (W - 1) + j, c);",
     "acc += d->w[c * W + (W - 1 - j)] * conv_input(s, d->u, own_from, halo, state, b, t - (W - 1) + j, c);"),
    ("causal window shifted by one token",
     "acc += d->w[c * W + j] * conv_input(s, d->u, own_from, halo, state, b, t - (W - 1) + j, c);",
     "acc += d->w[c * W + j] * conv_input(s, d->u, own_from, halo, state, b, t - W + j, c);"),
    ("reverse convolution not confined to the block", "const int64_t block_end = (t / T + 1) * T;",
     "const int64_t block_end = L;"),
    ("reverse taps reversed", "const int64_t tp = t + (W - 1) - j;", "const int64_t tp = t + j;"),
    ("bias dropped", "const double v = acc + (d->bias ? d->bias[c] : 0.0);", "const double v = acc;"),
    ("state rows read newest first",
     "if (state && tp >= -(W - 1)) return state[(b * (W - 1) + (W - 1 + tp)) * Cx + c];",
     "if (state && tp >= -(W - 1)) return state[(b * (W - 1) + (-1 - tp)) * Cx + c];"),
    ("noisy blocks continue from their own stream", "conv_causal(s, nf, cf->u, state_in);",
     "conv_causal(s, nf, NULL, state_in);"),
    ("state_out one row late",
     "conv_input(s, fwd->u, 0, NULL, state_in, b, s->seqlen - (W - 1) + r, c);",
     "conv_input(s, fwd->u, 0, NULL, state_in, b, s->seqlen - W + r, c);"),
]


@pytest.mark.parametrize("desc,old,new", MUTATIONS, ids=[m[0] for m in MUTATIONS])
def test_planted_conv_mistake_is_caught(desc, old, new, tmp_path):
    src = oracle.source_text()
    assert src.count(old) == 1, f"mutation anchor not found for: {desc}"
    lib = oracle.compile_variant(src.replace(old, new), str(tmp_path / "mutant.so"))
    variant = oracle.Variant(lib)
    failed = []
    for pin in pc.ALL_CONV_PINS:
        try:
            pin(variant)
        except (AssertionError, ValueError):
            failed.append(pin.__name__)
    assert failed, f"no pin caught the planted mistake: {desc}"
