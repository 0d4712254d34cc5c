"""CPU tests: the oracle's backward pass against its pins (finite differences of
the pinned forward, linearity, the clean-only case), and the pins against
planted mistakes in copies of the oracle source."""
import pytest

import oracle
import pins_backward as pb


@pytest.mark.parametrize("pin", pb.ALL_BACKWARD_PINS, ids=lambda f: f.__name__)
def test_backward_pin(pin):
    pin(oracle)


# (description, text in the oracle source, replacement)
MUTATIONS = [
    ("dB without the dt factor", "acc->dB[t * N + q] += dt * sb;", "acc->dB[t * N + q] += sb;"),
    ("dC from the state before the token", "if (dyt) sc += dyt[p] * ht[p * N + q];",
     "if (dyt) sc += dyt[p] * (prev ? prev[p * N + q] : 0.0);"),
    ("adjoint state not decayed", "for (int64_t e = 0; e < PN; ++e) G[e] *= a;", "(void)a;"),
    ("noisy gradient not passed to the clean states",
     "for (int64_t e = 0; e < PN; ++e) dsn[(k - 1) * PN + e] += G[e];", "(void)0;"),
    ("dA without dt", "dA += Gv * dt * a * hp;", "dA += Gv * a * hp;"),
    ("ddt without the decay term", "ddt += Gv * (A * a * hp + x[p] * Bt[q]);", "ddt += Gv * (x[p] * Bt[q]);"),
    ("dx without the D skip", "acc->dx[t * P + p] += dt * gb + (dyt ? d->D[h] * dyt[p] : 0.0);",
     "acc->dx[t * P + p] += dt * gb;"),
    ("state gradient one block late", "dat[i] = ((i + 1) % T == 0) ? dsn + (i / T) * PN : NULL;",
     "dat[i] = (i % T == 0 && i > 0) ? dsn + (i / T - 1) * PN : NULL;"),
]


@pytest.mark.parametrize("desc,old,new", MUTATIONS, ids=[m[0] for m in MUTATIONS])
def test_planted_backward_mistake_is_caught(desc, old, new, tmp_path):
    src = oracle.source_text()
    assert src.count(old) == 1, f"mutation anchor not found for: {desc}"
    lib = oracle.compile_variant(src.replace(old, new), str(tmp_path / "mutant.so"))
    variant = oracle.Variant(lib)
    failed = []
    for pin in pb.ALL_BACKWARD_PINS:
        try:
            pin(variant)
        except (AssertionError, ValueError):
            failed.append(pin.__name__)
    assert failed, f"no pin caught the planted mistake: {desc}"
