"""Planted mistakes in the oracle must each trip at least one pin.

The oracle's source carries no planted-mistake code.  Each mistake here is a textual patch of
a copy of ``oracle/kda_oracle.c`` (one snippet of the correct code and its wrong replacement),
compiled into a library of its own under ``oracle/_build/mutants/``; the pins then run against
that copy through ``oracle.use_library``.  Every snippet must occur exactly once in the source,
so a later edit of the oracle cannot silently retire a mistake.

Mistakes: 1 state decay dropped, 2 wrong sign in the delta correction, 3 output read before
the update, 4 transposed state in the output, 5 diagonal dropped from the q.k mask, 6
carry-over state not decayed, 7 dt_bias sign, 9 missing square root in the normalise, 10
beta sigmoid dropped; in the chunked form: 11 the key-key product transposed (K- K~^T for
K~ K-^T), 12 W built from K- instead of K~, 13 the chunk's decay taken at its first row
instead of its last, 14 the identity term dropped from the forward substitution, 15 beta
missing from U, 16 the state transposed in Delta; 17 the sign of A_log in the gate.
"""
import os

import pytest

import oracle
import oracle_pins as P

# id -> (correct snippet, wrong replacement), or a list of such pairs applied together
MUTANTS = {
    1: ("      for (int j = 0; j < Dk; ++j) S[(size_t)i * Dk + j] *= decay[j];",
        "      for (int j = 0; j < Dk; ++j) S[(size_t)i * Dk + j] *= 1.0;"),
    2: ("      const double c = beta[t] * (vt[i] - pred[i]);",
        "      const double c = beta[t] * (vt[i] + pred[i]);"),
    3: [("    /* S <- S Diag(exp(g_t)) */\n",
         "    for (int i = 0; i < Dv; ++i) {\n"
         "      double acc0 = 0.0;\n"
         "      for (int j = 0; j < Dk; ++j) acc0 += S[(size_t)i * Dk + j] * qt[j];\n"
         "      out[(size_t)t * Dv + i] = scale * acc0;\n"
         "    }\n"),
        ("      out[(size_t)t * Dv + i] = scale * acc;\n", "      (void)acc;\n")],
    4: ("      for (int j = 0; j < Dk; ++j) acc += S[(size_t)i * Dk + j] * qt[j];\n"
        "      out[(size_t)t * Dv + i] = scale * acc;",
        "      for (int j = 0; j < Dk; ++j) acc += S[(size_t)j * Dk + i] * qt[j];\n"
        "      out[(size_t)t * Dv + i] = scale * acc;"),
    5: ("        Aqk[(size_t)r * n + s] = (s <= r) ? tq : 0.0;",
        "        Aqk[(size_t)r * n + s] = (s < r) ? tq : 0.0;"),
    6: ("        Sn[(size_t)i * Dk + j] = S[(size_t)i * Dk + j] * gl + acc * gl;",
        "        Sn[(size_t)i * Dk + j] = S[(size_t)i * Dk + j] + acc * gl;"),
    7: ("      const double x = graw[(size_t)t * D + d] + dt_bias[d];",
        "      const double x = graw[(size_t)t * D + d] - dt_bias[d];"),
    9: ("    const double inv = 1.0 / sqrt(ss + eps);",
        "    const double inv = 1.0 / (ss + eps);"),
    10: ("    beta[t] = sigmoid(logit[t]);",
         "    beta[t] = logit[t];"),
    11: ("          tk += Kt[(size_t)r * Dk + j] * Kb[(size_t)s * Dk + j];",
         "          tk += Kb[(size_t)r * Dk + j] * Kt[(size_t)s * Dk + j];"),
    12: ("          acc += Ai[(size_t)r * n + s] * beta[c0 + s] * Kt[(size_t)s * Dk + j];",
         "          acc += Ai[(size_t)r * n + s] * beta[c0 + s] * Kb[(size_t)s * Dk + j];"),
    13: ("        const double gl = exp(G[(size_t)(n - 1) * Dk + j]);",
         "        const double gl = exp(G[(size_t)0 * Dk + j]);"),
    14: ("      for (int s = c; s < r; ++s)",
         "      for (int s = c + 1; s < r; ++s)"),
    15: ("          acc += Ai[(size_t)r * n + s] * beta[c0 + s] * v[(size_t)(c0 + s) * Dv + i];",
         "          acc += Ai[(size_t)r * n + s] * v[(size_t)(c0 + s) * Dv + i];"),
    16: ("        for (int j = 0; j < Dk; ++j) acc += W[(size_t)r * Dk + j] * S[(size_t)i * Dk + j];",
         "        for (int j = 0; j < Dk; ++j) acc += W[(size_t)r * Dk + j] * S[(size_t)j * Dk + i];"),
    17: ("  const double a = exp(A_log);",
         "  const double a = exp(-A_log);"),
}

_MUT_DIR = os.path.join(os.path.dirname(os.path.abspath(oracle.__file__)), "_build", "mutants")


def _mutant_library(m: int) -> str:
    pairs = MUTANTS[m] if isinstance(MUTANTS[m], list) else [MUTANTS[m]]
    src = oracle.source()
    for right, wrong in pairs:
        assert src.count(right) == 1, f"mistake {m}: a snippet no longer occurs once in the oracle"
        src = src.replace(right, wrong)
    return oracle.compile_source(src,
                                 os.path.join(_MUT_DIR, f"libkda_oracle_mut{m}_{os.getpid()}.so"))


def test_clean_source_has_no_mistake_switch():
    assert "mutation" not in oracle.source()


@pytest.mark.parametrize("m", sorted(MUTANTS))
def test_mutation_is_caught(m):
    failed = []
    with oracle.use_library(_mutant_library(m)):
        for pin in P.ALL_PINS:
            try:
                pin()
            except AssertionError:
                failed.append(pin.__name__)
    assert failed, f"mutation {m} slipped through every pin"


def test_oracle_restored_after_mutations():
    with oracle.use_library(_mutant_library(2)):
        pass
    P.pin_brute_force_tiny()
