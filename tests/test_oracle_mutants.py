"""Plant plausible mistakes in copies of the CPU oracle and check that the pins
catch every one of them.  Each mutant is a textual edit of oracle.c compiled
into a temporary library; the real oracle is untouched."""
import os

import pytest

import oracle
import oracle_pins as P

MUTANTS = {
    "accept_ratio_inverted": ("if (!(u * q < p))", "if (!(u * p < q))"),
    "accept_same_uniform_every_position": ("(double)j->u_accept[b * K + i]",
                                           "(double)j->u_accept[b * K]"),
    "residual_sign_flipped": ("r[v] = (p - q > 0.0) ? p - q : 0.0;",
                              "r[v] = (q - p > 0.0) ? q - p : 0.0;"),
    "residual_without_clamp": ("r[v] = (p - q > 0.0) ? p - q : 0.0;", "r[v] = p;"),
    "residual_from_first_row": ("double p = prob(j->target, j->dtype, toff[n], v, M[n], S[n], T);",
                                "double p = prob(j->target, j->dtype, toff[0], v, M[0], S[0], T);"),
    "bonus_from_row_K_minus_1": ("toff[K], v, M[K], S[K], T);",
                                 "toff[K - 1], v, M[K - 1], S[K - 1], T);"),
    "no_temperature_on_draft": (": row_sum(j->draft, j->dtype, doff[r - K - 1], V, M[r], T);",
                                ": row_sum(j->draft, j->dtype, doff[r - K - 1], V, M[r], 1.0);"),
    "no_temperature_on_draft_prob": ("x, M[K + 1 + i], S[K + 1 + i], T);",
                                     "x, M[K + 1 + i], S[K + 1 + i], 1.0);"),
    "inverse_cdf_off_by_one": ("if (C > t) {", "if (Cprev > t) {"),
    "inverse_cdf_unscaled_uniform": ("const double t = (double)j->u_resample[b] * Z;",
                                     "const double t = (double)j->u_resample[b];"),
    "no_stop_at_first_rejection": ("      n = i;\n      break;", "      n = i;\n      continue;"),
    "tail_not_padded": ("for (int i = n + 1; i <= K; ++i) out[i] = -1;", ""),
    "zero_residual_draws_from_bonus_row": (
        "r[v] = prob(j->target, j->dtype, toff[n], v, M[n], S[n], T);",
        "r[v] = prob(j->target, j->dtype, toff[K], v, M[K], S[K], T);"),
    "zero_residual_not_handled": ("if (Z == 0.0) { /* only reachable", "if (0) { /* only reachable"),
    "no_cell_reached_takes_last_index": ("      if (r[v] > 0.0) {\n        y = v;",
                                         "      if (1) {\n        y = v;"),
    "no_cell_reached_takes_first_positive": ("for (int64_t v = V - 1; v >= 0; --v)\n      if (r[v] > 0.0)",
                                             "for (int64_t v = 0; v < V; ++v)\n      if (r[v] > 0.0)"),
    "bf16_misread": ("uint32_t bits = (uint32_t)((const uint16_t *)base)[idx] << 16;",
                     "uint32_t bits = (uint32_t)((const uint16_t *)base)[idx] << 15;"),
}

# the Monte-Carlo check is the slowest; the exact checks run first
CHECKS = [c for c in P.ALL_CHECKS if c is not P.check_chi_square] + [P.check_chi_square]


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(tmp_path, name):
    old, new = MUTANTS[name]
    src = open(oracle.SRC).read()
    assert src.count(old) == 1, f"mutation site for {name} not found exactly once"
    path = os.path.join(tmp_path, "mutant.c")
    with open(path, "w") as f:
        f.write(src.replace(old, new))
    lib = oracle.build(path, os.path.join(tmp_path, "libmutant.so"))
    mutant = oracle.Oracle(lib)
    caught = []
    for check in CHECKS:
        try:
            check(mutant)
        except AssertionError:
            caught.append(check.__name__)
            break
    assert caught, f"mutant {name} passed every pin"
