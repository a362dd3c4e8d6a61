"""Planted mistakes in the chained two-stage verify oracle (oracle/chained.py)
must each fail its exact-enumeration losslessness pin.  Each mutant is a
textual edit of the module's source, loaded as a separate module; the real
oracle is untouched."""
import importlib.util
import os
import sys

import pytest

import test_oracle_chained as pins
from oracle import chained

MUTANTS = {
    # stage 2 draws from the final layer's row instead of max(0, p_f - q_i)
    "stage2_draws_from_final_row": ("r = np.maximum(0.0, p - q)", "r = p"),
    # stage 2 accepts with q_i / p_f instead of p_f / q_i
    "stage2_ratio_inverted": ("if not (u2[b, j] * q[tok] < p[tok]):",
                              "if not (u2[b, j] * p[tok] < q[tok]):"),
    # the token stage 1 drew is emitted without being verified against L_f
    "last_stage1_token_not_reverified": ("for j in range(m):", "for j in range(m - 1):"),
}


def _load_mutant(name, old, new, tmp_path):
    src = open(chained.__file__).read()
    assert src.count(old) == 1, f"mutation site for {name} not found exactly once"
    path = os.path.join(tmp_path, f"chained_{name}.py")
    with open(path, "w") as f:
        f.write(src.replace(old, new))
    spec = importlib.util.spec_from_file_location(f"oracle.chained_{name}", path,
                                                  submodule_search_locations=None)
    mod = importlib.util.module_from_spec(spec)
    mod.__package__ = "oracle"  # its relative imports resolve inside the oracle package
    sys.modules[spec.name] = mod
    spec.loader.exec_module(mod)
    return mod


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_chained_mutant_is_caught(name, tmp_path, monkeypatch):
    old, new = MUTANTS[name]
    mod = _load_mutant(name, old, new, str(tmp_path))
    monkeypatch.setattr(pins.chained, "verify_chained", mod.verify_chained)
    caught = False
    for seed, K, V, T in [(1, 1, 4, 1.0), (2, 2, 3, 0.7), (3, 1, 5, 1.3)]:
        try:
            pins._law_check(seed, K, V, T)
        except AssertionError:
            caught = True
            break
    assert caught, f"the losslessness pin misses the mutant '{name}'"
