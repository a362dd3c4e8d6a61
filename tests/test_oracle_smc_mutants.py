"""Planted mistakes in the SMC-SD oracle must each fail some pin of
tests/test_oracle_smc.py (the mutant is installed by monkeypatching oracle.smc
for the duration of one check)."""
import numpy as np
import pytest

import test_oracle_smc as pins
from oracle import smc

_orig_log_softmax_at = smc.log_softmax_at
_orig_systematic = smc.systematic
_orig_smc_step = smc.smc_step


def _ratio_inverted(*a, **k):
    r = _orig_smc_step(*a, **k)
    r = dict(r)
    r["dlogw"] = np.where(np.isfinite(r["dlogw"]), -r["dlogw"], r["dlogw"])
    return r


def _no_temperature(z, T, x):
    return _orig_log_softmax_at(z, 1.0, x)


def _targets_shifted(wbar, u):
    N = wbar.size
    C = np.cumsum(wbar)
    t = (np.arange(N) + 1.0 + float(u)) / N
    a = np.searchsorted(C, t, side="right")
    return np.minimum(a, N - 1).astype(np.int64)


def _weak_inequality(wbar, u):
    N = wbar.size
    C = np.cumsum(wbar)
    t = (np.arange(N) + float(u)) / N
    return np.minimum(np.searchsorted(C, t, side="left"), N - 1).astype(np.int64)


MUTANTS = {
    "ratio q/p instead of p/q": ("smc_step", _ratio_inverted),
    "temperature dropped": ("log_softmax_at", _no_temperature),
    "resampling targets (k+1+u)/N": ("systematic", _targets_shifted),
    "C_j >= target instead of >": ("systematic", _weak_inequality),
}
PINS = [getattr(pins, n) for n in dir(pins) if n.startswith("test_")]


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name, monkeypatch):
    attr, fn = MUTANTS[name]
    monkeypatch.setattr(smc, attr, fn)
    caught = []
    for pin in PINS:
        try:
            pin()
        except AssertionError:
            caught.append(pin.__name__)
    assert caught, f"no pin catches the mutant '{name}'"
