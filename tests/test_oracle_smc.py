"""Pins of the SMC-SD weight-step oracle (oracle/smc.py) to facts that do not
come from its own formulas: an importance-sampling identity checked by
exhaustive enumeration, hand-worked resampling cases, the defining property of
systematic resampling, its unbiasedness, agreement of the bonus draw with the
verify oracle (a separate C implementation), and invariances.  Each check is
chosen so that a plausible slip (p/q inverted, temperature on one model only,
an off-by-one in the resampling targets, a weak ">=") fails it."""
import numpy as np
import pytest

import oracle
from oracle import smc
from speculative_sampling_b200 import inputs


def _softmax(z, T):
    e = np.exp((z - z.max()) / T)
    return e / e.sum()


def test_importance_ratio_has_mean_one_under_the_draft():
    # E_{x ~ q}[exp(dlogw)] = sum_x q(x) p(x)/q(x) = 1, for every position:
    # enumerate all V tokens of a K = 1 round (one particle per token)
    rng = np.random.default_rng(5)
    V, T = 6, float(np.float32(0.8))  # the temperature is an fp32 input
    zt = rng.normal(0, 2, (1, 2, V)).astype(np.float32)
    zd = (zt[:, :1] + rng.normal(0, 1, (1, 1, V))).astype(np.float32)
    B = V
    tg = np.repeat(zt, B, 0)
    dr = np.repeat(zd, B, 0)
    tok = np.arange(V, dtype=np.int32)[:, None]
    r = smc.smc_step(tg, dr, tok, np.full(B, 0.5, np.float32), np.full(B, T, np.float32), None,
                     np.zeros(B // V, np.float32), 0.0, N=V)
    q = _softmax(zd[0, 0].astype(np.float64), T)
    assert abs(np.sum(q * np.exp(r["dlogw"])) - 1.0) < 1e-12
    # and E_{x ~ p}[exp(-dlogw)] = 1 (the ratio is p/q, not q/p)
    p = _softmax(zt[0, 0].astype(np.float64), T)
    assert abs(np.sum(p * np.exp(-r["dlogw"])) - 1.0) < 1e-12


def test_equal_models_give_equal_weights_and_no_resampling():
    x = inputs.generate("mix_b128_k4_v32000_bf16", B=8, V=501)
    x.draft[:] = x.target[:, :x.K]
    r = smc.smc_step(x.target, x.draft, x.tokens, x.u_resample, x.temperature, None,
                     np.array([0.3], np.float32), 0.99, N=8, dtype="bf16")
    assert np.all(r["dlogw"] == 0.0)
    assert r["ess"][0] == 8.0 and not r["resampled"][0]
    assert np.array_equal(r["ancestors"], np.arange(8))


def test_hand_worked_resampling_case():
    # normalised weights [1/2, 1/4, 1/4]: ESS = 1/(1/4 + 1/16 + 1/16) = 8/3;
    # targets (k + 0.1)/3 = 0.0333, 0.3667, 0.7 against C = [0.5, 0.75, 1]
    # give ancestors [0, 0, 1]
    wbar = np.array([0.5, 0.25, 0.25])
    assert np.array_equal(smc.systematic(wbar, 0.1), [0, 0, 1])
    assert np.array_equal(smc.systematic(wbar, 0.8), [0, 1, 2])  # 0.267, 0.6, 0.933
    # a target exactly on a running-sum value goes to the next particle (">")
    assert np.array_equal(smc.systematic(np.array([0.25, 0.25, 0.25, 0.25]), 0.0), [0, 1, 2, 3])
    lw = np.log(wbar) + 3.0
    B, V, K = 3, 4, 1
    z = np.zeros((B, K + 1, V), np.float32)
    tok = np.zeros((B, K), np.int32)
    r = smc.smc_step(z, z[:, :K], tok, np.full(B, 0.5, np.float32), np.ones(B, np.float32), lw,
                     np.array([0.1], np.float32), 1.0, N=3)
    assert abs(r["ess"][0] - 8.0 / 3.0) < 1e-12
    assert r["resampled"][0] and np.array_equal(r["ancestors"], [0, 0, 1])
    assert np.all(r["logw"] == 0.0)
    r = smc.smc_step(z, z[:, :K], tok, np.full(B, 0.5, np.float32), np.ones(B, np.float32), lw,
                     np.array([0.1], np.float32), 0.5, N=3)  # 8/3 >= 1.5: keep
    assert not r["resampled"][0] and np.allclose(r["logw"], lw)


def test_systematic_counts_are_floor_or_ceil():
    # the defining property of systematic resampling: particle j is copied
    # floor(N wbar_j) or ceil(N wbar_j) times, for any u
    rng = np.random.default_rng(9)
    for trial in range(300):
        N = int(rng.integers(2, 40))
        w = rng.gamma(0.3, 1.0, N) * (rng.random(N) < 0.8)
        if w.sum() == 0:
            continue
        wbar = w / w.sum()
        a = smc.systematic(wbar, float(rng.random()))
        cnt = np.bincount(a, minlength=N)
        assert np.all(cnt >= np.floor(N * wbar - 1e-9)) and np.all(cnt <= np.ceil(N * wbar + 1e-9))
        assert np.all(cnt[wbar == 0] == 0)


def test_systematic_is_unbiased_over_u():
    # E_u[count_j] = N wbar_j: average over a fine grid of u
    wbar = np.array([0.05, 0.4, 0.15, 0.0, 0.3, 0.1])
    N = wbar.size
    us = (np.arange(20000) + 0.5) / 20000
    mean = np.mean([np.bincount(smc.systematic(wbar, u), minlength=N) for u in us], axis=0)
    assert np.allclose(mean, N * wbar, atol=1e-3)


def test_bonus_draw_agrees_with_the_verify_oracle():
    # with draft == target every token is accepted and the verify oracle (C)
    # draws its bonus from p_K with u_resample: the same token as here
    x = inputs.generate("large_b256_k8_v151936_f32", B=6, K=3, V=2003)
    x.draft[:] = x.target[:, :x.K]
    v = oracle.verify(x.target, x.draft, x.tokens, x.u_accept, x.u_resample, x.temperature,
                      dtype="f32", diag=False)
    r = smc.smc_step(x.target, x.draft, x.tokens, x.u_resample, x.temperature, None,
                     np.array([0.5, 0.5], np.float32), 0.0, N=3)
    assert np.all(v["num_accepted"] == x.K)
    assert np.array_equal(r["out_tokens"], v["out_tokens"])


def test_temperature_applies_to_both_models():
    # scaling every logit and T by the same factor changes nothing
    x = inputs.generate("tiny_b1_k4_v1000_f32", B=4)
    args = (x.tokens, x.u_resample, x.temperature)
    r1 = smc.smc_step(x.target, x.draft, *args, None, np.array([0.2], np.float32), 0.5, N=4)
    r2 = smc.smc_step(x.target * 2, x.draft * 2, x.tokens, x.u_resample, x.temperature * 2,
                      None, np.array([0.2], np.float32), 0.5, N=4)
    assert np.allclose(r1["dlogw"], r2["dlogw"], rtol=1e-12, atol=1e-12)
    assert np.array_equal(r1["ancestors"], r2["ancestors"])
    # while scaling only the draft's logits changes the weights
    r3 = smc.smc_step(x.target, x.draft * 2, *args, None, np.array([0.2], np.float32), 0.5, N=4)
    assert not np.allclose(r1["dlogw"], r3["dlogw"])


def test_invalid_particles_get_zero_weight():
    x = inputs.generate("tiny_b1_k4_v1000_f32", B=4)
    x.tokens[1, 2] = 1000
    r = smc.smc_step(x.target, x.draft, x.tokens, x.u_resample, x.temperature, None,
                     np.array([0.2], np.float32), 1.0, N=4)
    assert r["dlogw"][1] == -np.inf and np.all(r["out_tokens"][1] == -1)
    assert np.all(r["ancestors"] != 1)  # weight 0 is never drawn
