"""Pins of the chained two-stage verify oracle (oracle/chained.py): the
losslessness the HiSpec page claims, checked by exact enumeration of the
output law (every draft tuple, every accept / reject decision and draw cell of
both stages); the reduction to a single verify when the intermediate and the
final layer agree; invalid inputs."""
import itertools
import math

import numpy as np
import pytest

import oracle
from oracle import chained
from oracle_pins import _mid_inside, softmax64


def _enumerate(zf, zi, zd, T):
    """All cases of both stages at cell midpoints, with their probabilities."""
    K, V = zd.shape
    pi = [softmax64(zi[i], T) for i in range(K + 1)]
    qd = [softmax64(zd[i], T) for i in range(K)]
    pf = [softmax64(zf[i], T) for i in range(K + 1)]
    cases = []  # (tokens, u1[K], ur1, u2[K+1], ur2, weight, emitted seq)
    for x in itertools.product(range(V), repeat=K):
        wx = math.prod(qd[i][x[i]] for i in range(K))
        a1 = [min(1.0, pi[i][x[i]] / qd[i][x[i]]) for i in range(K)]
        for n1 in range(K + 1):
            w1 = wx * math.prod(a1[:n1]) * ((1.0 - a1[n1]) if n1 < K else 1.0)
            if w1 <= 0.0:
                continue
            u1 = [_mid_inside(0.0, a1[i]) for i in range(n1)]
            if n1 < K:
                u1 += [_mid_inside(a1[n1], 1.0)] + [0.5] * (K - n1 - 1)
            r1 = np.maximum(0.0, pi[n1] - qd[n1]) if n1 < K else pi[K]
            e1 = np.concatenate([[0.0], np.cumsum(r1) / r1.sum()])
            e1[-1] = 1.0
            for y1 in range(V):
                c1 = e1[y1 + 1] - e1[y1]
                if c1 <= 0.0:
                    continue
                ur1 = _mid_inside(e1[y1], e1[y1 + 1])
                s = list(x[:n1]) + [y1]
                m = n1 + 1
                a2 = [min(1.0, pf[j][s[j]] / pi[j][s[j]]) for j in range(m)]
                for n2 in range(m + 1):
                    w2 = w1 * c1 * math.prod(a2[:n2]) * ((1.0 - a2[n2]) if n2 < m else 1.0)
                    if w2 <= 0.0:
                        continue
                    u2 = [_mid_inside(0.0, a2[j]) for j in range(n2)]
                    if n2 < m:
                        u2 += [_mid_inside(a2[n2], 1.0)]
                    u2 += [0.5] * (K + 1 - len(u2))
                    if n2 == m:
                        cases.append((x, u1, ur1, u2, 0.5, w2, tuple(s)))
                        continue
                    r2 = np.maximum(0.0, pf[n2] - pi[n2])
                    e2 = np.concatenate([[0.0], np.cumsum(r2) / r2.sum()])
                    e2[-1] = 1.0
                    for y2 in range(V):
                        c2 = e2[y2 + 1] - e2[y2]
                        if c2 <= 0.0:
                            continue
                        cases.append((x, u1, ur1, u2, _mid_inside(e2[y2], e2[y2 + 1]), w2 * c2,
                                      tuple(s[:n2]) + (y2,)))
    return cases, pf


def _law_check(seed, K, V, T):
    rng = np.random.default_rng(seed)
    zf = rng.normal(0, 1.5, (K + 1, V)).astype(np.float32)
    zi = (zf + rng.normal(0, 0.8, (K + 1, V))).astype(np.float32)
    zd = (zi[:K] + rng.normal(0, 0.8, (K, V))).astype(np.float32)
    cases, pf = _enumerate(zf, zi, zd, T)
    n = len(cases)
    r = chained.verify_chained(
        np.broadcast_to(zf, (n, K + 1, V)), np.broadcast_to(zi, (n, K + 1, V)),
        np.broadcast_to(zd, (n, K, V)), np.array([c[0] for c in cases], np.int32),
        np.array([c[1] for c in cases], np.float32), np.array([c[2] for c in cases], np.float32),
        np.array([c[3] for c in cases], np.float32), np.array([c[4] for c in cases], np.float32),
        np.full(n, T, np.float32))
    w = np.array([c[5] for c in cases])
    assert abs(w.sum() - 1.0) < 1e-12
    for i, c in enumerate(cases):  # each case emits the sequence its cells say
        e = c[6]
        assert r["num_emitted"][i] == len(e)
        assert tuple(r["out_tokens"][i, :len(e)]) == e and np.all(r["out_tokens"][i, len(e):] == -1)
    # lossless: the emitted token at position i, given the emitted prefix, has law p_f,i
    for i in range(K + 1):
        for prefix in itertools.product(range(V), repeat=i):
            joint = np.zeros(V)
            for c, wc in zip(cases, w):
                e = c[6]
                if len(e) > i and e[:i] == prefix:
                    joint[e[i]] += wc
            if joint.sum() <= 1e-300:
                continue
            assert np.max(np.abs(joint / joint.sum() - pf[i])) < 1e-12, (i, prefix)


@pytest.mark.parametrize("seed,K,V,T", [(1, 1, 4, 1.0), (2, 2, 3, 0.7), (3, 1, 5, 1.3)])
def test_two_stage_output_law_is_the_final_layers(seed, K, V, T):
    _law_check(seed, K, V, T)


def test_equal_intermediate_and_final_reduce_to_one_verify():
    from speculative_sampling_b200 import inputs
    x = inputs.generate("mix_b128_k4_v32000_bf16", B=16, V=2001)
    rng = np.random.default_rng(4)
    u2 = rng.random((16, x.K + 1)).astype(np.float32)
    r = chained.verify_chained(x.target, x.target, x.draft, x.tokens, x.u_accept, x.u_resample,
                               u2, x.u_resample, x.temperature, dtype="bf16")
    v = oracle.verify(x.target, x.draft, x.tokens, x.u_accept, x.u_resample, x.temperature,
                      dtype="bf16", diag=False)
    assert np.array_equal(r["out_tokens"], v["out_tokens"])
    assert np.array_equal(r["num_emitted"], v["num_accepted"] + 1)


def test_invalid_final_row_invalidates():
    from speculative_sampling_b200 import inputs
    x = inputs.generate("tiny_b1_k4_v1000_f32", B=3)
    fin = x.target.copy()
    fin[1, x.K, 5] = np.nan  # even a row past the emitted tokens
    r = chained.verify_chained(fin, x.target, x.draft, x.tokens, x.u_accept, x.u_resample,
                               np.zeros((3, x.K + 1), np.float32), x.u_resample, x.temperature)
    assert r["num_emitted"][1] == -1 and np.all(r["out_tokens"][1] == -1)
    assert r["num_emitted"][0] >= 1


def test_stage2_diagnostics_match_the_verify_oracle():
    """With the intermediate layer equal to the final one, the second stage's
    row statistics are those the C verify oracle computes for the same rows,
    every tested token has p_f = q_i (so it is accepted), and no residual is
    drawn."""
    from speculative_sampling_b200 import inputs
    x = inputs.generate("mix_b128_k4_v32000_bf16", B=12, V=1999)
    rng = np.random.default_rng(7)
    u2 = rng.random((12, x.K + 1)).astype(np.float32)
    r = chained.verify_chained(x.target, x.target, x.draft, x.tokens, x.u_accept, x.u_resample,
                               u2, x.u_resample, x.temperature, dtype="bf16")
    v = oracle.verify(x.target, x.draft, x.tokens, x.u_accept, x.u_resample, x.temperature,
                      dtype="bf16", diag=True)
    ok = v["num_accepted"] >= 0
    K1 = x.K + 1
    assert np.array_equal(r["row_max_f"][ok], v["row_max"][ok, :K1])
    assert np.allclose(r["row_sum_f"][ok], v["row_sum"][ok, :K1], rtol=1e-12, atol=0)
    tested = np.isfinite(r["p2_x"])
    assert np.array_equal(tested[ok].sum(axis=1), v["num_accepted"][ok] + 1)
    assert np.allclose(r["p2_x"][tested], r["q2_x"][tested], rtol=1e-12, atol=0)
    assert np.all(np.isnan(r["Z2"]))
