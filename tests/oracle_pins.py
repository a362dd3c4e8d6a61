"""Checks that pin the fp64 CPU oracle to facts fixed by the pages and by the
mathematics, not by the oracle itself.

Each ``check_*`` takes an ``oracle.Oracle`` (the real one, or a deliberately
broken copy built by test_oracle_mutants.py) and raises AssertionError when the
oracle disagrees with the fact it checks.

Facts used:
  * exactness (speculative decoding blog, section "The mathematical definition
    from Leviathan et al.": the algorithm returns exactly the target's output
    distribution, no approximation): the oracle's output law, computed by exact
    enumeration over every draft tuple and every cell of the uniforms, equals
    softmax(z/T) of the target rows;
  * P(accept at i) = sum_x q(x) min(1, p(x)/q(x)) = sum_x min(p(x), q(x)), and
    the residual mass Z = sum max(0, p - q) = 1 - sum min(p, q);
  * E[accepted] = sum_{i=1..K} prod_{j<i} a_j (acceptance compounds across
    positions, blog section "Working code on vLLM 0.6+", the note on K);
  * draft == target: every draft token is accepted and the bonus token is the
    textbook inverse-CDF sample of the target's last row (numpy cumsum +
    searchsorted);
  * a chi-square Monte-Carlo test of the law with 10^6 draws;
  * hand-derived worked cases (tests/golden/hand_cases.json);
  * closed forms of the softmax normaliser, exact bf16 widening, temperature
    scaling invariance, invalid-input handling.
"""
from __future__ import annotations

import itertools
import json
import math
import os

import numpy as np

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "hand_cases.json")


def softmax64(z32: np.ndarray, T: float) -> np.ndarray:
    """Textbook softmax(z/T) in fp64 of fp32 logits (exact widening)."""
    z = np.asarray(z32, dtype=np.float32).astype(np.float64)
    e = np.exp((z - z.max()) / float(np.float32(T)))
    return e / e.sum()


def _call(orc, zt, zd, tokens, u_acc, u_res, T, diag=True):
    """One oracle call where every case shares the same logit rows."""
    n = len(tokens)
    K1, V = zt.shape
    tgt = np.broadcast_to(zt.astype(np.float32), (n, K1, V))
    drf = np.broadcast_to(zd.astype(np.float32), (n, K1 - 1, V))
    return orc.verify(tgt, drf, np.asarray(tokens, np.int32), np.asarray(u_acc, np.float32),
                      np.asarray(u_res, np.float32), np.full(n, T, np.float32), dtype="f32",
                      diag=diag)


def _mid_inside(lo: float, hi: float) -> float:
    """fp32 midpoint of [lo, hi), checked to lie strictly inside the cell."""
    m = float(np.float32(0.5 * (lo + hi)))
    assert lo < m < hi, (lo, m, hi)
    return m


def enumerate_law(orc, zt: np.ndarray, zd: np.ndarray, T: float):
    """Exact output law of the oracle for fixed rows.

    Enumerates every draft tuple x in V^K (weight prod q_i(x_i)), every reject
    position n (weight prod_{i<n} alpha_i * (1 - alpha_n)), and every cell of
    the draw's uniform (weight = cell width).  The oracle is called once per
    combination at the cell midpoints.  Returns (cases, weights, outputs)."""
    K = zd.shape[0]
    V = zd.shape[1]
    p = [softmax64(zt[i], T) for i in range(K + 1)]
    q = [softmax64(zd[i], T) for i in range(K)]
    toks, uacc, ures, wts, meta = [], [], [], [], []
    for x in itertools.product(range(V), repeat=K):
        wx = math.prod(q[i][x[i]] for i in range(K))
        alpha = [min(1.0, p[i][x[i]] / q[i][x[i]]) for i in range(K)]
        for n in range(K + 1):
            w = wx * math.prod(alpha[:n])
            if n < K:
                w *= 1.0 - alpha[n]
            if w <= 0.0:
                continue
            ua = [_mid_inside(0.0, alpha[i]) for i in range(n)]
            if n < K:
                ua.append(_mid_inside(alpha[n], 1.0))
                ua += [0.5] * (K - n - 1)
            r = np.maximum(0.0, p[n] - q[n]) if n < K else p[K]
            edges = np.concatenate([[0.0], np.cumsum(r) / r.sum()])
            edges[-1] = 1.0
            for j in range(V):
                width = edges[j + 1] - edges[j]
                if width <= 0.0:
                    continue
                toks.append(x)
                uacc.append(ua)
                ures.append(_mid_inside(edges[j], edges[j + 1]))
                wts.append(w * width)
                meta.append((x, n, j))
    res = _call(orc, zt, zd, toks, uacc, ures, T)
    return meta, np.array(wts), res, p, q


def check_enumerated_law(orc, zt, zd, T, tol=1e-12):
    K = zd.shape[0]
    V = zd.shape[1]
    meta, w, res, p, q = enumerate_law(orc, zt, zd, T)
    out = res["out_tokens"]
    nacc = res["num_accepted"]
    assert abs(w.sum() - 1.0) < tol
    # the walk stops where the uniforms say it must, and emits the cell's token
    for c, (x, n, j) in enumerate(meta):
        assert nacc[c] == n, ("accept/reject decision", x, n, nacc[c])
        assert list(out[c, :n]) == list(x[:n]), "accepted tokens"
        assert out[c, n] == j, ("drawn token", x, n, j, out[c, n])
        assert all(out[c, n + 1:] == -1), "tail padding"
    # emitted token at position i given the emitted prefix: law = p_i
    emitted = [[(x[i] if n > i else j) for i in range(n + 1)] for (x, n, j) in meta]
    for i in range(K + 1):
        for prefix in itertools.product(range(V), repeat=i):
            joint = np.zeros(V)
            for c, e in enumerate(emitted):
                if len(e) > i and tuple(e[:i]) == prefix:
                    joint[e[i]] += w[c]
            tot = joint.sum()
            if tot <= 1e-300:
                continue
            assert np.max(np.abs(joint / tot - p[i])) < tol, ("law at position", i, prefix,
                                                              joint / tot, p[i])
    # acceptance probability and E[n]
    a = [np.minimum(p[i], q[i]).sum() for i in range(K)]
    reach = [w[[k for k, m in enumerate(meta) if m[1] >= i]].sum() for i in range(K + 1)]
    for i in range(K):
        assert abs(reach[i + 1] / reach[i] - a[i]) < tol, ("P(accept)", i)
    En = float(np.dot(w, [m[1] for m in meta]))
    En_closed = sum(math.prod(a[:i]) for i in range(1, K + 1))
    assert abs(En - En_closed) < tol, ("E[n]", En, En_closed)
    # residual mass identity Z = 1 - sum min(p, q) at the rejection row
    for c, (x, n, j) in enumerate(meta):
        if n < K:
            assert abs(res["Z"][c] - (1.0 - a[n])) < tol, ("Z", n)
        else:
            assert abs(res["Z"][c] - 1.0) < tol
    # diagnostic acceptance probabilities
    assert np.max(np.abs(res["accept_prob"][0] - np.array(a))) < tol


def law_rows(seed: int, K: int, V: int, T: float, spread: float = 1.5):
    rng = np.random.default_rng(seed)
    zt = (spread * rng.standard_normal((K + 1, V))).astype(np.float32)
    zd = (zt[:K] + 0.8 * rng.standard_normal((K, V))).astype(np.float32)
    return zt, zd


def hand_rows(T: float):
    """A hand-chosen pair of rows with a clear disagreement."""
    pt = np.array([[0.4, 0.3, 0.2, 0.1], [0.1, 0.2, 0.3, 0.4], [0.25, 0.25, 0.25, 0.25]])
    pd = np.array([[0.1, 0.2, 0.3, 0.4], [0.45, 0.1, 0.1, 0.35]])
    return (T * np.log(pt)).astype(np.float32), (T * np.log(pd)).astype(np.float32)


def check_law_suite(orc):
    zt, zd = hand_rows(1.0)
    check_enumerated_law(orc, zt, zd, 1.0)
    zt, zd = hand_rows(0.7)
    check_enumerated_law(orc, zt, zd, 0.7)
    for seed, K, V, T in [(1, 1, 6, 1.0), (2, 2, 5, 0.7), (3, 3, 4, 1.3), (4, 3, 6, 1.0)]:
        zt, zd = law_rows(seed, K, V, T)
        check_enumerated_law(orc, zt, zd, T)


def check_identities_random(orc, n_rows=40, V=50, tol=1e-12):
    """Z = 1 - sum min(p,q) after a forced rejection and the acceptance
    diagnostic sum min(p,q), on random rows of a larger vocabulary."""
    rng = np.random.default_rng(11)
    for _ in range(n_rows):
        T = float(rng.choice([0.3, 0.7, 1.0, 1.3]))
        zt = (2.0 * rng.standard_normal((2, V))).astype(np.float32)
        zd = (zt[:1] + rng.standard_normal((1, V))).astype(np.float32)
        p, q = softmax64(zt[0], T), softmax64(zd[0], T)
        x = int(np.argmax(q / p))  # alpha = p/q < 1 here
        alpha = p[x] / q[x]
        u = float(np.float32(0.5 * (alpha + 1.0)))
        res = _call(orc, zt, zd, [[x]], [[u]], [0.5], T)
        assert res["num_accepted"][0] == 0
        a = np.minimum(p, q).sum()
        assert abs(res["Z"][0] - (1.0 - a)) < tol
        assert abs(res["accept_prob"][0, 0] - a) < tol
        assert abs(res["p_x"][0, 0] - p[x]) < tol * 10 and abs(res["q_x"][0, 0] - q[x]) < tol * 10


def check_equal_rows_reduce_to_inverse_cdf(orc, n=2000):
    """draft == target: n = K for every uniform, and the bonus token is numpy's
    inverse-CDF sample of the target's row K."""
    rng = np.random.default_rng(5)
    K, V, T = 3, 37, 0.8
    zt = (2.0 * rng.standard_normal((K + 1, V))).astype(np.float32)
    zd = zt[:K].copy()
    toks = rng.integers(0, V, size=(n, K))
    ua = rng.random((n, K)).astype(np.float32)
    ur = rng.random(n).astype(np.float32)
    res = _call(orc, zt, zd, toks, ua, ur, T)
    assert np.all(res["num_accepted"] == K)
    assert np.array_equal(res["out_tokens"][:, :K], toks)
    pK = softmax64(zt[K], T)
    cdf = np.cumsum(pK)
    y = np.searchsorted(cdf, ur.astype(np.float64) * cdf[-1], side="right")
    assert np.array_equal(res["out_tokens"][:, K], y)


def check_chi_square(orc, N=1_000_000, chunks=5, pmin=1e-4):
    """Monte-Carlo law at V=8, K=2 with 10^6 draws: the emitted token at
    position 0, and at position 1 given an accepted x_0, follow the target."""
    from scipy import stats
    rng = np.random.default_rng(2024)
    K, V, T = 2, 8, 0.8
    zt = (1.2 * rng.standard_normal((K + 1, V))).astype(np.float32)
    zd = (zt[:K] + 0.9 * rng.standard_normal((K, V))).astype(np.float32)
    p = [softmax64(zt[i], T) for i in range(K + 1)]
    q = [softmax64(zd[i], T) for i in range(K)]
    h0 = np.zeros(V)
    v0 = int(np.argmax(np.minimum(p[0], q[0])))
    h1 = np.zeros(V)
    for _ in range(chunks):
        m = N // chunks
        toks = np.stack([rng.choice(V, size=m, p=q[i]) for i in range(K)], axis=1)
        k = rng.integers(0, 1 << 24, size=(m, K + 1))
        u = (k * 2.0 ** -24).astype(np.float32)
        res = _call(orc, zt, zd, toks, u[:, :K], u[:, K], T, diag=False)
        out, n = res["out_tokens"], res["num_accepted"]
        h0 += np.bincount(out[:, 0], minlength=V)
        sel = (n >= 1) & (out[:, 0] == v0)
        h1 += np.bincount(out[sel, 1], minlength=V)
    for h, pi in ((h0, p[0]), (h1, p[1])):
        pv = stats.chisquare(h, h.sum() * pi).pvalue
        assert pv > pmin, ("chi-square", pv)


def check_hand_cases(orc, tol=1e-6):
    with open(GOLDEN) as f:
        cases = json.load(f)["cases"]
    for c in cases:
        T = float(c["T"])
        zt = (T * np.log(np.array(c["target"]))).astype(np.float32)
        zd = (T * np.log(np.array(c["draft"]))).astype(np.float32)
        res = _call(orc, zt, zd, [c["tokens"]], [c["u_accept"]], [c["u_resample"]], T)
        assert list(res["out_tokens"][0]) == c["expect_tokens"], c["name"]
        assert res["num_accepted"][0] == c["expect_n"], c["name"]
        n = c["expect_n"]
        reached = min(n + 1, len(c["tokens"]))
        assert np.allclose(res["p_x"][0, :reached], c["expect_p_x"][:reached], rtol=tol), c["name"]
        assert np.allclose(res["q_x"][0, :reached], c["expect_q_x"][:reached], rtol=tol), c["name"]
        assert abs(res["Z"][0] - c["expect_Z"]) < tol, c["name"]


def check_normaliser_closed_forms(orc):
    # all-equal logits: max is the value, S = V exactly
    V = 1000
    zt = np.full((2, V), 3.25, np.float32)
    zd = np.full((1, V), -1.5, np.float32)
    res = _call(orc, zt, zd, [[7]], [[0.5]], [0.5], 0.9)
    assert np.all(res["row_max"][0] == [3.25, 3.25, -1.5])
    assert np.all(res["row_sum"][0] == V)
    assert res["num_accepted"][0] == 1 and res["out_tokens"][0, 1] == int(0.5 * V)
    # logits (0, -1, -2) at T = 1: S = 1 + e^-1 + e^-2
    zt = np.array([[0.0, -1.0, -2.0], [-2.0, -1.0, 0.0]], np.float32)
    res = _call(orc, zt, zt[:1], [[0]], [[0.5]], [0.5], 1.0)
    s = 1.0 + math.exp(-1.0) + math.exp(-2.0)
    assert abs(res["row_sum"][0, 0] - s) < 1e-15 and abs(res["row_sum"][0, 1] - s) < 1e-15
    # T = 2 on logits (0, -2): S = 1 + e^-1
    zt = np.array([[0.0, -2.0], [0.0, -2.0]], np.float32)
    res = _call(orc, zt, zt[:1], [[0]], [[0.5]], [0.5], 2.0)
    assert abs(res["row_sum"][0, 0] - (1.0 + math.exp(-1.0))) < 1e-15


def check_bf16_widening(orc):
    """bf16 bit patterns are read exactly: 0x3F80 = 1, 0x3F81 = 1 + 2^-7,
    0xC000 = -2; the verify on bf16 equals the verify on the widened fp32."""
    bits = np.array([[0x3F80, 0x3F81, 0xC000], [0x0000, 0x4000, 0xBF80]], np.uint16)
    f32 = np.array([[1.0, 1.0 + 2 ** -7, -2.0], [0.0, 2.0, -1.0]], np.float32)
    r_b = orc.verify(np.ascontiguousarray(bits[None]), np.ascontiguousarray(bits[None, :1]),
                     np.array([[1]]), np.array([[0.6]]), np.array([0.4]), np.array([1.0]),
                     dtype="bf16")
    r_f = orc.verify(f32[None], f32[None, :1], np.array([[1]]), np.array([[0.6]]),
                     np.array([0.4]), np.array([1.0]), dtype="f32")
    assert r_b["row_max"][0, 0] == 1.0 + 2 ** -7 and r_b["row_max"][0, 1] == 2.0
    for k in ("out_tokens", "num_accepted", "row_sum", "p_x", "q_x", "Z"):
        assert np.array_equal(r_b[k], r_f[k]), k


def check_temperature_scaling(orc):
    """Scaling every logit and T by the same power of two changes nothing."""
    from speculative_sampling_b200 import inputs
    x = inputs.generate("tiny_b1_k4_v1000_f32", B=64)
    r1 = orc.verify(x.target, x.draft, x.tokens, x.u_accept, x.u_resample, x.temperature)
    r2 = orc.verify(x.target * 4, x.draft * 4, x.tokens, x.u_accept, x.u_resample,
                    x.temperature * 4)
    assert np.array_equal(r1["out_tokens"], r2["out_tokens"])
    assert np.array_equal(r1["num_accepted"], r2["num_accepted"])
    # and dropping T changes results on this workload (T = 1 here, so use 0.5)
    r3 = orc.verify(x.target, x.draft, x.tokens, x.u_accept, x.u_resample, x.temperature * 0.5)
    assert not np.array_equal(r1["out_tokens"], r3["out_tokens"])


def check_invalid_inputs(orc):
    K, V = 2, 6
    rng = np.random.default_rng(3)
    zt = rng.standard_normal((K + 1, V)).astype(np.float32)
    zd = rng.standard_normal((K, V)).astype(np.float32)

    def run(zt_, zd_, toks, T=1.0):
        return _call(orc, zt_, zd_, [toks], [[0.5, 0.5]], [0.5], T)

    ok = run(zt, zd, [1, 2])
    assert ok["num_accepted"][0] >= 0
    for toks in ([V, 0], [0, -1]):
        r = run(zt, zd, toks)
        assert r["num_accepted"][0] == -1 and np.all(r["out_tokens"][0] == -1)
    for T in (0.0, -1.0, float("nan"), float("inf")):
        r = run(zt, zd, [1, 2], T)
        assert r["num_accepted"][0] == -1
    for bad in (np.nan, np.inf):
        z2 = zt.copy()
        z2[2, 3] = bad  # even the bonus row, which this draw may not reach
        assert run(z2, zd, [1, 2])["num_accepted"][0] == -1
    z3 = zd.copy()
    z3[1, :] = -np.inf
    assert run(zt, z3, [1, 2])["num_accepted"][0] == -1
    # -inf entries in an otherwise valid row are legal (probability zero)
    z4 = zt.copy()
    z4[0, 0] = -np.inf
    assert run(z4, zd, [1, 2])["num_accepted"][0] >= 0


def check_diagnostics_do_not_change_results(orc):
    """Outputs with and without the diagnostic arrays are identical (T != 1)."""
    from speculative_sampling_b200 import inputs
    x = inputs.generate("mix_b128_k4_v32000_bf16", B=32, V=2000)
    r1 = orc.verify(x.target, x.draft, x.tokens, x.u_accept, x.u_resample, x.temperature,
                    diag=True)
    r0 = orc.verify(x.target, x.draft, x.tokens, x.u_accept, x.u_resample, x.temperature,
                    diag=False)
    assert np.array_equal(r1["out_tokens"], r0["out_tokens"])
    assert np.array_equal(r1["num_accepted"], r0["num_accepted"])


def check_thread_invariance(orc):
    from speculative_sampling_b200 import inputs
    x = inputs.generate("mix_b128_k4_v32000_bf16", B=24, V=3000)
    r1 = orc.verify(x.target, x.draft, x.tokens, x.u_accept, x.u_resample, x.temperature,
                    nthreads=1)
    r8 = orc.verify(x.target, x.draft, x.tokens, x.u_accept, x.u_resample, x.temperature,
                    nthreads=8)
    for k in r1:
        assert np.array_equal(r1[k], r8[k], equal_nan=True), k


def check_zero_residual_draws_from_target_row(orc):
    """Z = 0 after a rejection (reachable only through rounding) draws from p_n.

    Draft row 0 equals target row 0, so p_0 = q_0 exactly; the draft token's
    logit is so low that p_0(x) = q_0(x) = 0 in fp64, so u*q < p fails and the
    walk rejects at n = 0.  The residual max(0, p_0 - q_0) is then zero
    everywhere.  The reading for this case draws from p_0 itself; the result must
    be numpy's inverse CDF of p_0 (cumsum + searchsorted, side='right'), not a
    draw from another row, and not -1."""
    T = 1.0
    z0 = np.array([0.3, -0.2, 1.1, 0.0, -0.7, -1000.0], np.float32)
    zt = np.stack([z0, np.array([2.0, -1.0, 0.5, 0.1, 0.0, 1.5], np.float32),
                   np.array([-0.5, 0.9, 0.2, 3.0, -2.0, 0.4], np.float32)])
    zd = np.stack([z0, zt[1] + np.float32(0.5)])
    us = [0.0, 0.1, 0.35, 0.6, 0.9, 0.999]
    res = _call(orc, zt, zd, [[5, 0]] * len(us), [[0.5, 0.5]] * len(us), us, T)
    p0 = softmax64(zt[0], T)
    assert p0[5] == 0.0  # the draft token has probability 0 in both rows
    cdf = np.cumsum(p0)
    want = np.searchsorted(cdf, np.asarray(us, np.float64) * cdf[-1], side="right")
    assert np.all(res["num_accepted"] == 0)
    assert np.array_equal(res["out_tokens"][:, 0], want), (res["out_tokens"][:, 0], want)
    assert np.all(res["out_tokens"][:, 1:] == -1)
    assert np.allclose(res["Z"], 1.0, rtol=0, atol=1e-12)  # mass of p_0
    assert np.all(res["margin_sample"] == 0.0)             # counted as a boundary draw


def check_no_cell_reached_takes_last_positive(orc):
    """When no running sum exceeds u*Z (u = 1 reaches this exactly: t equals the
    total), the draw is the largest index with positive weight: the limit of the
    inverse CDF as u -> 1.  Checked on a bonus row and on a residual whose last
    entries have zero weight, against the draw at the largest fp32 uniform below
    1 (whose cell is the same last positive one)."""
    T = 1.0
    V = 8
    # bonus draw: draft = target, every token accepted; p_1 is zero on 6, 7
    zb = np.array([[0.1, 0.4, -0.3, 0.8, 0.0, 0.2, -np.inf, -np.inf],
                   [0.5, -0.1, 0.3, 0.0, 0.9, 0.2, -np.inf, -np.inf]], np.float32)
    u_top = float(np.float32(1.0) - np.float32(2.0 ** -24))
    res = _call(orc, zb, zb[:1], [[3], [3]], [[0.5], [0.5]], [1.0, u_top], T)
    assert np.all(res["num_accepted"] == 1)
    assert list(res["out_tokens"][:, 1]) == [5, 5], res["out_tokens"]
    # residual draw: p - q is positive only on tokens 0 and 2 (so index 2 is last)
    pt = np.array([0.30, 0.05, 0.25, 0.10, 0.10, 0.10, 0.05, 0.05])
    pd = np.array([0.10, 0.10, 0.10, 0.15, 0.15, 0.15, 0.125, 0.125])
    zt = np.log(np.stack([pt, np.full(V, 1.0 / V)])).astype(np.float32)
    zd = np.log(pd[None]).astype(np.float32)
    res = _call(orc, zt, zd, [[6], [6]], [[0.99], [0.99]], [1.0, u_top], T)
    assert np.all(res["num_accepted"] == 0)
    assert list(res["out_tokens"][:, 0]) == [2, 2], res["out_tokens"]


ALL_CHECKS = [
    check_hand_cases,
    check_law_suite,
    check_identities_random,
    check_equal_rows_reduce_to_inverse_cdf,
    check_normaliser_closed_forms,
    check_bf16_widening,
    check_temperature_scaling,
    check_invalid_inputs,
    check_thread_invariance,
    check_diagnostics_do_not_change_results,
    check_zero_residual_draws_from_target_row,
    check_no_cell_reached_takes_last_positive,
    check_chi_square,
]
