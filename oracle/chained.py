"""fp64 CPU oracle of the chained two-stage verify (test infrastructure).

Only tests/, __graft_entry__.smoke() and bench.py's CPU legs use this module;
the CUDA path never calls it.

Source: the HiSpec page "HiSpec: Hierarchical Speculative Decoding for LLMs",
section 2 ("Methodology"): one early-exit model with a draft exit L_d, an
intermediate verifier exit L_i and the final layer L_f; the intermediate
verifier accepts draft tokens that agree with its distribution and rejects the
inaccurate ones early, without relaxing the final acceptance criterion; the
output is lossless because the lossless speculative-decoding argument is
applied in turn at both stages (L_d -> L_i -> L_f).

Readings taken where the page is silent:
  * stage 1 is the verify step with target L_i and draft L_d: the accepted
    prefix x_0..x_{n1-1} and the token y1 drawn at n1 (from max(0, p_i - q_d),
    or from L_i's row K when every draft token is accepted);
  * stage 2 verifies the m = n1 + 1 tokens s = (x_0..x_{n1-1}, y1) against
    L_f with L_i as their proposal distribution: s_j is accepted iff
    u2_j * q_i,j(s_j) < p_f,j(s_j); at the first rejection n2 a token is drawn
    from max(0, p_f,n2 - q_i,n2) / Z with u2_resample (from p_f,n2 if Z = 0);
    when all m are accepted they are emitted with no further token (L_f's row
    after them is not among the inputs);
  * emitted = n2 + 1 tokens after a rejection, m otherwise; then -1;
  * every row of the three logit tensors and every draft token is checked
    (invalid -> emitted -1 and all tokens -1), as the verify step does.
The first stage is the verify oracle (oracle.c); the second is written here in
plain numpy fp64.
"""
from __future__ import annotations

import numpy as np

from . import smc as _smc  # exact widening and the inverse-CDF rule


def _softmax(z: np.ndarray, T: float) -> np.ndarray:
    e = np.exp((z - np.max(z)) / T)
    return e / np.sum(e)


def verify_chained(final, inter, draft, tokens, u_accept1, u_resample1, u_accept2, u_resample2,
                   temperature, dtype: str = "f32", orc=None) -> dict:
    """final, inter [B, K+1, V]; draft [B, K, V]; tokens [B, K]; u_accept1 [B, K];
    u_resample1 [B]; u_accept2 [B, K+1]; u_resample2 [B]; temperature [B].
    Returns out_tokens [B, K+1], num_emitted [B], stage1 tokens and n1, the
    margins of the stage-2 decisions (for counting boundary cases), and the
    stage-2 diagnostics: the final layer's row maxima and normalisers
    sum_v exp((z_v - max)/T) [B, K+1], p_f,j(s_j) and q_i,j(s_j) for the tested
    positions j (NaN elsewhere) [B, K+1], and the mass Z2 = sum max(0, p_f - q_i)
    of the stage-2 residual draw (NaN when nothing is drawn) [B]."""
    from . import default as _default_oracle
    orc = orc or _default_oracle()
    # (with diagnostics: the decision margins count stage-1 boundary cases)
    r1 = orc.verify(inter, draft, tokens, u_accept1, u_resample1, temperature, dtype=dtype,
                    diag=True)
    n1 = r1["num_accepted"]
    s = r1["out_tokens"]
    zf = _smc._widen(final, dtype)
    zi = _smc._widen(inter, dtype)
    B, K1, V = zf.shape
    Tv = np.asarray(temperature, np.float32).astype(np.float64)
    u2 = np.asarray(u_accept2, np.float32).astype(np.float64)
    ur2 = np.asarray(u_resample2, np.float32).astype(np.float64)
    out = np.full((B, K1), -1, np.int64)
    emitted = np.full(B, -1, np.int64)
    margin = np.full(B, np.inf)
    f_max = np.full((B, K1), np.nan)
    f_sum = np.full((B, K1), np.nan)
    p2 = np.full((B, K1), np.nan)
    q2 = np.full((B, K1), np.nan)
    z2 = np.full(B, np.nan)
    for b in range(B):
        if n1[b] < 0 or not all(_smc._row_ok(zf[b, j]) for j in range(K1)):
            continue
        T = Tv[b]
        for j in range(K1):  # diagnostics of the final layer's rows
            f_max[b, j] = np.max(zf[b, j])
            f_sum[b, j] = np.sum(np.exp((zf[b, j] - f_max[b, j]) / T))
        m = int(n1[b]) + 1
        n2 = m
        for j in range(m):
            p = _softmax(zf[b, j], T)
            q = _softmax(zi[b, j], T)
            tok = int(s[b, j])
            p2[b, j] = p[tok]
            q2[b, j] = q[tok]
            a = p[tok] / q[tok] if q[tok] > 0 else np.inf
            if a < 1.0:
                margin[b] = min(margin[b], abs(u2[b, j] - a))
            if not (u2[b, j] * q[tok] < p[tok]):
                n2 = j
                break
        out[b, :n2] = s[b, :n2]
        if n2 < m:
            p = _softmax(zf[b, n2], T)
            q = _softmax(zi[b, n2], T)
            r = np.maximum(0.0, p - q)
            z2[b] = np.sum(r)
            if not (np.sum(r) > 0.0):
                r = p
            y = _smc.inverse_cdf(r, ur2[b])
            out[b, n2] = y
            C = np.cumsum(r)
            t = ur2[b] * C[-1]
            lo = C[y - 1] if y > 0 else 0.0
            # (in probability units: see oracle.boundary_mask)
            margin[b] = min(margin[b], min(abs(t - lo), abs(C[y] - t)))
            emitted[b] = n2 + 1
        else:
            emitted[b] = m
    return {"out_tokens": out, "num_emitted": emitted, "stage1_tokens": s, "stage1_n": n1,
            "stage1": r1, "margin2": margin, "row_max_f": f_max, "row_sum_f": f_sum,
            "p2_x": p2, "q2_x": q2, "Z2": z2}
