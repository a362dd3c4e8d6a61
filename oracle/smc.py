"""fp64 CPU oracle of the SMC-SD weight step (test infrastructure).

Only tests/, __graft_entry__.smoke() and bench.py's CPU legs use this module;
the CUDA path never calls it.

Source: the SMC-SD page "Faster LLM Inference via Sequential Monte Carlo",
section 2 ("Methodology", the round of draft / scoring / resampling) and
"Key differences from standard SD".  Per round, each of N draft particles is
extended by K tokens drawn from the draft model q; the target model p scores
all N x (K+1) positions in one batched pass and yields one bonus token per
particle; instead of rejecting, every particle keeps its K tokens and is
re-weighted by the ratio of target to draft probabilities; when the effective
sample size falls below a threshold, low-weight particles are dropped and
high-weight ones copied.

Readings taken where the page is silent:
  * temperature softmax on both models, as in the verify step;
  * the weight of a particle is the importance ratio of its K new tokens,
    log w += sum_i [log p_i(x_i) - log q_i(x_i)] (the tokens were drawn from q,
    the target is p; the K+1-th, bonus, token is drawn from p itself and
    carries ratio 1);
  * the bonus token is drawn from p_K by the verify step's inverse-CDF rule
    (strict ">" on the running sum in ascending token order, one uniform);
  * ESS = 1 / sum_n wbar_n^2 of the normalised weights of a group of N;
  * resampling (when ESS < threshold * N) is systematic: one uniform u per
    group, particle k takes the ancestor a_k = min{j : C_j > (k + u) / N},
    C the running sum of the normalised weights in particle order; after it
    every log-weight is 0, otherwise the log-weights carry over and a_k = k;
  * an invalid particle (draft token outside [0, V), temperature not finite
    and > 0, a logit row with NaN / +Inf or only -Inf) gets tokens -1 and
    log-weight -inf (weight 0).
All arithmetic is fp64 numpy; logits are widened exactly (bf16 bit patterns
through fp32).
"""
from __future__ import annotations

import numpy as np


def _widen(a, dtype: str) -> np.ndarray:
    if dtype == "bf16":
        a = np.asarray(a)
        if a.dtype != np.uint16:
            a = a.view(np.uint16)
        return (a.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    return np.asarray(a, np.float32).astype(np.float64)


def _row_ok(z: np.ndarray) -> bool:
    return not (np.any(np.isnan(z)) or np.any(z == np.inf) or np.all(z == -np.inf))


def log_softmax_at(z: np.ndarray, T: float, x: int) -> float:
    """log p(x) with p = softmax(z / T): (z_x - M)/T - log sum_v exp((z_v - M)/T)."""
    M = np.max(z)
    s = np.sum(np.exp((z - M) / T))
    return (z[x] - M) / T - np.log(s)


def inverse_cdf(w: np.ndarray, u: float) -> int:
    """min{j : sum_{v<=j} w_v > u * sum_v w_v}, ascending order; if rounding
    leaves no such j, the last j with w_j > 0."""
    C = np.cumsum(w)
    t = u * C[-1]
    j = int(np.searchsorted(C, t, side="right"))
    if j >= w.size:
        pos = np.nonzero(w > 0)[0]
        j = int(pos[-1]) if pos.size else 0
    return j


def systematic(wbar: np.ndarray, u: float) -> np.ndarray:
    """Ancestors a_k = min{j : C_j > (k + u)/N} for k = 0..N-1 (C the running
    sum of the normalised weights); clamped to the last particle with positive
    weight when rounding leaves C_{N-1} below a target."""
    N = wbar.size
    C = np.cumsum(wbar)
    t = (np.arange(N, dtype=np.float64) + float(u)) / N
    a = np.searchsorted(C, t, side="right")
    pos = np.nonzero(wbar > 0)[0]
    last = int(pos[-1]) if pos.size else 0
    return np.where(a >= N, last, a).astype(np.int64)


def smc_step(target, draft, tokens, u_bonus, temperature, logw_in, u_resample,
             ess_threshold: float, N: int, dtype: str = "f32") -> dict:
    """One SMC-SD round over B = G*N particles (G groups of N).

    target [B, K+1, V], draft [B, K, V] (fp32 or bf16 bit patterns), tokens
    [B, K], u_bonus [B], temperature [B], logw_in [B] (or None: zeros),
    u_resample [G].  Returns tokens [B, K+1] (x_0..x_{K-1}, bonus), dlogw [B]
    (this round's increment), logw [B] (after the round), ess [G] (before
    resampling), resampled [G], ancestors [B] (index within the group), and the
    margins of the ancestor decisions (distance of each (k+u)/N to the nearest
    C_j) and of the bonus draws (distance of u*Z to the drawn cell's edges, over
    Z), for counting boundary cases."""
    tokens = np.asarray(tokens)
    B, K = tokens.shape
    if B % N:
        raise ValueError("B must be a multiple of N")
    G = B // N
    zt = _widen(target, dtype)
    zd = _widen(draft, dtype)
    V = zt.shape[2]
    Tv = np.asarray(temperature, np.float32).astype(np.float64)
    ub = np.asarray(u_bonus, np.float32).astype(np.float64)
    lw0 = np.zeros(B) if logw_in is None else np.asarray(logw_in, np.float64)
    out = np.full((B, K + 1), -1, np.int64)
    dlogw = np.zeros(B)
    bonus_margin = np.full(B, np.inf)
    for b in range(B):
        T = Tv[b]
        ok = np.isfinite(T) and T > 0
        ok = ok and all(_row_ok(zt[b, i]) for i in range(K + 1))
        ok = ok and all(_row_ok(zd[b, i]) for i in range(K))
        ok = ok and all(0 <= tokens[b, i] < V for i in range(K))
        if not ok:
            dlogw[b] = -np.inf
            continue
        d = 0.0
        for i in range(K):
            x = int(tokens[b, i])
            d += log_softmax_at(zt[b, i], T, x) - log_softmax_at(zd[b, i], T, x)
        dlogw[b] = d
        pK = np.exp((zt[b, K] - np.max(zt[b, K])) / T)
        out[b, :K] = tokens[b]
        y = inverse_cdf(pK, ub[b])
        out[b, K] = y
        C = np.cumsum(pK)
        t = ub[b] * C[-1]
        lo = C[y - 1] if y > 0 else 0.0
        bonus_margin[b] = min(abs(t - lo), abs(C[y] - t)) / C[-1]
    logw = lw0 + dlogw
    ess = np.zeros(G)
    resampled = np.zeros(G, bool)
    anc = np.tile(np.arange(N, dtype=np.int64), G)
    logw_out = logw.copy()
    margin = np.full(B, np.inf)
    ur = np.asarray(u_resample, np.float32).astype(np.float64)
    for g in range(G):
        lw = logw[g * N:(g + 1) * N]
        m = np.max(lw)
        if not np.isfinite(m):
            ess[g] = 0.0
            anc[g * N:(g + 1) * N] = -1
            logw_out[g * N:(g + 1) * N] = -np.inf
            continue
        w = np.exp(lw - m)
        wbar = w / np.sum(w)
        ess[g] = 1.0 / np.sum(wbar * wbar)
        if ess[g] < ess_threshold * N:
            resampled[g] = True
            anc[g * N:(g + 1) * N] = systematic(wbar, ur[g])
            logw_out[g * N:(g + 1) * N] = 0.0
            C = np.cumsum(wbar)
            t = (np.arange(N) + ur[g]) / N
            margin[g * N:(g + 1) * N] = np.min(np.abs(t[:, None] - C[None, :]), axis=1)
    return {"out_tokens": out, "dlogw": dlogw, "logw": logw_out, "ess": ess,
            "resampled": resampled, "ancestors": anc, "ancestor_margin": margin,
            "bonus_margin": bonus_margin}
