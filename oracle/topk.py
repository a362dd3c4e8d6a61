"""CPU oracle of the top-k-excluding-one candidate step (test infrastructure).

Only tests/, __graft_entry__.smoke() and bench.py's CPU legs use this module;
the CUDA path never calls it.

Source: the LogitSpec page "LogitSpec: Accelerating Retrieval-based
Speculative Decoding via Next Next Token Speculation", section 2 (the
LogitSpec workflow, step 2): after the model predicts the next token x_{i+1},
the top k entries of the last logit row, excluding x_{i+1}, are taken as the
candidates for the next-next token (the page reports the true next-next token
inside the top 60 in more than half of the decoding steps).

Readings taken where the page is silent:
  * order: by logit, largest first; equal logits by ascending token id (so the
    result is unique);
  * the excluded token is never returned; exclude = -1 excludes nothing;
  * when fewer than k tokens remain, the rest of the row of outputs is -1
    (index) and -inf (value);
  * a row holding a NaN is invalid: every index -1, every value NaN;
    -inf and +inf are ordinary (smallest / largest) values;
  * the ranking uses the logits themselves (temperature does not change the
    order), widened exactly from bf16 / fp32.
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


def topk_exclude(logits, exclude, k: int, dtype: str = "f32"):
    """logits [R, V] (fp32, or bf16 bit patterns), exclude [R] (token id or -1).
    Returns (idx [R, k] int64, val [R, k] float64)."""
    z = _widen(logits, dtype)
    R, V = z.shape
    idx = np.full((R, k), -1, np.int64)
    val = np.full((R, k), -np.inf)
    for r in range(R):
        row = z[r]
        if np.any(np.isnan(row)):
            val[r] = np.nan
            continue
        cand = np.arange(V)
        if 0 <= exclude[r] < V:
            cand = cand[cand != exclude[r]]
        order = np.lexsort((cand, -row[cand]))  # by -value, then by index
        take = cand[order[:k]]
        idx[r, :take.size] = take
        val[r, :take.size] = row[take]
    return idx, val
