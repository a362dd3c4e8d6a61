"""Helpers shared by the GPU tests: move seeded inputs to the device, run the
CUDA path through the C-ABI, run the oracle, and compare them."""
from __future__ import annotations

import numpy as np

import oracle
import speculative_sampling_b200 as sd

# Tolerance for probabilities (row normalisers, p(x), q(x), Z): 1e-5 relative.
# The kernels widen logits exactly, carry log2(e)/T as two fp32 parts, evaluate
# 2^x with ex2.approx (about 2 ulp, i.e. ~2.4e-7 relative per element), sum
# each thread's elements in fp32 and every combine in fp64, so the expected
# error of a normaliser is a few 1e-7 relative; 1e-5 leaves a wide margin while
# still catching any dropped term or wrong scale.
RTOL = 1e-5
# Z (the residual mass, in probability units) is a difference of probabilities:
# sum max(0, p - q).  p and q carry the relative error of their normalisers
# (~1.6e-7 measured), so Z's absolute error is up to ~3e-7 however small Z is;
# when p and q nearly agree (Z of a few 1e-6, met by the fuzzed shapes) that is
# several percent of Z.  Z is compared within RTOL relative plus Z_ATOL.
Z_ATOL = 1e-6
# Decisions whose oracle margin is below this band may legitimately differ.
BAND = 1e-6
# Canary bands: every device output of the parity tests sits between two bands
# of CANARY_BYTES filled with a known pattern, checked after each call (an
# out-of-bounds write by a kernel would change them).
CANARY_BYTES = 4096
CANARY_BYTE = 0xA5


def require_cuda():
    import torch
    if not torch.cuda.is_available():
        raise RuntimeError("this test needs a CUDA device (B200)")
    return torch


def to_device(x):
    torch = require_cuda()
    dev = torch.device("cuda", 0)
    if x.dtype == "bf16":
        tg = torch.from_numpy(x.target.view(np.int16)).to(dev).view(torch.bfloat16)
        dr = torch.from_numpy(x.draft.view(np.int16)).to(dev).view(torch.bfloat16)
    else:
        tg = torch.from_numpy(x.target).to(dev)
        dr = torch.from_numpy(x.draft).to(dev)
    return dict(
        target=tg, draft=dr,
        tokens=torch.from_numpy(np.ascontiguousarray(x.tokens)).to(dev),
        u_accept=torch.from_numpy(x.u_accept).to(dev),
        u_resample=torch.from_numpy(x.u_resample).to(dev),
        temperature=torch.from_numpy(x.temperature).to(dev))


class Guarded:
    """A device tensor of the given shape and dtype carved out of a larger
    buffer, with CANARY_BYTES of CANARY_BYTE before and after it."""

    def __init__(self, shape, dtype, fill, device):
        torch = require_cuda()
        n = int(np.prod(shape)) * torch.empty((), dtype=dtype).element_size()
        self.n = n
        self.raw = torch.full((CANARY_BYTES + n + CANARY_BYTES,), CANARY_BYTE, dtype=torch.uint8,
                              device=device)
        self.t = self.raw[CANARY_BYTES:CANARY_BYTES + n].view(dtype).view(shape)
        self.t.fill_(fill)

    def check(self, name):
        lo = self.raw[:CANARY_BYTES]
        hi = self.raw[CANARY_BYTES + self.n:]
        assert bool((lo == CANARY_BYTE).all()) and bool((hi == CANARY_BYTE).all()), \
            f"canary band around {name} was overwritten"


def gpu_verify(x, debug=True, dev_inputs=None, garbage_workspace=False, early_exit=False):
    """CUDA path through specdec_verify_ex (with diagnostics) or specdec_verify
    (their early-exit forms with ``early_exit``).  Every output buffer is
    guarded by canary bands, checked after the call."""
    torch = require_cuda()
    d = dev_inputs if dev_inputs is not None else to_device(x)
    B, K = x.B, x.K
    R = 2 * K + 1
    dev = d["target"].device
    out = {}
    g_ot = Guarded((B, K + 1), torch.int32, -7, dev)
    g_on = Guarded((B,), torch.int32, -7, dev)
    guards = {"out_tokens": g_ot, "num_accepted": g_on}
    if debug:
        nan = float("nan")
        guards.update(row_max=Guarded((B, R), torch.float32, nan, dev),
                      row_sum=Guarded((B, R), torch.float64, nan, dev),
                      p_x=Guarded((B, K), torch.float64, nan, dev),
                      q_x=Guarded((B, K), torch.float64, nan, dev),
                      Z=Guarded((B,), torch.float64, nan, dev))
        dbg = {k: guards[k].t for k in ("row_max", "row_sum", "p_x", "q_x", "Z")}
        ws = None
        if garbage_workspace:
            dt = sd.SPECDEC_BF16 if x.dtype == "bf16" else sd.SPECDEC_F32
            n = sd.specdec_workspace_bytes(B, K, x.V, dt)
            ws = torch.randint(0, 255, (n,), dtype=torch.uint8, device=dev)
        ot, on = sd.verify(d["target"], d["draft"], d["tokens"], d["u_accept"], d["u_resample"],
                           d["temperature"], out_tokens=g_ot.t, out_num_accepted=g_on.t,
                           debug=dbg, workspace=ws, early_exit=early_exit)
        torch.cuda.synchronize()
        for k, v in dbg.items():
            out[k] = v.cpu().numpy()
    else:
        ot, on = sd.verify(d["target"], d["draft"], d["tokens"], d["u_accept"], d["u_resample"],
                           d["temperature"], out_tokens=g_ot.t, out_num_accepted=g_on.t,
                           early_exit=early_exit)
        torch.cuda.synchronize()
    for k, gd in guards.items():
        gd.check(k)
    out["out_tokens"] = ot.cpu().numpy()
    out["num_accepted"] = on.cpu().numpy()
    return out


def oracle_verify(x, seqs=None, nthreads=None):
    import os
    nthreads = nthreads or max(1, os.cpu_count() or 1)
    if seqs is None:
        return oracle.verify(x.target, x.draft, x.tokens, x.u_accept, x.u_resample,
                             x.temperature, dtype=x.dtype, nthreads=nthreads)
    s = np.asarray(seqs)
    return oracle.verify(x.target[s], x.draft[s], x.tokens[s], x.u_accept[s], x.u_resample[s],
                         x.temperature[s], dtype=x.dtype, nthreads=nthreads)


def rel(a, b):
    """Relative difference; probabilities below 1e-200 count as equal to 0."""
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    return np.abs(a - b) / np.maximum(np.abs(b), 1e-200)


def rows_read(o: dict, early_split) -> np.ndarray:
    """[B, 2K+1] mask of the rows a call reads: all of them, or with early exit
    (first sweep over positions < early_split) those of positions < early_split
    plus every row of the sequences that accepted all of those."""
    on = o["num_accepted"]
    B, K1 = o["out_tokens"].shape
    K = K1 - 1
    j = np.arange(2 * K + 1)
    pos = np.where(j <= K, j, j - K - 1)
    if early_split is None:
        return np.ones((B, 2 * K + 1), bool)
    return (pos[None, :] < early_split) | (on[:, None] >= early_split)


def compare(g: dict, o: dict, seqs=None, rtol=RTOL, band=BAND, stats=True,
            early_split=None) -> dict:
    """Element-by-element comparison of the CUDA path (g) with the oracle (o).

    Integer outputs: bit-exact on every sequence whose oracle decisions are not
    within ``band`` of a threshold; such boundary draws are counted.  Invalid
    sequences (n = -1) must agree exactly.  Probabilities: within ``rtol``, on
    the rows the call reads (``early_split``: see rows_read)."""
    if seqs is not None:
        g = {k: v[np.asarray(seqs)] for k, v in g.items()}
    on, gn = o["num_accepted"], g["num_accepted"]
    assert np.array_equal(on < 0, gn < 0), "invalid-sequence verdicts differ"
    assert np.all(g["out_tokens"][gn < 0] == -1)
    valid = on >= 0
    bnd = oracle.boundary_mask(o, band) & valid
    exact = valid & ~bnd
    mism = np.nonzero(exact & (np.any(g["out_tokens"] != o["out_tokens"], axis=1) | (gn != on)))[0]
    assert mism.size == 0, (f"{mism.size} non-boundary sequences differ, e.g. seq {mism[:5]}: "
                            f"gpu n={gn[mism[:5]]} oracle n={on[mism[:5]]} "
                            f"gpu={g['out_tokens'][mism[:2]]} oracle={o['out_tokens'][mism[:2]]}")
    K = o["out_tokens"].shape[1] - 1
    # draws per valid sequence: min(n+1, K) acceptance tests + one token draw
    draws = int(np.sum(np.minimum(on[valid] + 1, K) + 1))
    differ = valid & (np.any(g["out_tokens"] != o["out_tokens"], axis=1) | (gn != on))
    # boundary sequences over valid ones, and the count of their boundary draws
    # (an acceptance test or the token draw within `band` of its threshold)
    nb_acc = int(np.sum(valid & (o["margin_accept"] < band)))
    nb_smp = int(np.sum(valid & (o["margin_sample"] * np.where(np.isfinite(o["Z"]), o["Z"], 1.0)
                                 < band)))
    res = {"sequences": int(on.size), "valid": int(valid.sum()), "boundary": int(bnd.sum()),
           "draws": draws, "mismatched": int(differ.sum()),
           "boundary_rate": float(bnd.sum()) / max(int(valid.sum()), 1),
           "boundary_accept_tests": nb_acc, "boundary_token_draws": nb_smp}
    # Disagreements are allowed only on boundary draws (asserted above: every
    # sequence without one is bit-exact); they are counted and reported.  A
    # token draw within 1e-6 of a CDF cell edge can go either way between fp32
    # weights and the oracle's fp64, so no cap on them can hold at every size.
    res["mismatched_boundary"] = int((differ & bnd).sum())
    assert res["mismatched"] == res["mismatched_boundary"], res
    if not stats or "row_sum" not in g:
        return res
    v = valid[:, None] & rows_read(o, early_split)
    assert np.array_equal(g["row_max"][v].astype(np.float64), o["row_max"][v]), "row max"
    e_s = rel(g["row_sum"][v], o["row_sum"][v])
    assert e_s.max(initial=0) <= rtol, ("row sum", e_s.max())
    same = exact | (valid & (gn == on))
    reach = (np.arange(K)[None, :] <= on[:, None]) & same[:, None]
    e_p = rel(g["p_x"][reach], o["p_x"][reach])
    e_q = rel(g["q_x"][reach], o["q_x"][reach])
    assert e_p.max(initial=0) <= rtol, ("p(x)", e_p.max())
    assert e_q.max(initial=0) <= rtol, ("q(x)", e_q.max())
    zg, zo = g["Z"][same], o["Z"][same]
    e_z = rel(zg, zo)
    assert np.all(np.abs(zg - zo) <= rtol * np.abs(zo) + Z_ATOL), ("Z", e_z.max(initial=0))
    res.update(max_rel_row_sum=float(e_s.max(initial=0)), max_rel_px=float(e_p.max(initial=0)),
               max_rel_qx=float(e_q.max(initial=0)), max_rel_Z=float(e_z.max(initial=0)))
    return res
