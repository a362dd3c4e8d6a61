"""Python handle on the fp64 CPU oracle (oracle.c).

TEST INFRASTRUCTURE ONLY: imported by tests/, by the smoke check and by the
benchmark's CPU-baseline / reference leg.  The product path never imports it.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "oracle.c")
LIB = os.path.join(HERE, "liboracle.so")

CFLAGS = ["-O2", "-fPIC", "-shared", "-std=c11", "-fno-fast-math", "-ffp-contract=off",
          "-Wall", "-Wextra"]


def build(src: str = SRC, out: str = LIB) -> str:
    """Compile oracle.c with gcc (plain IEEE fp64, no contraction)."""
    cmd = ["gcc", *CFLAGS, "-o", out, src, "-lm", "-lpthread"]
    subprocess.run(cmd, check=True)
    return out


class _Diag(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in (
        "row_max", "row_sum", "p_x", "q_x", "accept_prob", "Z", "margin_accept",
        "margin_sample")]


class Oracle:
    """Loaded oracle library (the default build, or any other path)."""

    def __init__(self, path: str = LIB):
        if path == LIB and (not os.path.exists(LIB) or
                            os.path.getmtime(LIB) < os.path.getmtime(SRC)):
            build()
        self.path = path
        self.lib = ctypes.CDLL(path)
        f = self.lib.oracle_verify
        f.restype = ctypes.c_int
        f.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int, ctypes.c_void_p,
                      ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int64,
                      ctypes.c_int, ctypes.c_int64, ctypes.c_void_p, ctypes.c_void_p,
                      ctypes.c_void_p, ctypes.c_int]

    def verify(self, target: np.ndarray, draft: np.ndarray, tokens: np.ndarray,
               u_accept: np.ndarray, u_resample: np.ndarray, temperature: np.ndarray,
               dtype: Optional[str] = None, diag: bool = True, nthreads: int = 1) -> dict:
        """Run the oracle.  target [B,K+1,V], draft [B,K,V] as uint16 (bf16 bits)
        or float32.  Returns out_tokens [B,K+1], num_accepted [B] and, with
        ``diag``, the fp64 diagnostics."""
        if dtype is None:
            dtype = "bf16" if target.dtype == np.uint16 else "f32"
        store = np.uint16 if dtype == "bf16" else np.float32
        target = np.ascontiguousarray(target, dtype=store)
        draft = np.ascontiguousarray(draft, dtype=store)
        B, K1, V = target.shape
        K = K1 - 1
        if draft.shape != (B, K, V):
            raise ValueError("draft shape")
        tokens = np.ascontiguousarray(tokens, dtype=np.int32).reshape(B, K)
        u_accept = np.ascontiguousarray(u_accept, dtype=np.float32).reshape(B, K)
        u_resample = np.ascontiguousarray(u_resample, dtype=np.float32).reshape(B)
        temperature = np.ascontiguousarray(temperature, dtype=np.float32).reshape(B)
        out_tokens = np.zeros((B, K + 1), dtype=np.int32)
        out_n = np.zeros((B,), dtype=np.int32)
        res = {"out_tokens": out_tokens, "num_accepted": out_n}
        dptr = None
        if diag:
            R = 2 * K + 1
            arrs = {"row_max": (B, R), "row_sum": (B, R), "p_x": (B, K), "q_x": (B, K),
                    "accept_prob": (B, K), "Z": (B,), "margin_accept": (B,),
                    "margin_sample": (B,)}
            d = _Diag()
            for name, shape in arrs.items():
                a = np.full(shape, np.nan, dtype=np.float64)
                res[name] = a
                setattr(d, name, a.ctypes.data)
            dptr = ctypes.byref(d)
        rc = self.lib.oracle_verify(
            target.ctypes.data, draft.ctypes.data, 1 if dtype == "bf16" else 0,
            tokens.ctypes.data, u_accept.ctypes.data, u_resample.ctypes.data,
            temperature.ctypes.data, B, K, V, out_tokens.ctypes.data, out_n.ctypes.data,
            dptr, int(nthreads))
        if rc != 0:
            raise ValueError("oracle_verify rejected its arguments")
        return res


_default: Optional[Oracle] = None


def default() -> Oracle:
    global _default
    if _default is None:
        _default = Oracle()
    return _default


def verify(*args, **kw) -> dict:
    return default().verify(*args, **kw)


def boundary_mask(res: dict, band: float = 1e-6) -> np.ndarray:
    """Sequences whose acceptance or sampling decision lies within ``band`` of a
    threshold (the decisions a correct lower-precision implementation may take
    either way).

    Acceptance: |u - p/q| < band.  Token draw: the distance from u*Z to the
    nearer edge of the chosen cell of the cumulative sum, in probability units
    (margin_sample is that distance divided by Z, so it is multiplied back):
    the residual max(0, p - q) is a difference of probabilities, which any
    implementation whose normalisers carry a relative error of order 1e-7 knows
    only to that absolute precision, however small Z is.  For the bonus row
    Z = 1 and both readings agree."""
    draw = np.asarray(res["margin_sample"]) * np.where(np.isfinite(res["Z"]), res["Z"], 1.0)
    return (res["margin_accept"] < band) | (draw < band)
