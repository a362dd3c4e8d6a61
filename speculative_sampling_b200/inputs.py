"""Seeded synthetic inputs for the batched speculative-sampling verify step.

This module is the one piece shared by the CUDA path's tests/bench and the fp64
CPU oracle's tests.  It only draws random numbers and shapes them into the
tensors the verify step consumes; it holds none of the verify arithmetic (no
softmax normaliser, no acceptance ratio, no residual distribution, no inverse
CDF).  Draft tokens are drawn with the Gumbel-max trick, which needs no
normalised probabilities.

Workloads follow the shapes the pages talk about: the Llama-3 vocabulary
(V=128256) with K=5 draft tokens as in the vLLM example of the speculative
decoding blog ("Speculative Decoding ... Llama 70B x2.4", section "Working code
on vLLM 0.6+", num_speculative_tokens=5, temperature=0.7), batch sizes from 1 to
hundreds, a Qwen-size vocabulary (V=151936) with deeper speculation (K=8), and
an edge-case mix.  Logits are built as

    target z[v]  = 3 * N(0,1) - 1.1 * ln(rank[v])     (rank = 1 + a seeded
                                                        permutation of the
                                                        vocabulary, per sequence)
    draft  z'[v] = z[v] + sigma * N(0,1)

then rounded to the workload's dtype (bf16 with round-to-nearest-even, or
fp32).  Every sequence b draws from its own seed stream
``SeedSequence(entropy=seed, spawn_key=(b,))`` so any contiguous shard of the
batch can be generated on its own and equals the same slice of the whole batch.

Uniforms are k * 2**-24 for k in [0, 2**24): exact in fp32, never 1.0.
"""
from __future__ import annotations

import dataclasses
from typing import Optional

import numpy as np

__all__ = [
    "Workload",
    "WORKLOADS",
    "WORKLOAD_ORDER",
    "VerifyInputs",
    "generate",
    "f32_to_bf16_bits",
    "bf16_bits_to_f32",
    "elem_size",
]


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int
    K: int
    V: int
    dtype: str  # "f32" or "bf16"
    seed: int
    temperature: tuple  # choices; one per sequence is drawn when len > 1
    sigma: object  # float, or ("uniform", lo, hi) per sequence
    mix: str  # "random" | "equal10" | "edge"
    description: str


# Draft-noise sigma for the single-stream Llama-3-vocabulary workload: chosen so
# that the mean per-position acceptance probability of its K=5 positions is
# about 0.75 (the blog's measured acceptance rates are 67-84% at K=5).  The value
# was found by bisection with oracle/calibrate_sigma.py, which calls only the
# CPU oracle.
LLAMA_SINGLE_SIGMA = 0.881

WORKLOADS = {
    "tiny_b1_k4_v1000_f32": Workload(
        "tiny_b1_k4_v1000_f32", 1, 4, 1000, "f32", 0, (1.0,), 0.5, "random",
        "tiny verify: B=1 K=4 V=1000 fp32, draft noise 0.5, T=1.0"),
    "llama3_single_b1_k5_v128256_bf16": Workload(
        "llama3_single_b1_k5_v128256_bf16", 1, 5, 128256, "bf16", 1, (0.7,),
        LLAMA_SINGLE_SIGMA, "random",
        "single stream, Llama-3 vocabulary: B=1 K=5 V=128256 bf16, T=0.7"),
    "batched_b64_k5_v128256_bf16": Workload(
        "batched_b64_k5_v128256_bf16", 64, 5, 128256, "bf16", 2, (0.7,),
        ("uniform", 0.2, 1.5), "random",
        "batched serving: B=64 K=5 V=128256 bf16, per-sequence draft noise U(0.2,1.5), T=0.7"),
    "large_b256_k8_v151936_f32": Workload(
        "large_b256_k8_v151936_f32", 256, 8, 151936, "f32", 3, (1.0,), 0.5,
        "equal10",
        "large batch, deep speculation: B=256 K=8 V=151936 fp32, noise 0.5, T=1.0, "
        "10% of sequences with draft == target"),
    "mix_b128_k4_v32000_bf16": Workload(
        "mix_b128_k4_v32000_bf16", 128, 4, 32000, "bf16", 4, (0.3, 0.7, 1.3), 0.5,
        "edge",
        "edge mix: B=128 K=4 V=32000 bf16; 25% draft == target, 25% disjoint top-1, "
        "50% random; T in {0.3,0.7,1.3} per sequence"),
}
WORKLOAD_ORDER = list(WORKLOADS)


def elem_size(dtype: str) -> int:
    return {"f32": 4, "bf16": 2}[dtype]


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round fp32 values to bf16 (round to nearest, ties to even); return the bits."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    bias = ((u >> np.uint32(16)) & np.uint32(1)) + np.uint32(0x7FFF)
    return ((u + bias) >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns to fp32."""
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


@dataclasses.dataclass
class VerifyInputs:
    """Host arrays for one verify call.

    target   [B, K+1, V]  uint16 (bf16 bits) or float32, row-major, V contiguous
    draft    [B, K,   V]  same dtype
    tokens   [B, K]       int32 draft tokens
    u_accept [B, K]       float32 uniforms for the acceptance tests
    u_resample [B]        float32 uniform for the residual or bonus draw
    temperature [B]       float32
    """
    workload: str
    dtype: str
    B: int
    K: int
    V: int
    target: np.ndarray
    draft: np.ndarray
    tokens: np.ndarray
    u_accept: np.ndarray
    u_resample: np.ndarray
    temperature: np.ndarray
    seq_kind: np.ndarray  # per sequence: 0 random, 1 draft==target, 2 disjoint top-1
    sigma: np.ndarray  # per sequence draft noise

    def logits_f32(self, which: str) -> np.ndarray:
        a = getattr(self, which)
        return bf16_bits_to_f32(a) if self.dtype == "bf16" else a

    @property
    def floor_bytes(self) -> int:
        return self.B * (2 * self.K + 1) * self.V * elem_size(self.dtype)


def _round(x32: np.ndarray, dtype: str) -> np.ndarray:
    if dtype == "bf16":
        return f32_to_bf16_bits(x32)
    return np.ascontiguousarray(x32, dtype=np.float32)


def _uniform24(rng: np.random.Generator, n: int) -> np.ndarray:
    k = rng.integers(0, 1 << 32, size=n, dtype=np.uint64) >> np.uint64(8)
    return (k.astype(np.float64) * 2.0 ** -24).astype(np.float32)


def generate(name: str, seq_begin: int = 0, seq_end: Optional[int] = None,
             B: Optional[int] = None, V: Optional[int] = None,
             K: Optional[int] = None, sigma: Optional[float] = None) -> VerifyInputs:
    """Generate sequences [seq_begin, seq_end) of workload ``name``.

    ``B``/``V``/``K`` override the workload's sizes (same recipe, other shape)
    and ``sigma`` its draft noise; sequence b always uses seed stream
    (workload seed, b).
    """
    w = WORKLOADS[name]
    sigma_override = sigma
    Bw = w.B if B is None else B
    Vw = w.V if V is None else V
    Kw = w.K if K is None else K
    if seq_end is None:
        seq_end = Bw
    nb = seq_end - seq_begin
    if nb < 0 or seq_begin < 0:
        raise ValueError("bad sequence range")
    store = np.uint16 if w.dtype == "bf16" else np.float32
    target = np.empty((nb, Kw + 1, Vw), dtype=store)
    draft = np.empty((nb, Kw, Vw), dtype=store)
    tokens = np.empty((nb, Kw), dtype=np.int32)
    u_acc = np.empty((nb, Kw), dtype=np.float32)
    u_res = np.empty((nb,), dtype=np.float32)
    temp = np.empty((nb,), dtype=np.float32)
    kind = np.zeros((nb,), dtype=np.int8)
    sig = np.zeros((nb,), dtype=np.float64)
    for j, b in enumerate(range(seq_begin, seq_end)):
        ss = np.random.SeedSequence(entropy=w.seed, spawn_key=(b,))
        r_perm, r_tn, r_dn, r_tok, r_u, r_par = [np.random.default_rng(s) for s in ss.spawn(6)]
        # per-sequence parameters
        if isinstance(w.sigma, tuple):
            sigma = float(r_par.uniform(w.sigma[1], w.sigma[2]))
        else:
            sigma = float(w.sigma)
        if sigma_override is not None:
            sigma = float(sigma_override)
        T = float(w.temperature[int(r_par.integers(len(w.temperature)))]) if len(w.temperature) > 1 \
            else float(w.temperature[0])
        if w.mix == "equal10":
            k = 1 if b % 10 == 0 else 0
        elif w.mix == "edge":
            k = {0: 1, 1: 2}.get(b % 4, 0)
        else:
            k = 0
        kind[j] = k
        sig[j] = sigma
        temp[j] = np.float32(T)
        # target rows 0..K share the Zipf bias of this sequence
        rank = 1.0 + r_perm.permutation(Vw).astype(np.float64)
        bias = (-1.1 * np.log(rank)).astype(np.float32)
        zt = 3.0 * r_tn.standard_normal((Kw + 1, Vw), dtype=np.float32) + bias
        target[j] = _round(zt, w.dtype)
        if k == 1:
            draft[j] = target[j, :Kw]
        else:
            zd = zt[:Kw] + np.float32(sigma) * r_dn.standard_normal((Kw, Vw), dtype=np.float32)
            if k == 2:
                # "disjoint top-1": the draft's favourite is the target's least
                # likely token of that row
                tgt_rounded = bf16_bits_to_f32(target[j, :Kw]) if w.dtype == "bf16" else target[j, :Kw]
                vstar = np.argmin(tgt_rounded, axis=1)
                zd[np.arange(Kw), vstar] = zd.max(axis=1) + np.float32(8.0)
            draft[j] = _round(zd, w.dtype)
        # draft tokens x_i ~ softmax(z'_i / T) by Gumbel-max on the rounded logits
        zr = bf16_bits_to_f32(draft[j]) if w.dtype == "bf16" else draft[j]
        g = -np.log(-np.log(r_tok.random((Kw, Vw))))
        tokens[j] = np.argmax(zr.astype(np.float64) / T + g, axis=1).astype(np.int32)
        u = _uniform24(r_u, Kw + 1)
        u_acc[j] = u[:Kw]
        u_res[j] = u[Kw]
    return VerifyInputs(name, w.dtype, nb, Kw, Vw, target, draft, tokens, u_acc, u_res,
                        temp, kind, sig)
