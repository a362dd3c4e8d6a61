"""Chained two-stage verify (specdec_verify_chained) against its oracle
(oracle/chained.py).  The intermediate exit's logits are the final ones plus
seeded noise (rounded to the workload dtype); the draft exit's are the
workload's draft.  Emitted tokens and counts are compared exactly except on
boundary cases of either stage (a decision or draw within 1e-6 of its
threshold, counted as in the verify tests).  The second stage's diagnostics
(the final layer's row statistics, p_f(s_j) and q_i(s_j) of the tested
tokens, and the residual mass of its draw) are compared with the oracle's fp64
values at the tests' tolerance."""
import numpy as np
import pytest

import gpu_helpers as H
import oracle
import speculative_sampling_b200 as sd
from oracle import chained
from speculative_sampling_b200 import inputs

pytestmark = pytest.mark.gpu


def _make(name, B=None, V=None, K=None, sigma_i=0.3, seed=11):
    x = inputs.generate(name, B=B, V=V, K=K)
    rng = np.random.default_rng(seed)
    if x.dtype == "bf16":
        zf = inputs.bf16_bits_to_f32(x.target)
        inter = inputs.f32_to_bf16_bits((zf + sigma_i * rng.normal(size=zf.shape)).astype(np.float32))
    else:
        inter = (x.target + sigma_i * rng.normal(size=x.target.shape)).astype(np.float32)
    u2 = (rng.integers(0, 2 ** 24, (x.B, x.K + 1)).astype(np.float32) * np.float32(2.0 ** -24))
    ur2 = (rng.integers(0, 2 ** 24, x.B).astype(np.float32) * np.float32(2.0 ** -24))
    return x, inter, u2, ur2


def _gpu(x, inter, u2, ur2):
    torch = H.require_cuda()
    d = H.to_device(x)
    dv = lambda a: (torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).cuda()
                    .view(torch.bfloat16) if x.dtype == "bf16"
                    else torch.from_numpy(np.ascontiguousarray(a)).cuda())
    B, K = x.B, x.K
    nan = float("nan")
    dbg = dict(row_max=torch.full((B, 2 * K + 1), nan, dtype=torch.float32, device="cuda"),
               row_sum=torch.full((B, 2 * K + 1), nan, dtype=torch.float64, device="cuda"),
               p_x=torch.full((B, K + 1), nan, dtype=torch.float64, device="cuda"),
               q_x=torch.full((B, K + 1), nan, dtype=torch.float64, device="cuda"),
               Z=torch.full((B,), nan, dtype=torch.float64, device="cuda"))
    out = sd.verify_chained(d["target"], dv(inter), d["draft"], d["tokens"], d["u_accept"],
                            d["u_resample"], torch.from_numpy(u2).cuda(),
                            torch.from_numpy(ur2).cuda(), d["temperature"], debug2=dbg)
    torch.cuda.synchronize()
    res = {k: v.cpu().numpy() for k, v in out.items()}
    res.update({"dbg_" + k: v.cpu().numpy() for k, v in dbg.items()})
    return res


def _check(x, inter, u2, ur2):
    g = _gpu(x, inter, u2, ur2)
    o = chained.verify_chained(x.target, inter, x.draft, x.tokens, x.u_accept, x.u_resample, u2,
                               ur2, x.temperature, dtype=x.dtype)
    bnd = oracle.boundary_mask(o["stage1"], H.BAND) | (o["margin2"] < H.BAND)
    firm = ~bnd
    assert np.array_equal(g["stage1_n"][firm], o["stage1_n"][firm])
    assert np.array_equal(g["num_emitted"][firm], o["num_emitted"][firm])
    assert np.array_equal(g["out_tokens"][firm], o["out_tokens"][firm])
    print("chained", x.workload, "boundary sequences", int(np.sum(~firm)), "of", x.B)
    # second-stage diagnostics on the sequences both sides decided alike
    ok = firm & (o["num_emitted"] >= 0)
    K1 = x.K + 1
    assert np.array_equal(g["dbg_row_max"][ok, :K1].astype(np.float64), o["row_max_f"][ok])
    assert H.rel(g["dbg_row_sum"][ok, :K1], o["row_sum_f"][ok]).max(initial=0) <= H.RTOL
    tested = ok[:, None] & np.isfinite(o["p2_x"])
    assert H.rel(g["dbg_p_x"][tested], o["p2_x"][tested]).max(initial=0) <= H.RTOL
    assert H.rel(g["dbg_q_x"][tested], o["q2_x"][tested]).max(initial=0) <= H.RTOL
    drew = ok & np.isfinite(o["Z2"])
    zg, zo = g["dbg_Z"][drew], o["Z2"][drew]
    assert np.all(np.abs(zg - zo) <= H.RTOL * np.abs(zo) + H.Z_ATOL), \
        ("Z2", H.rel(zg, zo).max(initial=0))
    return g, o


@pytest.mark.parametrize("name,B,V,K", [
    ("batched_b64_k5_v128256_bf16", None, None, None),
    ("mix_b128_k4_v32000_bf16", 64, None, None),
    ("large_b256_k8_v151936_f32", 24, 30011, None),
    ("tiny_b1_k4_v1000_f32", None, None, None),
    ("large_b256_k8_v151936_f32", 16, 4099, 1),
])
def test_chained_matches_oracle(name, B, V, K):
    x, inter, u2, ur2 = _make(name, B=B, V=V, K=K)
    g, o = _check(x, inter, u2, ur2)
    # both stages do something on the larger batches
    if x.B >= 16:
        assert np.any(o["num_emitted"] < o["stage1_n"] + 1)


def test_equal_intermediate_and_final_is_one_verify():
    x, _, u2, ur2 = _make("mix_b128_k4_v32000_bf16", B=32, V=5003)
    g, o = _check(x, x.target.copy(), u2, ur2)
    v = H.oracle_verify(x)
    firm = ~oracle.boundary_mask(v, H.BAND)
    assert np.array_equal(g["num_emitted"][firm], v["num_accepted"][firm] + 1)


def test_chained_invalid_inputs():
    x, inter, u2, ur2 = _make("mix_b128_k4_v32000_bf16", B=8, V=3001)
    tgt = x.target.copy()
    nan = inputs.f32_to_bf16_bits(np.array([np.nan], np.float32))[0]
    tgt[2, x.K, 9] = nan          # a final-layer row (the last one)
    x.tokens[5, 0] = x.V          # a draft token
    x.target = tgt
    sd.specdec_device_errors(None)
    g, o = _check(x, inter, u2, ur2)
    assert g["num_emitted"][2] == -1 and g["num_emitted"][5] == -1
    assert np.all(g["out_tokens"][[2, 5]] == -1)
    sd.specdec_device_errors(None)


def _chained_fuzz(n=12, seed=77):
    rng = np.random.default_rng(seed)
    names = ["tiny_b1_k4_v1000_f32", "batched_b64_k5_v128256_bf16", "mix_b128_k4_v32000_bf16",
             "large_b256_k8_v151936_f32"]
    out = []
    for i in range(n):
        B = int(rng.integers(1, 33))
        K = int(rng.integers(1, 13))
        V = max(1, int(np.exp(rng.uniform(0.0, np.log(40000.0)))))
        T = np.exp(rng.uniform(np.log(0.2), np.log(4.0), B)).astype(np.float32)
        sig = float(rng.uniform(0.05, 1.0))
        out.append((i, names[i % 4], B, K, V, sig, T))
    return out


@pytest.mark.parametrize("case", _chained_fuzz(), ids=lambda c: "cfuzz%02d_%s_B%d_K%d_V%d" % c[:5])
def test_chained_fuzzed_shapes(case):
    """Seeded random shapes, intermediate-exit noise and per-sequence
    temperatures: both stages against the oracle (boundary cases of either
    stage excluded and counted, as above)."""
    _, name, B, K, V, sig, T = case
    x, inter, u2, ur2 = _make(name, B=B, V=V, K=K, sigma_i=sig, seed=B * 131 + V)
    x.temperature[:] = T
    _check(x, inter, u2, ur2)
