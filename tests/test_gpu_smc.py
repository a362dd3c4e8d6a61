"""SMC-SD weight step on the GPU (specdec_smc_step) against the fp64 oracle
(oracle/smc.py).  Integers (tokens, ancestors, the resample decision) are
compared exactly except where the oracle's own decision is within a band of a
threshold: the bonus draw within 1e-6 of a CDF edge (as in the verify tests),
and an ancestor or the ESS test within 1e-5 (the weights carry the row sums'
1e-7-level rounding, amplified by exp).  Log-weight increments agree within
2e-5 per draft token (1e-5 relative on each probability), ESS within 1e-5
relative."""
import numpy as np
import pytest

import gpu_helpers as H
import speculative_sampling_b200 as sd
from oracle import smc
from speculative_sampling_b200 import inputs

pytestmark = pytest.mark.gpu


def _run(x, N, thr, lw_in, u_res):
    torch = H.require_cuda()
    d = H.to_device(x)
    lw = None if lw_in is None else torch.from_numpy(lw_in).cuda()
    ur = torch.from_numpy(u_res).cuda()
    out = sd.smc_step(d["target"], d["draft"], d["tokens"], d["u_resample"], d["temperature"],
                      ur, N, ess_threshold=thr, log_weights_in=lw)
    torch.cuda.synchronize()
    return {k: v.cpu().numpy() for k, v in out.items()}


def _check(x, N, thr, lw_in, u_res):
    g = _run(x, N, thr, lw_in, u_res)
    o = smc.smc_step(x.target, x.draft, x.tokens, x.u_resample, x.temperature, lw_in, u_res,
                     thr, N, dtype=x.dtype)
    K = x.K
    # draft tokens are copied; the bonus is exact away from CDF edges
    assert np.array_equal(g["out_tokens"][:, :K], o["out_tokens"][:, :K])
    ok_bonus = o["bonus_margin"] >= H.BAND
    assert np.array_equal(g["out_tokens"][ok_bonus, K], o["out_tokens"][ok_bonus, K])
    # increments
    fin = np.isfinite(o["dlogw"])
    assert np.array_equal(np.isfinite(g["increment"]), fin)
    assert np.max(np.abs(g["increment"][fin] - o["dlogw"][fin]), initial=0) <= 2e-5 * K
    # ESS and the resample decision
    assert np.all(H.rel(g["ess"], o["ess"]) <= 1e-5)
    # (the resample decision shows in the ancestors and the log-weights below;
    # groups whose ESS is within 1e-5 of the threshold may go either way)
    near = np.abs(o["ess"] - thr * N) <= 1e-5 * N
    # ancestors: exact away from the running-sum edges
    firm = (o["ancestor_margin"] >= 1e-5) & ~np.repeat(near, N)
    assert np.array_equal(g["ancestors"][firm], o["ancestors"][firm])
    # log-weights after the round
    lwf = np.isfinite(o["logw"]) & ~np.repeat(near, N)
    assert np.max(np.abs(g["log_weights"][lwf] - o["logw"][lwf]), initial=0) <= 2e-5 * K + 1e-12
    return g, o


def _uniforms(G, seed):
    rng = np.random.default_rng(seed)
    return ((rng.integers(0, 2 ** 24, G)).astype(np.float32) * np.float32(2.0 ** -24))


@pytest.mark.parametrize("name,B,N,thr", [
    ("batched_b64_k5_v128256_bf16", None, 8, 0.5),
    ("mix_b128_k4_v32000_bf16", None, 16, 0.9),
    ("large_b256_k8_v151936_f32", 32, 4, 1.0),
    ("tiny_b1_k4_v1000_f32", None, 1, 0.5),
])
def test_smc_step_matches_oracle(name, B, N, thr):
    x = inputs.generate(name, B=B)
    G = x.B // N
    _check(x, N, thr, None, _uniforms(G, 1))


def test_smc_step_carries_log_weights_and_never_or_always_resamples():
    x = inputs.generate("mix_b128_k4_v32000_bf16", B=64, V=5003)
    rng = np.random.default_rng(3)
    lw = rng.normal(0, 2, x.B)
    u = _uniforms(8, 2)
    g, o = _check(x, 8, 0.0, lw, u)   # never resamples: ancestors identity, weights carried
    assert not np.any(o["resampled"])
    assert np.array_equal(g["ancestors"], np.tile(np.arange(8), 8))
    g, o = _check(x, 8, 1.0, lw, u)   # resamples every group whose weights differ
    assert np.all(o["resampled"])
    assert np.all(g["log_weights"] == 0.0)


def test_smc_step_invalid_particles():
    x = inputs.generate("mix_b128_k4_v32000_bf16", B=16, V=3001)
    x.tokens[3, 1] = -5
    x.temperature[9] = float("nan")
    sd.specdec_device_errors(None)
    g, o = _check(x, 4, 0.5, None, _uniforms(4, 5))
    assert np.all(g["out_tokens"][[3, 9]] == -1)
    assert np.all(np.isneginf(g["increment"][[3, 9]]))
    st, flags = sd.specdec_device_errors(None)
    assert flags & sd.SPECDEC_ERR_TOKEN and flags & sd.SPECDEC_ERR_TEMPERATURE


def test_smc_step_rejects_bad_arguments():
    torch = H.require_cuda()
    t = torch.zeros(64, dtype=torch.float32, device="cuda")
    p = t.data_ptr()
    s = torch.cuda.current_stream().cuda_stream
    # B not a multiple of N; N too large; negative threshold
    assert sd.specdec_smc_step(p, p, p, p, p, None, p, 0.5, 6, 4, 2, 8, sd.SPECDEC_F32, p, p, p,
                               p, None, s) == sd.SPECDEC_EINVAL
    assert sd.specdec_smc_step(p, p, p, p, p, None, p, 0.5, 8192, 8192, 2, 8, sd.SPECDEC_F32, p,
                               p, p, p, None, s) == sd.SPECDEC_EINVAL
    assert sd.specdec_smc_step(p, p, p, p, p, None, p, -1.0, 4, 4, 2, 8, sd.SPECDEC_F32, p, p, p,
                               p, None, s) == sd.SPECDEC_EINVAL


def _smc_fuzz(n=12, seed=99):
    rng = np.random.default_rng(seed)
    names = ["tiny_b1_k4_v1000_f32", "batched_b64_k5_v128256_bf16", "mix_b128_k4_v32000_bf16",
             "large_b256_k8_v151936_f32"]
    out = []
    for i in range(n):
        N = int(rng.choice([1, 2, 3, 4, 8, 16]))
        G = int(rng.integers(1, 9))
        K = int(rng.integers(1, 13))
        V = max(1, int(np.exp(rng.uniform(0.0, np.log(40000.0)))))
        thr = float(rng.choice([0.0, 0.3, 0.7, 1.0]))
        T = np.exp(rng.uniform(np.log(0.2), np.log(4.0), N * G)).astype(np.float32)
        lw = rng.normal(0, 1.5, N * G) if i % 2 else None
        out.append((i, names[i % 4], N, G, K, V, thr, T, lw))
    return out


@pytest.mark.parametrize("case", _smc_fuzz(), ids=lambda c: "sfuzz%02d_%s_N%d_G%d_K%d_V%d" % c[:6])
def test_smc_step_fuzzed_shapes(case):
    """Seeded random group sizes, shapes, thresholds, temperatures and
    incoming log-weights against the oracle."""
    i, name, N, G, K, V, thr, T, lw = case
    x = inputs.generate(name, B=N * G, K=K, V=V)
    x.temperature[:] = T
    _check(x, N, thr, lw, _uniforms(G, 100 + i))
