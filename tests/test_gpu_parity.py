"""CUDA path (through the C-ABI) against the fp64 CPU oracle on the same
seeded inputs: the five workloads, ragged and degenerate shapes, invalid
inputs, determinism and the alternative entry points."""
import numpy as np
import pytest

import gpu_helpers as H
import speculative_sampling_b200 as sd
from speculative_sampling_b200 import inputs

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("name", ["tiny_b1_k4_v1000_f32", "llama3_single_b1_k5_v128256_bf16",
                                  "batched_b64_k5_v128256_bf16", "mix_b128_k4_v32000_bf16"])
def test_parity_full_workload(name):
    x = inputs.generate(name)
    g = H.gpu_verify(x)
    o = H.oracle_verify(x)
    r = H.compare(g, o)
    print(name, r)


def test_parity_large_batch_full():
    """B=256, K=8, V=151936 fp32 (2.6 GB of logits): every sequence against the
    oracle (on all host cores), plus the structural properties of the output."""
    x = inputs.generate("large_b256_k8_v151936_f32")
    g = H.gpu_verify(x)
    o = H.oracle_verify(x)
    r = H.compare(g, o)
    print("large_b256_k8_v151936_f32", r)
    assert r["valid"] == x.B
    eq = x.seq_kind == 1
    assert eq.sum() >= 25 and np.all(g["num_accepted"][eq] == x.K)
    n = g["num_accepted"]
    assert np.all((n >= 0) & (n <= x.K))
    ot = g["out_tokens"]
    for b in range(x.B):
        assert np.array_equal(ot[b, :n[b]], x.tokens[b, :n[b]])
        assert 0 <= ot[b, n[b]] < x.V
        assert np.all(ot[b, n[b] + 1:] == -1)


@pytest.mark.parametrize("name,B,K,V", [
    ("batched_b64_k5_v128256_bf16", 6, 5, 33333),   # odd V: rows alternate alignment
    ("large_b256_k8_v151936_f32", 5, 3, 10007),    # ragged fp32 rows
    ("mix_b128_k4_v32000_bf16", 16, 4, 4099),      # ragged, several tiles
    ("batched_b64_k5_v128256_bf16", 3, 2, 5),      # V smaller than one vector
    ("tiny_b1_k4_v1000_f32", 3, 2, 3),
    ("tiny_b1_k4_v1000_f32", 2, 1, 1),             # V = 1: everything is certain
    ("batched_b64_k5_v128256_bf16", 4, 1, 2000),   # K = 1
    ("batched_b64_k5_v128256_bf16", 3, 32, 2000),  # K = 32 (a full warp of positions)
    ("mix_b128_k4_v32000_bf16", 40, 4, 32000),     # all three edge kinds
])
def test_parity_shapes(name, B, K, V):
    x = inputs.generate(name, B=B, K=K, V=V)
    g = H.gpu_verify(x)
    o = H.oracle_verify(x)
    print(name, B, K, V, H.compare(g, o))


def test_draft_equals_target_takes_bonus_path():
    x = inputs.generate("mix_b128_k4_v32000_bf16", B=32)
    x.draft[:] = x.target[:, :x.K]
    g = H.gpu_verify(x)
    o = H.oracle_verify(x)
    H.compare(g, o)
    assert np.all(g["num_accepted"] == x.K)


@pytest.mark.parametrize("T", [0.05, 0.3, 3.0, 8.0])
def test_temperature_extremes(T):
    x = inputs.generate("mix_b128_k4_v32000_bf16", B=24, V=8000)
    x.temperature[:] = T
    g = H.gpu_verify(x)
    o = H.oracle_verify(x)
    print(T, H.compare(g, o))


def test_invalid_inputs_flagged_not_faulted():
    x = inputs.generate("mix_b128_k4_v32000_bf16", B=12, V=3000)
    K = x.K
    x.tokens[1, 2] = x.V           # token out of range
    x.tokens[2, 0] = -5
    x.temperature[3] = 0.0         # bad temperatures
    x.temperature[4] = -1.0
    x.temperature[5] = np.nan
    nan_bf16 = np.uint16(0x7FC0)
    pinf_bf16 = np.uint16(0x7F80)
    ninf_bf16 = np.uint16(0xFF80)
    x.target[6, K, 17] = nan_bf16  # NaN in the bonus row
    x.draft[7, 1, 5] = pinf_bf16   # +Inf in a draft row
    x.draft[8, 0, :] = ninf_bf16   # a row of only -Inf
    x.target[9, 0, :100] = ninf_bf16  # -Inf entries in a valid row are legal
    H.require_cuda()
    sd.specdec_device_errors(None)  # clear
    g = H.gpu_verify(x)
    o = H.oracle_verify(x)
    H.compare(g, o)
    bad = [1, 2, 3, 4, 5, 6, 7, 8]
    assert np.all(g["num_accepted"][bad] == -1)
    assert np.all(g["num_accepted"][[0, 9, 10, 11]] >= 0)
    st, flags = sd.specdec_device_errors(None)
    assert st == sd.SPECDEC_EDEVICE
    assert flags == (sd.SPECDEC_ERR_TOKEN | sd.SPECDEC_ERR_TEMPERATURE | sd.SPECDEC_ERR_LOGITS)
    assert sd.specdec_device_errors(None) == (sd.SPECDEC_OK, 0)


def test_deterministic_and_entry_points_agree():
    torch = H.require_cuda()
    x = inputs.generate("batched_b64_k5_v128256_bf16")
    d = H.to_device(x)
    g1 = H.gpu_verify(x, dev_inputs=d)
    g2 = H.gpu_verify(x, dev_inputs=d, garbage_workspace=True)
    g3 = H.gpu_verify(x, dev_inputs=d, debug=False)
    for k in g1:
        assert np.array_equal(g1[k], g2[k], equal_nan=True), k
    for k in ("out_tokens", "num_accepted"):
        assert np.array_equal(g1[k], g3[k]), k
    # dtype-fixed entry point
    ot = torch.empty((x.B, x.K + 1), dtype=torch.int32, device="cuda")
    on = torch.empty((x.B,), dtype=torch.int32, device="cuda")
    st = sd.specdec_verify_bf16(d["target"].data_ptr(), d["draft"].data_ptr(),
                                d["tokens"].data_ptr(), d["u_accept"].data_ptr(),
                                d["u_resample"].data_ptr(), d["temperature"].data_ptr(),
                                x.B, x.K, x.V, ot.data_ptr(), on.data_ptr(),
                                torch.cuda.current_stream().cuda_stream)
    assert st == sd.SPECDEC_OK
    torch.cuda.synchronize()
    assert np.array_equal(ot.cpu().numpy(), g1["out_tokens"])
    # end-to-end host entry point from pinned memory
    pin = {k: torch.from_numpy(np.ascontiguousarray(getattr(x, k))).pin_memory()
           for k in ("target", "draft", "tokens", "u_accept", "u_resample", "temperature")}
    hot = torch.empty((x.B, x.K + 1), dtype=torch.int32).pin_memory()
    hon = torch.empty((x.B,), dtype=torch.int32).pin_memory()
    sd.verify_host(pin["target"], pin["draft"], pin["tokens"], pin["u_accept"],
                   pin["u_resample"], pin["temperature"], hot, hon)
    assert np.array_equal(hot.numpy(), g1["out_tokens"])
    assert np.array_equal(hon.numpy(), g1["num_accepted"])


def test_workspace_reuse_across_sizes():
    """The library-owned workspace is reused by calls of different sizes."""
    for name, B, V in [("batched_b64_k5_v128256_bf16", 64, None), ("mix_b128_k4_v32000_bf16", 7, 999),
                       ("large_b256_k8_v151936_f32", 3, 5003), ("batched_b64_k5_v128256_bf16", 9, None)]:
        x = inputs.generate(name, B=B, V=V)
        g = H.gpu_verify(x, debug=False)
        o = H.oracle_verify(x)
        H.compare(g, o, stats=False)


def test_empty_batch():
    torch = H.require_cuda()
    e = torch.empty
    ot, on = sd.verify(e((0, 6, 100), dtype=torch.bfloat16, device="cuda"),
                       e((0, 5, 100), dtype=torch.bfloat16, device="cuda"),
                       e((0, 5), dtype=torch.int32, device="cuda"),
                       e((0, 5), dtype=torch.float32, device="cuda"),
                       e((0,), dtype=torch.float32, device="cuda"),
                       e((0,), dtype=torch.float32, device="cuda"))
    assert ot.shape == (0, 6) and on.shape == (0,)


def _fuzz_cases(n=24, seed=2026):
    """Seeded random shapes over the four recipes: B in [1, 48], K in [1, 12],
    V log-uniform in [1, 70000] (odd and even, so rows take every alignment),
    per-sequence temperatures in [0.2, 4]."""
    rng = np.random.default_rng(seed)
    names = ["tiny_b1_k4_v1000_f32", "batched_b64_k5_v128256_bf16", "mix_b128_k4_v32000_bf16",
             "large_b256_k8_v151936_f32"]
    cases = []
    for i in range(n):
        name = names[i % len(names)]
        B = int(rng.integers(1, 49))
        K = int(rng.integers(1, 13))
        V = int(np.exp(rng.uniform(0.0, np.log(70000.0))))
        T = np.exp(rng.uniform(np.log(0.2), np.log(4.0), B)).astype(np.float32)
        cases.append((i, name, B, K, max(V, 1), T))
    return cases


@pytest.mark.parametrize("case", _fuzz_cases(), ids=lambda c: "fuzz%02d_%s_B%d_K%d_V%d" % c[:5])
def test_parity_fuzzed_shapes(case):
    """The full call and early exit against the oracle on seeded random shapes:
    every sequence without a boundary draw bit-exact, statistics within the
    tolerance, canaries intact (gpu_helpers)."""
    _, name, B, K, V, T = case
    x = inputs.generate(name, B=B, K=K, V=V)
    x.temperature[:] = T
    o = H.oracle_verify(x)
    H.compare(H.gpu_verify(x), o)
    H.compare(H.gpu_verify(x, debug=False, early_exit=True), o, stats=False)


def test_parity_many_sequences():
    """B = 2048 (the finish grid takes several waves of CTAs, one CTA per
    sequence; each sweep CTA holds many rows), every sequence against the
    oracle, for the full call and early exit."""
    x = inputs.generate("mix_b128_k4_v32000_bf16", B=2048, V=16000)
    o = H.oracle_verify(x)
    print("B=2048", H.compare(H.gpu_verify(x), o))
    H.compare(H.gpu_verify(x, debug=False, early_exit=True), o, stats=False)
