"""Top-k candidates excluding one token (specdec_topk_exclude) against the
CPU oracle (oracle/topk.py): indices and logits are compared exactly (it is
index work on exactly widened values).  Cases: the bench workload's target
rows (k = 60, the LogitSpec page's figure, excluding the draft tokens), fp32
rows of 151936, k = 1 and 256, quantised logits with many ties (the fast
path), constant rows (ties overflow the candidate buffer: the radix-select
path), -inf entries, rows shorter than k, odd V with misaligned rows, rows
picked by index, NaN rows (also a NaN among values far below the top k
of a long row), exclusions at vector-group edges, bad arguments."""
import numpy as np
import pytest

import gpu_helpers as H
import speculative_sampling_b200 as sd
from oracle import topk
from speculative_sampling_b200 import inputs

pytestmark = pytest.mark.gpu


def _dev(a, dtype):
    torch = H.require_cuda()
    if dtype == "bf16":
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).cuda().view(torch.bfloat16)
    return torch.from_numpy(np.ascontiguousarray(a, np.float32)).cuda()


def _check(rows, dtype, k, exclude):
    torch = H.require_cuda()
    ex_t = None if exclude is None else torch.from_numpy(exclude.astype(np.int32)).cuda()
    idx, val = sd.topk_exclude(_dev(rows, dtype), k, exclude=ex_t)
    torch.cuda.synchronize()
    ex = np.full(rows.shape[0], -1) if exclude is None else exclude
    oi, ov = topk.topk_exclude(rows, ex, k, dtype=dtype)
    gi, gv = idx.cpu().numpy(), val.cpu().numpy().astype(np.float64)
    assert np.array_equal(gi, oi)
    assert np.array_equal(np.isnan(gv), np.isnan(ov))
    ok = ~np.isnan(ov)
    assert np.array_equal(gv[ok], ov[ok])


def test_bench_rows_top60_excluding_draft_tokens():
    x = inputs.generate("batched_b64_k5_v128256_bf16", B=16)
    rows = x.target[:, :x.K].reshape(-1, x.V)
    _check(rows, "bf16", 60, x.tokens.reshape(-1))


@pytest.mark.parametrize("k", [1, 60, 256])
def test_fp32_rows(k):
    x = inputs.generate("large_b256_k8_v151936_f32", B=4)
    rows = x.target.reshape(-1, x.V)[:12]
    ex = np.arange(12) * 997 % x.V
    _check(rows, "f32", k, ex)


def test_ties_constant_rows_and_inf():
    rng = np.random.default_rng(8)
    V = 20011
    q = np.round(rng.normal(0, 2, (6, V))).astype(np.float32)  # about 15 distinct values
    q[1] = 1.5                                                   # constant: radix path
    q[2, ::3] = -np.inf
    q[3] = -np.inf
    q[3, 100:105] = 2.0
    q[4, ::2] = 0.0                                              # +0 and -0 are equal
    q[4, 1::2] = -0.0
    ex = np.array([-1, 7, 3, 100, V - 1, 0])
    _check(q, "f32", 60, ex)
    _check(inputs.f32_to_bf16_bits(q), "bf16", 200, ex)


def test_short_rows_odd_lengths_and_row_index():
    torch = H.require_cuda()
    rng = np.random.default_rng(2)
    for V in (1, 5, 100, 33333):
        rows = rng.normal(0, 1, (5, V)).astype(np.float32)
        _check(rows, "f32", 256, np.full(5, V // 2))
        _check(inputs.f32_to_bf16_bits(rows), "bf16", 60, None)
    # rows picked by index out of a [B, K+1, V] tensor: the bonus / resampled rows
    x = inputs.generate("mix_b128_k4_v32000_bf16", B=8, V=3001)
    t = _dev(x.target, "bf16")
    sel = np.array([0 * 5 + 2, 3 * 5 + 4, 7 * 5 + 0], np.int64)
    idx, val = sd.topk_exclude(t, 60, row_index=torch.from_numpy(sel).cuda())
    oi, _ = topk.topk_exclude(x.target.reshape(-1, x.V)[sel], np.full(3, -1), 60, dtype="bf16")
    assert np.array_equal(idx.cpu().numpy(), oi)


def test_nan_rows_and_bad_arguments():
    torch = H.require_cuda()
    rows = np.ones((3, 1000), np.float32)
    rows[1, 500] = np.nan
    sd.specdec_device_errors(None)
    _check(rows, "f32", 10, None)
    st, flags = sd.specdec_device_errors(None)
    assert flags & sd.SPECDEC_ERR_LOGITS
    t = torch.zeros(64, dtype=torch.float32, device="cuda")
    p, s = t.data_ptr(), torch.cuda.current_stream().cuda_stream
    for k, stride in ((0, 8), (257, 8), (4, 7)):
        assert sd.specdec_topk_exclude(p, stride, None, 2, 8, sd.SPECDEC_F32, None, k, p, p, s) \
            == sd.SPECDEC_EINVAL


def test_long_rows_nan_outside_the_top_groups_then_clean_call():
    """Long rows (fp32, 12500 vectors: 7 rounds of 4 vectors per thread, one
    vector group per round): a NaN among values far below the top k and one
    in the last element make those rows invalid (the first pass, which reads
    every element, finds them); exclusions sit on round edges.  A following
    clean call must be exact."""
    rng = np.random.default_rng(11)
    V = 50000
    rows = rng.normal(0, 3, (4, V)).astype(np.float32)
    rows[1, 24992:25008] = -50.0
    rows[1, 25000] = np.nan
    rows[2, V - 1] = np.nan
    seg = 4 * 512 * 4          # elements of one round of the 512 threads
    ex = np.array([seg, 2 * seg - 1, 0, V - 1])
    sd.specdec_device_errors(None)
    _check(rows, "f32", 60, ex)
    st, flags = sd.specdec_device_errors(None)
    assert flags & sd.SPECDEC_ERR_LOGITS
    clean = rng.normal(0, 3, (2, V)).astype(np.float32)
    _check(clean, "f32", 60, np.array([seg * 4 * 3, 5]))
    st, flags = sd.specdec_device_errors(None)
    assert not (flags & sd.SPECDEC_ERR_LOGITS)
    _check(inputs.f32_to_bf16_bits(rows[[0, 3]]), "bf16", 256, ex[[0, 3]])
