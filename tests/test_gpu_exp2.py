"""Accuracy of the statistics sweep's FMA-pipe exponential (2^a by argument
reduction and a degree-5 minimax polynomial, see specdec.cu) on the GPU,
through its test entry point: against fp64 exp2 (the mathematics) and against
CUDA's own exp2f (torch.exp2 on a float32 CUDA tensor).  The bound is 4 ulp
relative (2^-22): the polynomial's own error is 3.6 ulp in fp32 arithmetic,
and the MUFU ex2.approx.f32 it stands in for is documented at about 2 ulp."""
import numpy as np
import pytest

import gpu_helpers as H
import speculative_sampling_b200 as sd

pytestmark = pytest.mark.gpu

ULP = 2.0 ** -24


def _exp2_poly(a_np, torch):
    a = torch.from_numpy(a_np).cuda()
    y = torch.empty_like(a)
    st = sd.specdec_test_exp2(a.data_ptr(), y.data_ptr(), a.numel(),
                              torch.cuda.current_stream().cuda_stream)
    assert st == sd.SPECDEC_OK
    torch.cuda.synchronize()
    return a, y


def test_fma_exp2_within_4_ulp():
    torch = H.require_cuda()
    rng = np.random.default_rng(0)
    a_np = np.concatenate([
        np.linspace(-125.0, 64.0, 4_000_001, dtype=np.float32),
        rng.uniform(-40.0, 1.0, 2_000_000).astype(np.float32),
        # near the rounding points of the reduction and around 0
        (np.arange(-125, 64, dtype=np.float32)[:, None] +
         np.array([-0.5, -0.4999999, 0.4999999, 0.5, 0.0], np.float32)).ravel(),
        np.array([0.0, -0.0, 1e-30, -1e-30, 63.99999], np.float32)])
    a_np = a_np[(a_np >= -125.0) & (a_np <= 64.0)]
    a, y = _exp2_poly(a_np, torch)
    y_np = y.cpu().numpy().astype(np.float64)
    ref = np.exp2(a_np.astype(np.float64))
    rel = np.abs(y_np - ref) / ref
    assert rel.max() <= 4 * ULP, (rel.max() / ULP, a_np[np.argmax(rel)])
    # against CUDA's exp2f on the same arguments
    cu = torch.exp2(a).cpu().numpy().astype(np.float64)
    d = np.abs(y_np - cu) / cu
    assert d.max() <= 5 * ULP, d.max() / ULP
    print("max error", rel.max() / ULP, "ulp vs fp64;", d.max() / ULP, "ulp vs exp2f")


def test_fma_exp2_small_and_odd_arguments():
    torch = H.require_cuda()
    a_np = np.array([-125.5, -126.0, -200.0, -1e30, -np.inf, 3.0, 0.25], np.float32)
    _, y = _exp2_poly(a_np, torch)
    y_np = y.cpu().numpy().astype(np.float64)
    # below -125: about 2^-125 (a negligible term, never more than 2^-124.5)
    assert np.all((y_np[:5] > 0) & (y_np[:5] <= 2.0 ** -124.5))
    assert abs(y_np[5] - 8.0) <= 4 * ULP * 8.0 and abs(y_np[6] - 2 ** 0.25) <= 4 * ULP * 2 ** 0.25
    # odd length (the last element is handled alone) and empty input
    _, y3 = _exp2_poly(np.array([1.0, 2.0, 3.0], np.float32), torch)
    assert np.allclose(y3.cpu().numpy(), [2.0, 4.0, 8.0], rtol=4 * ULP, atol=0)
    assert sd.specdec_test_exp2(None, None, 0, None) == sd.SPECDEC_OK
    assert sd.specdec_test_exp2(None, None, -1, None) == sd.SPECDEC_EINVAL
