"""Early-exit verify (specdec_verify_early_exit*) against the oracle.

The early-exit call reads the rows of positions 0 and 1 first and the rest of
a sequence's rows only when both of its first draft tokens are accepted; its
results are those of the oracle (the same rule as the full call: bit-exact
integers outside counted boundary draws, probabilities within 1e-5 on the rows
it reads).  The edge cases cover every route through the two passes: all
sequences stopping in the first pass, all going on to the second, K = 1 and
K = 2 (the second pass holds only the bonus row, or one position and the bonus
row), rows of odd length, and input errors inside the rows that are read.
"""
import numpy as np
import pytest

import gpu_helpers as H
import speculative_sampling_b200 as sd
from speculative_sampling_b200 import inputs

pytestmark = pytest.mark.gpu


def _split(K):
    return K if K < 2 else 2


@pytest.mark.parametrize("name,B,V", [
    ("tiny_b1_k4_v1000_f32", None, None),
    ("llama3_single_b1_k5_v128256_bf16", None, None),
    ("batched_b64_k5_v128256_bf16", None, None),
    ("mix_b128_k4_v32000_bf16", None, None),
    ("large_b256_k8_v151936_f32", 48, None),
])
def test_early_exit_matches_oracle(name, B, V):
    x = inputs.generate(name, B=B, V=V)
    g = H.gpu_verify(x, early_exit=True)
    o = H.oracle_verify(x)
    H.compare(g, o, early_split=_split(x.K))


@pytest.mark.parametrize("K,V,sigma", [(1, 4099, 0.5), (2, 4099, 0.5), (6, 33333, 0.3),
                                       (3, 5, 1.0)])
def test_early_exit_shapes(K, V, sigma):
    x = inputs.generate("large_b256_k8_v151936_f32", B=24, K=K, V=V, sigma=sigma)
    g = H.gpu_verify(x, early_exit=True)
    o = H.oracle_verify(x)
    H.compare(g, o, early_split=_split(K))


def test_early_exit_all_stop_early_and_all_go_on():
    # draft == target: every token accepted, every sequence takes the second pass
    x = inputs.generate("mix_b128_k4_v32000_bf16", B=32, V=7001)
    x.draft[:] = x.target[:, :x.K]
    o = H.oracle_verify(x)
    assert np.all(o["num_accepted"] == x.K)
    H.compare(H.gpu_verify(x, early_exit=True), o, early_split=2)
    # a uniform of 1 - 2^-24 rejects every draft token with p < q: most stop at 0
    y = inputs.generate("batched_b64_k5_v128256_bf16", B=16)
    y.u_accept[:] = np.float32(1.0 - 2.0 ** -24)
    o = H.oracle_verify(y)
    assert np.mean(o["num_accepted"] < 2) > 0.5
    H.compare(H.gpu_verify(y, early_exit=True), o, early_split=2)


def test_early_exit_agrees_with_full_call():
    x = inputs.generate("batched_b64_k5_v128256_bf16")
    d = H.to_device(x)
    a = H.gpu_verify(x, dev_inputs=d, debug=False)
    b = H.gpu_verify(x, dev_inputs=d, debug=False, early_exit=True)
    o = H.oracle_verify(x)
    bnd = H.oracle.boundary_mask(o, H.BAND)
    same = ~bnd
    assert np.array_equal(a["out_tokens"][same], b["out_tokens"][same])
    assert np.array_equal(a["num_accepted"][same], b["num_accepted"][same])
    # repeated early-exit calls are bit-identical
    c = H.gpu_verify(x, dev_inputs=d, debug=False, early_exit=True)
    assert np.array_equal(b["out_tokens"], c["out_tokens"])


def test_early_exit_invalid_inputs_in_read_rows():
    torch = H.require_cuda()
    x = inputs.generate("mix_b128_k4_v32000_bf16", B=12, V=3001)
    x.tokens[1, 0] = x.V            # token out of range at position 0 (first pass)
    x.temperature[2] = 0.0          # temperature (first pass)
    nan = inputs.f32_to_bf16_bits(np.array([np.nan], np.float32))[0]
    x.target[3, 1, 17] = nan        # NaN in the target row of position 1 (first pass)
    o = H.oracle_verify(x)
    assert np.all(o["num_accepted"][[1, 2, 3]] == -1)
    sd.specdec_device_errors(None)
    g = H.gpu_verify(x, early_exit=True)
    H.compare(g, o, early_split=2)
    st, flags = sd.specdec_device_errors(None)
    assert st == sd.SPECDEC_EDEVICE
    assert flags == (sd.SPECDEC_ERR_TOKEN | sd.SPECDEC_ERR_TEMPERATURE | sd.SPECDEC_ERR_LOGITS)
