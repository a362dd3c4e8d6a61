"""The two rounding fallbacks of the draw on the GPU, against the oracle:

  * Z = 0 after a rejection: draft row n equals target row n and the draft
    token has probability 0 under both, so the walk rejects there and the
    residual max(0, p - q) vanishes; the draw then comes from p_n.  The
    uniforms are in [0, 1) as usual; the expected tokens are the oracle's, and
    also numpy's inverse CDF of p_n.
  * no running sum exceeds u*Z: with u_resample = 1 the target t equals the
    total exactly, and the draw is the last index with positive weight (the
    limit of the inverse CDF as u -> 1).  The rows end in -inf logits (bonus
    case) or in entries where p < q (residual case), so the last positive index
    is not V - 1.
"""
import numpy as np
import pytest

import gpu_helpers as H
from speculative_sampling_b200 import inputs

pytestmark = pytest.mark.gpu


def _softmax64(z, T):
    z = np.asarray(z, np.float64)
    e = np.exp((z - z.max()) / T)
    return e / e.sum()


@pytest.mark.parametrize("V", [6, 4099, 40000])
def test_zero_residual_draws_from_target_row(V):
    x = inputs.generate("large_b256_k8_v151936_f32", B=16, K=3, V=V)
    rng = np.random.default_rng(V)
    for b in range(x.B):
        n = b % x.K                              # the position that rejects
        x.draft[b, n] = x.target[b, n]
        x.tokens[b, n] = (7 * b) % V
        x.target[b, n, x.tokens[b, n]] = -1000.0   # p(x) = q(x) = 0 in fp64
        x.draft[b, n, x.tokens[b, n]] = -1000.0
        x.tokens[b, :n] = np.argmax(x.draft[b, :n], axis=1)  # earlier positions: likely accepted
        x.u_accept[b, :n] = 0.0                  # u = 0 accepts any token with p > 0
    x.u_resample[:] = rng.integers(0, 2 ** 24, x.B).astype(np.float32) * np.float32(2.0 ** -24)
    g = H.gpu_verify(x)
    o = H.oracle_verify(x)
    n = o["num_accepted"]
    assert np.array_equal(g["num_accepted"], n)
    assert np.all(n == np.arange(x.B) % x.K)
    for b in range(x.B):
        p = _softmax64(x.target[b, n[b]], float(x.temperature[b]))
        cdf = np.cumsum(p)
        t = float(x.u_resample[b]) * cdf[-1]
        y = int(np.searchsorted(cdf, t, side="right"))
        assert o["out_tokens"][b, n[b]] == y
        # the GPU agrees wherever the draw is not within 1e-6 of a cell edge
        lo = cdf[y - 1] if y > 0 else 0.0
        if min(t - lo, cdf[y] - t) / cdf[-1] > H.BAND:
            assert g["out_tokens"][b, n[b]] == y, (b, g["out_tokens"][b], y)
        assert np.array_equal(g["out_tokens"][b, :n[b]], x.tokens[b, :n[b]])
        assert np.all(g["out_tokens"][b, n[b] + 1:] == -1)


@pytest.mark.parametrize("V", [8, 5003])
def test_no_cell_reached_takes_last_positive(V):
    x = inputs.generate("large_b256_k8_v151936_f32", B=8, K=2, V=V)
    last = V - 3
    for b in range(x.B):
        if b % 2 == 0:   # bonus draw: every token accepted, row K ends in -inf
            x.draft[b] = x.target[b, :x.K]
            x.u_accept[b] = 0.5
            x.target[b, x.K, last + 1:] = -np.inf
        else:            # residual at position 0 with p < q on the last entries
            x.target[b, 0, last + 1:] = -30.0
            x.draft[b, 0, last + 1:] = 5.0
            x.tokens[b, 0] = V - 1       # q(x) >> p(x): rejected for u = 0.99
            x.u_accept[b, 0] = 0.99
    x.u_resample[:] = 1.0
    g = H.gpu_verify(x, debug=False)
    o = H.oracle_verify(x)
    assert np.array_equal(g["num_accepted"], o["num_accepted"])
    n = o["num_accepted"]
    for b in range(x.B):
        assert n[b] == (x.K if b % 2 == 0 else 0)
        if b % 2 == 0:
            want = last
        else:
            p = _softmax64(x.target[b, 0], float(x.temperature[b]))
            q = _softmax64(x.draft[b, 0], float(x.temperature[b]))
            want = int(np.nonzero(p - q > 0)[0].max())
        assert o["out_tokens"][b, n[b]] == want
        assert g["out_tokens"][b, n[b]] == want, (b, g["out_tokens"][b], want)
