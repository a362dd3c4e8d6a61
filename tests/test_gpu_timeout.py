"""A bounded on-chip wait that runs out, on purpose and without a fault.

The test hook makes the statistics sweep's producer skip the copy of one tile
and sets every wait's bound to 1 ms.  The consumer warps' waits for that tile
then run out: the kernel sets SPECDEC_ERR_TIMEOUT, marks the statistics it
could not finish as incomplete and winds down (after its own copies in flight
have landed); the sequence whose row held the tile gets outputs -1, the others
are verified as usual, and the next call (hook cleared) is exact again."""
import numpy as np
import pytest

import gpu_helpers as H
import speculative_sampling_b200 as sd
from speculative_sampling_b200 import inputs

pytestmark = pytest.mark.gpu


def test_wait_runs_out_and_the_device_recovers():
    H.require_cuda()
    x = inputs.generate("batched_b64_k5_v128256_bf16", B=8)  # one wave: one sweep launch
    o = H.oracle_verify(x)
    d = H.to_device(x)
    tpr = -(-(-(-x.V // 8)) // 1024)          # 16 KB tiles of 1024 vectors of 8 bf16
    rps = 2 * x.K + 1
    skip = 7 * tpr + 3                        # a tile of row 7, which belongs to sequence 0
    assert skip // tpr // rps == 0
    sd.specdec_device_errors(None)            # clear
    assert sd.specdec_test_set_wait_fault(skip, 1_000_000) == sd.SPECDEC_OK
    try:
        g = H.gpu_verify(x, dev_inputs=d, debug=False)
    finally:
        assert sd.specdec_test_set_wait_fault(-1, 2_000_000_000) == sd.SPECDEC_OK
    st, flags = sd.specdec_device_errors(None)
    assert st == sd.SPECDEC_EDEVICE and flags == sd.SPECDEC_ERR_TIMEOUT, (st, flags)
    n = g["num_accepted"]
    assert n[0] == -1 and np.all(g["out_tokens"][0] == -1)
    hit = np.nonzero(n < 0)[0]
    assert hit.size <= 2, hit                 # the CTA holding the tile spans <= 2 sequences
    ok = n >= 0
    H.compare({k: v[ok] for k, v in g.items()}, {k: v[ok] for k, v in o.items()}, stats=False)
    # hook cleared: the same inputs verify exactly and no error is flagged
    g2 = H.gpu_verify(x, dev_inputs=d)
    H.compare(g2, o)
    assert sd.specdec_device_errors(None) == (sd.SPECDEC_OK, 0)


def test_hook_arguments_checked():
    H.require_cuda()
    assert sd.specdec_test_set_wait_fault(-2, 1000) == sd.SPECDEC_EINVAL
    assert sd.specdec_test_set_wait_fault(5, 0) == sd.SPECDEC_EINVAL
    assert sd.specdec_test_set_wait_fault(-1, 2_000_000_000) == sd.SPECDEC_OK


def test_get_error_and_error_string():
    torch = H.require_cuda()
    x = inputs.generate("mix_b128_k4_v32000_bf16", B=4, V=3000)
    x.tokens[2, 1] = x.V                      # out of range: flagged on the device
    sd.specdec_get_error()                    # clear
    g = H.gpu_verify(x, debug=False)
    assert g["num_accepted"][2] == -1
    assert sd.specdec_get_error() == sd.SPECDEC_EDEVICE
    assert sd.specdec_get_error() == sd.SPECDEC_OK   # read and cleared
    assert sd.specdec_error_string(sd.SPECDEC_EDEVICE) == sd.status_string(sd.SPECDEC_EDEVICE)
    torch.cuda.synchronize()
