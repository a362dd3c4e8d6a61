"""Calls on two streams whose kernels overlap on the GPU.  The library keeps
one workspace per (device, stream), so the calls share no partials, chunk
sums or arrival tickets: each result must equal the same call made alone, and
the oracle's."""
import numpy as np
import pytest

import gpu_helpers as H
import speculative_sampling_b200 as sd
from speculative_sampling_b200 import inputs

pytestmark = pytest.mark.gpu

FIELDS = ("target", "draft", "tokens", "u_accept", "u_resample", "temperature")


def test_two_streams_back_to_back():
    torch = H.require_cuda()
    xa = inputs.generate("batched_b64_k5_v128256_bf16", seq_begin=0, seq_end=48)
    xb = inputs.generate("batched_b64_k5_v128256_bf16", seq_begin=48, seq_end=96)
    da, db = H.to_device(xa), H.to_device(xb)
    want = {}
    for key, d in (("a", da), ("b", db)):
        ot, on = sd.verify(*[d[k] for k in FIELDS])
        torch.cuda.synchronize()
        want[key] = (ot.cpu().numpy(), on.cpu().numpy())
    s1, s2 = torch.cuda.Stream(), torch.cuda.Stream()
    for s in (s1, s2):
        s.wait_stream(torch.cuda.current_stream())
    # size each stream's workspace, then issue calls on both with no
    # synchronisation between them
    for s, d in ((s1, da), (s2, db)):
        with torch.cuda.stream(s):
            sd.verify(*[d[k] for k in FIELDS], stream=s.cuda_stream)
    torch.cuda.synchronize()
    outs = []
    for rep in range(4):
        for key, s, d in (("a", s1, da), ("b", s2, db)):
            with torch.cuda.stream(s):
                ot, on = sd.verify(*[d[k] for k in FIELDS], stream=s.cuda_stream)
            outs.append((key, ot, on))
    torch.cuda.synchronize()
    for key, ot, on in outs:
        assert np.array_equal(ot.cpu().numpy(), want[key][0]), key
        assert np.array_equal(on.cpu().numpy(), want[key][1]), key
    for key, x in (("a", xa), ("b", xb)):
        H.compare({"out_tokens": want[key][0], "num_accepted": want[key][1]}, H.oracle_verify(x),
                  stats=False)
