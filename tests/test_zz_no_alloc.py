"""specdec_verify_static, the allocation-free entry point.

Some callers of this library may not allocate device memory: a serving engine
that has handed nearly all of HBM to its own pools (KV cache) and forbids
allocations outside them, or a latency-critical loop that cannot pay for
cudaMalloc's device-wide synchronisation.  specdec_verify_static serves them by
keeping its workspace in a fixed array inside the library.  These tests call it
through the C-ABI and check that it returns exactly what specdec_verify returns
on the same inputs, on two calls in a row (the array keeps the previous call's
contents, which must not matter), and that sizes beyond the array are refused
without touching the outputs.

This file is named so that pytest collects it last.
"""
import numpy as np
import pytest

import gpu_helpers as H
import speculative_sampling_b200 as sd
from speculative_sampling_b200 import inputs

pytestmark = pytest.mark.gpu


def _call(fn, x, d, torch):
    ot = torch.full((x.B, x.K + 1), -7, dtype=torch.int32, device="cuda")
    on = torch.full((x.B,), -7, dtype=torch.int32, device="cuda")
    dt = sd.SPECDEC_BF16 if x.dtype == "bf16" else sd.SPECDEC_F32
    st = fn(d["target"].data_ptr(), d["draft"].data_ptr(), d["tokens"].data_ptr(),
            d["u_accept"].data_ptr(), d["u_resample"].data_ptr(), d["temperature"].data_ptr(),
            x.B, x.K, x.V, dt, ot.data_ptr(), on.data_ptr(),
            torch.cuda.current_stream().cuda_stream)
    torch.cuda.synchronize()
    return st, ot.cpu().numpy(), on.cpu().numpy()


@pytest.mark.parametrize("name,B,V", [
    ("batched_b64_k5_v128256_bf16", None, None),   # the benchmarked batch
    ("mix_b128_k4_v32000_bf16", None, None),
    ("large_b256_k8_v151936_f32", 24, 30011),      # fp32, ragged rows
])
def test_static_scratch_matches_allocating_entry_point(name, B, V):
    torch = H.require_cuda()
    x = inputs.generate(name, B=B, V=V)
    d = H.to_device(x)
    st, ref_tok, ref_n = _call(sd.specdec_verify, x, d, torch)
    assert st == sd.SPECDEC_OK
    # integer outputs: the tests' tolerance for them is bit-exact
    for _ in range(2):
        st, tok, n = _call(sd.specdec_verify_static, x, d, torch)
        assert st == sd.SPECDEC_OK, sd.status_string(st)
        assert np.array_equal(tok, ref_tok)
        assert np.array_equal(n, ref_n)
    # and the allocating path still agrees with the CPU oracle
    o = H.oracle_verify(x)
    H.compare({"out_tokens": tok, "num_accepted": n}, o, stats=False)


def test_static_scratch_after_other_sizes():
    """A call after calls of other sizes (stale scratch contents) is unaffected."""
    torch = H.require_cuda()
    a = inputs.generate("mix_b128_k4_v32000_bf16", B=40, V=7001)
    b = inputs.generate("batched_b64_k5_v128256_bf16", B=9)
    da, db = H.to_device(a), H.to_device(b)
    _, ref_tok, ref_n = _call(sd.specdec_verify, a, da, torch)
    for x, d in ((b, db), (a, da), (b, db), (a, da)):
        st, tok, n = _call(sd.specdec_verify_static, x, d, torch)
        assert st == sd.SPECDEC_OK
    assert np.array_equal(tok, ref_tok) and np.array_equal(n, ref_n)


def test_static_scratch_refuses_oversized_batches():
    torch = H.require_cuda()
    K, V = 8, 151936
    B = 256
    while sd.specdec_workspace_bytes(B, K, V, sd.SPECDEC_F32) <= sd.SPECDEC_STATIC_SCRATCH_BYTES:
        B *= 2
    assert sd.specdec_workspace_bytes(B, K, V, sd.SPECDEC_F32) > sd.SPECDEC_STATIC_SCRATCH_BYTES
    # tiny real buffers: the call must refuse before reading or writing any
    t = torch.zeros(64, dtype=torch.float32, device="cuda")
    out = torch.full((16,), -7, dtype=torch.int32, device="cuda")
    p = t.data_ptr()
    st = sd.specdec_verify_static(p, p, p, p, p, p, B, K, V, sd.SPECDEC_F32, out.data_ptr(),
                                  out.data_ptr(), torch.cuda.current_stream().cuda_stream)
    torch.cuda.synchronize()
    assert st == sd.SPECDEC_ESIZE
    assert "fixed scratch" in sd.status_string(st)
    assert torch.all(out == -7)
