"""The verify entry points inside CUDA graphs: a serving loop captures the
step once and replays it with new inputs copied into the same buffers.  The
replays must give exactly what direct calls give.  The library-owned
workspace cannot grow while a stream is being captured: such a call returns
SPECDEC_ESTATE and launches nothing."""
import numpy as np
import pytest

import gpu_helpers as H
import speculative_sampling_b200 as sd
from speculative_sampling_b200 import inputs

pytestmark = pytest.mark.gpu


def _bufs(x, torch):
    d = H.to_device(x)
    d["ot"] = torch.full((x.B, x.K + 1), -7, dtype=torch.int32, device="cuda")
    d["on"] = torch.full((x.B,), -7, dtype=torch.int32, device="cuda")
    return d


def _args(x, d, stream):
    return (d["target"].data_ptr(), d["draft"].data_ptr(), d["tokens"].data_ptr(),
            d["u_accept"].data_ptr(), d["u_resample"].data_ptr(), d["temperature"].data_ptr(),
            x.B, x.K, x.V, sd.SPECDEC_BF16, d["ot"].data_ptr(), d["on"].data_ptr(), stream)


@pytest.mark.parametrize("entry", ["specdec_verify", "specdec_verify_early_exit"])
def test_graph_replay_matches_direct_calls(entry):
    torch = H.require_cuda()
    fn = getattr(sd, entry)
    a = inputs.generate("batched_b64_k5_v128256_bf16", B=16)
    b = inputs.generate("mix_b128_k4_v32000_bf16", B=16, V=a.V, K=a.K)
    d = _bufs(a, torch)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        # a direct call first: sizes the workspace
        assert fn(*_args(a, d, s.cuda_stream)) == sd.SPECDEC_OK
        s.synchronize()
        want_a = (d["ot"].cpu().numpy().copy(), d["on"].cpu().numpy().copy())
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=s):
            st = fn(*_args(a, d, s.cuda_stream))
        assert st == sd.SPECDEC_OK
    # replay on the captured inputs, then on new inputs copied into the buffers
    d["ot"].fill_(-7)
    g.replay()
    torch.cuda.synchronize()
    assert np.array_equal(d["ot"].cpu().numpy(), want_a[0])
    assert np.array_equal(d["on"].cpu().numpy(), want_a[1])
    nb = H.to_device(b)
    for k in ("target", "draft", "tokens", "u_accept", "u_resample", "temperature"):
        d[k].copy_(nb[k])
    g.replay()
    torch.cuda.synchronize()
    got = (d["ot"].cpu().numpy(), d["on"].cpu().numpy())
    db = _bufs(b, torch)
    assert fn(*_args(b, db, torch.cuda.current_stream().cuda_stream)) == sd.SPECDEC_OK
    torch.cuda.synchronize()
    assert np.array_equal(got[0], db["ot"].cpu().numpy())
    assert np.array_equal(got[1], db["on"].cpu().numpy())
    o = H.oracle_verify(b)
    H.compare({"out_tokens": got[0], "num_accepted": got[1]}, o, stats=False)


def test_workspace_growth_is_refused_during_capture():
    torch = H.require_cuda()
    sd.specdec_release()  # the next call has to allocate
    x = inputs.generate("tiny_b1_k4_v1000_f32", B=4)
    d = H.to_device(x)
    ot = torch.empty((x.B, x.K + 1), dtype=torch.int32, device="cuda")
    on = torch.empty((x.B,), dtype=torch.int32, device="cuda")
    s = torch.cuda.Stream()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(s):
        with torch.cuda.graph(g, stream=s):
            st = sd.specdec_verify_f32(d["target"].data_ptr(), d["draft"].data_ptr(),
                                       d["tokens"].data_ptr(), d["u_accept"].data_ptr(),
                                       d["u_resample"].data_ptr(), d["temperature"].data_ptr(),
                                       x.B, x.K, x.V, ot.data_ptr(), on.data_ptr(), s.cuda_stream)
    assert st == sd.SPECDEC_ESTATE
