"""Calls issued back to back on one stream, with no synchronisation between
them.  Every kernel of a call is launched with programmatic dependent launch:
a call's statistics sweep may be placed on the GPU while the kernel before it
(the previous call's k_finish, or the copy that writes this call's inputs) is
still running, and it must neither read its inputs nor touch the library's
workspace before that kernel has completed.  Each call's result must equal
what the same call gives alone."""
import numpy as np
import pytest

import gpu_helpers as H
import speculative_sampling_b200 as sd
from speculative_sampling_b200 import inputs

pytestmark = pytest.mark.gpu

FIELDS = ("target", "draft", "tokens", "u_accept", "u_resample", "temperature")


def _batches(name, n, B, **kw):
    """n batches of the same shape with different sequences (seed streams)."""
    return [inputs.generate(name, seq_begin=i * B, seq_end=(i + 1) * B, **kw) for i in range(n)]


def _args(d):
    return [d[k] for k in FIELDS]


@pytest.mark.parametrize("name,B,kw", [
    ("batched_b64_k5_v128256_bf16", 64, {}),
    ("mix_b128_k4_v32000_bf16", 16, {"V": 4099}),
    ("large_b256_k8_v151936_f32", 8, {"V": 10007}),
])
def test_inputs_rewritten_between_calls(name, B, kw):
    """One set of device buffers; before each call a copy kernel writes the
    next batch into them.  The sweep of each call must see its own batch."""
    torch = H.require_cuda()
    xs = _batches(name, 4, B, **kw)
    srcs = [H.to_device(x) for x in xs]
    want = []
    for d in srcs:  # each batch alone
        ot, on = sd.verify(*_args(d))
        torch.cuda.synchronize()
        want.append((ot.cpu().numpy(), on.cpu().numpy()))
    buf = {k: torch.empty_like(srcs[0][k]) for k in FIELDS}
    outs = []
    for rnd in range(2):
        for i, d in enumerate(srcs):
            for k in FIELDS:
                buf[k].copy_(d[k])
            ot, on = sd.verify(*_args(buf))
            outs.append((i, ot.clone(), on.clone()))
    torch.cuda.synchronize()
    for i, ot, on in outs:
        assert np.array_equal(ot.cpu().numpy(), want[i][0])
        assert np.array_equal(on.cpu().numpy(), want[i][1])
    o = H.oracle_verify(xs[0])
    H.compare({"out_tokens": want[0][0], "num_accepted": want[0][1]}, o, stats=False)


def test_entry_points_interleaved():
    """The verify (full and early exit), the SMC-SD step, the chained verify
    and the top-k candidates, one after another on one stream, sharing the
    library workspace, twice over; then each compared with a call made alone."""
    torch = H.require_cuda()
    xa, xb = _batches("batched_b64_k5_v128256_bf16", 2, 32)
    da, db = H.to_device(xa), H.to_device(xb)
    B, K = xa.B, xa.K
    ur_g = torch.full((B // 8,), 0.37, dtype=torch.float32, device="cuda")
    u2 = torch.full((B, K + 1), 0.5, dtype=torch.float32, device="cuda")
    ridx = torch.arange(B * (K + 1), dtype=torch.int64, device="cuda")

    def run_all():
        r = {}
        r["full_a"] = sd.verify(*_args(da))
        r["early_b"] = sd.verify(*_args(db), early_exit=True)
        s = sd.smc_step(da["target"], da["draft"], da["tokens"], da["u_resample"],
                        da["temperature"], ur_g, 8, ess_threshold=0.9)
        r["smc_a"] = (s["out_tokens"], s["increment"], s["ancestors"])
        c = sd.verify_chained(db["target"], db["target"], db["draft"], db["tokens"],
                              db["u_accept"], db["u_resample"], u2, db["u_resample"],
                              db["temperature"])
        r["chained_b"] = (c["out_tokens"], c["num_emitted"])
        r["topk_a"] = sd.topk_exclude(da["target"].reshape(-1, xa.V), 60, row_index=ridx)
        r["full_b"] = sd.verify(*_args(db))
        return {k: tuple(t.clone() for t in v) for k, v in r.items()}

    run_all()  # sizes the library workspace
    torch.cuda.synchronize()
    alone = {}
    # each entry point alone, synchronised
    alone["full_a"] = sd.verify(*_args(da))
    torch.cuda.synchronize()
    alone["early_b"] = sd.verify(*_args(db), early_exit=True)
    torch.cuda.synchronize()
    s = sd.smc_step(da["target"], da["draft"], da["tokens"], da["u_resample"], da["temperature"],
                    ur_g, 8, ess_threshold=0.9)
    torch.cuda.synchronize()
    alone["smc_a"] = (s["out_tokens"], s["increment"], s["ancestors"])
    c = sd.verify_chained(db["target"], db["target"], db["draft"], db["tokens"], db["u_accept"],
                          db["u_resample"], u2, db["u_resample"], db["temperature"])
    torch.cuda.synchronize()
    alone["chained_b"] = (c["out_tokens"], c["num_emitted"])
    alone["topk_a"] = sd.topk_exclude(da["target"].reshape(-1, xa.V), 60, row_index=ridx)
    torch.cuda.synchronize()
    alone["full_b"] = sd.verify(*_args(db))
    torch.cuda.synchronize()
    alone = {k: tuple(t.cpu().numpy() for t in v) for k, v in alone.items()}
    for rnd in range(2):
        got = run_all()
        torch.cuda.synchronize()
        for k, v in got.items():
            for a, b in zip(v, alone[k]):
                assert np.array_equal(a.cpu().numpy(), b), (rnd, k)
    # the two full calls are also the oracle's
    for x, key in ((xa, "full_a"), (xb, "full_b")):
        H.compare({"out_tokens": alone[key][0], "num_accepted": alone[key][1]},
                  H.oracle_verify(x), stats=False)
