"""Multi-rank host logic on CPU (gloo, world size 2): batch sharding, the max
of per-rank times, and gathering outputs.  The per-rank verify here is the CPU
oracle (test infrastructure), which lets the sharded pipeline be checked end
to end without a GPU: the gathered outputs must equal one whole-batch run."""
import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp

WORKLOAD = "mix_b128_k4_v32000_bf16"
PER_RANK = 6
V = 3001


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, result_q):
    import datetime

    import torch
    import torch.distributed as dist

    import oracle
    from speculative_sampling_b200 import dist as sdist
    from speculative_sampling_b200 import inputs

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        w = inputs.WORKLOADS[WORKLOAD]
        b0, b1 = sdist.shard_range(PER_RANK, rank)
        x = inputs.generate(WORKLOAD, seq_begin=b0, seq_end=b1, B=PER_RANK * world, V=V)
        r = oracle.verify(x.target, x.draft, x.tokens, x.u_accept, x.u_resample,
                          x.temperature, dtype=w.dtype, diag=False)
        t_max = sdist.max_over_ranks(1.5 + rank)  # a stand-in per-rank time
        toks, ns = sdist.gather_outputs(torch.from_numpy(r["out_tokens"]),
                                        torch.from_numpy(r["num_accepted"]))
        dist.barrier()
        if rank == 0:
            result_q.put(("ok", t_max, toks.numpy(), ns.numpy()))
        else:
            result_q.put(("rank", rank, toks is None and ns is None))
    except Exception as e:  # pragma: no cover - reported to the parent
        result_q.put(("error", repr(e)))
    finally:
        dist.destroy_process_group()


def test_shards_match_whole_batch_generation():
    from speculative_sampling_b200 import dist as sdist
    from speculative_sampling_b200 import inputs
    whole = inputs.generate(WORKLOAD, B=3 * PER_RANK, V=V)
    parts = [inputs.generate(WORKLOAD, *sdist.shard_range(PER_RANK, r), B=3 * PER_RANK, V=V)
             for r in range(3)]
    cat = sdist.concat_inputs(parts)
    for k, a in cat.items():
        assert np.array_equal(a, getattr(whole, k), equal_nan=True), k
    assert sdist.shard_range(64, 3) == (192, 256)
    with pytest.raises(ValueError):
        sdist.shard_range(-1, 0)


def test_gloo_two_ranks_shard_verify_gather():
    import oracle
    from speculative_sampling_b200 import inputs
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    msgs = [q.get(timeout=180) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    errs = [m for m in msgs if m[0] == "error"]
    assert not errs, errs
    ok = [m for m in msgs if m[0] == "ok"][0]
    others = [m for m in msgs if m[0] == "rank"]
    assert all(m[2] for m in others), "non-destination ranks get no gathered output"
    _, t_max, toks, ns = ok
    assert t_max == 2.5
    w = inputs.WORKLOADS[WORKLOAD]
    whole = inputs.generate(WORKLOAD, B=world * PER_RANK, V=V)
    ref = oracle.verify(whole.target, whole.draft, whole.tokens, whole.u_accept,
                        whole.u_resample, whole.temperature, dtype=w.dtype, diag=False)
    assert np.array_equal(toks, ref["out_tokens"])
    assert np.array_equal(ns, ref["num_accepted"])


def test_helpers_without_process_group():
    import torch

    from speculative_sampling_b200 import dist as sdist
    assert sdist.max_over_ranks(3.0) == 3.0
    a, b = torch.zeros(2, 3), torch.zeros(2)
    assert sdist.gather_outputs(a, b)[0] is a
