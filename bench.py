"""Benchmark of the batched speculative-sampling verify step on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl {cuda,reference}]
                    [--workload NAME]

One step = one specdec_verify call (the whole hot path: row statistics,
acceptance, residual/bonus draw) over one batch of the workload, by default
B=64 sequences, K=5 draft tokens, V=128256 (Llama-3 vocabulary), bf16 logits.
Under torchrun every rank verifies its own batch of B sequences (rank r takes
sequences [r*B, (r+1)*B) of the same seeded stream: weak scaling, no collective
on the data path; NCCL only carries the barrier and the max-over-ranks time).

Prints one JSON line (rank 0).  ``value`` is the whole-job verify throughput in
GB/s of algorithmic bytes (one read of both logit tensors) with the inputs
resident in HBM; ``e2e`` is the same metric through specdec_verify_host with
pinned host buffers (host->device copies and the result read-back inside the
timed region).  ``--impl reference`` times the fp64 CPU oracle on the host
cores on the same workload (one sequence per step).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from speculative_sampling_b200 import inputs  # noqa: E402

METRIC = "verify GB/s (% of HBM peak) and rows/s at B=64 K=5 V=128256 bf16"
NOMINAL_HBM_GBS = 8000.0
FALLBACK_HBM_GBS = 6650.0
L2_BYTES = 126 * 2 ** 20
# Device cycles of a delay queued on the stream just before a timed region's
# start event (about 0.3 ms at 2 GHz): while the device waits, the host queues
# the region's first launches, so the events bracket the device's time for the
# K steps and not the host's issue of the first one.  Nothing of the verify
# runs during the delay, which lies outside the region.
QUEUE_DELAY_CYCLES = 600_000


def start_region(torch, ev, stream):
    with torch.cuda.stream(stream):
        torch.cuda._sleep(QUEUE_DELAY_CYCLES)
    ev.record(stream)


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["cuda", "reference"], default="cuda")
    ap.add_argument("--workload", default="batched_b64_k5_v128256_bf16")
    ap.add_argument("--e2e-steps", type=int, default=20)
    ap.add_argument("--cpu-seconds", type=float, default=10.0,
                    help="minimum oracle time for the cpu_baseline leg")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--kernel-timing", choices=["on", "off"], default="on")
    ap.add_argument("--early-exit", choices=["on", "off"], default="on",
                    help="also time specdec_verify_early_exit on the same steps")
    ap.add_argument("--chained", choices=["on", "off"], default="on",
                    help="also time specdec_verify_chained (an intermediate tensor of the "
                         "target's shape, the target logits as the final layer)")
    ap.add_argument("--early-exit-large", choices=["on", "off"], default="on",
                    help="also time the full call and early exit on the large fp32 workload's "
                         "shape (K=8, V=151936) at 64 sequences per rank")
    ap.add_argument("--topk", choices=["on", "off"], default="on",
                    help="also time specdec_topk_exclude (k=60) over the target's draft rows")
    ap.add_argument("--smc", choices=["on", "off"], default="on",
                    help="also time specdec_smc_step (groups of 8 particles) on the same steps")
    return ap.parse_args()


def measured_peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def stored_traffic():
    """DRAM bytes (read + write) of one verify step of the bench workload from
    the committed ncu capture (profiles/verify_step_traffic.json): per launch of
    the sweep, and of the whole step (every kernel).  Valid only while the
    kernel source is unchanged since the capture (checked by hash); None
    otherwise."""
    p = os.path.join(ROOT, "profiles", "verify_step_traffic.json")
    src = os.path.join(ROOT, "speculative_sampling_b200", "csrc", "specdec.cu")
    try:
        with open(p) as f:
            d = json.load(f)
        h = hashlib.sha256(open(src, "rb").read()).hexdigest()
        if d.get("source_sha256") != h:
            return None
        return d
    except Exception:
        return None


class ClockSampler:
    """SM clock and throttle reasons of one GPU, sampled via NVML while running:
    every 10 ms, and back to back (no sleep) while ``fast`` is set, so that a
    timed region of a millisecond still gets samples."""

    REASONS = {
        "gpu_idle": 0x1, "applications_clocks_setting": 0x2, "sw_power_cap": 0x4,
        "hw_slowdown": 0x8, "sync_boost": 0x10, "sw_thermal_slowdown": 0x20,
        "hw_thermal_slowdown": 0x40, "hw_power_brake_slowdown": 0x80,
        "display_clock_setting": 0x100,
    }

    def __init__(self, index: int):
        self.samples = []
        self.window = None
        self.max_mhz = None
        self.err = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        except Exception as e:  # pragma: no cover - depends on the box
            self.nv = None
            self.err = str(e)
        self._stop = threading.Event()
        self._wake = threading.Event()
        self._t = None
        self.fast = False

    def _run(self):
        nv = self.nv
        while not self._stop.is_set():
            try:
                mhz = nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM)
                try:
                    r = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                except Exception:
                    r = nv.nvmlDeviceGetCurrentClocksThrottleReasons(self.h)
                self.samples.append((time.perf_counter(), mhz, r))
            except Exception as e:  # pragma: no cover
                self.err = str(e)
            if not self.fast:
                self._wake.wait(0.01)
                self._wake.clear()

    def start(self):
        if self.nv is not None:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()

    def go_fast(self):
        """Sample back to back from now on; returns once a fresh sample exists."""
        self.fast = True
        self._wake.set()
        if self.nv is None or self._t is None:
            return
        t = time.perf_counter()
        while (not self.samples or self.samples[-1][0] < t) and time.perf_counter() - t < 0.05:
            time.sleep(0)

    def stop(self):
        if self._t is not None:
            self._stop.set()
            self._wake.set()
            self._t.join()

    def summary(self):
        if self.nv is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0,
                    "note": f"NVML unavailable: {self.err}"}
        s = self.samples
        note = None
        if self.window:
            t0, t1 = self.window
            inside = [x for x in s if t0 <= x[0] <= t1]
            if inside:
                s = inside
            else:
                note = "timed region shorter than the sampling period; samples span warm-up too"
        mhz = [x[1] for x in s]
        bits = 0
        for x in s:
            bits |= int(x[2])
        reasons = [k for k, v in self.REASONS.items() if bits & v and k != "gpu_idle"]
        out = {"sm_mhz": statistics.median(mhz) if mhz else None, "sm_max_mhz": self.max_mhz,
               "reasons": reasons, "samples": len(s)}
        if note:
            out["note"] = note
        return out


# ---------------------------------------------------------------------------
def run_reference(args):
    """fp64 CPU oracle on the host cores, one sequence of the workload per step."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    import oracle
    w = inputs.WORKLOADS[args.workload]
    x = inputs.generate(args.workload)
    o = oracle.default()
    es = inputs.elem_size(w.dtype)
    per_seq = (2 * w.K + 1) * w.V * es

    def step(i):
        b = i % x.B
        s = slice(b, b + 1)
        o.verify(x.target[s], x.draft[s], x.tokens[s], x.u_accept[s], x.u_resample[s],
                 x.temperature[s], dtype=w.dtype, diag=False, nthreads=1)

    for i in range(args.warmup):
        step(i)
    t0 = time.perf_counter()
    for i in range(args.steps):
        step(args.warmup + i)
    dt = time.perf_counter() - t0
    gbs = per_seq * args.steps / dt / 1e9
    line = {
        "impl": "reference", "metric": METRIC, "value": gbs, "unit": "GB/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": dt / args.steps * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": args.workload, "B": w.B, "K": w.K, "V": w.V,
                   "logits_dtype": w.dtype},
        "cpu_baseline": {"value": gbs, "unit": "GB/s", "cores": 1, "kind": "oracle",
                         "sample": f"one sequence ({2 * w.K + 1} rows x {w.V}) of the workload "
                                   f"per step, rotating over its {w.B} sequences"},
        "e2e": {"value": gbs, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def cpu_baseline(x, w, seconds):
    import oracle
    o = oracle.default()
    cores = os.cpu_count() or 1
    per_batch = x.floor_bytes
    t0 = time.perf_counter()
    reps = 0
    while True:
        o.verify(x.target, x.draft, x.tokens, x.u_accept, x.u_resample, x.temperature,
                 dtype=w.dtype, diag=False, nthreads=cores)
        reps += 1
        if time.perf_counter() - t0 >= seconds:
            break
    dt = time.perf_counter() - t0
    return {"value": per_batch * reps / dt / 1e9, "unit": "GB/s", "cores": cores,
            "kind": "oracle",
            "sample": f"the whole {x.B}-sequence batch of the workload, repeated {reps}x "
                      f"({dt:.1f} s), sequences split over {cores} threads"}


def run_cuda(args):
    import torch
    import speculative_sampling_b200 as sd
    from speculative_sampling_b200 import dist as sdist

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        if world == 1 and args.gpus > 1:
            raise SystemExit("--gpus N > 1 must be launched with torchrun (one rank per GPU)")
    torch.cuda.set_device(local)
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    dev = torch.device("cuda", local)
    w = inputs.WORKLOADS[args.workload]
    # weak scaling: rank r verifies sequences [r*B, (r+1)*B)
    x = sdist.generate_shard(args.workload, rank, world)
    B, K, V = x.B, x.K, x.V
    dt_code = sd.SPECDEC_BF16 if w.dtype == "bf16" else sd.SPECDEC_F32
    floor = x.floor_bytes
    # device copies: enough rotating copies that each step's inputs were last
    # touched more than L2's capacity ago
    ncopies = max(2, int(np.ceil(2 * L2_BYTES / floor)) + 1)
    tview = (lambda a: torch.from_numpy(a.view(np.int16)).view(torch.bfloat16)) \
        if w.dtype == "bf16" else (lambda a: torch.from_numpy(a))
    bufs = []
    for _ in range(ncopies):
        bufs.append(dict(
            t=tview(x.target).to(dev), d=tview(x.draft).to(dev),
            tok=torch.from_numpy(x.tokens).to(dev), ua=torch.from_numpy(x.u_accept).to(dev),
            ur=torch.from_numpy(x.u_resample).to(dev), T=torch.from_numpy(x.temperature).to(dev),
            ot=torch.empty((B, K + 1), dtype=torch.int32, device=dev),
            on=torch.empty((B,), dtype=torch.int32, device=dev)))
    stream = torch.cuda.current_stream(dev)
    sp = stream.cuda_stream
    calls = [(b["t"].data_ptr(), b["d"].data_ptr(), b["tok"].data_ptr(), b["ua"].data_ptr(),
              b["ur"].data_ptr(), b["T"].data_ptr(), B, K, V, dt_code, b["ot"].data_ptr(),
              b["on"].data_ptr(), sp) for b in bufs]
    L = sd.lib()
    fn = L.specdec_verify

    def step(i):
        st = fn(*calls[i % ncopies])
        if st != 0:
            raise RuntimeError(f"specdec_verify failed: {sd.status_string(st)}")

    def barrier():
        if dist is not None:
            dist.barrier()

    sampler = ClockSampler(torch.cuda.current_device() if world == 1 else local)
    sampler.start()
    for i in range(max(3, args.warmup)):
        step(i)
    torch.cuda.synchronize()
    # one verify result must agree with itself across copies (sanity, untimed)
    ref_tok = bufs[0]["ot"].cpu()
    if not torch.equal(ref_tok, bufs[1]["ot"].cpu()):
        raise RuntimeError("rotating input copies produced different outputs")

    nk = L.specdec_kernel_count()
    before = [L.specdec_launch_count(i) for i in range(nk)]
    # headline region: K steps exactly as a caller runs them (no per-kernel
    # events between the launches, which would break their programmatic overlap)
    barrier()
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    sampler.go_fast()
    tw0 = time.perf_counter()
    start_region(torch, e0, stream)
    for i in range(args.steps):
        step(i)
    e1.record(stream)
    torch.cuda.synchronize()
    tw1 = time.perf_counter()
    sampler.fast = False
    barrier()
    sampler.window = (tw0, tw1)
    sampler.stop()
    after = [L.specdec_launch_count(i) for i in range(nk)]
    ms = sdist.max_over_ranks(e0.elapsed_time(e1), dev)
    # step distribution: the same K steps again, each bracketed by its own pair
    # of events on the stream (back to back, no synchronisation between steps)
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(args.steps)]
    for i in range(args.steps):
        evs[i][0].record(stream)
        step(i)
        evs[i][1].record(stream)
    torch.cuda.synchronize()
    per_step = np.array([a.elapsed_time(b) for a, b in evs]) * 1e3  # us
    # single-call latency: one call at a time, synchronised before the next
    lat = []
    for i in range(min(args.steps, 100)):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        step(i)
        b.record(stream)
        torch.cuda.synchronize()
        lat.append(a.elapsed_time(b) * 1e3)
    lat = np.array(lat)
    # kernel region: the same K steps again with every launch bracketed by CUDA
    # events on its stream; gives each kernel's mean device time (roofline)
    kern = {}
    # launches of each kernel per step (the sweep runs once per wave of sequences)
    lps = [(a - b) / args.steps for a, b in zip(after, before)]
    if args.kernel_timing == "on":
        sd.profile_begin(int(args.steps * max(lps)) + 1)
        for i in range(args.steps):
            step(i)
        torch.cuda.synchronize()
        kern = sd.profile_end()
    ms_step = ms / args.steps
    total_bytes = floor * world
    gbs = total_bytes / (ms_step * 1e-3) / 1e9

    # ---- early exit: the same steps through specdec_verify_early_exit -------
    early = None
    if args.early_exit == "on":
        fe = L.specdec_verify_early_exit
        for i in range(3):
            if fe(*calls[i % ncopies]) != 0:
                raise RuntimeError("specdec_verify_early_exit failed")
        torch.cuda.synchronize()
        barrier()
        torch.cuda.synchronize()
        f0 = torch.cuda.Event(enable_timing=True)
        f1 = torch.cuda.Event(enable_timing=True)
        start_region(torch, f0, stream)
        for i in range(args.steps):
            fe(*calls[i % ncopies])
        f1.record(stream)
        torch.cuda.synchronize()
        barrier()
        ms_ee = sdist.max_over_ranks(f0.elapsed_time(f1), dev) / args.steps
        n_ee = bufs[0]["on"].cpu().numpy()
        same_tokens = bool(np.array_equal(bufs[0]["ot"].cpu().numpy(), ref_tok.numpy()))
        P = 2 if K >= 2 else K
        rows_read = int(np.sum(np.where(n_ee >= P, 2 * K + 1, 2 * P)))
        read_bytes = rows_read * V * (2 if w.dtype == "bf16" else 4)
        early = {"ms_per_step": ms_ee, "value": total_bytes / (ms_ee * 1e-3) / 1e9, "unit": "GB/s",
                 "rows_read_fraction": rows_read / (B * (2 * K + 1)),
                 "read_GBs": read_bytes * world / (ms_ee * 1e-3) / 1e9,
                 "tokens_equal_full_call": same_tokens,
                 "note": "value counts the full two-tensor floor per step, as the headline "
                         "does; read_GBs counts the rows this call actually reads"}
        # the same shape at low acceptance (draft noise 1.5 for every sequence):
        # the full call and early exit, each timed over the K steps
        xl = sdist.generate_shard(args.workload, rank, world, sigma=1.5)
        lb = [dict(t=tview(xl.target).to(dev), d=tview(xl.draft).to(dev),
                   tok=torch.from_numpy(xl.tokens).to(dev),
                   ua=torch.from_numpy(xl.u_accept).to(dev),
                   ur=torch.from_numpy(xl.u_resample).to(dev),
                   T=torch.from_numpy(xl.temperature).to(dev),
                   ot=torch.empty((B, K + 1), dtype=torch.int32, device=dev),
                   on=torch.empty((B,), dtype=torch.int32, device=dev)) for _ in range(ncopies)]
        lcalls = [(b["t"].data_ptr(), b["d"].data_ptr(), b["tok"].data_ptr(), b["ua"].data_ptr(),
                   b["ur"].data_ptr(), b["T"].data_ptr(), B, K, V, dt_code, b["ot"].data_ptr(),
                   b["on"].data_ptr(), sp) for b in lb]
        low = {}
        for key, f in (("full_ms_per_step", fn), ("early_exit_ms_per_step", fe)):
            for i in range(3):
                if f(*lcalls[i % ncopies]) != 0:
                    raise RuntimeError("verify failed on the low-acceptance batch")
            torch.cuda.synchronize()
            barrier()
            torch.cuda.synchronize()
            g0 = torch.cuda.Event(enable_timing=True)
            g1 = torch.cuda.Event(enable_timing=True)
            start_region(torch, g0, stream)
            for i in range(args.steps):
                f(*lcalls[i % ncopies])
            g1.record(stream)
            torch.cuda.synchronize()
            barrier()
            low[key] = sdist.max_over_ranks(g0.elapsed_time(g1), dev) / args.steps
            if key == "full_ms_per_step":
                low_tok = lb[0]["ot"].cpu().numpy().copy()
        n_l = lb[0]["on"].cpu().numpy()
        rows_l = int(np.sum(np.where(n_l >= P, 2 * K + 1, 2 * P)))
        low.update(rows_read_fraction=rows_l / (B * (2 * K + 1)),
                   mean_accepted=float(np.mean(n_l)),
                   tokens_equal_full_call=bool(np.array_equal(lb[0]["ot"].cpu().numpy(), low_tok)),
                   note="the bench shape with draft noise 1.5 for every sequence")
        early["low_acceptance"] = low
        del lb, lcalls

        # a workload where the rows early exit leaves unread outweigh its second
        # finish chain: the large fp32 workload's shape (K = 8, V = 151936) at
        # 64 sequences per rank, at its own draft noise and at 1.5
        if args.early_exit_large == "on":
            big = {}
            LB = 64
            for tag, sig in (("default_noise", None), ("noise_1.5", 1.5)):
                xb = sdist.generate_shard("large_b256_k8_v151936_f32", rank, world, per_rank=LB,
                                          sigma=sig)
                wb = inputs.WORKLOADS["large_b256_k8_v151936_f32"]
                tvb = tview if wb.dtype == w.dtype else (
                    (lambda a: torch.from_numpy(a.view(np.int16)).view(torch.bfloat16))
                    if wb.dtype == "bf16" else (lambda a: torch.from_numpy(a)))
                dtb = sd.SPECDEC_BF16 if wb.dtype == "bf16" else sd.SPECDEC_F32
                bb = [dict(t=tvb(xb.target).to(dev), d=tvb(xb.draft).to(dev),
                           tok=torch.from_numpy(xb.tokens).to(dev),
                           ua=torch.from_numpy(xb.u_accept).to(dev),
                           ur=torch.from_numpy(xb.u_resample).to(dev),
                           T=torch.from_numpy(xb.temperature).to(dev),
                           ot=torch.empty((LB, xb.K + 1), dtype=torch.int32, device=dev),
                           on=torch.empty((LB,), dtype=torch.int32, device=dev)) for _ in range(2)]
                bc = [(b["t"].data_ptr(), b["d"].data_ptr(), b["tok"].data_ptr(), b["ua"].data_ptr(),
                       b["ur"].data_ptr(), b["T"].data_ptr(), LB, xb.K, xb.V, dtb,
                       b["ot"].data_ptr(), b["on"].data_ptr(), sp) for b in bb]
                leg = {}
                for key, f in (("full_ms_per_step", fn), ("early_exit_ms_per_step", fe)):
                    for i in range(3):
                        if f(*bc[i % 2]) != 0:
                            raise RuntimeError("verify failed on the large-shape batch")
                    torch.cuda.synchronize()
                    barrier()
                    torch.cuda.synchronize()
                    h0 = torch.cuda.Event(enable_timing=True)
                    h1 = torch.cuda.Event(enable_timing=True)
                    start_region(torch, h0, stream)
                    for i in range(args.steps):
                        f(*bc[i % 2])
                    h1.record(stream)
                    torch.cuda.synchronize()
                    barrier()
                    leg[key] = sdist.max_over_ranks(h0.elapsed_time(h1), dev) / args.steps
                    if key == "full_ms_per_step":
                        big_tok = bb[0]["ot"].cpu().numpy().copy()
                Pb = 2 if xb.K >= 2 else xb.K
                n_b = bb[0]["on"].cpu().numpy()
                rows_b = int(np.sum(np.where(n_b >= Pb, 2 * xb.K + 1, 2 * Pb)))
                leg.update(rows_read_fraction=rows_b / (LB * (2 * xb.K + 1)),
                           mean_accepted=float(np.mean(n_b)),
                           tokens_equal_full_call=bool(np.array_equal(bb[0]["ot"].cpu().numpy(),
                                                                       big_tok)))
                big[tag] = leg
                del bb, bc, xb
                torch.cuda.empty_cache()
            early["large_fp32_shape"] = dict(
                big, workload="large_b256_k8_v151936_f32 recipe, B=%d per rank" % LB,
                bytes_per_step=LB * world * 17 * 151936 * 4)

    # ---- SMC-SD weight step on the same logits (groups of 8 particles) -------
    smc_line = None
    if args.smc == "on" and B % 8 == 0:
        Np = 8
        G = B // Np
        ur_g = torch.full((G,), 0.5, dtype=torch.float32, device=dev)
        lw_out = torch.empty((B,), dtype=torch.float64, device=dev)
        ess_o = torch.empty((G,), dtype=torch.float64, device=dev)
        anc = torch.empty((B,), dtype=torch.int32, device=dev)
        fs = L.specdec_smc_step

        def smc(i):
            b = bufs[i % ncopies]
            return fs(b["t"].data_ptr(), b["d"].data_ptr(), b["tok"].data_ptr(),
                      b["ur"].data_ptr(), b["T"].data_ptr(), None, ur_g.data_ptr(), 0.5, B, Np,
                      K, V, dt_code, b["ot"].data_ptr(), lw_out.data_ptr(), ess_o.data_ptr(),
                      anc.data_ptr(), None, sp)
        for i in range(3):
            if smc(i) != 0:
                raise RuntimeError("specdec_smc_step failed")
        torch.cuda.synchronize()
        barrier()
        torch.cuda.synchronize()
        s0 = torch.cuda.Event(enable_timing=True)
        s1 = torch.cuda.Event(enable_timing=True)
        start_region(torch, s0, stream)
        for i in range(args.steps):
            smc(i)
        s1.record(stream)
        torch.cuda.synchronize()
        barrier()
        ms_smc = sdist.max_over_ranks(s0.elapsed_time(s1), dev) / args.steps
        smc_line = {"ms_per_step": ms_smc, "value": total_bytes / (ms_smc * 1e-3) / 1e9,
                    "unit": "GB/s", "particles_per_group": Np, "groups": G * world,
                    "note": "one SMC-SD round over the same logits: statistics sweep, log "
                            "importance ratios and bonus draws, ESS and systematic resampling"}

    # ---- chained two-stage verify: final = the target, intermediate = its copy
    # one position later in the rotation (distinct logits of the same shape) -----
    chained_line = None
    if args.chained == "on" and K <= 31:
        u2 = torch.rand((B, K + 1), dtype=torch.float32, device=dev,
                        generator=torch.Generator(device=dev).manual_seed(5))
        o_tok = torch.empty((B, K + 1), dtype=torch.int32, device=dev)
        o_em = torch.empty((B,), dtype=torch.int32, device=dev)
        fch = L.specdec_verify_chained

        def ch(i):
            b = bufs[i % ncopies]
            inter = bufs[(i + 1) % ncopies]["t"]
            return fch(b["t"].data_ptr(), inter.data_ptr(), b["d"].data_ptr(), b["tok"].data_ptr(),
                       b["ua"].data_ptr(), b["ur"].data_ptr(), u2.data_ptr(), b["ur"].data_ptr(),
                       b["T"].data_ptr(), B, K, V, dt_code, o_tok.data_ptr(), o_em.data_ptr(),
                       None, None, sp)
        for i in range(3):
            if ch(i) != 0:
                raise RuntimeError("specdec_verify_chained failed")
        torch.cuda.synchronize()
        barrier()
        torch.cuda.synchronize()
        c0 = torch.cuda.Event(enable_timing=True)
        c1 = torch.cuda.Event(enable_timing=True)
        start_region(torch, c0, stream)
        for i in range(args.steps):
            ch(i)
        c1.record(stream)
        torch.cuda.synchronize()
        barrier()
        ms_ch = sdist.max_over_ranks(c0.elapsed_time(c1), dev) / args.steps
        ch_bytes = (2 * (K + 1) + K) * V * (2 if w.dtype == "bf16" else 4) * B
        chained_line = {"ms_per_step": ms_ch, "unit": "GB/s",
                        "value": ch_bytes * world / (ms_ch * 1e-3) / 1e9,
                        "bytes_per_step": ch_bytes * world,
                        "note": "two sweeps: intermediate + draft (stage 1), then the final "
                                "layer's rows (stage 2, with the intermediate's row statistics "
                                "kept from stage 1); value counts one read of the three "
                                "tensors"}

    # ---- LogitSpec candidates: top 60 of each target row, draft token left out
    topk_line = None
    if args.topk == "on":
        kk = 60
        nrows = B * K  # the target rows of the K draft positions
        ridx = [torch.tensor([b * (K + 1) + i for b in range(B) for i in range(K)],
                             dtype=torch.int64, device=dev)]
        oidx = torch.empty((nrows, kk), dtype=torch.int32, device=dev)
        oval = torch.empty((nrows, kk), dtype=torch.float32, device=dev)
        ftk = L.specdec_topk_exclude

        def tk(i):
            b = bufs[i % ncopies]
            return ftk(b["t"].data_ptr(), V, ridx[0].data_ptr(), nrows, V, dt_code,
                       b["tok"].data_ptr(), kk, oidx.data_ptr(), oval.data_ptr(), sp)
        for i in range(3):
            if tk(i) != 0:
                raise RuntimeError("specdec_topk_exclude failed")
        torch.cuda.synchronize()
        barrier()
        torch.cuda.synchronize()
        k0 = torch.cuda.Event(enable_timing=True)
        k1 = torch.cuda.Event(enable_timing=True)
        start_region(torch, k0, stream)
        for i in range(args.steps):
            tk(i)
        k1.record(stream)
        torch.cuda.synchronize()
        barrier()
        ms_tk = sdist.max_over_ranks(k0.elapsed_time(k1), dev) / args.steps
        row_bytes = V * (2 if w.dtype == "bf16" else 4)
        topk_line = {"ms_per_call": ms_tk, "k": kk, "rows": nrows * world,
                     "value": nrows * row_bytes * world / (ms_tk * 1e-3) / 1e9, "unit": "GB/s",
                     "rows_per_s": nrows * world / (ms_tk * 1e-3),
                     "note": "one read of each row counted; the candidate pass re-reads it "
                             "from L2"}

    # ---- end to end through the host entry point (pinned buffers) ----------
    pin = {k: torch.from_numpy(np.ascontiguousarray(getattr(x, k))).pin_memory()
           for k in ("target", "draft", "tokens", "u_accept", "u_resample", "temperature")}
    hot = torch.empty((B, K + 1), dtype=torch.int32).pin_memory()
    hon = torch.empty((B,), dtype=torch.int32).pin_memory()
    hargs = (pin["target"].data_ptr(), pin["draft"].data_ptr(), pin["tokens"].data_ptr(),
             pin["u_accept"].data_ptr(), pin["u_resample"].data_ptr(),
             pin["temperature"].data_ptr(), B, K, V, dt_code, hot.data_ptr(), hon.data_ptr(), sp)
    for _ in range(2):
        if L.specdec_verify_host(*hargs) != 0:
            raise RuntimeError("specdec_verify_host failed")
    h2d = sum(int(t.numel() * t.element_size()) for t in pin.values())
    d2h = int(hot.numel() * 4 + hon.numel() * 4)
    barrier()
    torch.cuda.synchronize()
    ee0 = torch.cuda.Event(enable_timing=True)
    ee1 = torch.cuda.Event(enable_timing=True)
    ee0.record(stream)
    for _ in range(args.e2e_steps):
        L.specdec_verify_host(*hargs)
    ee1.record(stream)
    torch.cuda.synchronize()
    ms_e2e = sdist.max_over_ranks(ee0.elapsed_time(ee1), dev)
    barrier()
    if not np.array_equal(hot.numpy(), ref_tok.numpy()):
        raise RuntimeError("end-to-end outputs differ from the device-resident run")
    e2e_gbs = total_bytes / (ms_e2e / args.e2e_steps * 1e-3) / 1e9

    if rank != 0:
        if dist is not None:
            dist.destroy_process_group()
        return 0

    peak, peak_kind = measured_peaks()
    launches = int(sum(a - b for a, b in zip(after, before)))
    rows = B * (2 * K + 1) * world
    line = {
        "metric": METRIC, "value": gbs, "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": max(3, args.warmup), "ms_per_step": ms_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": {"workload": args.workload, "B": B, "K": K, "V": V, "logits_dtype": w.dtype,
                   "B_total": B * world, "parallelism": f"dp{world}",
                   "l2": f"inputs rotate over {ncopies} device copies "
                         f"({ncopies * floor / 1e6:.0f} MB) > 126 MB L2"},
        "timing": "CUDA events around the K steps on their stream; a device delay queued "
                  "before the start event lets the host queue the first launches",
        "rows_per_s": rows / (ms_step * 1e-3),
        "sequences_per_s": B * world / (ms_step * 1e-3),
        "pct_of_hbm_peak": {f"of_{peak_kind}_{peak:.0f}GBs": 100.0 * gbs / world / peak,
                            "of_nominal_8000GBs": 100.0 * gbs / world / NOMINAL_HBM_GBS},
        "gpu_launches": launches,
    }
    if kern:
        # launches of the sweep per step (one for the full call); the achieved
        # rate is the algorithmic bytes of a launch over its mean time
        st_ms, st_n = kern["k_row_stats"]
        per_launch = floor * args.steps / max(st_n, 1)
        avg = st_ms / max(st_n, 1)
        ach = per_launch / (avg * 1e-3) / 1e9
        tr = stored_traffic() if args.workload == "batched_b64_k5_v128256_bf16" else None
        line["roofline"] = {"bound": "hbm", "kernel": "k_row_stats", "achieved": ach,
                            "peak": peak, "peak_kind": peak_kind, "unit": "GB/s",
                            "frac": ach / peak,
                            "traffic": tr["sweep_bytes_per_launch"] if tr else None,
                            "algorithmic_bytes_per_launch": per_launch,
                            "launches_per_step": st_n / args.steps,
                            "launches_timed": st_n,
                            "timing": "CUDA events around each launch on its stream, over a "
                                      "second run of the K steps"}
        if tr:
            line["step_traffic"] = {"dram_bytes_per_step": tr["step_bytes"],
                                    "algorithmic_bytes_per_step": floor,
                                    "ratio": tr["step_bytes"] / floor,
                                    "per_kernel": tr["per_kernel_bytes_per_step"],
                                    "source": "profiles/verify_step_traffic.json"}
        line["kernel_us"] = {k: (v[0] / max(v[1], 1) * 1e3) for k, v in kern.items()}
    if early is not None:
        line["early_exit"] = early
    if smc_line is not None:
        line["smc_step"] = smc_line
    if topk_line is not None:
        line["topk_exclude"] = topk_line
    if chained_line is not None:
        line["verify_chained"] = chained_line
    line["e2e"] = {"value": e2e_gbs, "unit": "GB/s", "h2d_bytes_per_step": h2d,
                   "d2h_bytes_per_step": d2h, "steps": args.e2e_steps}
    line["step_us"] = {"median": float(np.median(per_step)), "p10": float(np.percentile(per_step, 10)),
                       "p90": float(np.percentile(per_step, 90)), "steps": int(per_step.size),
                       "note": "each of K back-to-back steps bracketed by its own events"}
    line["latency_us"] = {"median": float(np.median(lat)), "p10": float(np.percentile(lat, 10)),
                          "p90": float(np.percentile(lat, 90)), "calls": int(lat.size),
                          "note": "one call at a time, the stream synchronised between calls"}
    line["clocks"] = sampler.summary()
    if line["clocks"].get("sm_mhz"):
        line["clocks"]["sm_mhz_x_us_per_step"] = line["clocks"]["sm_mhz"] * ms_step * 1e3
    if world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(x, w, args.cpu_seconds)
    print(json.dumps(line), flush=True)
    if dist is not None:
        dist.destroy_process_group()
    return 0


def main():
    args = parse()
    if args.impl == "reference":
        return run_reference(args)
    return run_cuda(args)


if __name__ == "__main__":
    sys.exit(main())
