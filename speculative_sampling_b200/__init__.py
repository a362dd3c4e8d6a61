"""Python binding of libspecdec.so (the batched speculative-sampling verify
step for B200).

The functions named ``specdec_*`` mirror the C-ABI in include/specdec.h one to
one and take raw pointers (ints) -- argument marshalling only.  ``verify`` and
``verify_host`` are conveniences that take torch tensors / numpy arrays, check
shapes and dtypes and call the C entry points.  Every step of the computation
runs in the CUDA kernels of libspecdec.so; when the library is missing the
import of this binding fails loudly instead of falling back to anything else.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "libspecdec.so")

SPECDEC_OK, SPECDEC_EINVAL, SPECDEC_ECUDA, SPECDEC_EDEVICE, SPECDEC_ESTATE, SPECDEC_ESIZE = range(6)
SPECDEC_STATIC_SCRATCH_BYTES = 4 << 20
SPECDEC_F32, SPECDEC_BF16 = 0, 1
SPECDEC_ERR_TOKEN, SPECDEC_ERR_TEMPERATURE, SPECDEC_ERR_LOGITS, SPECDEC_ERR_TIMEOUT = 1, 2, 4, 8

_P = ctypes.c_void_p
_I = ctypes.c_int
_SIGS = {
    "specdec_verify": (_I, [_P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _P, _P, _P]),
    "specdec_verify_bf16": (_I, [_P, _P, _P, _P, _P, _P, _I, _I, _I, _P, _P, _P]),
    "specdec_verify_f32": (_I, [_P, _P, _P, _P, _P, _P, _I, _I, _I, _P, _P, _P]),
    "specdec_workspace_bytes": (ctypes.c_size_t, [_I, _I, _I, _I]),
    "specdec_verify_ex": (_I, [_P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _P, ctypes.c_size_t, _P,
                               _P, _P, _P]),
    "specdec_verify_host": (_I, [_P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _P, _P, _P]),
    "specdec_verify_early_exit": (_I, [_P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _P, _P, _P]),
    "specdec_verify_early_exit_ex": (_I, [_P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _P,
                                          ctypes.c_size_t, _P, _P, _P, _P]),
    "specdec_verify_static": (_I, [_P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _P, _P, _P]),
    "specdec_smc_step": (_I, [_P, _P, _P, _P, _P, _P, _P, ctypes.c_double, _I, _I, _I, _I, _I,
                              _P, _P, _P, _P, _P, _P]),
    "specdec_topk_exclude": (_I, [_P, ctypes.c_longlong, _P, _I, _I, _I, _P, _I, _P, _P, _P]),
    "specdec_verify_chained": (_I, [_P, _P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _P, _P,
                                    _P, _P, _P]),
    "specdec_verify_chained_ex": (_I, [_P, _P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _P,
                                       _P, _P, _P, _P, _P]),
    "specdec_device_errors": (_I, [_P, ctypes.POINTER(ctypes.c_uint32)]),
    "specdec_get_error": (_I, []),
    "specdec_error_string": (ctypes.c_char_p, [_I]),
    "specdec_test_set_wait_fault": (_I, [ctypes.c_longlong, ctypes.c_ulonglong]),
    "specdec_test_exp2": (_I, [_P, _P, _I, _P]),
    "specdec_release": (None, []),
    "specdec_status_string": (ctypes.c_char_p, [_I]),
    "specdec_kernel_count": (_I, []),
    "specdec_kernel_name": (ctypes.c_char_p, [_I]),
    "specdec_launch_count": (ctypes.c_uint64, [_I]),
    "specdec_profile_begin": (_I, [_I]),
    "specdec_profile_end": (_I, [ctypes.POINTER(ctypes.c_double), ctypes.POINTER(_I), _I]),
}


class SpecdecError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)} (status {status})")


class _Debug(ctypes.Structure):
    _fields_ = [("row_max", _P), ("row_sum", _P), ("p_x", _P), ("q_x", _P), ("Z", _P)]


_lib = None


def lib() -> ctypes.CDLL:
    """The loaded libspecdec.so.  Raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"{LIB_PATH} is missing: build it with `python -m speculative_sampling_b200.build`"
                " (there is no fallback implementation)")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGS.items():
            f = getattr(L, name)
            f.restype = res
            f.argtypes = args
        _lib = L
    return _lib


def status_string(status: int) -> str:
    return lib().specdec_status_string(int(status)).decode()


def _chk(status: int, where: str) -> int:
    if status != SPECDEC_OK:
        raise SpecdecError(status, where)
    return status


# ---- one-to-one wrappers of the C-ABI (pointers as ints) -------------------
def specdec_verify(target, draft, tokens, u_accept, u_resample, temperature, B, K, V, dtype,
                   out_tokens, out_num_accepted, stream) -> int:
    return lib().specdec_verify(target, draft, tokens, u_accept, u_resample, temperature, B, K,
                                V, dtype, out_tokens, out_num_accepted, stream)


def specdec_verify_bf16(target, draft, tokens, u_accept, u_resample, temperature, B, K, V,
                        out_tokens, out_num_accepted, stream) -> int:
    return lib().specdec_verify_bf16(target, draft, tokens, u_accept, u_resample, temperature,
                                     B, K, V, out_tokens, out_num_accepted, stream)


def specdec_verify_f32(target, draft, tokens, u_accept, u_resample, temperature, B, K, V,
                       out_tokens, out_num_accepted, stream) -> int:
    return lib().specdec_verify_f32(target, draft, tokens, u_accept, u_resample, temperature,
                                    B, K, V, out_tokens, out_num_accepted, stream)


def specdec_workspace_bytes(B, K, V, dtype) -> int:
    return lib().specdec_workspace_bytes(B, K, V, dtype)


def specdec_verify_ex(target, draft, tokens, u_accept, u_resample, temperature, B, K, V, dtype,
                      workspace, workspace_bytes, dbg, out_tokens, out_num_accepted,
                      stream) -> int:
    return lib().specdec_verify_ex(target, draft, tokens, u_accept, u_resample, temperature, B,
                                   K, V, dtype, workspace, workspace_bytes, dbg, out_tokens,
                                   out_num_accepted, stream)


def specdec_verify_early_exit(target, draft, tokens, u_accept, u_resample, temperature, B, K,
                              V, dtype, out_tokens, out_num_accepted, stream) -> int:
    return lib().specdec_verify_early_exit(target, draft, tokens, u_accept, u_resample,
                                           temperature, B, K, V, dtype, out_tokens,
                                           out_num_accepted, stream)


def specdec_verify_early_exit_ex(target, draft, tokens, u_accept, u_resample, temperature, B, K,
                                 V, dtype, workspace, workspace_bytes, dbg, out_tokens,
                                 out_num_accepted, stream) -> int:
    return lib().specdec_verify_early_exit_ex(target, draft, tokens, u_accept, u_resample,
                                              temperature, B, K, V, dtype, workspace,
                                              workspace_bytes, dbg, out_tokens,
                                              out_num_accepted, stream)


def specdec_verify_host(target, draft, tokens, u_accept, u_resample, temperature, B, K, V,
                        dtype, out_tokens, out_num_accepted, stream) -> int:
    return lib().specdec_verify_host(target, draft, tokens, u_accept, u_resample, temperature,
                                     B, K, V, dtype, out_tokens, out_num_accepted, stream)


def specdec_verify_static(target, draft, tokens, u_accept, u_resample, temperature, B, K, V,
                          dtype, out_tokens, out_num_accepted, stream) -> int:
    """specdec_verify with the library's fixed scratch instead of an allocated
    workspace, for callers that may not allocate device memory (see the header
    for the size limit and the no-overlap rule)."""
    return lib().specdec_verify_static(target, draft, tokens, u_accept, u_resample, temperature,
                                       B, K, V, dtype, out_tokens, out_num_accepted, stream)


def specdec_smc_step(target, draft, tokens, u_bonus, temperature, log_weights_in, u_resample,
                     ess_threshold, B, N, K, V, dtype, out_tokens, log_weights_out, ess,
                     ancestors, log_weight_increment, stream) -> int:
    return lib().specdec_smc_step(target, draft, tokens, u_bonus, temperature, log_weights_in,
                                  u_resample, float(ess_threshold), B, N, K, V, dtype,
                                  out_tokens, log_weights_out, ess, ancestors,
                                  log_weight_increment, stream)


def smc_step(target, draft, tokens, u_bonus, temperature, u_resample, N, ess_threshold=0.5,
             log_weights_in=None, stream=None) -> dict:
    """One SMC-SD round on CUDA tensors (see specdec_smc_step): target
    [B,K+1,V], draft [B,K,V], tokens [B,K] int32, u_bonus [B] / temperature [B]
    float32, u_resample [B//N] float32, log_weights_in [B] float64 or None.
    Returns a dict of CUDA tensors: out_tokens, log_weights, ess, ancestors,
    increment."""
    import torch
    B, K1, V = target.shape
    K = K1 - 1
    if B % N:
        raise ValueError("B must be a multiple of N")
    dev = target.device
    out = dict(out_tokens=torch.empty((B, K + 1), dtype=torch.int32, device=dev),
               log_weights=torch.empty((B,), dtype=torch.float64, device=dev),
               ess=torch.empty((B // N,), dtype=torch.float64, device=dev),
               ancestors=torch.empty((B,), dtype=torch.int32, device=dev),
               increment=torch.empty((B,), dtype=torch.float64, device=dev))
    _check_dev(target, draft, tokens, u_bonus, temperature, u_resample)
    if stream is None:
        stream = torch.cuda.current_stream(dev).cuda_stream
    st = specdec_smc_step(target.data_ptr(), draft.data_ptr(), tokens.data_ptr(),
                          u_bonus.data_ptr(), temperature.data_ptr(),
                          None if log_weights_in is None else log_weights_in.data_ptr(),
                          u_resample.data_ptr(), ess_threshold, B, N, K, V, _dtype_code(target),
                          out["out_tokens"].data_ptr(), out["log_weights"].data_ptr(),
                          out["ess"].data_ptr(), out["ancestors"].data_ptr(),
                          out["increment"].data_ptr(), stream)
    _chk(st, "specdec_smc_step")
    return out


def specdec_topk_exclude(logits, row_stride, row_index, rows, V, dtype, exclude, k, out_idx,
                         out_val, stream) -> int:
    return lib().specdec_topk_exclude(logits, row_stride, row_index, rows, V, dtype, exclude, k,
                                      out_idx, out_val, stream)


def topk_exclude(logits, k, exclude=None, row_index=None, stream=None):
    """Top-k token ids (and logits) of each row of a [R, V] CUDA tensor (or of
    the rows named by int64 ``row_index`` of a [*, V] tensor), leaving out
    ``exclude[r]`` (int32, -1 = none).  Returns (idx [R', k] int32, val [R', k]
    float32)."""
    import torch
    V = logits.shape[-1]
    flat = logits.reshape(-1, V)
    rows = flat.shape[0] if row_index is None else row_index.numel()
    dev = logits.device
    idx = torch.empty((rows, k), dtype=torch.int32, device=dev)
    val = torch.empty((rows, k), dtype=torch.float32, device=dev)
    if stream is None:
        stream = torch.cuda.current_stream(dev).cuda_stream
    st = specdec_topk_exclude(flat.data_ptr(), flat.stride(0),
                              None if row_index is None else row_index.data_ptr(), rows, V,
                              _dtype_code(logits), None if exclude is None else exclude.data_ptr(),
                              k, idx.data_ptr(), val.data_ptr(), stream)
    _chk(st, "specdec_topk_exclude")
    return idx, val


def specdec_verify_chained(final, inter, draft, tokens, u_accept1, u_resample1, u_accept2,
                           u_resample2, temperature, B, K, V, dtype, out_tokens,
                           out_num_emitted, stage1_tokens, stage1_num_accepted, stream) -> int:
    return lib().specdec_verify_chained(final, inter, draft, tokens, u_accept1, u_resample1,
                                        u_accept2, u_resample2, temperature, B, K, V, dtype,
                                        out_tokens, out_num_emitted, stage1_tokens,
                                        stage1_num_accepted, stream)


def specdec_verify_chained_ex(final, inter, draft, tokens, u_accept1, u_resample1, u_accept2,
                              u_resample2, temperature, B, K, V, dtype, out_tokens,
                              out_num_emitted, stage1_tokens, stage1_num_accepted, dbg2,
                              stream) -> int:
    return lib().specdec_verify_chained_ex(final, inter, draft, tokens, u_accept1, u_resample1,
                                           u_accept2, u_resample2, temperature, B, K, V, dtype,
                                           out_tokens, out_num_emitted, stage1_tokens,
                                           stage1_num_accepted, dbg2, stream)


def verify_chained(final, inter, draft, tokens, u_accept1, u_resample1, u_accept2, u_resample2,
                   temperature, stream=None, debug2: Optional[dict] = None) -> dict:
    """Chained two-stage verify on CUDA tensors (see specdec_verify_chained).
    Returns a dict of CUDA int32 tensors: out_tokens [B,K+1], num_emitted [B],
    stage1_tokens [B,K+1], stage1_n [B].  With ``debug2`` (a dict of
    preallocated tensors named as specdec_debug's fields) the call goes through
    specdec_verify_chained_ex and fills the second stage's diagnostics."""
    import torch
    B, K1, V = final.shape
    K = K1 - 1
    dev = final.device
    out = dict(out_tokens=torch.empty((B, K1), dtype=torch.int32, device=dev),
               num_emitted=torch.empty((B,), dtype=torch.int32, device=dev),
               stage1_tokens=torch.empty((B, K1), dtype=torch.int32, device=dev),
               stage1_n=torch.empty((B,), dtype=torch.int32, device=dev))
    _check_dev(final, inter, draft, tokens, u_accept1, u_resample1, u_accept2, u_resample2,
               temperature)
    if stream is None:
        stream = torch.cuda.current_stream(dev).cuda_stream
    dbg = None
    if debug2 is not None:
        d = _Debug()
        for f, _ in _Debug._fields_:
            t = debug2.get(f)
            setattr(d, f, t.data_ptr() if t is not None else None)
        dbg = ctypes.byref(d)
    st = specdec_verify_chained_ex(final.data_ptr(), inter.data_ptr(), draft.data_ptr(),
                                   tokens.data_ptr(), u_accept1.data_ptr(), u_resample1.data_ptr(),
                                   u_accept2.data_ptr(), u_resample2.data_ptr(),
                                   temperature.data_ptr(), B, K, V, _dtype_code(final),
                                   out["out_tokens"].data_ptr(), out["num_emitted"].data_ptr(),
                                   out["stage1_tokens"].data_ptr(), out["stage1_n"].data_ptr(),
                                   dbg, stream)
    _chk(st, "specdec_verify_chained_ex")
    return out


def specdec_device_errors(stream=None) -> tuple:
    flags = ctypes.c_uint32(0)
    st = lib().specdec_device_errors(stream, ctypes.byref(flags))
    return st, int(flags.value)


def specdec_get_error() -> int:
    return lib().specdec_get_error()


def specdec_error_string(status: int) -> str:
    return lib().specdec_error_string(int(status)).decode()


def specdec_test_set_wait_fault(skip_tile: int, wait_ns: int) -> int:
    return lib().specdec_test_set_wait_fault(int(skip_tile), int(wait_ns))


def specdec_test_exp2(a, y, n, stream) -> int:
    return lib().specdec_test_exp2(a, y, n, stream)


def specdec_release() -> None:
    lib().specdec_release()


def kernel_names() -> list:
    L = lib()
    return [L.specdec_kernel_name(i).decode() for i in range(L.specdec_kernel_count())]


def launch_counts() -> list:
    L = lib()
    return [int(L.specdec_launch_count(i)) for i in range(L.specdec_kernel_count())]


def profile_begin(max_launches: int) -> None:
    _chk(lib().specdec_profile_begin(int(max_launches)), "specdec_profile_begin")


def profile_end() -> dict:
    n = lib().specdec_kernel_count()
    ms = (ctypes.c_double * n)()
    cnt = (ctypes.c_int * n)()
    _chk(lib().specdec_profile_end(ms, cnt, n), "specdec_profile_end")
    return {name: (ms[i], cnt[i]) for i, name in enumerate(kernel_names())}


# ---- torch / numpy conveniences --------------------------------------------
def _dtype_code(t) -> int:
    import torch
    if t.dtype in (torch.bfloat16, torch.uint16, torch.int16):
        return SPECDEC_BF16
    if t.dtype == torch.float32:
        return SPECDEC_F32
    raise TypeError(f"logits must be bfloat16 (or its 16-bit pattern) or float32, got {t.dtype}")


def _check_dev(*ts):
    dev = ts[0].device
    for t in ts:
        if not t.is_cuda or t.device != dev:
            raise ValueError("all tensors must be on the same CUDA device")
        if not t.is_contiguous():
            raise ValueError("tensors must be contiguous")


def verify(target, draft, tokens, u_accept, u_resample, temperature, out_tokens=None,
           out_num_accepted=None, stream=None, workspace=None, debug: Optional[dict] = None,
           early_exit: bool = False):
    """Run the verify step on CUDA tensors.

    target [B,K+1,V] and draft [B,K,V] (bfloat16 or float32), tokens [B,K]
    int32, u_accept [B,K] / u_resample [B] / temperature [B] float32.  Returns
    (out_tokens [B,K+1] int32, out_num_accepted [B] int32), written
    asynchronously on ``stream`` (default: torch's current stream).  With
    ``workspace`` (a uint8 CUDA tensor of specdec_workspace_bytes bytes) or
    ``debug`` (dict of preallocated tensors named as specdec_debug's fields)
    the call goes through specdec_verify_ex.  ``early_exit`` selects the
    early-exit entry points (same results, fewer rows read)."""
    import torch
    B, K1, V = target.shape
    K = K1 - 1
    if tuple(draft.shape) != (B, K, V) or draft.dtype != target.dtype:
        raise ValueError("draft must be [B,K,V] with the target's dtype")
    if tuple(tokens.shape) != (B, K) or tokens.dtype != torch.int32:
        raise ValueError("tokens must be int32 [B,K]")
    for t, shp in ((u_accept, (B, K)), (u_resample, (B,)), (temperature, (B,))):
        if tuple(t.shape) != shp or t.dtype != torch.float32:
            raise ValueError("uniforms and temperature must be float32 of shape [B,K], [B], [B]")
    if out_tokens is None:
        out_tokens = torch.empty((B, K + 1), dtype=torch.int32, device=target.device)
    if out_num_accepted is None:
        out_num_accepted = torch.empty((B,), dtype=torch.int32, device=target.device)
    _check_dev(target, draft, tokens, u_accept, u_resample, temperature, out_tokens,
               out_num_accepted)
    if stream is None:
        stream = torch.cuda.current_stream(target.device).cuda_stream
    dt = _dtype_code(target)
    args = (target.data_ptr(), draft.data_ptr(), tokens.data_ptr(), u_accept.data_ptr(),
            u_resample.data_ptr(), temperature.data_ptr(), B, K, V, dt)
    if workspace is None and debug is None:
        f, name = ((specdec_verify_early_exit, "specdec_verify_early_exit") if early_exit
                   else (specdec_verify, "specdec_verify"))
        st = f(*args, out_tokens.data_ptr(), out_num_accepted.data_ptr(), stream)
        _chk(st, name)
        return out_tokens, out_num_accepted
    need = specdec_workspace_bytes(B, K, V, dt)
    if workspace is None:
        workspace = torch.empty((need,), dtype=torch.uint8, device=target.device)
    dbg = None
    if debug is not None:
        d = _Debug()
        for f, _ in _Debug._fields_:
            t = debug.get(f)
            setattr(d, f, t.data_ptr() if t is not None else None)
        dbg = ctypes.byref(d)
    f, name = ((specdec_verify_early_exit_ex, "specdec_verify_early_exit_ex") if early_exit
               else (specdec_verify_ex, "specdec_verify_ex"))
    st = f(*args, workspace.data_ptr(), workspace.numel(), dbg, out_tokens.data_ptr(),
           out_num_accepted.data_ptr(), stream)
    _chk(st, name)
    return out_tokens, out_num_accepted


def verify_host(target, draft, tokens, u_accept, u_resample, temperature, out_tokens,
                out_num_accepted, stream=None):
    """End-to-end call on HOST arrays (numpy or CPU torch tensors, ideally
    pinned): copies in, verifies, copies out, synchronises."""
    def ptr(a):
        return a.data_ptr() if hasattr(a, "data_ptr") else a.ctypes.data
    B, K1, V = target.shape
    K = K1 - 1
    dt = SPECDEC_BF16 if str(target.dtype) in ("uint16", "torch.uint16", "torch.bfloat16",
                                               "torch.int16", "int16") else SPECDEC_F32
    st = specdec_verify_host(ptr(target), ptr(draft), ptr(tokens), ptr(u_accept),
                             ptr(u_resample), ptr(temperature), B, K, V, dt, ptr(out_tokens),
                             ptr(out_num_accepted), stream)
    _chk(st, "specdec_verify_host")
    return out_tokens, out_num_accepted
