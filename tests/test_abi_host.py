"""Host-side checks of the C-ABI that need no GPU: the library loads, exports
every function include/specdec.h declares, and rejects invalid arguments on
the host (SPECDEC_EINVAL) before any launch."""
import ctypes
import os
import re

import pytest

import speculative_sampling_b200 as sd
from speculative_sampling_b200 import build as sd_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    sd_build.build()
    return sd.lib()


def declared_functions():
    names = set()
    inc = os.path.join(ROOT, "include")
    for fn in os.listdir(inc):
        if fn.endswith(".h"):
            src = open(os.path.join(inc, fn)).read()
            src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
            names |= set(re.findall(r"\b(specdec_\w+)\s*\(", src))
    return sorted(names)


def test_every_declared_symbol_is_exported(L):
    names = declared_functions()
    assert "specdec_verify" in names and len(names) >= 10
    for n in names:
        assert hasattr(L, n), n
        assert n in sd._SIGS, f"binding lacks {n}"


def test_status_strings_and_kernel_names(L):
    assert sd.status_string(sd.SPECDEC_OK) == "ok"
    assert "invalid" in sd.status_string(sd.SPECDEC_EINVAL)
    assert sd.kernel_names() == ["k_row_stats", "k_finish", "k_smc_resample", "k_topk_exclude"]
    assert len(sd.launch_counts()) == 4


# fake, never-dereferenced addresses: validation must reject before any use
A16 = 0x10000


@pytest.mark.parametrize("B,K,V,dtype", [
    (-1, 5, 100, sd.SPECDEC_BF16), (2, 0, 100, sd.SPECDEC_BF16), (2, 33, 100, sd.SPECDEC_BF16),
    (2, 5, 0, sd.SPECDEC_BF16), (2, 5, 100, 7), (2, 5, -3, sd.SPECDEC_F32)])
def test_bad_sizes_rejected(L, B, K, V, dtype):
    st = sd.specdec_verify(A16, A16, A16, A16, A16, A16, B, K, V, dtype, A16, A16, None)
    assert st == sd.SPECDEC_EINVAL


def test_null_and_misaligned_pointers_rejected(L):
    args = [A16] * 6
    for i in range(6):
        a = list(args)
        a[i] = None
        assert sd.specdec_verify(*a, 2, 3, 64, sd.SPECDEC_F32, A16, A16, None) == sd.SPECDEC_EINVAL
    assert sd.specdec_verify(*args, 2, 3, 64, sd.SPECDEC_F32, None, A16, None) == sd.SPECDEC_EINVAL
    # fp32 logits at an odd address, bf16 logits at an odd address
    assert sd.specdec_verify(A16 + 2, A16, A16, A16, A16, A16, 2, 3, 64, sd.SPECDEC_F32, A16, A16,
                             None) == sd.SPECDEC_EINVAL
    assert sd.specdec_verify(A16, A16 + 1, A16, A16, A16, A16, 2, 3, 64, sd.SPECDEC_BF16, A16,
                             A16, None) == sd.SPECDEC_EINVAL


def test_empty_batch_is_a_no_op(L):
    for f in (sd.specdec_verify, sd.specdec_verify_host):
        assert f(None, None, None, None, None, None, 0, 5, 128256, sd.SPECDEC_BF16, None, None,
                 None) == sd.SPECDEC_OK


def test_workspace_size_is_monotone(L):
    w1 = sd.specdec_workspace_bytes(1, 5, 128256, sd.SPECDEC_BF16)
    w64 = sd.specdec_workspace_bytes(64, 5, 128256, sd.SPECDEC_BF16)
    assert 0 < w1 <= w64 and w64 % 256 == 0
    assert sd.specdec_workspace_bytes(64, 0, 128256, sd.SPECDEC_BF16) == 0


def test_profile_api_without_launches(L):
    sd.profile_begin(4)
    res = sd.profile_end()
    assert set(res) == {"k_row_stats", "k_finish", "k_smc_resample", "k_topk_exclude"}
    assert all(c == 0 for _, c in res.values())
    assert L.specdec_profile_begin(0) == sd.SPECDEC_EINVAL


def test_binding_fails_loudly_without_library(monkeypatch, tmp_path):
    monkeypatch.setattr(sd, "LIB_PATH", str(tmp_path / "missing.so"))
    monkeypatch.setattr(sd, "_lib", None)
    with pytest.raises(RuntimeError, match="no fallback"):
        sd.lib()
