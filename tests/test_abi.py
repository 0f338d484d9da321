"""The C-ABI library loads, exports every symbol the header declares, and its
host-side checks return the documented status codes (no GPU needed: every
call here fails validation before touching a device)."""

import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "mla_decode.h")


def _declared():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(mla_[a-z0-9_]+)\s*\(", src)))


@pytest.fixture(scope="module")
def L():
    import mla_decode_attention_16_b200 as m
    return m.lib


def test_header_declares_expected_calls():
    names = _declared()
    for n in ("mla_get_metadata", "mla_decode_fwd", "mla_get_num_sm_parts", "mla_get_workspace_size"):
        assert n in names


def test_library_exports_every_declared_symbol(L):
    missing = [n for n in _declared() if not hasattr(L, n)]
    assert not missing, missing


def test_status_strings(L):
    assert L.mla_status_string(0) == b"MLA_OK"
    assert L.mla_status_string(3) == b"MLA_ERR_WORKSPACE"
    assert L.mla_status_string(99) == b"MLA_ERR_UNKNOWN"


def test_workspace_size_formula(L):
    out = ctypes.c_size_t()
    assert L.mla_get_workspace_size(64, 16, 74, ctypes.byref(out)) == 0
    chunks = 64 + 74
    lse_end = 256 + chunks * 16 * 4
    o_off = (lse_end + 255) // 256 * 256
    assert out.value == o_off + chunks * 16 * 512 * 4
    assert L.mla_get_workspace_size(0, 16, 74, ctypes.byref(out)) == 1
    assert L.mla_get_workspace_size(1, 2048, 74, ctypes.byref(out)) == 2


def test_host_validation_before_any_launch(L):
    vp = ctypes.c_void_p
    fake = vp(256)  # never dereferenced: validation fails first
    # null q / outputs
    rc = L.mla_decode_fwd(None, fake, 1, fake, 1, fake, 1, 1, 16, 0, 0.1, 0, fake, fake, 1, fake, 1 << 30,
                          fake, fake, None)
    assert rc == 1
    # bad dtype
    rc = L.mla_decode_fwd(fake, fake, 1, fake, 1, fake, 1, 1, 16, 7, 0.1, 0, fake, fake, 1, fake, 1 << 30,
                          fake, fake, None)
    assert rc == 1
    # too many rows
    rc = L.mla_decode_fwd(fake, fake, 1, fake, 1, fake, 1, 2, 1024, 0, 0.1, 0, fake, fake, 1, fake, 1 << 30,
                          fake, fake, None)
    assert rc == 2
    # workspace too small
    rc = L.mla_decode_fwd(fake, fake, 1, fake, 1, fake, 4, 1, 16, 0, 0.1, 0, fake, fake, 1, fake, 16,
                          fake, fake, None)
    assert rc == 3
    # non-finite scale
    rc = L.mla_decode_fwd(fake, fake, 1, fake, 1, fake, 1, 1, 16, 0, float("nan"), 0, fake, fake, 1, fake,
                          1 << 30, fake, fake, None)
    assert rc == 1
    # misaligned out
    rc = L.mla_decode_fwd(fake, fake, 1, fake, 1, fake, 1, 1, 16, 0, 0.1, 0, fake, fake, 1, fake, 1 << 30,
                          vp(258), fake, None)
    assert rc == 1
    # metadata: null and oversize batch
    assert L.mla_get_metadata(None, 4, 16, 1, fake, fake, None) == 1
    assert L.mla_get_metadata(fake, 20000, 16, 1, fake, fake, None) == 2
    parts = ctypes.c_int()
    assert L.mla_get_num_sm_parts(0, 0, ctypes.byref(parts)) == 1
    assert L.mla_get_num_sm_parts(0, 4096, ctypes.byref(parts)) == 2


def test_fp8_cache_flag_validation(L):
    """MLA_KV_FP8_E5M2 (0x100) is accepted only OR-ed into bf16 / fp16; checks run before any launch."""
    vp = ctypes.c_void_p
    fake = vp(256)
    flag = 0x100
    # a bad base dtype with the flag, or a stray bit, is rejected as an invalid argument
    for bad in (flag | 7, 0x200, flag | 0x200):
        rc = L.mla_decode_fwd(fake, fake, 1, fake, 1, fake, 1, 1, 16, bad, 0.1, 0, fake, fake, 1, fake, 1 << 30,
                              fake, fake, None)
        assert rc == 1, hex(bad)
    # a valid flagged dtype gets as far as the workspace check
    rc = L.mla_decode_fwd(fake, fake, 1, fake, 1, fake, 4, 1, 16, flag | 1, 0.1, 0, fake, fake, 1, fake, 16,
                          fake, fake, None)
    assert rc == 3
    parts = ctypes.c_int()
    L.mla_get_num_sm_parts_dtype.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.POINTER(ctypes.c_int)]
    assert L.mla_get_num_sm_parts_dtype(0, 16, 7, ctypes.byref(parts)) == 1
    assert L.mla_get_num_sm_parts_dtype(0, 0, flag, ctypes.byref(parts)) == 1
    assert L.mla_get_num_sm_parts_dtype(0, 4096, flag, ctypes.byref(parts)) == 2
    assert L.mla_get_num_sm_parts_dtype(0, 16, flag, None) == 1
