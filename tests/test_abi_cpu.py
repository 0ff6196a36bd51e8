"""CPU-side checks of the C ABI: the library builds and loads, exports every entry point
the public header declares, and host-only calls validate their arguments."""

import ctypes
import os
import re

import pytest

import deepseek_mla_decode_b200 as mla

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "mla_decode.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(mla_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_expected_api():
    fns = declared_functions()
    assert set(mla.EXPORTED_SYMBOLS) == set(fns), fns


def test_library_exports_every_declared_symbol():
    L = mla.load_library()
    for name in declared_functions():
        assert hasattr(L, name), name
    # exported with C linkage (no mangling)
    out = os.popen(f"nm -D --defined-only {mla.LIB_PATH}").read()
    for name in declared_functions():
        assert re.search(rf"\bT {name}\b", out), name


def test_status_strings():
    L = mla.load_library()
    for code, name in [(0, "MLA_OK"), (1, "MLA_ERR_INVALID_ARG"), (2, "MLA_ERR_UNSUPPORTED"),
                       (3, "MLA_ERR_CUDA"), (4, "MLA_ERR_WORKSPACE_TOO_SMALL"), (5, "MLA_ERR_DEVICE")]:
        assert L.mla_status_string(code).decode() == name
    assert L.mla_status_string(99).decode() == "MLA_ERR_UNKNOWN"


def test_metadata_size_host_only():
    n = mla.metadata_size(256, 1, 128)
    assert n == (16 + 4 * 256 + 4 * 256) * 4
    assert mla.metadata_size(1, 2, 16) == (16 + 4 * 256 + 4) * 4


@pytest.mark.parametrize("B,s_q,H", [(0, 1, 128), (1, 0, 128), (1, 5, 128), (1, 1, 48), (1, 1, 256)])
def test_unsupported_shapes_rejected(B, s_q, H):
    with pytest.raises(mla.MLAError) as e:
        mla.metadata_size(B, s_q, H)
    assert e.value.code == 2


def test_null_pointers_rejected_before_any_device_call():
    L = mla.load_library()
    # every pointer NULL: must return INVALID_ARG without touching a device
    rc = L.mla_decode(None, None, None, 1, None, 1, None, 1, 1, 16, 0.1, 0, None, 0, None, 0, None, None, None,
                      None)
    assert rc == 1
    rc = L.mla_get_metadata(None, 1, 1, 16, None, 0, None)
    assert rc == 1
    assert L.mla_metadata_size(1, 1, 16, None) == 1


def test_fp8_and_prefill_entry_points_validate_before_any_device_call():
    L = mla.load_library()
    rc = L.mla_decode_fp8(None, None, None, 1, None, 1, None, None, 1, 1, 16, 0.1, 0, None, 0, None, 0, None, None,
                          None, None)
    assert rc == 1
    rc = L.mla_decode_fp8_attention(None, None, None, 1, None, 1, None, None, 1, 1, 16, 0.1, 0, None, 0, None, 0,
                                    None, None, None, None)
    assert rc == 1
    assert L.mla_quantize_kv_fp8(None, None, 1, None) == 1
    n = ctypes.c_size_t()
    assert L.mla_sage_workspace_size(0, 1, ctypes.byref(n)) == 1
    assert L.mla_sage_workspace_size(1, 0, ctypes.byref(n)) == 1
    assert L.mla_sage_workspace_size(1, 1, None) == 1
    assert L.mla_sage_quantize(None, None, None, 10, 2, None, 0, None) == 1
    assert L.mla_sage_attention(10, 2, 0.1, None, 0, None, None, None, None) == 1
    assert L.mla_sage_prefill(None, None, None, 10, 2, 0.1, None, 0, None, None, None, None) == 1


def test_prefill_workspace_size_host_only():
    # codes (2 x 192 + 128 bytes per token and head, tokens padded to 128) + token scales
    # (8 bytes per token and head) + channel scale and scratch (8 bytes per channel and head)
    S, H = 300, 3
    sp = 384
    assert mla.sage_workspace_size(S, H) == H * sp * (2 * 192 + 128) + 2 * H * sp * 4 + 2 * H * 128 * 4
