"""C-ABI checks that need no GPU: the library loads, exports every function
include/thd_attn.h declares, and rejects bad arguments on the host before any
CUDA call."""
import ctypes
import os
import re

import numpy as np
import pytest

import sliding_window_gqa_cu_b200 as swa
from sliding_window_gqa_cu_b200 import build

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include",
                      "thd_attn.h")


@pytest.fixture(scope="module")
def lib():
    build.build()
    return swa.load_library()


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?\w+\s*\*?\s*(thd_\w+)\s*\(", src, flags=re.M)))


def test_header_declares_the_entry_points():
    names = declared_functions()
    for want in ("thd_attn_fwd", "thd_attn_get_error", "thd_attn_status_string", "thd_attn_plan",
                 "thd_attn_abi_version"):
        assert want in names


def test_library_exports_every_declared_symbol(lib):
    for name in declared_functions():
        assert hasattr(lib, name), f"{name} declared in thd_attn.h but not exported"


def test_abi_version_and_status_strings(lib):
    assert lib.thd_attn_abi_version() >> 16 == 1
    for code in (0, -1, -2, -3, -4, -5):
        assert lib.thd_attn_status_string(code) not in (None, b"", b"unknown status")
    assert lib.thd_attn_status_string(7) == b"unknown status"


def _fwd(lib, cu, Hq=4, Hkv=2, D=64, window=0, scale=0.125, ptr=0x10000, lse=None, sinks=None):
    cu = np.asarray(cu, dtype=np.int32)
    return lib.thd_attn_fwd(ptr, ptr, ptr, cu.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)),
                            cu.size - 1, Hq, Hkv, D, window, scale, sinks, ptr, lse, None)


@pytest.mark.parametrize("kw,code", [
    (dict(cu=[0, 5, 3]), -1),                 # decreasing boundaries
    (dict(cu=[1, 5]), -1),                    # does not start at 0
    (dict(cu=[0, 5], Hq=3, Hkv=2), -1),       # Hq % Hkv != 0
    (dict(cu=[0, 5], Hkv=0), -1),
    (dict(cu=[0, 5], window=-1), -1),
    (dict(cu=[0, 5], scale=0.0), -1),
    (dict(cu=[0, 5], scale=-1.0), -1),
    (dict(cu=[0, 5], scale=float("nan")), -1),
    (dict(cu=[0, 5], scale=float("inf")), -1),
    (dict(cu=[0, 5], ptr=0x10008), -1),       # not 16-byte aligned
    (dict(cu=[0, 5], ptr=0), -1),             # null
    (dict(cu=[0, 5], lse=0x10002), -1),       # misaligned lse
    (dict(cu=[0, 5], D=96), -2),              # unsupported head dim
    (dict(cu=[0, 5], D=32), -2),
])
def test_fwd_rejects_bad_arguments_without_touching_cuda(lib, kw, code):
    assert _fwd(lib, **kw) == code


def test_empty_pack_is_a_noop(lib):
    assert _fwd(lib, [0]) == 0
    assert _fwd(lib, [0, 0, 0]) == 0
    assert _fwd(lib, [0, 0], ptr=0) == 0      # nothing to read or write


def test_negative_doc_count_rejected(lib):
    cu = np.zeros(1, dtype=np.int32)
    rc = lib.thd_attn_fwd(16, 16, 16, cu.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)), -1,
                          4, 2, 64, 0, 0.1, None, 16, None, None)
    assert rc == -1


def test_plan_binding_errors(lib):
    with pytest.raises(swa.ThdAttnError) as e:
        swa.thd_attn_plan([0, 4, 2], 4, 2, 64, 0)
    assert e.value.code == -1
    with pytest.raises(swa.ThdAttnError) as e:
        swa.thd_attn_plan([0, 4], 4, 2, 48, 0)
    assert e.value.code == -2


def test_missing_library_fails_loudly(monkeypatch, tmp_path):
    monkeypatch.setattr(swa, "_lib", None)
    monkeypatch.setattr(swa, "_PKG", str(tmp_path))
    with pytest.raises(ImportError):
        swa.load_library()
