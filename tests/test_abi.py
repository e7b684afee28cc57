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
                 "thd_attn_abi_version", "thd_attn_bwd", "thd_attn_bwd_workspace_bytes",
                 "thd_qk_norm_rope", "thd_sparse_mla_fwd", "thd_sparse_mla_workspace_bytes"):
        assert want in names


def test_library_exports_every_declared_symbol(lib):
    for name in declared_functions():
        assert hasattr(lib, name), f"{name} declared in thd_attn.h but not exported"


def test_abi_version_and_status_strings(lib):
    assert lib.thd_attn_abi_version() >> 16 == 1
    for code in (0, -1, -2, -3, -4, -5, -6, -7):
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


# --------------------------------------------------------------- backward ---

def _bwd(lib, cu, Hq=4, Hkv=2, D=64, window=0, scale=0.125, ptr=0x10000, lse=0x10000,
         ws=0x10000, ws_bytes=1 << 30, dq=0x10000):
    cu = np.asarray(cu, dtype=np.int32)
    lib.thd_attn_bwd.argtypes = [ctypes.c_void_p] * 6 + [ctypes.POINTER(ctypes.c_int32)] + \
        [ctypes.c_int] * 5 + [ctypes.c_float] + [ctypes.c_void_p] * 6 + [ctypes.c_size_t, ctypes.c_void_p]
    return lib.thd_attn_bwd(ptr, ptr, ptr, ptr, lse, ptr,
                            cu.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)), cu.size - 1,
                            Hq, Hkv, D, window, scale, None, dq, ptr, ptr, None, ws, ws_bytes, None)


def test_bwd_workspace_size(lib):
    lib.thd_attn_bwd_workspace_bytes.argtypes = [ctypes.c_int64, ctypes.c_int]
    lib.thd_attn_bwd_workspace_bytes.restype = ctypes.c_size_t
    assert lib.thd_attn_bwd_workspace_bytes(1000, 6) == 2 * 24064  # 2 x 24000 rounded up to 256
    assert lib.thd_attn_bwd_workspace_bytes(0, 6) == 0


@pytest.mark.parametrize("kw,code", [
    (dict(cu=[0, 5, 3]), -1),                 # decreasing boundaries
    (dict(cu=[0, 5], D=256, lse=None), -1),   # D = 256 is supported; lse still required
    (dict(cu=[0, 5], D=48), -2),
    (dict(cu=[0, 5], scale=0.0), -1),
    (dict(cu=[0, 5], lse=None), -1),          # the forward's lse is required
    (dict(cu=[0, 5], lse=0x10002), -1),       # misaligned fp32 pointer
    (dict(cu=[0, 5], dq=0x10008), -1),        # misaligned bf16 pointer
    (dict(cu=[0, 5], ws=None), -1),
    (dict(cu=[0, 5], ws_bytes=100), -1),      # workspace smaller than needed
])
def test_bwd_rejects_bad_arguments_before_any_launch(lib, kw, code):
    assert _bwd(lib, **kw) == code


# --------------------------------------------------------------- prologue ---

def _pro(lib, cu, Hq=4, Hkv=2, D=128, eps=1e-5, theta=500000.0, rope=1, ptr=0x10000, kptr=0x10000,
         pos=None):
    cu = np.asarray(cu, dtype=np.int32)
    lib.thd_qk_norm_rope.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.POINTER(ctypes.c_int32),
                                     ctypes.c_int, ctypes.c_void_p, ctypes.c_int, ctypes.c_int,
                                     ctypes.c_int, ctypes.c_float, ctypes.c_float, ctypes.c_int,
                                     ctypes.c_void_p]
    return lib.thd_qk_norm_rope(ptr, kptr, cu.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)),
                                cu.size - 1, pos, Hq, Hkv, D, eps, theta, rope, None)


@pytest.mark.parametrize("kw,code", [
    (dict(cu=[0, 5, 3]), -1),
    (dict(cu=[2, 5]), -1),
    (dict(cu=[0, 5], D=96), -2),
    (dict(cu=[0, 5], eps=0.0), -1),
    (dict(cu=[0, 5], theta=0.5), -1),
    (dict(cu=[0, 5], ptr=0x10008), -1),       # misaligned q
    (dict(cu=[0, 5], pos=0x10002), -1),       # misaligned positions
    (dict(cu=[0, 5], kptr=None), -1),         # k missing with Hkv > 0
    (dict(cu=[0, 0]), 0),                     # empty pack: nothing to do
])
def test_prologue_rejects_bad_arguments_before_any_launch(lib, kw, code):
    assert _pro(lib, **kw) == code


# ------------------------------------------------------------- sparse MLA ---

def _smla(lib, T=4, Tg=4, H=128, K=64, vd=128, scale=0.1, ptr=0x10000, idx=0x10000, ws=0x10000,
          ws_bytes=1 << 30, out=0x10000):
    lib.thd_sparse_mla_fwd.argtypes = [ctypes.c_void_p] * 4 + [ctypes.c_int64, ctypes.c_int64] + \
        [ctypes.c_int] * 3 + [ctypes.c_float, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_size_t,
                              ctypes.c_void_p]
    return lib.thd_sparse_mla_fwd(ptr, ptr, idx, ptr, T, Tg, H, K, vd, scale, out, ws, ws_bytes, None)


@pytest.mark.parametrize("kw,code", [
    (dict(H=64), -2),              # heads in groups of 128
    (dict(K=50), -2),              # slots in chunks of 64 (pad with -1)
    (dict(vd=100), -2),
    (dict(scale=float("nan")), -1),
    (dict(T=-1), -1),
    (dict(idx=0x10002), -1),       # misaligned int32 indices
    (dict(out=0x10008), -1),       # misaligned bf16 output
    (dict(ws_bytes=100), -1),      # workspace smaller than the latent
    (dict(T=0), 0),                # nothing to do
])
def test_sparse_mla_rejects_bad_arguments_before_any_launch(lib, kw, code):
    assert _smla(lib, **kw) == code


def test_sparse_mla_workspace_size(lib):
    lib.thd_sparse_mla_workspace_bytes.argtypes = [ctypes.c_int64, ctypes.c_int, ctypes.c_int]
    lib.thd_sparse_mla_workspace_bytes.restype = ctypes.c_size_t
    # latent 10*128*512*2, indices 10*64*4 -> 2560 (256-aligned), counts 40 -> 256
    assert lib.thd_sparse_mla_workspace_bytes(10, 128, 64) == 1310720 + 2560 + 256


def _host(lib, cu=(0, 5, 9), n_chunks=4, sinks_h=None, sinks_d=None, q_h=0x10000, out_d=0x20000):
    lib.thd_attn_fwd_host.argtypes = [ctypes.c_void_p] * 3 + [ctypes.POINTER(ctypes.c_int32)] + \
        [ctypes.c_int] * 5 + [ctypes.c_float] + [ctypes.c_void_p] * 9 + [ctypes.c_int, ctypes.c_void_p]
    arr = (ctypes.c_int32 * len(cu))(*cu)
    p = 0x30000
    return lib.thd_attn_fwd_host(q_h, p, p, arr, len(cu) - 1, 4, 2, 64, 0, 0.125, sinks_h, p, p,
                                 p, p, p, sinks_d, out_d, p, n_chunks, None)


@pytest.mark.parametrize("kw,code", [
    (dict(n_chunks=0), -1),
    (dict(n_chunks=65), -1),
    (dict(sinks_h=0x40000), -1),          # host sinks without device sinks
    (dict(sinks_d=0x40000), -1),          # device sinks without host sinks
    (dict(cu=(1, 5, 9)), -1),             # cu_seqlens must start at 0
    (dict(cu=(0, 5, 3)), -1),             # and not decrease
    (dict(q_h=None), -1),
    (dict(out_d=None), -1),
    (dict(cu=(0, 0, 0)), 0),              # nothing to do
])
def test_host_pipeline_rejects_bad_arguments_before_any_cuda_call(lib, kw, code):
    assert _host(lib, **kw) == code


def test_stall_selftest_rejects_null_before_any_cuda_call(lib):
    lib.thd_attn_selftest_stall.argtypes = [ctypes.c_void_p]
    assert lib.thd_attn_selftest_stall(None) == -1


# ----------------------------------------------- key-bounded range and merge ---

def _range_keys(lib, cu=(0, 5, 9), qb=0, qe=9, k_end=5, D=64, ptr=0x10000):
    cu = np.asarray(cu, dtype=np.int32)
    lib.thd_attn_fwd_range_keys.argtypes = [ctypes.c_void_p] * 3 + [ctypes.POINTER(ctypes.c_int32)] + \
        [ctypes.c_int, ctypes.c_int64, ctypes.c_int64, ctypes.c_int64] + [ctypes.c_int] * 4 + \
        [ctypes.c_float] + [ctypes.c_void_p] * 4
    return lib.thd_attn_fwd_range_keys(ptr, ptr, ptr, cu.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)),
                                       cu.size - 1, qb, qe, k_end, 4, 2, D, 0, 0.125, None, ptr, None,
                                       None)


@pytest.mark.parametrize("kw,code", [
    (dict(k_end=10), -1),          # beyond the pack
    (dict(k_end=-1), -1),
    (dict(qb=5, qe=4), -1),        # empty-but-reversed row range
    (dict(qe=10), -1),
    (dict(cu=(0, 5, 3)), -1),
    (dict(ptr=0x10008), -1),       # misaligned
    (dict(D=96), -2),
    (dict(qb=4, qe=4), 0),         # no rows: nothing to do
    (dict(cu=(0,), qe=0, k_end=0), 0),
])
def test_range_keys_rejects_bad_arguments_before_any_cuda_call(lib, kw, code):
    assert _range_keys(lib, **kw) == code


def _merge(lib, rows=3, Hq=4, D=128, a=0x10000, la=0x20000, b=0x30000, lb=0x40000, o=0x50000,
           lo=0x60000):
    lib.thd_attn_merge.argtypes = [ctypes.c_void_p] * 4 + [ctypes.c_int64, ctypes.c_int, ctypes.c_int] + \
        [ctypes.c_void_p] * 3
    return lib.thd_attn_merge(a, la, b, lb, rows, Hq, D, o, lo, None)


@pytest.mark.parametrize("kw,code", [
    (dict(D=96), -2),
    (dict(rows=-1), -1),
    (dict(Hq=0), -1),
    (dict(a=None), -1),
    (dict(lo=None), -1),
    (dict(b=0x30008), -1),         # misaligned bf16 part
    (dict(la=0x20002), -1),        # misaligned fp32 LSE
    (dict(rows=0, a=None, la=None), 0),   # nothing to merge
])
def test_merge_rejects_bad_arguments_before_any_launch(lib, kw, code):
    assert _merge(lib, **kw) == code
