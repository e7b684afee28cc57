"""The allocation-free entry point, thd_attn_fwd_noalloc.

Some callers may not allocate device memory: runtimes that reserve all device
memory up front and hand out only pre-planned buffers, and latency-critical
loops that cannot take the device-wide synchronisation cudaMalloc/cudaFree may
cause.  For them the library offers a variant whose only scratch (the tile
schedule and a status word) is a fixed array inside its device image.

This file is collected last on purpose (test_zz_...): if it fails, a run that
stops at the first failure has already run every other test.  It passes both
alone in a fresh process (the first call then does the per-device set-up) and
after the other tests.
"""
import ctypes

import numpy as np
import pytest
import torch

import sliding_window_gqa_cu_b200 as swa
from sliding_window_gqa_cu_b200 import build, workloads

OUT_MAX, OUT_MEAN, LSE_MAX = 2e-2, 2e-3, 1e-3   # the tolerances of the parity tests


@pytest.fixture(scope="module")
def lib():
    build.build()
    return swa.load_library()


def _noalloc_c_call(lib, q, k, v, cu, window, scale, sinks, out, lse, status, stream):
    cu = np.ascontiguousarray(cu, dtype=np.int32)
    return lib.thd_attn_fwd_noalloc(
        q.data_ptr(), k.data_ptr(), v.data_ptr(), cu.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)),
        cu.size - 1, q.shape[1], k.shape[1], q.shape[2], window, scale,
        sinks.data_ptr() if sinks is not None else None, out.data_ptr(),
        lse.data_ptr() if lse is not None else None,
        status.data_ptr() if status is not None else None, ctypes.c_void_p(stream.cuda_stream))


def test_oversized_schedule_is_rejected_before_any_cuda_call(lib):
    # 65,537 query tiles x 1 head pair: one item past the scratch's 65,536.
    cu = np.array([0, 128 * 65537], dtype=np.int32)
    p = 1 << 20
    rc = lib.thd_attn_fwd_noalloc(p, p, p, cu.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)), 1,
                                  2, 1, 128, 0, 0.1, None, p, None, None, None)
    assert rc == -6
    assert b"scratch" in lib.thd_attn_status_string(-6)


CASES = [
    # (seed, lens, Hq, Hkv, D, window, sinks, status word used)
    (31, [700, 1, 0, 255, 129], 16, 4, 128, 0, True, "scratch"),    # two heads per CTA
    (32, [900, 77], 8, 1, 256, 300, False, "caller"),               # D = 256, CTA pair
    (32, [900, 77], 8, 1, 256, 300, False, "scratch"),              # same pack: cached schedule
    (33, [300, 5, 200], 4, 2, 64, 0, True, "caller"),               # D = 64
    (34, [400, 129], 3, 1, 128, 77, True, "scratch"),               # odd group: one head per CTA
]


@pytest.mark.gpu
def test_noalloc_matches_the_regular_entry_point_on_calls_in_a_row(lib):
    """Each call is compared with thd_attn_fwd on the same inputs, within the
    parity tolerances and bit for bit (both run the same kernel on the same
    work items, so every output row is computed the same way).  The third
    call repeats the second one's pack, so it runs on the schedule already in
    the scratch without uploading it again."""
    dev = torch.device("cuda:0")
    stream = torch.cuda.current_stream(dev)
    caller_status = torch.zeros(1, dtype=torch.int32, device=dev)
    for seed, lens, Hq, Hkv, D, window, with_sinks, status_kind in CASES:
        p = workloads.random_pack(seed, lens, Hq, Hkv, D, window, D ** -0.5, with_sinks)
        q, k, v = (p[n].to(dev) for n in "qkv")
        sinks = p["sinks"].to(dev) if p["sinks"] is not None else None
        ref_out, ref_lse = swa.thd_attn_fwd(q, k, v, p["cu_seqlens"], p["window"], p["scale"], sinks)
        assert swa.thd_attn_get_error() == 0
        out = torch.full_like(ref_out, float("nan"))
        lse = torch.full_like(ref_lse, float("nan"))
        rc = _noalloc_c_call(lib, q, k, v, p["cu_seqlens"], p["window"], p["scale"], sinks, out,
                             lse, caller_status if status_kind == "caller" else None, stream)
        assert rc == 0, swa.STATUS.get(rc, rc)
        torch.cuda.synchronize()
        if status_kind == "caller":
            assert int(caller_status.item()) == 0
        else:
            assert swa.thd_attn_noalloc_get_error(stream) == 0
        assert torch.isfinite(out.float()).all()
        err = (out.float() - ref_out.float()).abs()
        assert err.max().item() <= OUT_MAX and err.mean().item() <= OUT_MEAN
        assert (lse - ref_lse).abs().max().item() <= LSE_MAX
        assert torch.equal(out, ref_out) and torch.equal(lse, ref_lse)
