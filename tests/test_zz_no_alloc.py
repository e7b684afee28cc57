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


@pytest.mark.gpu
def test_noalloc_matches_the_regular_entry_point_on_two_calls_in_a_row(lib):
    dev = torch.device("cuda:0")
    stream = torch.cuda.current_stream(dev)
    packs = [
        workloads.random_pack(31, [700, 1, 0, 255, 129], 16, 4, 128, 0, 128 ** -0.5, True),
        workloads.random_pack(32, [900, 77], 8, 1, 256, 300, 256 ** -0.5, False),
    ]
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    for i, p in enumerate(packs):
        q, k, v = (p[n].to(dev) for n in "qkv")
        sinks = p["sinks"].to(dev) if p["sinks"] is not None else None
        ref_out, ref_lse = swa.thd_attn_fwd(q, k, v, p["cu_seqlens"], p["window"], p["scale"], sinks)
        assert swa.thd_attn_get_error() == 0
        out = torch.full_like(ref_out, float("nan"))
        lse = torch.full_like(ref_lse, float("nan"))
        # first call: the scratch's own status word; second: a caller-owned one
        rc = _noalloc_c_call(lib, q, k, v, p["cu_seqlens"], p["window"], p["scale"], sinks, out,
                             lse, status if i == 1 else None, stream)
        assert rc == 0, swa.STATUS.get(rc, rc)
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        err = (out.float() - ref_out.float()).abs()
        assert torch.isfinite(out.float()).all()
        assert err.max().item() <= OUT_MAX and err.mean().item() <= OUT_MEAN
        assert (lse - ref_lse).abs().max().item() <= LSE_MAX
