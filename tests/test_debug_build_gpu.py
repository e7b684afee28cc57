"""The debug build (THD_DEBUG=1): every forward CTA checks its work items
against the schedule's invariants before touching memory and records
THD_ERR_BAD_ITEM instead of trapping.  On the schedules the library builds the
checks must all pass, and the debug build must compute exactly what the
regular build does (the checks only read)."""
import ctypes
import os

import pytest
import torch

import sliding_window_gqa_cu_b200 as swa
from sliding_window_gqa_cu_b200 import build, workloads

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def debug_lib():
    build.build()
    swa.load_library()
    out = os.path.join(os.path.dirname(swa.library_path()), "libthdattn_debug.so")
    return swa.bind(ctypes.CDLL(build.build(out=out, defines=("THD_DEBUG=1",))))


@pytest.mark.parametrize("lens,Hq,Hkv,D,window,sinks", [
    ([300, 1, 0, 129, 77], 4, 2, 64, 100, True),   # one CTA, two heads
    ([390, 5, 128, 1, 200], 8, 2, 128, 0, True),   # one CTA, two heads, G = 4
    ([400, 77], 4, 2, 128, 0, False),               # one CTA, two heads
    ([300, 9], 6, 2, 128, 50, True),                # one head per item
    ([520, 3], 16, 1, 256, 0, True),                # CTA pair, key-split softmax
    ([300, 45], 3, 1, 256, 64, False),              # one CTA, D = 256
])
def test_debug_build_matches_the_regular_build(debug_lib, lens, Hq, Hkv, D, window, sinks):
    p = workloads.random_pack(41, lens, Hq, Hkv, D, window, D ** -0.5, sinks)
    dev = torch.device("cuda:0")
    q, k, v = (p[n].to(dev) for n in "qkv")
    s = p["sinks"].to(dev) if sinks else None
    ref_o, ref_l = swa.thd_attn_fwd(q, k, v, p["cu_seqlens"], window, p["scale"], s)
    assert swa.thd_attn_get_error() == 0
    regular = swa._lib
    try:
        swa._lib = debug_lib
        out, lse = swa.thd_attn_fwd(q, k, v, p["cu_seqlens"], window, p["scale"], s)
        assert swa.thd_attn_get_error() == 0
    finally:
        swa._lib = regular
    assert torch.equal(out, ref_o) and torch.equal(lse, ref_l)
