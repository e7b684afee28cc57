"""The forward from host buffers with overlapped copies (thd_attn_fwd_host).

Its token ranges are computed as thd_attn_fwd_range computes them, so the
result must equal, bit for bit, the same ranges run one after another on the
device.  (The range schedule aligns tiles to the range end, so a row's keys
are grouped into tiles differently than in the whole-pack forward and the
lazily rescaled running max, hence the bf16 rounding of P, can differ: against
thd_attn_fwd and the fp64 oracle the forward's tolerances apply.)"""
import numpy as np
import pytest
import torch

import oracle
import sliding_window_gqa_cu_b200 as swa
from sliding_window_gqa_cu_b200 import build, workloads

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build.build()
    swa.load_library()


def _pinned(t):
    return t.contiguous().pin_memory()


@pytest.mark.parametrize("lens,Hq,Hkv,D,window,sinks,n_chunks", [
    ([300, 1, 0, 129, 77], 4, 2, 64, 0, False, 3),
    ([390, 5, 128, 1, 200], 8, 2, 128, 127, True, 8),
    ([1000], 16, 1, 256, 300, True, 5),
    ([70, 3], 4, 4, 128, 0, False, 64),    # more ranges than some documents have rows
])
def test_host_pipeline_equals_device_forward(lens, Hq, Hkv, D, window, sinks, n_chunks):
    p = workloads.random_pack(5, lens, Hq, Hkv, D, window, D ** -0.5, sinks)
    dev = torch.device("cuda:0")
    q, k, v = (p[n].to(dev) for n in "qkv")
    s_d = p["sinks"].to(dev) if p["sinks"] is not None else None
    T = q.shape[0]
    ranges = [(T * c // n_chunks, T * (c + 1) // n_chunks) for c in range(n_chunks)]
    parts = [swa.thd_attn_fwd_range(q[a:b].contiguous(), k, v, p["cu_seqlens"], a, b, window,
                                    p["scale"], s_d) for a, b in ranges if b > a]
    out_rng = torch.cat([o for o, _ in parts]).cpu()
    lse_rng = torch.cat([l for _, l in parts]).cpu()
    out_full, lse_full = swa.thd_attn_fwd(q, k, v, p["cu_seqlens"], window, p["scale"], s_d)
    out_h, lse_h = swa.thd_attn_fwd_host(_pinned(p["q"]), _pinned(p["k"]), _pinned(p["v"]),
                                         p["cu_seqlens"], window, p["scale"],
                                         p["sinks"] if sinks else None, n_chunks=n_chunks)
    torch.cuda.synchronize()
    assert swa.thd_attn_get_error() == 0
    assert torch.equal(out_h, out_rng)
    assert torch.equal(lse_h, lse_rng)
    assert (out_h.float() - out_full.cpu().float()).abs().max() <= 1.6e-2
    assert (lse_h - lse_full.cpu()).abs().max() <= 1e-3
    ro, rl = oracle.attention(p["q"], p["k"], p["v"], p["cu_seqlens"], window, p["scale"], p["sinks"])
    err = np.abs(out_h.double().numpy() - ro)
    assert err.max() <= 2e-2 and err.mean() <= 2e-3
    assert np.abs(lse_h.double().numpy() - rl).max() <= 1e-3


def test_host_pipeline_reuses_device_buffers_across_calls():
    p = workloads.random_pack(6, [500, 260, 33], 8, 2, 128, 0, 128 ** -0.5, True)
    dev = torch.device("cuda:0")
    T = p["q"].shape[0]
    bufs = {"q": torch.empty_like(p["q"], device=dev), "k": torch.empty_like(p["k"], device=dev),
            "v": torch.empty_like(p["v"], device=dev),
            "out": torch.empty((T, 8, 128), dtype=torch.bfloat16, device=dev),
            "lse": torch.empty((T, 8), dtype=torch.float32, device=dev),
            "sinks": torch.empty(8, dtype=torch.float32, device=dev)}
    qh, kh, vh = _pinned(p["q"]), _pinned(p["k"]), _pinned(p["v"])
    outs = []
    for _ in range(3):  # each call gets fresh host outputs; the device buffers are shared
        outs.append(swa.thd_attn_fwd_host(qh, kh, vh, p["cu_seqlens"], 0, p["scale"], p["sinks"],
                                          device_buffers=bufs, n_chunks=4))
    torch.cuda.synchronize()
    for o, l in outs[1:]:
        assert torch.equal(o, outs[0][0]) and torch.equal(l, outs[0][1])
