"""Packs with hundreds of work items of mixed lengths.

Long runs of one-tile items (one-token documents) mixed with long documents,
windows and sinks, for every one-CTA shape of the forward (two heads per CTA
with one S buffer, one head with two, head dims 64, 128 and 256): more work
items than SMs, so CTAs of different lengths run back to back on every SM.
Checked

  * against the oracle on every row (the tolerances of the parity tests);
  * under launches of two packs on two streams at once, and alternately on one
    stream (the schedule cache serves both): every result equals that pack's
    result from a quiet GPU, bit for bit;
  * through the allocation-free entry point, bit for bit against thd_attn_fwd.
"""
import numpy as np
import pytest
import torch

import oracle
import sliding_window_gqa_cu_b200 as swa
from sliding_window_gqa_cu_b200 import build, workloads

OUT_MAX, OUT_MEAN, LSE_MAX = 2e-2, 2e-3, 1e-3   # the tolerances of the parity tests

pytestmark = pytest.mark.gpu

_RNG_LENS = np.random.default_rng(7)
MIXED = ([1] * 40 + [130, 257, 700, 1025, 2048, 5, 64, 128, 129, 0, 3]
         + [int(x) for x in _RNG_LENS.integers(1, 400, size=20)])

CASES = [
    # (seed, lens, Hq, Hkv, D, window, sinks): more items than the 148 SMs in every case
    (51, MIXED, 16, 2, 128, 0, True),      # two heads per CTA, one S buffer
    (52, MIXED, 16, 2, 128, 300, False),   # same, sliding window
    (53, MIXED, 6, 6, 128, 0, True),       # G = 1: one head per CTA, two S buffers
    (54, MIXED, 8, 2, 64, 129, True),      # D = 64, two heads per CTA
    (55, MIXED, 6, 2, 64, 0, False),       # D = 64, odd group
    (56, [3000, 900, 64, 2] + [1] * 30 + [200] * 10, 3, 1, 256, 300, True),  # D = 256, one CTA
]


def _n_items(p):
    return len(swa.thd_attn_plan(p["cu_seqlens"], p["Hq"], p["Hkv"], p["D"], p["window"]))


@pytest.fixture(scope="module")
def libs():
    build.build()
    return swa.load_library()


def _run(p, dev, stream=None):
    q, k, v = (p[n].to(dev) for n in "qkv")
    s = p["sinks"].to(dev) if p["sinks"] is not None else None
    return swa.thd_attn_fwd(q, k, v, p["cu_seqlens"], p["window"], p["scale"], s, stream=stream)


@pytest.mark.parametrize("case", CASES, ids=[f"D{c[4]}_Hq{c[2]}_Hkv{c[3]}_w{c[5]}" for c in CASES])
def test_many_items_parity(libs, case):
    seed, lens, Hq, Hkv, D, window, sinks = case
    p = workloads.random_pack(seed, lens, Hq, Hkv, D, window, D ** -0.5, sinks)
    assert _n_items(p) > 148
    dev = torch.device("cuda:0")
    out, lse = _run(p, dev)
    assert swa.thd_attn_get_error() == 0
    ref_out, ref_lse = oracle.attention(p["q"], p["k"], p["v"], p["cu_seqlens"], window,
                                        p["scale"], p["sinks"])
    o = out.cpu().double().numpy().reshape(ref_out.shape)
    err = np.abs(o - ref_out)
    assert np.isfinite(o).all()
    assert err.max() <= OUT_MAX and err.mean() <= OUT_MEAN, (err.max(), err.mean())
    assert np.abs(lse.cpu().double().numpy().reshape(ref_lse.shape) - ref_lse).max() <= LSE_MAX


def test_two_streams_at_once_and_alternating_packs(libs):
    """Two packs launched back to back on two streams without synchronising
    (their launches may overlap on the GPU), then alternately on one stream:
    every result equals that pack's result from a quiet GPU."""
    dev = torch.device("cuda:0")
    pa = workloads.random_pack(61, MIXED, 16, 2, 128, 0, 128 ** -0.5, True)
    pb = workloads.random_pack(62, MIXED[::-1], 8, 8, 128, 200, 128 ** -0.5, False)
    ref = [_run(pa, dev), _run(pb, dev)]
    torch.cuda.synchronize()
    assert swa.thd_attn_get_error() == 0
    s1, s2 = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    tensors = []
    for p in (pa, pb):
        q, k, v = (p[n].to(dev) for n in "qkv")
        s = p["sinks"].to(dev) if p["sinks"] is not None else None
        tensors.append((q, k, v, s))
    torch.cuda.synchronize()
    results = []
    for rep in range(4):
        for idx, st in ((0, s1), (1, s2)):
            q, k, v, s = tensors[idx]
            p = (pa, pb)[idx]
            with torch.cuda.stream(st):
                results.append((idx, swa.thd_attn_fwd(q, k, v, p["cu_seqlens"], p["window"],
                                                      p["scale"], s, stream=st)))
    torch.cuda.synchronize()
    for rep in range(3):  # one stream, alternating packs
        for idx in (0, 1):
            q, k, v, s = tensors[idx]
            p = (pa, pb)[idx]
            results.append((idx, swa.thd_attn_fwd(q, k, v, p["cu_seqlens"], p["window"],
                                                  p["scale"], s)))
    torch.cuda.synchronize()
    assert swa.thd_attn_get_error() == 0
    for idx, (o, l) in results:
        assert torch.equal(o, ref[idx][0]) and torch.equal(l, ref[idx][1])


def test_noalloc_many_items_matches_regular(libs):
    dev = torch.device("cuda:0")
    stream = torch.cuda.current_stream(dev)
    for seed, lens, Hq, Hkv, D, window, sinks in (CASES[0], CASES[2], CASES[5], CASES[0]):
        p = workloads.random_pack(seed, lens, Hq, Hkv, D, window, D ** -0.5, sinks)
        q, k, v = (p[n].to(dev) for n in "qkv")
        s = p["sinks"].to(dev) if p["sinks"] is not None else None
        ref_out, ref_lse = swa.thd_attn_fwd(q, k, v, p["cu_seqlens"], window, p["scale"], s)
        assert swa.thd_attn_get_error() == 0
        out = torch.full_like(ref_out, float("nan"))
        lse = torch.full_like(ref_lse, float("nan"))
        swa.thd_attn_fwd_noalloc(q, k, v, p["cu_seqlens"], out, lse, window, p["scale"], s,
                                 stream=stream)
        assert swa.thd_attn_noalloc_get_error(stream) == 0
        assert torch.equal(out, ref_out) and torch.equal(lse, ref_lse)
