"""GPU parity: the CUDA path (through the C ABI) against the fp64 CPU oracle.

Tolerances (from the hot path's numerical contract): bf16 output max-abs
error 2e-2 and mean-abs error 2e-3; fp32 log-sum-exp max-abs error 1e-3.
Small packs, the 8k and the 32k benchmark packs are compared element by
element on every row.  The 64k pack and the 128k document are compared on a
dense subset of rows the oracle computes one by one (two full query heads,
1/61 of all rows, document, tile and window edges), in the same launch
configuration the benchmark times; tests/test_full_oracle_gpu.py checks every
row of those two on request.
"""
import numpy as np
import pytest
import torch

import oracle
import sliding_window_gqa_cu_b200 as swa
from sliding_window_gqa_cu_b200 import build, workloads

OUT_MAX, OUT_MEAN, LSE_MAX = 2e-2, 2e-3, 1e-3

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build.build()
    swa.load_library()


def run_gpu(p, with_lse=True):
    dev = torch.device("cuda:0")
    q, k, v = (p[n].to(dev) for n in "qkv")
    sinks = p["sinks"].to(dev) if p["sinks"] is not None else None
    out, lse = swa.thd_attn_fwd(q, k, v, p["cu_seqlens"], p["window"], p["scale"], sinks,
                                return_lse=with_lse)
    assert swa.thd_attn_get_error() == 0
    torch.cuda.synchronize()
    return out.cpu(), (lse.cpu() if lse is not None else None)


def assert_close(out_gpu, lse_gpu, out_ref, lse_ref, what=""):
    o = out_gpu.double().numpy().reshape(out_ref.shape)
    err = np.abs(o - out_ref)
    assert np.isfinite(o).all(), f"{what}: non-finite output"
    assert err.max() <= OUT_MAX, f"{what}: max abs err {err.max():.3e}"
    assert err.mean() <= OUT_MEAN, f"{what}: mean abs err {err.mean():.3e}"
    if lse_gpu is not None:
        l = lse_gpu.double().numpy().reshape(lse_ref.shape)
        lerr = np.abs(l - lse_ref)
        assert lerr.max() <= LSE_MAX, f"{what}: lse max abs err {lerr.max():.3e}"


def full_parity(p, what=""):
    out, lse = run_gpu(p)
    ref_out, ref_lse = oracle.attention(p["q"], p["k"], p["v"], p["cu_seqlens"], p["window"],
                                        p["scale"], p["sinks"])
    assert_close(out, lse, ref_out, ref_lse, what)
    return out, lse


# ------------------------------------------------------------ small packs ----

def test_tiny_pack_all_rows():
    cfg = workloads.CONFIGS["tiny_2doc_gqa2_d64"]
    full_parity(workloads.make_pack(cfg, 0), cfg.name)


CASES = [
    # (lens, Hq, Hkv, D, window, sinks)
    ([300, 1, 0, 129, 77], 4, 2, 64, 0, False),
    ([300, 1, 0, 129, 77], 4, 2, 64, 100, True),
    ([255, 2, 130], 3, 1, 64, 0, True),           # odd group: one head per item
    ([390, 5, 128, 1, 200], 8, 2, 128, 0, False),
    ([390, 5, 128, 1, 200], 8, 2, 128, 0, True),
    ([390, 5, 128, 1, 200], 8, 2, 128, 1, False),
    ([390, 5, 128, 1, 200], 8, 2, 128, 2, True),
    ([390, 5, 128, 1, 200], 8, 2, 128, 127, False),
    ([390, 5, 128, 1, 200], 8, 2, 128, 128, True),
    ([390, 5, 128, 1, 200], 8, 2, 128, 129, False),
    ([600], 4, 4, 128, 0, True),                  # MHA, G = 1
    ([333, 64], 6, 2, 128, 50, False),            # G = 3
    ([520, 3], 16, 1, 256, 0, True),              # MQA, D = 256 (CTA pair)
    ([520, 3], 4, 2, 256, 65, False),
    ([700, 0, 0], 2, 1, 256, 64, True),
    ([400, 77], 4, 2, 128, 0, True),              # one CTA, two heads (group 2)
    ([300, 9], 12, 2, 128, 100, True),            # group 6: one CTA, two heads
    ([500, 130], 16, 2, 128, 0, True),            # group 8
    ([300, 45], 3, 1, 256, 0, True),              # odd group at D = 256: one CTA, one head
]


@pytest.mark.parametrize("lens,Hq,Hkv,D,window,sinks", CASES)
def test_small_pack_parity(lens, Hq, Hkv, D, window, sinks):
    p = workloads.random_pack(1, lens, Hq, Hkv, D, window, D ** -0.5, sinks)
    full_parity(p, f"{lens} Hq{Hq} Hkv{Hkv} D{D} W{window} sinks{sinks}")


def test_window_at_least_doc_equals_causal_on_gpu():
    p = workloads.random_pack(2, [200, 50], 4, 2, 128, 0, 128 ** -0.5, True)
    out0, lse0 = run_gpu(p)
    p2 = dict(p, window=200)
    out1, lse1 = run_gpu(p2)
    assert torch.equal(out0, out1) and torch.equal(lse0, lse1)


def test_gqa_equals_mha_on_expanded_kv_on_gpu():
    p = workloads.random_pack(3, [300, 40], 8, 2, 128, 0, 128 ** -0.5, False)
    out_g, _ = run_gpu(p)
    pm = dict(p, k=p["k"].repeat_interleave(4, 1).contiguous(), v=p["v"].repeat_interleave(4, 1).contiguous(),
              Hkv=8)
    out_m, _ = run_gpu(pm)
    assert (out_g.float() - out_m.float()).abs().max() <= 1e-2


def test_zero_query_gives_window_mean_on_gpu():
    p = workloads.random_pack(4, [260, 9], 4, 2, 64, 0, 0.125, False)
    p["q"] = torch.zeros_like(p["q"])
    full_parity(p, "q=0")


def test_without_lse_and_out_canary():
    p = workloads.random_pack(5, [140, 3, 90], 4, 2, 128, 0, 128 ** -0.5, True)
    T, Hq, D = p["q"].shape
    dev = torch.device("cuda:0")
    pad = 4096
    buf = torch.full((T * Hq * D + 2 * pad,), 7.0, dtype=torch.bfloat16, device=dev)
    out = buf[pad:pad + T * Hq * D].view(T, Hq, D)
    swa.thd_attn_fwd(p["q"].to(dev), p["k"].to(dev), p["v"].to(dev), p["cu_seqlens"], 0,
                     p["scale"], p["sinks"].to(dev), out=out, return_lse=False)
    torch.cuda.synchronize()
    assert (buf[:pad] == 7.0).all() and (buf[-pad:] == 7.0).all(), "wrote outside out"
    ref, _ = oracle.attention(p["q"], p["k"], p["v"], p["cu_seqlens"], 0, p["scale"], p["sinks"])
    assert_close(out.cpu(), None, ref, None, "no-lse")


def test_empty_packs_are_noops():
    dev = torch.device("cuda:0")
    e = torch.empty((0, 4, 64), dtype=torch.bfloat16, device=dev)
    ek = torch.empty((0, 2, 64), dtype=torch.bfloat16, device=dev)
    out, lse = swa.thd_attn_fwd(e, ek, ek, [0], 0, 0.125)
    out, lse = swa.thd_attn_fwd(e, ek, ek, [0, 0, 0], 0, 0.125)
    assert out.shape == (0, 4, 64) and swa.thd_attn_get_error() == 0


def test_single_token_documents():
    p = workloads.random_pack(6, [1] * 300, 4, 2, 128, 0, 128 ** -0.5, False)
    out, lse = run_gpu(p)
    want = p["v"].repeat_interleave(2, 1).float()
    assert (out.float() - want).abs().max() == 0     # exactly its own value row, rounded once
    full_parity(p, "single-token docs")


def test_repeat_calls_reuse_cached_schedule():
    p = workloads.random_pack(7, [333, 444], 8, 2, 128, 0, 128 ** -0.5, True)
    a, la = run_gpu(p)
    b, lb = run_gpu(p)
    assert torch.equal(a, b) and torch.equal(la, lb)


# ------------------------------------------------- full-size benchmark packs -

def sample_rows(cu, window, Hq, rng, n_random=384):
    rows = set()
    cu = [int(x) for x in cu]
    for d in range(len(cu) - 1):
        s, e = cu[d], cu[d + 1]
        if e == s:
            continue
        for t in (s, s + 1, e - 1, e - 2, e - 128, e - 129, e - 127, s + window - 1, s + window,
                  s + window + 1):
            if s <= t < e:
                rows.add((t, int(rng.integers(Hq))))
    for t in rng.integers(0, cu[-1], size=n_random):
        rows.add((int(t), int(rng.integers(Hq))))
    return np.array(sorted(rows), dtype=np.int64)


@pytest.mark.parametrize("name", ["pack8k_gqa4_d128_causal", "pack32k_gqa4_d128_w4096"])
def test_full_size_pack_every_row(name):
    """Every (token, head) row of the 8k and 32k benchmark packs, element by
    element, against the full oracle (FlintMagiPlan.attention's window and
    sink semantics, "flint.magi" page)."""
    cfg = workloads.CONFIGS[name]
    p = workloads.make_pack(cfg, 0)
    full_parity(p, name)


def dense_subset_rows(cu, window, Hq, Hkv, stride=61):
    """Every row of the first query head of the first kv group and of the last
    query head of the last kv group, every stride-th (token, head) row of the
    flattened pack (stride prime to the head counts, so all heads and token
    positions mod 128 are hit), plus document, tile and window edges."""
    T = int(cu[-1])
    rows = {(t, h) for h in (0, Hq - 1) for t in range(T)}
    rows.update((r // Hq, r % Hq) for r in range(7, T * Hq, stride))
    rows.update(map(tuple, sample_rows(cu, window, Hq, np.random.default_rng(0))))
    return np.array(sorted(rows), dtype=np.int64)


@pytest.mark.parametrize("name", ["pack64k_gqa8_d128_causal_sink", "doc128k_mqa_d256_w8192_sink"])
def test_full_size_pack_dense_subset(name):
    """The 64k pack and the 128k document, in the launch configuration the
    benchmark times: two full query heads (one at each end of the kv groups)
    and 1/61 of all other rows, element by element against the oracle."""
    cfg = workloads.CONFIGS[name]
    p = workloads.make_pack(cfg, 0)
    out, lse = run_gpu(p)
    assert torch.isfinite(out.float()).all() and torch.isfinite(lse).all()
    rows = dense_subset_rows(p["cu_seqlens"], cfg.window, cfg.Hq, cfg.Hkv)
    ref_o, ref_l = oracle.attention_rows(p["q"], p["k"], p["v"], p["cu_seqlens"], cfg.window,
                                         cfg.scale, rows, p["sinks"])
    got_o = out[rows[:, 0], rows[:, 1]]
    got_l = lse[rows[:, 0], rows[:, 1]]
    assert_close(got_o, got_l, ref_o, ref_l, name)
