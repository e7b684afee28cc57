"""GPU parity of the backward (dq, dk, dv, dsink) against the fp64 CPU oracle.

Tolerance.  The pages fix no precision for the gradient; the forward's
contract is max-abs 2e-2 and mean-abs 2e-3 on outputs of order one.  The
backward rounds P and dS to bf16 (unit roundoff 2^-9) before its three
products and rounds its outputs to bf16, accumulating in fp32, so each
gradient element carries a relative error of a few 2^-9 of the magnitude of
its terms.  The forward's tolerances are therefore applied relative to each
gradient tensor's largest magnitude: max |err| <= 2e-2 * max |ref| and
mean |err| <= 2e-3 * max |ref| (max |ref| floored at 1e-3 for tensors that
vanish exactly).

Small packs are compared element by element on every row; the full-size
benchmark packs on sampled dq rows and sampled dk / dv rows (each computed one
by one by the oracle: dq per query row, dk and dv per key row), on exact sum
invariants of dk and dv where there is no sink, and on the sink gradient of a
4,096-token slice against the oracle's whole-slice value.
"""
import numpy as np
import pytest
import torch

import oracle
import sliding_window_gqa_cu_b200 as swa
from sliding_window_gqa_cu_b200 import build, workloads

REL_MAX, REL_MEAN = 2e-2, 2e-3
# Gradients that vanish exactly (window 1: one key per query, so dq = dk = 0)
# are computed as rounding-level residues; the scale has this floor.
SCALE_FLOOR = 1e-3

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build.build()
    swa.load_library()


def dout_for(p, seed):
    g = torch.Generator().manual_seed(seed)
    return torch.randn(p["q"].shape, generator=g).to(torch.bfloat16)


def run_gpu_bwd(p, dout):
    dev = torch.device("cuda:0")
    q, k, v = (p[n].to(dev) for n in "qkv")
    sinks = p["sinks"].to(dev) if p["sinks"] is not None else None
    out, lse = swa.thd_attn_fwd(q, k, v, p["cu_seqlens"], p["window"], p["scale"], sinks)
    dq, dk, dv, ds = swa.thd_attn_bwd(q, k, v, out, lse, dout.to(dev), p["cu_seqlens"],
                                      p["window"], p["scale"], sinks)
    torch.cuda.synchronize()
    assert swa.thd_attn_get_error() == 0
    return dq.cpu(), dk.cpu(), dv.cpu(), (ds.cpu() if ds is not None else None)


def assert_grad_close(got, ref, what):
    g = got.double().numpy().reshape(ref.shape)
    assert np.isfinite(g).all(), f"{what}: non-finite"
    scale = max(np.abs(ref).max(), SCALE_FLOOR)
    err = np.abs(g - ref)
    assert err.max() <= REL_MAX * scale, f"{what}: max err {err.max():.3e} vs max|ref| {scale:.3e}"
    assert err.mean() <= REL_MEAN * scale, f"{what}: mean err {err.mean():.3e} vs max|ref| {scale:.3e}"


def full_bwd_parity(p, seed, what):
    dout = dout_for(p, seed)
    dq, dk, dv, ds = run_gpu_bwd(p, dout)
    rq, rk, rv, rs = oracle.attention_bwd(p["q"], p["k"], p["v"], dout, p["cu_seqlens"],
                                          p["window"], p["scale"], p["sinks"])
    assert_grad_close(dq, rq, f"{what} dq")
    assert_grad_close(dk, rk, f"{what} dk")
    assert_grad_close(dv, rv, f"{what} dv")
    if rs is None:
        assert ds is None
    else:
        assert_grad_close(ds, rs, f"{what} dsink")


BWD_CASES = [
    # (lens, Hq, Hkv, D, window, sinks)
    ([300, 1, 0, 129, 77], 4, 2, 64, 0, False),
    ([300, 1, 0, 129, 77], 4, 2, 64, 100, True),
    ([255, 2, 130], 3, 1, 64, 0, True),            # odd group
    ([390, 5, 128, 1, 200], 8, 2, 128, 0, False),
    ([390, 5, 128, 1, 200], 8, 2, 128, 0, True),
    ([390, 5, 128, 1, 200], 8, 2, 128, 1, False),  # window 1: own token only
    ([390, 5, 128, 1, 200], 8, 2, 128, 127, True),
    ([390, 5, 128, 1, 200], 8, 2, 128, 129, False),
    ([600], 4, 4, 128, 0, True),                   # MHA
    ([333, 64], 6, 2, 128, 50, False),             # G = 3
    ([520, 3], 16, 1, 128, 0, True),               # MQA, G = 16
    ([500, 130], 16, 2, 128, 300, True),           # G = 8
    ([520, 3], 16, 1, 256, 0, True),               # D = 256, MQA
    ([300, 45, 1], 3, 1, 256, 0, True),            # D = 256, odd group
    ([400, 77], 4, 2, 256, 65, False),             # D = 256, window
    ([200, 1, 130], 2, 2, 256, 0, True),           # D = 256, MHA
    ([700], 4, 1, 256, 129, True),                 # D = 256, several key and query tiles
]


@pytest.mark.parametrize("lens,Hq,Hkv,D,window,sinks", BWD_CASES)
def test_small_pack_bwd_parity(lens, Hq, Hkv, D, window, sinks):
    p = workloads.random_pack(11, lens, Hq, Hkv, D, window, D ** -0.5, sinks)
    full_bwd_parity(p, 1, f"{lens} Hq{Hq} Hkv{Hkv} D{D} W{window} sinks{sinks}")


def test_mid_pack_bwd_parity():
    # several 128-tiles per document on both sides, ragged tails, a sink
    p = workloads.random_pack(12, [1500, 700, 3, 900], 8, 2, 128, 0, 128 ** -0.5, True)
    full_bwd_parity(p, 2, "mid pack")


def test_single_token_documents_bwd():
    p = workloads.random_pack(13, [1] * 200, 4, 2, 128, 0, 128 ** -0.5, False)
    dout = dout_for(p, 3)
    dq, dk, dv, _ = run_gpu_bwd(p, dout)
    # One key per query: dq and dk vanish exactly; the kernel leaves only the
    # fp32 rounding residue of dP - D (an O(1) dot product minus its own value).
    assert dq.float().abs().max() <= 1e-4 and dk.float().abs().max() <= 1e-4
    want = dout.float().reshape(200, 2, 2, 128).sum(2)
    assert (dv.float() - want).abs().max() <= 2e-2 * want.abs().max()


def test_bwd_is_deterministic():
    p = workloads.random_pack(14, [700, 300], 8, 2, 128, 0, 128 ** -0.5, True)
    dout = dout_for(p, 4)
    a = run_gpu_bwd(p, dout)
    b = run_gpu_bwd(p, dout)
    for x, y in zip(a, b):
        assert torch.equal(x, y)


def test_mid_pack_bwd_parity_d256():
    # head dim 256: several 64-key and 64-query tiles per document, a sink
    p = workloads.random_pack(15, [1100, 300, 2], 8, 2, 256, 0, 256 ** -0.5, True)
    full_bwd_parity(p, 7, "mid pack D256")


# ------------------------------------------------- full-size benchmark packs -

def sample_rows(cu, window, Hq, rng, n_random=256):
    rows = set()
    cu = [int(x) for x in cu]
    for d in range(len(cu) - 1):
        s, e = cu[d], cu[d + 1]
        for t in (s, s + 1, e - 1, e - 128, e - 129, s + window, s + window - 1):
            if s <= t < e:
                rows.add((t, int(rng.integers(Hq))))
    for t in rng.integers(0, cu[-1], size=n_random):
        rows.add((int(t), int(rng.integers(Hq))))
    return np.array(sorted(rows), dtype=np.int64)


def kv_sample_rows(cu, window, Hkv, rng, starts=True):
    """(key token, kv head) rows for the key-side check: keys at each
    document's end and its last tile edges (few queries see them, so the
    oracle stays cheap), every tile edge of the two shortest documents, and
    the first key of the two longest (seen by a whole window, or document, of
    queries when that is short enough)."""
    cu = [int(x) for x in cu]
    docs = [(cu[d], cu[d + 1]) for d in range(len(cu) - 1) if cu[d + 1] > cu[d]]
    rows = set()
    for s, e in docs:
        for t in (e - 1, e - 2, e - 64, e - 127, e - 128, e - 129, e - 200):
            if s <= t < e:
                rows.add((t, int(rng.integers(Hkv))))
    for s, e in sorted(docs, key=lambda d: d[1] - d[0])[:2]:
        for t in (s, s + 1, s + 127, s + 128, s + 129):
            if s <= t < e:
                rows.add((t, int(rng.integers(Hkv))))
    if window > 0 and starts:
        for s, e in sorted(docs, key=lambda d: d[0] - d[1])[:2]:
            rows.add((s, int(rng.integers(Hkv))))
            rows.add((s + (e - s) // 2, int(rng.integers(Hkv))))
    return np.array(sorted(rows), dtype=np.int64)


def assert_sample_close(got, ref, what):
    scale = max(np.abs(ref).max(), SCALE_FLOOR)
    err = np.abs(got - ref)
    assert np.isfinite(got).all(), f"{what}: non-finite"
    assert err.max() <= REL_MAX * scale, f"{what}: max err {err.max():.3e} vs {scale:.3e}"
    assert err.mean() <= REL_MEAN * scale, f"{what}: mean err {err.mean():.3e} vs {scale:.3e}"


@pytest.mark.parametrize("name", ["pack64k_gqa8_d128_causal_sink", "pack32k_gqa4_d128_w4096",
                                  "doc128k_mqa_d256_w8192_sink"])
def test_full_size_pack_bwd(name):
    cfg = workloads.CONFIGS[name]
    p = workloads.make_pack(cfg, 0)
    dout = dout_for(p, 5)
    dq, dk, dv, ds = run_gpu_bwd(p, dout)
    for t in (dq, dk, dv):
        assert torch.isfinite(t.float()).all()
    rows = sample_rows(p["cu_seqlens"], cfg.window, cfg.Hq, np.random.default_rng(1))
    ref = oracle.attention_bwd_q_rows(p["q"], p["k"], p["v"], dout, p["cu_seqlens"], cfg.window,
                                      cfg.scale, rows, p["sinks"])
    assert_sample_close(dq[rows[:, 0], rows[:, 1]].double().numpy(), ref, f"{name} dq rows")
    # key side, element by element on sampled (key, kv head) rows
    # (a key in the middle of the 128k document is seen by 8,192 queries of
    # all 16 heads, too many for the oracle here: only its end-of-document keys)
    krows = kv_sample_rows(p["cu_seqlens"], cfg.window, cfg.Hkv, np.random.default_rng(2),
                           starts=cfg.D != 256)
    rk, rv = oracle.attention_bwd_kv_rows(p["q"], p["k"], p["v"], dout, p["cu_seqlens"],
                                          cfg.window, cfg.scale, krows, p["sinks"])
    assert_sample_close(dk[krows[:, 0], krows[:, 1]].double().numpy(), rk, f"{name} dk rows")
    assert_sample_close(dv[krows[:, 0], krows[:, 1]].double().numpy(), rv, f"{name} dv rows")
    if p["sinks"] is None:
        # Exact invariants without a sink: softmax is shift invariant, so the
        # key gradients of a (document, kv head) sum to zero, and the value
        # gradients sum to the sum of dO over the document and the group.
        cu = np.asarray(p["cu_seqlens"])
        G = cfg.Hq // cfg.Hkv
        dkf, dvf, dof = dk.double(), dv.double(), dout.double()
        for d in range(len(cu) - 1):
            a, b = int(cu[d]), int(cu[d + 1])
            for g in range(cfg.Hkv):
                want_v = dof[a:b, g * G:(g + 1) * G].sum((0, 1))
                got_v = dvf[a:b, g].sum(0)
                assert (got_v - want_v).abs().max() <= 2e-2 * want_v.abs().max() + 1e-3 * (b - a) ** 0.5
                ksum = dkf[a:b, g].sum(0).abs().max()
                assert ksum <= 2e-2 * dkf[a:b, g].abs().sum(0).max()


def test_sink_gradient_on_a_4k_slice():
    """dsink sums over every query row, so it is checked on the first 4,096
    tokens of the 64k pack (its sinks, heads and scale) against the oracle's
    sink gradient of the whole slice."""
    cfg = workloads.CONFIGS["pack64k_gqa8_d128_causal_sink"]
    p = workloads.make_pack(cfg, 0, T_override=4096)
    dout = dout_for(p, 6)
    _, _, _, ds = run_gpu_bwd(p, dout)
    ref = oracle.attention_dsink(p["q"], p["k"], p["v"], dout, p["cu_seqlens"], cfg.window,
                                 cfg.scale, p["sinks"])
    assert_sample_close(ds.double().numpy(), ref, "dsink (4k slice)")
