"""Pins for the CPU oracle: checks against what the pages and mathematics fix.

Nothing here compares the oracle with itself.  Each check is either a
hand-derived worked example (tests/golden/), a closed form, a special case
that reduces to a textbook/library routine, an invariant of the definition,
or a second independent formulation (the dense-mask brute force).
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
from sliding_window_gqa_cu_b200 import workloads

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "hand_examples.json")


def _pack(seed, lens, Hq, Hkv, D, window, scale=None, sinks=False, std=1.0):
    scale = D ** -0.5 if scale is None else scale
    return workloads.random_pack(seed, lens, Hq, Hkv, D, window, scale, sinks, std)


def _run(p, **over):
    args = dict(q=p["q"], k=p["k"], v=p["v"], cu_seqlens=p["cu_seqlens"], window=p["window"],
                scale=p["scale"], sinks=p["sinks"])
    args.update(over)
    return oracle.attention(**args)


# ---------------------------------------------------------------- golden ----

def _golden_cases():
    with open(GOLDEN) as f:
        return json.load(f)["cases"]


@pytest.mark.parametrize("case", _golden_cases(), ids=lambda c: c["name"])
def test_hand_worked_examples(case):
    env = {"e": math.e, "log": math.log}
    q = np.asarray(case["q"], dtype=np.float64)
    k = np.asarray(case["k"], dtype=np.float64)
    v = np.asarray(case["v"], dtype=np.float64)
    out, lse = oracle.attention(q, k, v, case["cu_seqlens"], case["window"], case["scale"],
                                case["sinks"])
    for row in case["expected"]:
        t, h = row["token"], row["head"]
        want = [eval(expr, {"__builtins__": {}}, env) for expr in row["out"]]
        np.testing.assert_allclose(out[t, h], want, rtol=1e-13, atol=1e-13, err_msg=row["why"])
        assert abs(lse[t, h] - eval(row["lse"], {"__builtins__": {}}, env)) < 1e-13, row["why"]


# ------------------------------------------------------------ brute force ---

@pytest.mark.parametrize("seed,lens,Hq,Hkv,D,window,sinks", [
    (0, [37, 91], 4, 2, 16, 0, False),
    (1, [5, 0, 17, 1, 40], 4, 1, 8, 0, True),
    (2, [64, 3, 29], 6, 3, 8, 7, False),
    (3, [50, 50], 2, 2, 12, 1, True),
    (4, [0, 33, 0], 8, 2, 8, 33, True),
    (5, [1, 1, 1], 2, 1, 8, 2, False),
    (6, [70], 4, 4, 8, 16, True),
])
def test_loop_oracle_matches_dense_brute_force(seed, lens, Hq, Hkv, D, window, sinks):
    p = _pack(seed, lens, Hq, Hkv, D, window, sinks=sinks)
    out, lse = _run(p)
    dout, dlse = oracle.dense_attention(p["q"], p["k"], p["v"], p["cu_seqlens"], window,
                                        p["scale"], p["sinks"])
    np.testing.assert_allclose(out, dout, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, dlse, rtol=0, atol=1e-12)


def test_dense_mask_small_case():
    # doc [0,3) and [3,5), window 2: row 2 sees 1,2; row 4 sees 3,4; row 3 sees 3 only.
    m = oracle.dense_mask([0, 3, 5], 2)
    want = np.zeros((5, 5), dtype=bool)
    for i, js in {0: [0], 1: [0, 1], 2: [1, 2], 3: [3], 4: [3, 4]}.items():
        want[i, js] = True
    assert (m == want).all()


# ------------------------------------------------------------ closed forms --

@pytest.mark.parametrize("window,sinks", [(0, False), (0, True), (5, False), (5, True), (1, True)])
def test_zero_query_closed_form(window, sinks):
    """q = 0 => every score is 0: out = sum_{V(i)} v / (|V(i)| + e^sink), lse = ln(|V(i)| + e^sink)."""
    lens = [9, 1, 14]
    p = _pack(11, lens, 4, 2, 8, window, sinks=sinks)
    q0 = torch.zeros_like(p["q"])
    out, lse = _run(p, q=q0)
    v = p["v"].double().numpy()
    cu = p["cu_seqlens"]
    for d in range(len(lens)):
        s, e = int(cu[d]), int(cu[d + 1])
        for i in range(s, e):
            lo = s if window == 0 else max(s, i - window + 1)
            n = i - lo + 1
            for h in range(4):
                extra = math.exp(float(p["sinks"][h])) if sinks else 0.0
                want = v[lo:i + 1, h // 2].sum(axis=0) / (n + extra)
                np.testing.assert_allclose(out[i, h], want, atol=1e-13)
                assert abs(lse[i, h] - math.log(n + extra)) < 1e-13


def test_single_token_document_returns_own_value_row():
    p = _pack(12, [4, 1, 6, 1], 4, 2, 16, 0)
    out, lse = _run(p)
    v = p["v"].double().numpy()
    for t in (4, 11):          # the two 1-token documents
        for h in range(4):
            np.testing.assert_allclose(out[t, h], v[t, h // 2], atol=1e-15)
    # the first token of every document also sees only itself
    for t in (0, 5):
        np.testing.assert_allclose(out[t], v[t, np.arange(4) // 2], atol=1e-15)


def test_window_one_returns_own_value_row():
    p = _pack(13, [20, 7], 4, 1, 8, 1)
    out, _ = _run(p)
    v = p["v"].double().numpy()
    np.testing.assert_allclose(out, np.repeat(v, 4, axis=1), atol=1e-15)


@pytest.mark.parametrize("sinks", [False, True])
def test_constant_value_document_returns_the_constant(sinks):
    p = _pack(14, [30, 12], 4, 2, 8, 0, sinks=sinks)
    c = torch.linspace(-2, 2, 8).to(torch.bfloat16)
    v = c.expand(42, 2, 8).contiguous()
    out, lse = _run(p, v=v)
    cd = c.double().numpy()
    if not sinks:
        np.testing.assert_allclose(out, np.broadcast_to(cd, out.shape), atol=1e-14)
    else:
        s = p["sinks"].double().numpy()
        frac = 1.0 - np.exp(s[None, :] - lse)          # share of Z not taken by the sink
        np.testing.assert_allclose(out, frac[..., None] * cd, atol=1e-13)


# -------------------------------------------------------------- invariants --

def test_window_at_least_doc_length_equals_full_causal():
    p = _pack(15, [17, 40, 3], 4, 2, 8, 0, sinks=True)
    full = _run(p)
    for w in (40, 41, 1000):
        o, l = _run(p, window=w)
        np.testing.assert_array_equal(o, full[0])
        np.testing.assert_array_equal(l, full[1])
    o, _ = _run(p, window=39)
    assert np.abs(o - full[0]).max() > 1e-6          # one shorter window must differ


def test_gqa_equals_mha_on_repeat_kv_expanded_kv():
    p = _pack(16, [25, 31], 8, 2, 8, 6, sinks=True)
    out, lse = _run(p)
    kx = p["k"].repeat_interleave(4, dim=1)
    vx = p["v"].repeat_interleave(4, dim=1)
    out2, lse2 = _run(p, k=kx, v=vx)
    np.testing.assert_array_equal(out, out2)
    np.testing.assert_array_equal(lse, lse2)


def test_very_negative_sink_equals_no_sink():
    p = _pack(17, [19, 23], 4, 2, 8, 0, sinks=True)
    o1, l1 = _run(p, sinks=np.full(4, -1e30, dtype=np.float32))
    o0, l0 = _run(p, sinks=None)
    np.testing.assert_allclose(o1, o0, atol=1e-15)
    np.testing.assert_allclose(l1, l0, atol=1e-15)


def test_document_permutation_invariance():
    lens = [13, 0, 29, 6]
    p = _pack(18, lens, 4, 2, 8, 5, sinks=True)
    out, lse = _run(p)
    cu = p["cu_seqlens"]
    perm = [2, 3, 0, 1]
    idx = np.concatenate([np.arange(cu[d], cu[d + 1]) for d in perm])
    cu2 = workloads.cu_seqlens_from_lengths([lens[d] for d in perm])
    o2, l2 = oracle.attention(p["q"][idx], p["k"][idx], p["v"][idx], cu2, 5, p["scale"], p["sinks"])
    np.testing.assert_array_equal(o2, out[idx])
    np.testing.assert_array_equal(l2, lse[idx])


def test_softmax_weights_and_sink_sum_to_one():
    """sum_{j in V(i)} exp(s_ij - lse) + exp(sink - lse) = 1 on every row."""
    lens = [11, 21]
    p = _pack(19, lens, 4, 2, 8, 4, sinks=True)
    _, lse = _run(p)
    q, k = p["q"].double().numpy(), p["k"].double().numpy()
    s = p["sinks"].double().numpy()
    cu = p["cu_seqlens"]
    for d in range(2):
        for i in range(cu[d], cu[d + 1]):
            lo = max(cu[d], i - 4 + 1)
            for h in range(4):
                sc = p["scale"] * (k[lo:i + 1, h // 2] @ q[i, h])
                tot = np.exp(sc - lse[i, h]).sum() + math.exp(s[h] - lse[i, h])
                assert abs(tot - 1.0) < 1e-13


# ------------------------------------------------- library special cases ----

@pytest.mark.parametrize("window", [0, 9])
def test_single_document_matches_torch_sdpa(window):
    """One document, no sink: torch's fp64 CPU scaled_dot_product_attention."""
    p = _pack(20, [57], 4, 2, 16, window)
    out, lse = _run(p)
    q = p["q"].double().permute(1, 0, 2)[None]
    k = p["k"].double().repeat_interleave(2, dim=1).permute(1, 0, 2)[None]
    v = p["v"].double().repeat_interleave(2, dim=1).permute(1, 0, 2)[None]
    T = 57
    i = torch.arange(T)[:, None]
    j = torch.arange(T)[None, :]
    allowed = (j <= i) & ((i - j < window) if window else torch.ones(T, T, dtype=torch.bool))
    ref = torch.nn.functional.scaled_dot_product_attention(q, k, v, attn_mask=allowed, scale=p["scale"])
    np.testing.assert_allclose(out, ref[0].permute(1, 0, 2).numpy(), atol=1e-12)
    sc = (q @ k.transpose(-1, -2)) * p["scale"]
    ref_lse = torch.logsumexp(sc.masked_fill(~allowed, float("-inf")), dim=-1)[0].T
    np.testing.assert_allclose(lse, ref_lse.numpy(), atol=1e-12)


# ------------------------------------------------------------- row access ---

def test_rows_entry_point_equals_full_forward():
    p = _pack(21, [40, 2, 33], 8, 4, 16, 10, sinks=True)
    out, lse = _run(p)
    rows = np.array([[0, 0], [39, 7], [40, 3], [41, 5], [74, 1], [60, 6]])
    o, l = oracle.attention_rows(p["q"], p["k"], p["v"], p["cu_seqlens"], 10, p["scale"], rows,
                                 p["sinks"])
    np.testing.assert_array_equal(o, out[rows[:, 0], rows[:, 1]])
    np.testing.assert_array_equal(l, lse[rows[:, 0], rows[:, 1]])


def test_valid_pair_count_matches_the_dense_mask():
    for cu, w in [([0, 37, 128], 0), ([0, 5, 5, 90], 7), ([0, 300], 64), ([0, 1, 2], 1)]:
        assert oracle.valid_pairs(cu, w) == int(oracle.dense_mask(cu, w).sum())
    # the tiny pack's count quoted for the benchmark workload table
    assert oracle.valid_pairs([0, 37, 128], 0) == 4889


def test_rejects_invalid_arguments():
    p = _pack(22, [4, 4], 4, 2, 8, 0)
    with pytest.raises(ValueError):
        oracle.attention(p["q"], p["k"], p["v"], [0, 5, 8], -1, 0.5)
    with pytest.raises(ValueError):
        oracle.attention(p["q"], p["k"], p["v"], [1, 5, 8], 0, 0.5)
    with pytest.raises(ValueError):
        oracle.attention(p["q"], p["k"], p["v"], [0, 6, 5, 8], 0, 0.5)
