"""Pins for the oracle's backward (dq, dk, dv, dsink), checked against things
other than its own formula:

* central finite differences of the (separately pinned) forward oracle, on
  tiny packs, for every input element and every sink;
* PyTorch's scaled_dot_product_attention autograd in fp64 on one document
  (repeat_kv-expanded K/V, so the kv-head gradients are sums over the group);
* exact invariants: without a sink, softmax is shift invariant, so the key
  gradients of a (document, kv head) sum to zero; the value gradients of a
  document sum to the sum over its queries of (1 - sink share) * dO;
* special cases: single-token documents, and the sampled-row entry point.

The backward is the derivative of the forward of FlintMagiPlan.attention
("flint.magi" page: window, sink) over MuseMagiPlan.attention's packed THD
tensors ("muse_spark.magi_cp" page), with repeat_kv's GQA mapping
("muse_glimmer.model" page).
"""
import numpy as np
import pytest
import torch

import oracle
from sliding_window_gqa_cu_b200 import workloads


def _f64_pack(seed, lens, Hq, Hkv, D, window, sinks):
    p = workloads.random_pack(seed, lens, Hq, Hkv, D, window, D ** -0.5, sinks)
    q, k, v = (p[n].double().numpy() for n in "qkv")
    s = p["sinks"].numpy().astype(np.float32) if p["sinks"] is not None else None
    dout = np.random.default_rng(seed + 100).standard_normal(q.shape)
    return p, q, k, v, s, dout


def _loss(q, k, v, s, dout, cu, window, scale):
    out, _ = oracle.attention(q, k, v, cu, window, scale, s)
    return float((out * dout).sum())


@pytest.mark.parametrize("lens,Hq,Hkv,window,sinks", [
    ([5, 0, 7, 1], 4, 2, 0, True),
    ([5, 0, 7, 1], 4, 2, 3, False),
    ([9, 4], 3, 1, 2, True),
])
def test_backward_matches_finite_differences(lens, Hq, Hkv, window, sinks):
    D = 4
    p, q, k, v, s, dout = _f64_pack(3, lens, Hq, Hkv, D, window, sinks)
    cu, scale = p["cu_seqlens"], p["scale"]
    dq, dk, dv, ds = oracle.attention_bwd(q, k, v, dout, cu, window, scale, s)
    h = 1e-5
    for name, x, g in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
        fd = np.zeros_like(x)
        for idx in np.ndindex(x.shape):
            xp, xm = x.copy(), x.copy()
            xp[idx] += h
            xm[idx] -= h
            args = {"q": q, "k": k, "v": v}
            args[name] = xp
            fp = _loss(args["q"], args["k"], args["v"], s, dout, cu, window, scale)
            args[name] = xm
            fm = _loss(args["q"], args["k"], args["v"], s, dout, cu, window, scale)
            fd[idx] = (fp - fm) / (2 * h)
        assert np.abs(fd - g).max() <= 1e-6 * max(1.0, np.abs(g).max()), name
    if sinks:
        for hh in range(Hq):
            sp, sm = s.copy(), s.copy()
            sp[hh] = np.float32(s[hh] + np.float32(1e-2))
            sm[hh] = np.float32(s[hh] - np.float32(1e-2))
            fd = (_loss(q, k, v, sp, dout, cu, window, scale) -
                  _loss(q, k, v, sm, dout, cu, window, scale)) / (float(sp[hh]) - float(sm[hh]))
            # central difference: error O(h^2) with h = 1e-2
            assert abs(fd - ds[hh]) <= 2e-4 * max(1.0, abs(ds[hh])), hh
    else:
        assert ds is None


@pytest.mark.parametrize("window", [0, 5])
def test_backward_matches_torch_sdpa_autograd(window):
    T, Hq, Hkv, D = 23, 4, 2, 16
    p, q, k, v, _, dout = _f64_pack(5, [T], Hq, Hkv, D, window, False)
    dq, dk, dv, _ = oracle.attention_bwd(q, k, v, dout, p["cu_seqlens"], window, p["scale"])
    qt = torch.tensor(q).permute(1, 0, 2).requires_grad_()          # [Hq, T, D]
    kt = torch.tensor(k).permute(1, 0, 2).requires_grad_()
    vt = torch.tensor(v).permute(1, 0, 2).requires_grad_()
    kx = kt.repeat_interleave(Hq // Hkv, 0)
    vx = vt.repeat_interleave(Hq // Hkv, 0)
    mask = torch.tensor(oracle.dense_mask(p["cu_seqlens"], window))
    out = torch.nn.functional.scaled_dot_product_attention(qt, kx, vx, attn_mask=mask,
                                                           scale=p["scale"])
    out.backward(torch.tensor(dout).permute(1, 0, 2))
    assert np.allclose(qt.grad.permute(1, 0, 2).numpy(), dq, atol=1e-10)
    assert np.allclose(kt.grad.permute(1, 0, 2).numpy(), dk, atol=1e-10)
    assert np.allclose(vt.grad.permute(1, 0, 2).numpy(), dv, atol=1e-10)


@pytest.mark.parametrize("sinks", [False, True])
def test_backward_invariants(sinks):
    lens = [40, 1, 0, 33, 60]
    Hq, Hkv, D, window = 6, 2, 8, 9
    p, q, k, v, s, dout = _f64_pack(7, lens, Hq, Hkv, D, window, sinks)
    cu = np.asarray(p["cu_seqlens"])
    dq, dk, dv, ds = oracle.attention_bwd(q, k, v, dout, cu, window, p["scale"], s)
    _, lse = oracle.attention(q, k, v, cu, window, p["scale"], s)
    G = Hq // Hkv
    for d in range(len(lens)):
        a, b = int(cu[d]), int(cu[d + 1])
        if a == b:
            continue
        for g in range(Hkv):
            heads = range(g * G, (g + 1) * G)
            share = np.zeros((b - a, G))
            if sinks:
                share = np.exp(s[list(heads)][None, :].astype(np.float64) - lse[a:b, list(heads)])
            want_dv = sum(((1 - share[:, n])[:, None] * dout[a:b, h]).sum(0) for n, h in enumerate(heads))
            assert np.allclose(dv[a:b, g].sum(0), want_dv, atol=1e-10)
            if not sinks:
                assert np.abs(dk[a:b, g].sum(0)).max() <= 1e-10


def test_single_token_documents():
    lens = [1, 1, 1, 1]
    p, q, k, v, _, dout = _f64_pack(8, lens, 4, 2, 8, 0, False)
    dq, dk, dv, _ = oracle.attention_bwd(q, k, v, dout, p["cu_seqlens"], 0, p["scale"])
    assert np.abs(dq).max() == 0 and np.abs(dk).max() == 0
    assert np.allclose(dv, dout.reshape(4, 2, 2, 8).sum(2))


def test_q_rows_entry_point_equals_full_backward():
    p, q, k, v, s, dout = _f64_pack(9, [50, 7, 30], 4, 2, 8, 6, True)
    dq, _, _, _ = oracle.attention_bwd(q, k, v, dout, p["cu_seqlens"], 6, p["scale"], s)
    rows = np.array([[0, 0], [49, 3], [50, 1], [56, 2], [86, 0], [60, 3]])
    got = oracle.attention_bwd_q_rows(q, k, v, dout, p["cu_seqlens"], 6, p["scale"], rows, s)
    assert np.allclose(got, dq[rows[:, 0], rows[:, 1]], atol=1e-13)


@pytest.mark.parametrize("lens,Hq,Hkv,window,sinks", [
    ([37, 0, 91, 1, 20], 4, 2, 0, True),
    ([37, 0, 91, 1, 20], 6, 2, 9, False),
    ([60, 33], 3, 3, 5, True),      # MHA
    ([80], 4, 1, 0, False),         # MQA
])
def test_kv_rows_entry_point_equals_full_backward(lens, Hq, Hkv, window, sinks):
    # Every (key token, kv head) row of small packs, with and without a window
    # or sink, equals the full backward's dk and dv (same derivative, summed
    # over the queries that see the key instead of scattered from each query).
    p, q, k, v, s, dout = _f64_pack(31, lens, Hq, Hkv, 16, window, sinks)
    _, rk, rv, _ = oracle.attention_bwd(q, k, v, dout, p["cu_seqlens"], window, p["scale"], s)
    T = q.shape[0]
    rows = np.array([(j, g) for j in range(T) for g in range(Hkv)], dtype=np.int64)
    dk, dv = oracle.attention_bwd_kv_rows(q, k, v, dout, p["cu_seqlens"], window, p["scale"], rows, s)
    assert np.abs(dk - rk[rows[:, 0], rows[:, 1]]).max() <= 1e-12
    assert np.abs(dv - rv[rows[:, 0], rows[:, 1]]).max() <= 1e-12
    # a shuffled subset in any order gives the same rows
    sub = rows[np.random.default_rng(0).permutation(len(rows))[:11]]
    dk2, dv2 = oracle.attention_bwd_kv_rows(q, k, v, dout, p["cu_seqlens"], window, p["scale"], sub, s)
    assert np.abs(dk2 - rk[sub[:, 0], sub[:, 1]]).max() <= 1e-12
    assert np.abs(dv2 - rv[sub[:, 0], sub[:, 1]]).max() <= 1e-12


@pytest.mark.parametrize("window", [0, 7])
def test_dsink_from_forward_equals_full_backward(window):
    p, q, k, v, s, dout = _f64_pack(32, [40, 3, 70], 6, 2, 16, window, True)
    _, _, _, rs = oracle.attention_bwd(q, k, v, dout, p["cu_seqlens"], window, p["scale"], s)
    got = oracle.attention_dsink(q, k, v, dout, p["cu_seqlens"], window, p["scale"], s)
    assert np.abs(got - rs).max() <= 1e-12 * max(1.0, np.abs(rs).max())


def test_kv_rows_rejects_out_of_range_rows():
    p, q, k, v, s, dout = _f64_pack(33, [10], 2, 1, 16, 0, False)
    with pytest.raises(ValueError):
        oracle.attention_bwd_kv_rows(q, k, v, dout, p["cu_seqlens"], 0, p["scale"],
                                     np.array([[0, 1]]), s)   # kv head 1 of 1
