"""Context-parallel forward on one GPU: every rank's local step
(thd_attn_fwd_range over its token shard, against the whole pack's K/V) is
run one after another, and the shards' outputs together must equal the fp64
oracle (forward tolerances) and the single-launch forward.  The steps do not
wait on each other, so running them in turn on one GPU is exactly what
separate GPUs would compute.  With a single process the cp module's gather
is the identity and cp_attention_fwd is the full forward.  The overlapped
form (each rank's own slice first, the keys before it after the gather,
merged by log-sum-exp) is checked the same way, with its key-bounded step
and its merge on their degenerate cases."""
import numpy as np
import pytest
import torch

import oracle
import sliding_window_gqa_cu_b200 as swa
from sliding_window_gqa_cu_b200 import build, cp, workloads

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build.build()
    swa.load_library()


@pytest.mark.parametrize("lens,Hq,Hkv,D,window,sinks,world", [
    ([390, 5, 128, 1, 200], 8, 2, 128, 0, True, 2),
    ([390, 5, 128, 1, 200], 8, 2, 128, 100, False, 3),
    ([700, 45], 8, 2, 64, 0, True, 4),
    ([520, 3], 16, 1, 256, 0, True, 3),     # CTA-pair kernel
    ([300, 45], 3, 1, 256, 64, True, 2),    # odd group at D = 256
    ([600], 6, 2, 128, 0, False, 5),        # G = 3
])
def test_sharded_forward_equals_the_oracle(lens, Hq, Hkv, D, window, sinks, world):
    p = workloads.random_pack(31, lens, Hq, Hkv, D, window, D ** -0.5, sinks)
    dev = torch.device("cuda:0")
    q, k, v = (p[n].to(dev) for n in "qkv")
    s = p["sinks"].to(dev) if sinks else None
    T = int(p["T"])
    outs, lses = [], []
    for b, e in cp.shard_bounds(T, world):
        o, l = swa.thd_attn_fwd_range(q[b:e].contiguous(), k, v, p["cu_seqlens"], b, e, window,
                                      p["scale"], s)
        outs.append(o)
        lses.append(l)
    out, lse = torch.cat(outs), torch.cat(lses)
    torch.cuda.synchronize()
    assert swa.thd_attn_get_error() == 0
    ref_o, ref_l = oracle.attention(p["q"], p["k"], p["v"], p["cu_seqlens"], window, p["scale"],
                                    p["sinks"])
    o = out.cpu().double().numpy()
    assert np.abs(o - ref_o).max() <= 2e-2 and np.abs(o - ref_o).mean() <= 2e-3
    assert np.abs(lse.cpu().double().numpy() - ref_l).max() <= 1e-3
    full_o, full_l = swa.thd_attn_fwd(q, k, v, p["cu_seqlens"], window, p["scale"], s)
    assert (full_o.float() - out.float()).abs().max() <= 1.6e-2
    assert (full_l - lse).abs().max() <= 1e-3


def test_single_process_cp_is_the_forward():
    p = workloads.random_pack(32, [400, 77], 8, 2, 128, 0, 128 ** -0.5, True)
    dev = torch.device("cuda:0")
    q, k, v = (p[n].to(dev) for n in "qkv")
    s = p["sinks"].to(dev)
    a, la = cp.cp_attention_fwd(q, k, v, p["cu_seqlens"], 0, p["scale"], s)
    b, lb = swa.thd_attn_fwd(q, k, v, p["cu_seqlens"], 0, p["scale"], s)
    assert torch.equal(a, b) and torch.equal(la, lb)


@pytest.mark.parametrize("lens,Hq,Hkv,D,window,sinks,world", [
    ([390, 5, 128, 1, 200], 16, 4, 128, 0, True, 4),    # whole kv groups per rank
    ([390, 5, 128, 1, 200], 16, 4, 128, 0, True, 2),
    ([520, 3], 16, 1, 256, 300, True, 8),              # MQA: query heads split, K/V replicated
    ([700, 45], 8, 2, 64, 0, False, 4),
])
def test_head_sharded_forward_equals_the_oracle(lens, Hq, Hkv, D, window, sinks, world):
    """Every rank's head slice (cp.head_shard) run in turn on one GPU: the
    slices side by side equal the oracle and, bit for bit, the whole-pack
    forward (each row is computed the same way whichever heads share it)."""
    p = workloads.random_pack(33, lens, Hq, Hkv, D, window, D ** -0.5, sinks)
    dev = torch.device("cuda:0")
    q, k, v = (p[n].to(dev) for n in "qkv")
    s = p["sinks"].to(dev) if sinks else None
    outs, lses = [], []
    for r in range(world):
        q_lo, q_hi, kv_lo, kv_hi = cp.head_shard(Hq, Hkv, world, r)
        o, l = cp.head_sharded_attention_fwd(q[:, q_lo:q_hi].contiguous(), k[:, kv_lo:kv_hi].contiguous(),
                                             v[:, kv_lo:kv_hi].contiguous(), p["cu_seqlens"], window,
                                             p["scale"], s[q_lo:q_hi].contiguous() if sinks else None)
        outs.append(o)
        lses.append(l)
    out, lse = torch.cat(outs, 1), torch.cat(lses, 1)
    torch.cuda.synchronize()
    assert swa.thd_attn_get_error() == 0
    ref_o, ref_l = oracle.attention(p["q"], p["k"], p["v"], p["cu_seqlens"], window, p["scale"],
                                    p["sinks"])
    o = out.cpu().double().numpy()
    assert np.abs(o - ref_o).max() <= 2e-2 and np.abs(o - ref_o).mean() <= 2e-3
    assert np.abs(lse.cpu().double().numpy() - ref_l).max() <= 1e-3
    full_o, full_l = swa.thd_attn_fwd(q, k, v, p["cu_seqlens"], window, p["scale"], s)
    assert (full_o.float() - out.float()).abs().max() <= 1.6e-2
    assert (full_l - lse).abs().max() <= 1e-3


@pytest.mark.parametrize("lens,Hq,Hkv,D,window,sinks,world", [
    ([390, 5, 128, 1, 200], 8, 2, 128, 0, True, 2),
    ([390, 5, 128, 1, 200], 8, 2, 128, 100, False, 3),
    ([390, 5, 128, 1, 200], 8, 2, 128, 30, True, 4),   # windows shorter than a shard
    ([700, 45], 8, 2, 64, 0, True, 4),
    ([520, 3], 16, 1, 256, 0, True, 3),     # CTA-pair kernel
    ([300, 45], 3, 1, 256, 64, True, 2),    # odd group at D = 256
    ([600], 6, 2, 128, 0, False, 5),        # G = 3
    ([256, 256], 8, 2, 128, 0, True, 2),    # shard boundary on a document start
    ([5], 4, 2, 128, 0, True, 7),           # empty shards
])
def test_overlapped_parts_equal_the_oracle(lens, Hq, Hkv, D, window, sinks, world):
    """Each rank's rows from their two key parts (the rank's slice as a pack
    of its own, then the crossing document's rows against the keys before
    the slice, merged by log-sum-exp), ranks run in turn on one GPU with the
    whole pack standing in for the gathered K/V: the fp64 oracle within the
    forward tolerances, and the single-launch forward within bf16 rounding
    of the merge."""
    p = workloads.random_pack(33, lens, Hq, Hkv, D, window, D ** -0.5, sinks)
    dev = torch.device("cuda:0")
    q, k, v = (p[n].to(dev) for n in "qkv")
    s = p["sinks"].to(dev) if sinks else None
    T = int(p["T"])
    outs, lses = [], []
    for b, e in cp.shard_bounds(T, world):
        o, l = cp.cp_rank_parts(q[b:e].contiguous(), k[b:e].contiguous(), v[b:e].contiguous(),
                                p["cu_seqlens"], b, e, window, p["scale"], s, kv_before=lambda: (k, v))
        outs.append(o)
        lses.append(l)
    out, lse = torch.cat(outs), torch.cat(lses)
    torch.cuda.synchronize()
    assert swa.thd_attn_get_error() == 0
    ref_o, ref_l = oracle.attention(p["q"], p["k"], p["v"], p["cu_seqlens"], window, p["scale"],
                                    p["sinks"])
    o = out.cpu().double().numpy()
    assert np.abs(o - ref_o).max() <= 2e-2 and np.abs(o - ref_o).mean() <= 2e-3
    assert np.abs(lse.cpu().double().numpy() - ref_l).max() <= 1e-3
    full_o, full_l = swa.thd_attn_fwd(q, k, v, p["cu_seqlens"], window, p["scale"], s)
    assert (full_o.float() - out.float()).abs().max() <= 1.6e-2
    assert (full_l - lse).abs().max() <= 1e-3


def test_key_bounded_rows_without_keys():
    """Rows whose window holds no key before k_end: out 0 and lse -inf
    (exactly); with a sink, lse is the sink logit."""
    lens, W, b = [400], 16, 200
    p = workloads.random_pack(34, lens, 8, 2, 128, W, 128 ** -0.5, True)
    dev = torch.device("cuda:0")
    q, k, v = (p[n].to(dev) for n in "qkv")
    o, l = swa.thd_attn_fwd_range(q[b:].contiguous(), k, v, p["cu_seqlens"], b, 400, W, p["scale"],
                                  None, k_end=b)
    torch.cuda.synchronize()
    assert swa.thd_attn_get_error() == 0
    far = slice(W - 1, None)  # rows b + W - 1 and on see no key before b
    assert torch.all(o[far] == 0) and torch.all(torch.isneginf(l[far]))
    assert torch.all(torch.isfinite(l[:W - 1]))
    s = p["sinks"].to(dev)
    _, ls = swa.thd_attn_fwd_range(q[b:].contiguous(), k, v, p["cu_seqlens"], b, 400, W, p["scale"],
                                   s, k_end=b)
    torch.cuda.synchronize()
    assert torch.allclose(ls[far], s.expand_as(ls[far]), rtol=0, atol=1e-5)


def test_merge_degenerate_parts_are_exact():
    """Merging with a part of lse -inf returns the other part bit for bit;
    merging a part with itself keeps out and adds log 2 to lse."""
    g = torch.Generator().manual_seed(35)
    dev = torch.device("cuda:0")
    a = torch.randn((77, 4, 128), generator=g).to(torch.bfloat16).to(dev)
    la = torch.randn((77, 4), generator=g).to(dev)
    z = torch.zeros_like(a)
    ninf = torch.full_like(la, float("-inf"))
    o, l = swa.thd_attn_merge(a, la, z, ninf)
    assert torch.equal(o, a) and torch.equal(l, la)
    o, l = swa.thd_attn_merge(z, ninf, a, la)
    assert torch.equal(o, a) and torch.equal(l, la)
    o, l = swa.thd_attn_merge(a, la, a, la)
    assert torch.equal(o, a) and torch.allclose(l, la + float(np.log(2.0)), rtol=0, atol=1e-6)
    o, l = swa.thd_attn_merge(z, ninf, z, ninf)
    assert torch.equal(o, z) and torch.all(torch.isneginf(l))
    # in place
    a2, la2 = a.clone(), la.clone()
    swa.thd_attn_merge(a2, la2, z, ninf, out=a2, lse=la2)
    assert torch.equal(a2, a) and torch.equal(la2, la)


def test_single_process_overlapped_cp_is_the_forward():
    p = workloads.random_pack(36, [400, 77], 8, 2, 128, 0, 128 ** -0.5, True)
    dev = torch.device("cuda:0")
    q, k, v = (p[n].to(dev) for n in "qkv")
    s = p["sinks"].to(dev)
    o, l = cp.cp_attention_fwd_overlapped(q, k, v, p["cu_seqlens"], 0, p["scale"], s)
    fo, fl = swa.thd_attn_fwd(q, k, v, p["cu_seqlens"], 0, p["scale"], s)
    torch.cuda.synchronize()
    assert torch.equal(o, fo) and torch.equal(l, fl)
