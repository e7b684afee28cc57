"""Context-parallel forward on one GPU: every rank's local step
(thd_attn_fwd_range over its token shard, against the whole pack's K/V) is
run one after another, and the shards' outputs together must equal the fp64
oracle (forward tolerances) and the single-launch forward.  The steps do not
wait on each other, so running them in turn on one GPU is exactly what
separate GPUs would compute.  With a single process the cp module's gather
is the identity and cp_attention_fwd is the full forward."""
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
