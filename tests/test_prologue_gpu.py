"""GPU parity of the Q/K prologue (scaleless RMSNorm, then split-half RoPE,
"muse_glimmer.model" page) against the fp64 oracle.

Tolerance: the kernel computes in fp32 (angles reduced in double) and rounds
once to bf16, so every element is within one bf16 rounding (2^-9 relative)
plus fp32 error of order 1e-6 of the unit-RMS row: |gpu - ref| <=
2^-8 |ref| + 1e-5.
"""
import numpy as np
import pytest
import torch

import oracle
from oracle import prologue as OP
import sliding_window_gqa_cu_b200 as swa
from sliding_window_gqa_cu_b200 import build, workloads

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build.build()
    swa.load_library()


def check(got, ref, what):
    g = got.float().double().cpu().numpy()
    err = np.abs(g - ref)
    bound = 2.0 ** -8 * np.abs(ref) + 1e-5
    assert np.isfinite(g).all(), what
    assert (err <= bound).all(), f"{what}: worst excess {(err - bound).max():.3e}"


@pytest.mark.parametrize("lens,Hq,Hkv,D,rope", [
    ([300, 1, 0, 129, 77], 4, 2, 64, True),
    ([300, 1, 0, 129, 77], 4, 2, 64, False),
    ([390, 5, 128, 1, 200], 8, 2, 128, True),
    ([600], 4, 4, 256, True),
    ([520, 3], 16, 1, 128, True),
])
def test_prologue_parity(lens, Hq, Hkv, D, rope):
    p = workloads.random_pack(21, lens, Hq, Hkv, D, 0, D ** -0.5, False)
    dev = torch.device("cuda:0")
    q, k = p["q"].to(dev), p["k"].to(dev)
    swa.thd_qk_norm_rope(q, k, p["cu_seqlens"], apply_rope=rope)
    torch.cuda.synchronize()
    check(q, OP.qk_norm_rope(p["q"], p["cu_seqlens"], apply_rope=rope), "q")
    check(k, OP.qk_norm_rope(p["k"], p["cu_seqlens"], apply_rope=rope), "k")


def test_prologue_explicit_large_positions():
    p = workloads.random_pack(22, [500], 4, 2, 128, 0, 128 ** -0.5, False)
    pos = np.random.default_rng(3).integers(0, 1 << 20, size=500).astype(np.int32)
    dev = torch.device("cuda:0")
    q, k = p["q"].to(dev), p["k"].to(dev)
    swa.thd_qk_norm_rope(q, k, p["cu_seqlens"], positions=torch.from_numpy(pos).to(dev))
    torch.cuda.synchronize()
    check(q, OP.qk_norm_rope(p["q"], p["cu_seqlens"], positions=pos), "q")
    check(k, OP.qk_norm_rope(p["k"], p["cu_seqlens"], positions=pos), "k")


def test_prologue_full_size_pack_sampled_tokens():
    cfg = workloads.CONFIGS["pack64k_gqa8_d128_causal_sink"]
    p = workloads.make_pack(cfg, 0)
    dev = torch.device("cuda:0")
    q, k = p["q"].to(dev), p["k"].to(dev)
    swa.thd_qk_norm_rope(q, k, p["cu_seqlens"])
    torch.cuda.synchronize()
    cu = np.asarray(p["cu_seqlens"])
    rows = set(int(x) for x in np.random.default_rng(4).integers(0, cu[-1], 1500))
    rows |= {int(c) for c in cu[:-1]} | {int(c) - 1 for c in cu[1:]}
    rows = np.array(sorted(r for r in rows if 0 <= r < cu[-1]))
    pos = OP.doc_positions(cu)[rows]
    check(q[rows], OP.qk_norm_rope(p["q"][rows], None, positions=pos), "q")
    check(k[rows], OP.qk_norm_rope(p["k"][rows], None, positions=pos), "k")


def test_prologue_then_attention_matches_the_oracle_chain():
    p = workloads.random_pack(23, [400, 90], 8, 2, 128, 0, 128 ** -0.5, True)
    dev = torch.device("cuda:0")
    q, k, v = (p[n].to(dev) for n in "qkv")
    swa.thd_qk_norm_rope(q, k, p["cu_seqlens"])
    out, lse = swa.thd_attn_fwd(q, k, v, p["cu_seqlens"], 0, p["scale"], p["sinks"].to(dev))
    torch.cuda.synchronize()
    # oracle chain: prologue in fp64, rounded to bf16 like the tensors the
    # attention reads, then the attention oracle
    qo = torch.from_numpy(OP.qk_norm_rope(p["q"], p["cu_seqlens"])).to(torch.bfloat16)
    ko = torch.from_numpy(OP.qk_norm_rope(p["k"], p["cu_seqlens"])).to(torch.bfloat16)
    ref_out, ref_lse = oracle.attention(qo, ko, p["v"], p["cu_seqlens"], 0, p["scale"], p["sinks"])
    o = out.cpu().double().numpy()
    assert np.abs(o - ref_out).max() <= 2e-2 and np.abs(o - ref_out).mean() <= 2e-3
    assert np.abs(lse.cpu().double().numpy() - ref_lse).max() <= 1e-3
