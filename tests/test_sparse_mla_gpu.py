"""GPU parity of sparse MLA ("mistral_large4.attention" page, sparse_mla)
against the fp64 oracle.

Tolerance: the kernel rounds P and the latent to bf16 (2^-9 each) and the
output once more; the attention forward's bounds are applied relative to the
output's largest magnitude: max |err| <= 2e-2 max|ref|, mean |err| <=
2e-3 max|ref|.  Rows without a valid slot must be exactly zero.
"""
import numpy as np
import pytest
import torch

from oracle import sparse_mla as SM
import sliding_window_gqa_cu_b200 as swa
from sliding_window_gqa_cu_b200 import build, workloads

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build.build()
    swa.load_library()


def run(c):
    dev = torch.device("cuda:0")
    out = swa.thd_sparse_mla_fwd(c["q"].to(dev), c["kv"].to(dev), c["indices"].to(dev),
                                 c["value_weight"].to(dev), c["scale"])
    torch.cuda.synchronize()
    assert swa.thd_sparse_mla_get_error() == 0
    return out.cpu()


def check(got, ref, what):
    g = got.double().numpy()
    scale = np.abs(ref).max()
    err = np.abs(g - ref)
    assert np.isfinite(g).all(), what
    assert err.max() <= 2e-2 * scale, f"{what}: max err {err.max():.3e} vs {scale:.3e}"
    assert err.mean() <= 2e-3 * scale, f"{what}: mean err {err.mean():.3e} vs {scale:.3e}"


@pytest.mark.parametrize("lens,H,K,vd", [
    ([150, 40], 128, 64, 128),      # one slot chunk
    ([300, 1, 77], 128, 192, 64),   # three chunks, a one-token document
    ([260], 256, 128, 256),         # two head groups, widest value head
    ([500, 20], 128, 512, 128),     # many chunks, partly empty
])
def test_sparse_mla_parity(lens, H, K, vd):
    c = workloads.sparse_mla_case(41, lens, H, K, vd)
    got = run(c)
    ref = SM.sparse_mla(c["q"], c["kv"], c["indices"], c["value_weight"], c["scale"])
    check(got, ref, f"{lens} H{H} K{K} vd{vd}")


def test_empty_rows_are_zero_and_out_of_range_slots_are_ignored():
    c = workloads.sparse_mla_case(42, [200], 128, 128, 128)
    idx = c["indices"].clone()
    idx[5] = -1                          # no valid slot
    idx[7, 3] = 10 ** 6                  # out of range: ignored like -1
    c["indices"] = idx
    got = run(c)
    assert got[5].float().abs().max() == 0
    ref_idx = idx.clone()
    ref_idx[7, 3] = -1
    ref = SM.sparse_mla(c["q"], c["kv"], ref_idx, c["value_weight"], c["scale"])
    check(got, ref, "masked")


def test_full_size_sampled_tokens():
    c = workloads.sparse_mla_case(0, [4096], 128, 2048, 128)
    got = run(c)
    rows = np.unique(np.concatenate([np.random.default_rng(5).integers(0, 4096, 48), [0, 1, 2047, 4095]]))
    ref = SM.sparse_mla(c["q"][rows], c["kv"], c["indices"][rows], c["value_weight"], c["scale"])
    check(got[rows], ref, "full size")
