"""The stall detector on the GPU, without a fault: a bounded wait on a
barrier that nothing signals gives up after its limit and records the timeout
status, a block waiting at the same time gives up early on seeing it, the
host reads and clears the status, and the context stays usable."""
import numpy as np
import pytest
import torch

import oracle
import sliding_window_gqa_cu_b200 as swa
from sliding_window_gqa_cu_b200 import build, workloads

pytestmark = pytest.mark.gpu

WAIT_LIMIT_NS = 2_000_000_000  # the kernels' wait limit
TIMEOUT = -4                   # THD_ERR_TIMEOUT


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build.build()
    swa.load_library()


def test_bounded_wait_times_out_and_the_context_survives():
    torch.zeros(1, device="cuda:0")
    assert swa.thd_attn_get_error() == 0
    waited0, waited1 = swa.thd_attn_selftest_stall()
    assert WAIT_LIMIT_NS <= waited0 < 2 * WAIT_LIMIT_NS      # gave up at its limit
    assert 0 < waited1 < WAIT_LIMIT_NS                        # gave up on the recorded status
    assert swa.thd_attn_get_error() == TIMEOUT               # read once ...
    assert swa.thd_attn_get_error() == 0                     # ... then cleared
    p = workloads.random_pack(3, [200, 1, 77], 8, 2, 128, 64, 128 ** -0.5, True)
    dev = torch.device("cuda:0")
    out, lse = swa.thd_attn_fwd(p["q"].to(dev), p["k"].to(dev), p["v"].to(dev), p["cu_seqlens"],
                                p["window"], p["scale"], p["sinks"].to(dev))
    assert swa.thd_attn_get_error() == 0
    ref_o, ref_l = oracle.attention(p["q"], p["k"], p["v"], p["cu_seqlens"], p["window"], p["scale"],
                                    p["sinks"])
    assert np.abs(out.cpu().double().numpy() - ref_o).max() <= 2e-2
    assert np.abs(lse.cpu().double().numpy() - ref_l).max() <= 1e-3
