"""Every row of the two largest benchmark packs against the full fp64 oracle.

These runs take about 15 minutes of host CPU per pack on a 16-thread host, so
they are opt-in: ``python -m pytest tests/test_full_oracle_gpu.py
--full-oracle -s``.  They are not marked ``gpu`` (a plain ``-m gpu`` run
leaves them out); the default GPU suite checks the same packs on a dense
subset of rows.  Each test prints its maximum and mean output error and its
maximum log-sum-exp error.

Definition: FlintMagiPlan.attention ("flint.magi" page: window, sink) on
MuseMagiPlan.attention's packed THD tensors ("muse_spark.magi_cp" page).
"""
import json
import time

import numpy as np
import pytest
import torch

import oracle
import sliding_window_gqa_cu_b200 as swa
from sliding_window_gqa_cu_b200 import build, workloads

OUT_MAX, OUT_MEAN, LSE_MAX = 2e-2, 2e-3, 1e-3
REL_MAX, REL_MEAN = 2e-2, 2e-3

pytestmark = pytest.mark.full_oracle


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build.build()
    swa.load_library()


@pytest.mark.parametrize("name", ["pack64k_gqa8_d128_causal_sink", "doc128k_mqa_d256_w8192_sink"])
def test_full_size_pack_every_row_full_oracle(name):
    cfg = workloads.CONFIGS[name]
    p = workloads.make_pack(cfg, 0)
    dev = torch.device("cuda:0")
    q, k, v = (p[n].to(dev) for n in "qkv")
    sinks = p["sinks"].to(dev) if p["sinks"] is not None else None
    out, lse = swa.thd_attn_fwd(q, k, v, p["cu_seqlens"], cfg.window, cfg.scale, sinks)
    assert swa.thd_attn_get_error() == 0
    out, lse = out.cpu(), lse.cpu()
    del q, k, v
    t0 = time.time()
    ref_o, ref_l = oracle.attention(p["q"], p["k"], p["v"], p["cu_seqlens"], cfg.window,
                                    cfg.scale, p["sinks"])
    secs = time.time() - t0
    err = np.abs(out.double().numpy() - ref_o)
    lerr = np.abs(lse.double().numpy() - ref_l)
    rec = {"workload": name, "rows": int(ref_l.size), "out_max_abs": float(err.max()),
           "out_mean_abs": float(err.mean()), "lse_max_abs": float(lerr.max()),
           "oracle_seconds": round(secs, 1), "oracle_threads": oracle.num_threads()}
    print("FULL_ORACLE " + json.dumps(rec), flush=True)
    assert np.isfinite(out.float().numpy()).all()
    assert err.max() <= OUT_MAX and err.mean() <= OUT_MEAN and lerr.max() <= LSE_MAX


@pytest.mark.parametrize("name", ["pack8k_gqa4_d128_causal", "pack32k_gqa4_d128_w4096"])
def test_full_size_pack_bwd_every_element_full_oracle(name):
    """dq, dk and dv of the 8k and 32k packs on every element against the
    full fp64 backward oracle (the derivative of the same definition), with
    the backward tolerances: max error 2e-2 and mean error 2e-3 of max|ref|
    per tensor.  The default GPU suite checks these packs' gradients on
    sampled rows."""
    cfg = workloads.CONFIGS[name]
    p = workloads.make_pack(cfg, 0)
    dev = torch.device("cuda:0")
    g = torch.Generator().manual_seed(5)
    dout = torch.randn(p["q"].shape, generator=g).to(torch.bfloat16)
    q, k, v = (p[n].to(dev) for n in "qkv")
    sinks = p["sinks"].to(dev) if p["sinks"] is not None else None
    out, lse = swa.thd_attn_fwd(q, k, v, p["cu_seqlens"], cfg.window, cfg.scale, sinks)
    dq, dk, dv, ds = swa.thd_attn_bwd(q, k, v, out, lse, dout.to(dev), p["cu_seqlens"], cfg.window,
                                      cfg.scale, sinks)
    torch.cuda.synchronize()
    assert swa.thd_attn_get_error() == 0
    got = {"dq": dq.cpu(), "dk": dk.cpu(), "dv": dv.cpu()}
    del q, k, v, out, lse, dq, dk, dv
    t0 = time.time()
    rq, rk, rv, rs = oracle.attention_bwd(p["q"], p["k"], p["v"], dout, p["cu_seqlens"], cfg.window,
                                          cfg.scale, p["sinks"])
    secs = time.time() - t0
    rec = {"workload": name, "oracle_seconds": round(secs, 1), "oracle_threads": oracle.num_threads()}
    ok = True
    for key, ref in (("dq", rq), ("dk", rk), ("dv", rv)):
        gv = got[key].double().numpy().reshape(ref.shape)
        scale = max(float(np.abs(ref).max()), 1e-3)
        err = np.abs(gv - ref)
        rec[key] = {"max_abs": float(err.max()), "mean_abs": float(err.mean()), "max_ref": scale}
        ok = ok and np.isfinite(gv).all() and err.max() <= REL_MAX * scale and err.mean() <= REL_MEAN * scale
    print("FULL_ORACLE_BWD " + json.dumps(rec), flush=True)
    assert ok, rec
