"""Planted mistakes in a copy of the CPU oracle must be caught by its pins.

Each mutant is a one-line textual change to a temporary copy of the oracle's
C source (a dropped term, a wrong index, a wrong sign or bound).  The pins
(hand-worked examples and the dense brute force) are run against the mutant,
and at least one of them must fail.  The real oracle source is never touched.
"""
import json
import math
import os

import numpy as np
import pytest

import oracle
from sliding_window_gqa_cu_b200 import workloads

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "hand_examples.json")

MUTANTS = {
    "window_off_by_one": ("lo = i - window + 1;", "lo = i - window;"),
    "gqa_modulo_map": ("const int g = h / G;", "const int g = h % Hkv;"),
    "sink_dropped_from_Z": ("double Z = has_sink ? exp(sink - m) : 0.0;", "double Z = 0.0;"),
    "scale_dropped": ("sc[j - lo] = scale * acc;", "sc[j - lo] = acc;"),
    "key_index_uses_query_token": ("load_elem(k, (j * Hkv + g)", "load_elem(k, (i * Hkv + g)"),
    "document_start_ignored": ("int64_t lo = s;", "int64_t lo = 0;"),
    "lse_without_max_shift": ("*lse_out = m + log(Z);", "*lse_out = log(Z);"),
    "value_head_modulo": ("load_elem(v, (j * Hkv + g)", "load_elem(v, (j * Hkv + h % Hkv)"),
    "sink_scaled_like_scores": ("(double)sinks[h] : -INFINITY;", "scale * (double)sinks[h] : -INFINITY;"),
}


def _pins_fail(lib) -> list[str]:
    failures = []
    env = {"e": math.e, "log": math.log}
    with open(GOLDEN) as f:
        cases = json.load(f)["cases"]
    for case in cases:
        q, k, v = (np.asarray(case[n], dtype=np.float64) for n in "qkv")
        try:
            out, lse = oracle.attention(q, k, v, case["cu_seqlens"], case["window"], case["scale"],
                                        case["sinks"], lib=lib)
        except ValueError:
            failures.append(case["name"])
            continue
        for row in case["expected"]:
            want = [eval(x, {"__builtins__": {}}, env) for x in row["out"]]
            if (not np.allclose(out[row["token"], row["head"]], want, atol=1e-12)
                    or abs(lse[row["token"], row["head"]] - eval(row["lse"], {"__builtins__": {}}, env)) > 1e-12):
                failures.append(case["name"])
                break
    for seed, lens, Hq, Hkv, D, w, s in [(0, [37, 91], 4, 2, 16, 0, False),
                                          (1, [5, 0, 17, 1, 40], 4, 1, 8, 0, True),
                                          (2, [64, 3, 29], 6, 3, 8, 7, True)]:
        p = workloads.random_pack(seed, lens, Hq, Hkv, D, w, D ** -0.5, s)
        o, l = oracle.attention(p["q"], p["k"], p["v"], p["cu_seqlens"], w, p["scale"], p["sinks"], lib=lib)
        do, dl = oracle.dense_attention(p["q"], p["k"], p["v"], p["cu_seqlens"], w, p["scale"], p["sinks"])
        if not (np.allclose(o, do, atol=1e-12) and np.allclose(l, dl, atol=1e-12)):
            failures.append(f"dense{seed}")
    return failures


def test_unmutated_copy_passes(tmp_path):
    src = open(oracle._SRC).read()
    path = tmp_path / "copy.c"
    path.write_text(src)
    lib = oracle.load(oracle.build(force=True, src=str(path), out=str(tmp_path / "copy.so")))
    assert _pins_fail(lib) == []


# The C source holds the forward first, then the backward after this marker,
# then the key-rows backward entry point after the second marker (pinned
# against the full backward in test_oracle_bwd_pins.py); a forward mutant
# changes the forward part only, a backward mutant the full backward only.
BWD_MARKER = " * Backward."
KV_ROWS_MARKER = " * dk and dv for selected"


def _mutate(old, new, backward):
    src = open(oracle._SRC).read()
    cut = src.index(BWD_MARKER)
    cut2 = src.index(KV_ROWS_MARKER)
    head, mid, rest = src[:cut], src[cut:cut2], src[cut2:]
    part = mid if backward else head
    assert part.count(old) == 1, f"mutation anchor {old[:40]!r} not unique"
    if backward:
        return head + mid.replace(old, new) + rest
    return head.replace(old, new) + mid + rest


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name, tmp_path):
    old, new = MUTANTS[name]
    path = tmp_path / f"{name}.c"
    path.write_text(_mutate(old, new, backward=False))
    lib = oracle.load(oracle.build(force=True, src=str(path), out=str(tmp_path / f"{name}.so")))
    assert _pins_fail(lib), f"mutant {name} survived every pin"


# ----------------------------------------------------------------- backward --
# Planted mistakes in the oracle's backward; caught by finite differences of
# the (unmutated-forward) copy, by PyTorch SDPA autograd, or by the invariants.

BWD_MUTANTS = {
    "bwd_D_term_dropped": ("const double dS = p[j - lo] * (dP - Di);\n                for (int c = 0; c < D; c++) {",
                           "const double dS = p[j - lo] * dP;\n                for (int c = 0; c < D; c++) {"),
    "bwd_dsink_sign": ("dsink_part[hh] -= psink * Di;", "dsink_part[hh] += psink * Di;"),
    "bwd_dk_uses_key": ("scale * dS * load_elem(q, (i * Hq + h) * (int64_t)D + c, dtype);",
                        "scale * dS * load_elem(k, (i * Hkv + g) * (int64_t)D + c, dtype);"),
    "bwd_dv_weighted_by_dS": ("p[j - lo] * load_elem(dout, (i * Hq + h) * (int64_t)D + c, dtype);",
                              "dS * load_elem(dout, (i * Hq + h) * (int64_t)D + c, dtype);"),
    "bwd_dq_scale_dropped": ("dq[(i * Hq + h) * (int64_t)D + c] +=\n                        scale * dS",
                             "dq[(i * Hq + h) * (int64_t)D + c] +=\n                        dS"),
    "bwd_dk_wrong_group": ("dk[(j * Hkv + g) * (int64_t)D + c] +=", "dk[(j * Hkv + h % Hkv) * (int64_t)D + c] +="),
}


def _bwd_pins_fail(lib) -> list[str]:
    import torch
    failures = []
    # finite differences of the forward on a tiny pack with a sink and a window
    p = workloads.random_pack(3, [5, 0, 7, 1], 4, 2, 4, 3, 0.5, True)
    q, k, v = (p[n].double().numpy() for n in "qkv")
    s = p["sinks"].numpy().astype(np.float32)
    dout = np.random.default_rng(103).standard_normal(q.shape)
    cu = p["cu_seqlens"]
    dq, dk, dv, ds = oracle.attention_bwd(q, k, v, dout, cu, 3, 0.5, s, lib=lib)

    def loss(q_, k_, v_, s_):
        o, _ = oracle.attention(q_, k_, v_, cu, 3, 0.5, s_)  # the real (pinned) forward
        return float((o * dout).sum())

    h = 1e-5
    for name, x, g in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
        for idx in list(np.ndindex(x.shape))[::3]:
            xp, xm = x.copy(), x.copy()
            xp[idx] += h
            xm[idx] -= h
            a = {"q": q, "k": k, "v": v}
            a[name] = xp
            fp = loss(a["q"], a["k"], a["v"], s)
            a[name] = xm
            fm = loss(a["q"], a["k"], a["v"], s)
            if abs((fp - fm) / (2 * h) - g[idx]) > 1e-6 * max(1.0, np.abs(g).max()):
                failures.append(f"fd_{name}")
                break
    for hh in range(4):
        sp, sm = s.copy(), s.copy()
        sp[hh] += np.float32(1e-2)
        sm[hh] -= np.float32(1e-2)
        fd = (loss(q, k, v, sp) - loss(q, k, v, sm)) / (float(sp[hh]) - float(sm[hh]))
        if abs(fd - ds[hh]) > 2e-4 * max(1.0, abs(ds[hh])):
            failures.append("fd_sink")
            break
    # SDPA autograd, one document, no sink
    p = workloads.random_pack(5, [23], 4, 2, 16, 0, 0.25, False)
    q, k, v = (p[n].double().numpy() for n in "qkv")
    dout = np.random.default_rng(105).standard_normal(q.shape)
    dq, dk, dv, _ = oracle.attention_bwd(q, k, v, dout, p["cu_seqlens"], 0, 0.25, lib=lib)
    qt, kt, vt = (torch.tensor(a).permute(1, 0, 2).requires_grad_() for a in (q, k, v))
    o = torch.nn.functional.scaled_dot_product_attention(
        qt, kt.repeat_interleave(2, 0), vt.repeat_interleave(2, 0), is_causal=True, scale=0.25)
    o.backward(torch.tensor(dout).permute(1, 0, 2))
    for name, t, g in (("q", qt, dq), ("k", kt, dk), ("v", vt, dv)):
        if not np.allclose(t.grad.permute(1, 0, 2).numpy(), g, atol=1e-10):
            failures.append(f"sdpa_{name}")
    return failures


def test_unmutated_backward_copy_passes(tmp_path):
    path = tmp_path / "copy_bwd.c"
    path.write_text(open(oracle._SRC).read())
    lib = oracle.load(oracle.build(force=True, src=str(path), out=str(tmp_path / "copy_bwd.so")))
    assert _bwd_pins_fail(lib) == []


@pytest.mark.parametrize("name", sorted(BWD_MUTANTS))
def test_backward_mutant_is_caught(name, tmp_path):
    old, new = BWD_MUTANTS[name]
    path = tmp_path / f"{name}.c"
    path.write_text(_mutate(old, new, backward=True))
    lib = oracle.load(oracle.build(force=True, src=str(path), out=str(tmp_path / f"{name}.so")))
    assert _bwd_pins_fail(lib), f"mutant {name} survived every pin"
