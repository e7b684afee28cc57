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


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name, tmp_path):
    old, new = MUTANTS[name]
    src = open(oracle._SRC).read()
    assert src.count(old) == 1, f"mutation anchor for {name} not unique in oracle source"
    path = tmp_path / f"{name}.c"
    path.write_text(src.replace(old, new))
    lib = oracle.load(oracle.build(force=True, src=str(path), out=str(tmp_path / f"{name}.so")))
    assert _pins_fail(lib), f"mutant {name} survived every pin"
