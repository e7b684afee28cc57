"""The host tile schedule covers every visible (query, key, head) triple
exactly as the kernel needs: each (token, head) row is owned by exactly one
work item, every visible key of the row lies in the item's key tiles, no key
tile is fully masked, and items run in chunks of kv groups whose K/V fits in
L2, longest first within a chunk, with the heads of one (query tile, kv group)
adjacent.  Checked by brute force against the window definition of
FlintMagiPlan.attention ("flint.magi" page)."""
import numpy as np
import pytest

import sliding_window_gqa_cu_b200 as swa
from sliding_window_gqa_cu_b200 import build, workloads


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build.build()
    swa.load_library()


def visible_range(i, s, window):
    lo = s if window == 0 else max(s, i - window + 1)
    return lo, i  # inclusive


def check_plan(cu, Hq, Hkv, D, window):
    plan = swa.thd_attn_plan(cu, Hq, Hkv, D, window)
    cu = np.asarray(cu)
    T = int(cu[-1])
    G = Hq // Hkv
    owner = np.full((T, Hq), -1, dtype=np.int64)
    for idx, it in enumerate(plan):
        q0, q1, s, h0 = int(it["q0"]), int(it["q1"]), int(it["doc_start"]), int(it["head0"])
        ks, nkv, nh, bn = int(it["kv_start"]), int(it["n_kv"]), int(it["n_heads"]), int(it["block_n"])
        d = int(np.searchsorted(cu, s, side="right") - 1)
        while cu[d + 1] == cu[d]:
            d += 1
        e = int(cu[d + 1])
        assert cu[d] == s and q1 - q0 == 128 and s < q1 <= e and nkv >= 1
        assert ks + nkv * bn == q1
        assert h0 // G == (h0 + nh - 1) // G, "heads of an item must share one kv head"
        rows = range(max(q0, s), q1)
        for h in range(h0, h0 + nh):
            for i in rows:
                assert owner[i, h] == -1, "row owned twice"
                owner[i, h] = idx
        tile_hit = np.zeros(nkv, dtype=bool)
        for i in rows:
            lo, hi = visible_range(i, s, window)
            assert ks <= lo and hi < ks + nkv * bn
            tile_hit[(lo - ks) // bn:(hi - ks) // bn + 1] = True
        assert tile_hit.all(), "a key tile with no visible pair was scheduled"
    assert (owner >= 0).all(), "some (token, head) row is not covered"
    # chunks of kv groups in order (as many groups per chunk as keep their
    # K/V within 48 MB), longest first within each chunk
    c = int(min(max((48 << 20) // max(T * D * 4, 1), 1), Hkv))
    chunk = plan["head0"] // G // c
    assert (np.diff(chunk) >= 0).all(), "kv group chunks interleaved"
    for g in np.unique(chunk):
        assert (np.diff(plan["n_kv"][chunk == g]) <= 0).all(), "not longest first within a chunk"
    return plan


def test_group_chunks_follow_the_l2_budget():
    # 64k tokens at D = 128: 32 MiB of K/V per kv head -> one group per chunk
    cu = workloads.cu_seqlens_from_lengths([30000, 35536])
    plan = swa.thd_attn_plan(cu, 16, 8, 128, 0)
    assert (np.diff(plan["head0"] // 2) >= 0).all()
    # 8k tokens: 4 MiB per kv head -> all 8 groups in one chunk (plain longest first)
    cu = workloads.cu_seqlens_from_lengths([5000, 3192])
    plan = swa.thd_attn_plan(cu, 16, 8, 128, 0)
    assert (np.diff(plan["n_kv"]) <= 0).all()
    assert len(set(plan["head0"][:8] // 2)) > 1


@pytest.mark.parametrize("lens,Hq,Hkv,D,window", [
    ([37, 91], 4, 2, 64, 0),
    ([5, 0, 300, 1, 129, 128, 127], 8, 2, 128, 0),
    ([5, 0, 300, 1, 129, 128, 127], 8, 2, 128, 7),
    ([700, 256, 3], 6, 2, 128, 128),       # G = 3: one head per item
    ([1000, 33], 16, 1, 256, 129),
    ([513], 2, 2, 64, 1),
    ([0, 0], 4, 2, 64, 0),
    ([250, 10, 777], 4, 4, 128, 300),      # MHA, G = 1
])
def test_plan_covers_every_visible_pair_once(lens, Hq, Hkv, D, window):
    plan = check_plan(workloads.cu_seqlens_from_lengths(lens), Hq, Hkv, D, window)
    assert len(plan) == 0 if sum(lens) == 0 else len(plan) > 0


def test_plan_random_packs():
    rng = np.random.default_rng(7)
    for trial in range(12):
        lens = list(rng.integers(0, 400, size=rng.integers(1, 6)))
        Hkv = int(rng.choice([1, 2, 4]))
        Hq = Hkv * int(rng.choice([1, 2, 3, 4]))
        D = int(rng.choice([64, 128, 256]))
        window = int(rng.choice([0, 1, 2, 127, 128, 129, 500]))
        check_plan(workloads.cu_seqlens_from_lengths(lens), Hq, Hkv, D, window)


def test_gqa_heads_adjacent_and_shapes():
    cu = workloads.cu_seqlens_from_lengths([1000, 400])
    # D = 128: one CTA per item, two heads of one kv group
    plan = swa.thd_attn_plan(cu, 32, 8, 128, 0)
    assert set(plan["n_heads"]) == {2} and set(plan["block_n"]) == {128}
    # consecutive items of one (query tile, kv head) form one run
    key = [(int(p["q0"]), int(p["head0"]) // 4) for p in plan]
    seen, prev = set(), None
    for k in key:
        if k != prev:
            assert k not in seen, "items of one (tile, kv group) are split apart"
            seen.add(k)
        prev = k
    # D = 256: CTA-pair items of two heads with 128-key tiles; odd groups fall
    # back to one head per CTA with 64-key tiles
    p256 = swa.thd_attn_plan(cu, 16, 1, 256, 64)
    assert set(p256["block_n"]) == {128} and set(p256["n_heads"]) == {2}
    assert set(swa.thd_attn_plan(cu, 3, 1, 256, 64)["block_n"]) == {64}
    assert set(swa.thd_attn_plan(cu, 3, 1, 128, 0)["n_heads"]) == {1}


def test_benchmark_pack_plan_sizes():
    cfg = workloads.CONFIGS["pack64k_gqa8_d128_causal_sink"]
    plan = swa.thd_attn_plan(workloads.pack_cu_seqlens(cfg, 0), cfg.Hq, cfg.Hkv, cfg.D, cfg.window)
    n_tiles = sum((L + 127) // 128 for L in np.diff(workloads.pack_cu_seqlens(cfg, 0)))
    assert len(plan) == n_tiles * cfg.Hq // 2
    assert plan["n_kv"][0] == (24218 + 127) // 128
