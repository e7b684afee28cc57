"""Context-parallel forward, host side (CPU): the token shards, the K/V
all-gather over a world-size-2 gloo group (blocking and asynchronous), the
range schedule of each rank's local step (every row of the shard owned
exactly once, no row outside it, every visible key in its items' key tiles)
and its key-bounded form, and the overlapped forward's split of a shard into
its own-slice pack and the rows with keys on earlier ranks, checked by brute
force against the window definition of FlintMagiPlan.attention ("flint.magi"
page); and the overlapped forward itself on two gloo ranks, its GPU calls
replaced by fp64 stand-ins, against the oracle."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

import sliding_window_gqa_cu_b200 as swa
from sliding_window_gqa_cu_b200 import build, cp, multirank, workloads


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build.build()
    swa.load_library()


@pytest.mark.parametrize("T,world", [(10, 3), (2, 4), (65536, 8), (1, 1), (129, 2)])
def test_shard_bounds_partition_the_pack(T, world):
    b = cp.shard_bounds(T, world)
    assert len(b) == world and b[0][0] == 0 and b[-1][1] == T
    assert all(b[r][1] == b[r + 1][0] for r in range(world - 1))
    assert all(0 <= e - s <= -(-T // world) for s, e in b)


def check_range_plan(cu, qb, qe, Hq, Hkv, D, window):
    plan = swa.thd_attn_plan_range(cu, qb, qe, Hq, Hkv, D, window)
    cu = np.asarray(cu)
    T, G = int(cu[-1]), Hq // Hkv
    owner = np.full((T, Hq), -1)
    for idx, it in enumerate(plan):
        q0, q1, s, h0 = int(it["q0"]), int(it["q1"]), int(it["doc_start"]), int(it["head0"])
        ks, nkv, nh, bn = int(it["kv_start"]), int(it["n_kv"]), int(it["n_heads"]), int(it["block_n"])
        assert 0 < q1 - q0 <= 128 and q1 <= qe and (q0 >= qb or qb == 0)
        assert ks + nkv * bn == q1
        d = int(np.searchsorted(cu, s, side="right") - 1)
        while cu[d + 1] == cu[d]:
            d += 1
        e = int(cu[d + 1])
        rows = range(max(q0, s, qb), q1)
        for h in range(h0, h0 + nh):
            for i in rows:
                assert owner[i, h] == -1
                owner[i, h] = idx
        for i in rows:
            lo = s if window == 0 else max(s, i - window + 1)
            assert ks <= lo and i < ks + nkv * bn and i < e
    assert (owner[qb:qe] >= 0).all(), "a row of the shard is not covered"
    assert (owner[:qb] < 0).all() and (owner[qe:] < 0).all(), "a row outside the shard is covered"


@pytest.mark.parametrize("lens,Hq,Hkv,D,window,world", [
    ([300, 1, 0, 129, 77], 4, 2, 128, 0, 2),
    ([300, 1, 0, 129, 77], 4, 2, 128, 100, 3),
    ([700, 256, 3], 6, 2, 128, 128, 4),
    ([1000, 33], 16, 1, 256, 129, 3),
    ([513], 2, 2, 64, 1, 5),
])
def test_range_plans_cover_each_shard_exactly(lens, Hq, Hkv, D, window, world):
    cu = workloads.cu_seqlens_from_lengths(lens)
    for qb, qe in cp.shard_bounds(int(cu[-1]), world):
        check_range_plan(cu, qb, qe, Hq, Hkv, D, window)


def check_key_bounded_plan(cu, qb, qe, k_end, Hq, Hkv, D, window):
    """Every row of [qb, qe) exactly once; an item's key tiles end at
    min(q1, k_end) (at least one tile); each row's keys below k_end inside
    them."""
    plan = swa.thd_attn_plan_range_keys(cu, qb, qe, k_end, Hq, Hkv, D, window)
    cu = np.asarray(cu)
    T = int(cu[-1])
    owner = np.zeros((T, Hq), dtype=int)
    for it in plan:
        q0, q1, s, h0 = int(it["q0"]), int(it["q1"]), int(it["doc_start"]), int(it["head0"])
        ks, nkv, nh, bn = int(it["kv_start"]), int(it["n_kv"]), int(it["n_heads"]), int(it["block_n"])
        assert nkv >= 1 and ks + nkv * bn == min(q1, k_end)
        rows = range(max(q0, s, qb), q1)
        owner[rows.start:rows.stop, h0:h0 + nh] += 1
        for i in rows:
            lo = s if window == 0 else max(s, i - window + 1)
            hi = min(i, k_end - 1)
            if lo <= hi:
                assert ks <= lo and hi < ks + nkv * bn
    assert (owner[qb:qe] == 1).all() and (owner[:qb] == 0).all() and (owner[qe:] == 0).all()


@pytest.mark.parametrize("lens,Hq,Hkv,D,window", [
    ([300, 1, 0, 129, 77], 4, 2, 128, 0),
    ([300, 1, 0, 129, 77], 4, 2, 128, 100),
    ([700, 256, 3], 6, 2, 128, 128),
    ([1000, 33], 16, 1, 256, 129),
    ([513], 2, 2, 64, 1),
])
def test_key_bounded_range_plans(lens, Hq, Hkv, D, window):
    """The schedule of the keys-before-the-rank part of an overlapped
    context-parallel row (thd_attn_fwd_range with k_end = the rank's first
    row), and k_end = T, which is the plain range plan."""
    cu = workloads.cu_seqlens_from_lengths(lens)
    T = int(cu[-1])
    for world in (2, 3, 5):
        for qb, qe in cp.shard_bounds(T, world):
            check_key_bounded_plan(cu, qb, qe, qb, Hq, Hkv, D, window)
            check_key_bounded_plan(cu, qb, qe, T, Hq, Hkv, D, window)
            assert np.array_equal(swa.thd_attn_plan_range_keys(cu, qb, qe, T, Hq, Hkv, D, window),
                                  swa.thd_attn_plan_range(cu, qb, qe, Hq, Hkv, D, window))
    with pytest.raises(swa.ThdAttnError):
        swa.thd_attn_plan_range_keys(cu, 0, T, T + 1, Hq, Hkv, D, window)


@pytest.mark.parametrize("seed", range(6))
def test_overlap_split_of_a_shard_by_brute_force(seed):
    """local_cu_seqlens cuts the pack's documents at the range start (row i
    of [b, e) keeps the keys of its document at or after b, from the pack's
    boundaries), and crossing_rows ends the rows whose document started
    before b -- the only rows with keys on earlier ranks."""
    rng = np.random.default_rng(seed)
    lens = [int(x) for x in rng.integers(0, 90, size=int(rng.integers(1, 7)))]
    cu = workloads.cu_seqlens_from_lengths(lens)
    T = int(cu[-1])
    doc_start = np.zeros(T, dtype=int)
    for d in range(len(lens)):
        doc_start[cu[d]:cu[d + 1]] = cu[d]
    for world in (1, 2, 3, 7):
        for b, e in cp.shard_bounds(T, world):
            lc = cp.local_cu_seqlens(cu, b, e)
            assert lc[0] == 0 and lc[-1] == e - b and (np.diff(lc) >= 0).all()
            x = cp.crossing_rows(cu, b, e)
            assert b <= x <= e
            for i in range(b, e):
                j = int(np.searchsorted(lc, i - b, side="right")) - 1
                while lc[j + 1] == lc[j]:
                    j += 1
                assert lc[j] + b == max(doc_start[i], b)
                assert (i < x) == (doc_start[i] < b)


def test_full_range_plan_is_the_forward_plan():
    cu = workloads.cu_seqlens_from_lengths([300, 1, 0, 129, 77])
    a = swa.thd_attn_plan(cu, 8, 2, 128, 0)
    b = swa.thd_attn_plan_range(cu, 0, int(cu[-1]), 8, 2, 128, 0)
    assert np.array_equal(a, b)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, result_dir):
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    multirank.init("gloo", timeout_s=60)
    p = workloads.random_pack(5, [300, 1, 0, 129, 78], 4, 2, 64, 0, 0.125, False)
    T = int(p["T"])
    b, e = cp.shard_bounds(T, world)[rank]
    k, v = p["k"].float(), p["v"].float()
    kf, vf = cp.gather_kv(k[b:e].contiguous(), v[b:e].contiguous(), T)
    ok = torch.equal(kf, k) and torch.equal(vf, v)
    # the asynchronous form (the overlapped forward's) gives the same tensors
    _, _, finish = cp.gather_kv_async(k[b:e].contiguous(), v[b:e].contiguous(), T)
    ka, va = finish()
    ok = ok and torch.equal(ka, k) and torch.equal(va, v)
    with open(os.path.join(result_dir, f"r{rank}.txt"), "w") as f:
        f.write("ok" if ok else "mismatch")
    multirank.shutdown()


def test_two_rank_gloo_kv_all_gather(tmp_path):
    port = _free_port()
    mp.spawn(_worker, args=(2, port, str(tmp_path)), nprocs=2, join=True)
    assert [open(tmp_path / f"r{r}.txt").read() for r in range(2)] == ["ok", "ok"]


# ------------------------------------- overlapped form, two gloo ranks on CPU --
# The kernels need a GPU; here the three calls the overlapped forward makes are
# replaced by fp64 stand-ins (the oracle's forward, a dense key-bounded
# softmax from the oracle's mask, the log-sum-exp merge) so that its host
# logic -- shard bounds, the own-slice pack, the crossing rows, k_end, the
# asynchronous all-gather and the in-place merge -- runs on two real ranks.

def _ref_fwd(q, k, v, cu_seqlens, window=0, scale=None, sinks=None, **_):
    import oracle
    o, l = oracle.attention(q.double().numpy(), k.double().numpy(), v.double().numpy(), cu_seqlens,
                            window, scale, sinks)
    return torch.from_numpy(o), torch.from_numpy(l)


def _ref_range(q, k, v, cu_seqlens, q_begin, q_end, window=0, scale=None, sinks=None, k_end=None, **_):
    """Rows [q_begin, q_end) against keys j < k_end (dense, fp64, no sinks)."""
    import oracle
    assert sinks is None
    qa, ka, va = (t.double().numpy() for t in (q, k, v))
    G = qa.shape[1] // ka.shape[1]
    mask = oracle.dense_mask(cu_seqlens, window)[q_begin:q_end, :k_end]         # [n, k_end]
    kx, vx = oracle.repeat_kv(ka[:k_end], G), oracle.repeat_kv(va[:k_end], G)
    sc = np.where(mask[None], scale * np.einsum("ihc,jhc->hij", qa, kx), -np.inf)  # [Hq, n, k_end]
    m = sc.max(axis=2, keepdims=True) if k_end > 0 else np.full(sc.shape[:2] + (1,), -np.inf)
    ms = np.where(np.isfinite(m), m, 0.0)
    w = np.exp(sc - ms)
    Z = w.sum(axis=2, keepdims=True)
    out = np.einsum("hij,jhc->ihc", np.where(Z > 0, w / np.where(Z > 0, Z, 1.0), 0.0), vx)
    lse = np.where(Z[..., 0] > 0, np.log(np.where(Z[..., 0] > 0, Z[..., 0], 1.0)) + ms[..., 0], -np.inf)
    return torch.from_numpy(out), torch.from_numpy(lse.T.copy())


def _ref_merge(out_a, lse_a, out_b, lse_b, out=None, lse=None, **_):
    m = torch.maximum(lse_a, lse_b)
    ms = torch.where(torch.isfinite(m), m, torch.zeros_like(m))
    wa, wb = torch.exp(lse_a - ms), torch.exp(lse_b - ms)
    s = wa + wb
    o = torch.where(s[..., None] > 0, (wa[..., None] * out_a + wb[..., None] * out_b) / s[..., None],
                    torch.zeros_like(out_a))
    l = torch.where(s > 0, ms + torch.log(s), torch.full_like(s, float("-inf")))
    out.copy_(o)
    lse.copy_(l)
    return out, lse


def _overlap_worker(rank, world, port, result_dir, lens, window, sinks):
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    multirank.init("gloo", timeout_s=60)
    import oracle
    swa.thd_attn_fwd, swa.thd_attn_fwd_range, swa.thd_attn_merge = _ref_fwd, _ref_range, _ref_merge
    p = workloads.random_pack(7, lens, 4, 2, 64, window, 0.125, sinks)
    T = int(p["T"])
    b, e = cp.shard_bounds(T, world)[rank]
    q, k, v = (p[n].double() for n in "qkv")
    o, l = cp.cp_attention_fwd_overlapped(q[b:e].contiguous(), k[b:e].contiguous(), v[b:e].contiguous(),
                                          p["cu_seqlens"], window, 0.125, p["sinks"])
    ref_o, ref_l = oracle.attention(p["q"], p["k"], p["v"], p["cu_seqlens"], window, 0.125, p["sinks"])
    ok = (o.shape[0] == e - b and np.abs(o.numpy() - ref_o[b:e]).max(initial=0.0) < 1e-9 and
          np.abs(l.numpy() - ref_l[b:e]).max(initial=0.0) < 1e-9)
    with open(os.path.join(result_dir, f"r{rank}.txt"), "w") as f:
        f.write("ok" if ok else "mismatch")
    multirank.shutdown()


@pytest.mark.parametrize("lens,window,sinks", [
    ([300, 1, 0, 129, 78], 0, True),    # the shard boundary inside the first document
    ([300, 1, 0, 129, 78], 40, False),  # a window shorter than the crossing part
    ([254, 254], 0, True),              # the boundary on a document start: no keys before it
])
def test_two_rank_gloo_overlapped_forward(tmp_path, lens, window, sinks):
    port = _free_port()
    mp.spawn(_overlap_worker, args=(2, port, str(tmp_path), lens, window, sinks), nprocs=2, join=True)
    assert [open(tmp_path / f"r{r}.txt").read() for r in range(2)] == ["ok", "ok"]


# ----------------------------------------------------------- head sharding --

@pytest.mark.parametrize("Hq,Hkv,world", [(64, 8, 8), (64, 8, 2), (32, 8, 4), (16, 1, 8),
                                          (16, 1, 2), (8, 2, 4), (4, 4, 4), (16, 2, 1)])
def test_head_shard_partitions_the_heads(Hq, Hkv, world):
    G = Hq // Hkv
    seen = np.zeros(Hq, dtype=int)
    for r in range(world):
        q_lo, q_hi, kv_lo, kv_hi = cp.head_shard(Hq, Hkv, world, r)
        assert q_hi - q_lo == Hq // world
        seen[q_lo:q_hi] += 1
        # every query head of the slice reads a kv head of the slice, and the
        # slice's own GQA mapping (local head // local group) is the global one
        for h in range(q_lo, q_hi):
            assert kv_lo <= h // G < kv_hi
            local_G = (q_hi - q_lo) // (kv_hi - kv_lo)
            assert (h - q_lo) // local_G == h // G - kv_lo
    assert (seen == 1).all()


@pytest.mark.parametrize("Hq,Hkv,world", [(12, 4, 8), (6, 3, 4), (8, 2, 3)])
def test_head_shard_rejects_uneven_splits(Hq, Hkv, world):
    with pytest.raises(ValueError):
        cp.head_shard(Hq, Hkv, world, 0)


def _head_shard_worker(rank, world, port, Hq, Hkv, out_q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    torch.distributed.init_process_group("gloo", rank=rank, world_size=world)
    try:
        mine = torch.tensor(cp.head_shard(Hq, Hkv, world, rank), dtype=torch.int64)
        got = [torch.zeros(4, dtype=torch.int64) for _ in range(world)]
        torch.distributed.all_gather(got, mine)
        if rank == 0:
            out_q.put([g.tolist() for g in got])
    finally:
        torch.distributed.destroy_process_group()


@pytest.mark.parametrize("Hq,Hkv", [(64, 8), (16, 1)])
def test_head_shard_over_two_gloo_ranks(Hq, Hkv):
    # Each rank derives its own slice; together they cover every query head once.
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        port = sk.getsockname()[1]
    ctx = mp.get_context("spawn")
    out_q = ctx.Queue()
    procs = [ctx.Process(target=_head_shard_worker, args=(r, 2, port, Hq, Hkv, out_q)) for r in range(2)]
    for p in procs:
        p.start()
    shards = out_q.get(timeout=120)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    heads = sorted(h for q_lo, q_hi, _, _ in shards for h in range(q_lo, q_hi))
    assert heads == list(range(Hq))
