"""World-size-2 CPU (gloo) test of the multi-rank host plumbing used by
bench.py: per-rank packs of one shape with different values, the barrier,
and the max-over-ranks timing reduction feeding the whole-job rate."""
import os
import socket
import time

import torch
import torch.multiprocessing as mp

from sliding_window_gqa_cu_b200 import multirank, workloads


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, result_dir):
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    info = multirank.init("gloo", timeout_s=60)
    assert (info.rank, info.world) == (rank, world)
    cfg = workloads.CONFIGS["tiny_2doc_gqa2_d64"]
    pack = workloads.make_pack(cfg, 0, tensor_seed=multirank.tensor_seed(0, rank))
    # identical shape and document boundaries on every rank ...
    cu = torch.tensor(pack["cu_seqlens"], dtype=torch.int64)
    cus = [torch.zeros_like(cu) for _ in range(world)]
    torch.distributed.all_gather(cus, cu)
    assert all(torch.equal(c, cus[0]) for c in cus)
    # ... but different tensor values
    sig = pack["q"].float().sum().reshape(1)
    sigs = [torch.zeros(1) for _ in range(world)]
    torch.distributed.all_gather(sigs, sig)
    assert len({float(s) for s in sigs}) == world
    multirank.barrier()
    t0 = time.perf_counter()
    time.sleep(0.05 * (rank + 1))  # rank 1 is the slow one
    dt = time.perf_counter() - t0
    mx = multirank.max_over_ranks(dt)
    assert mx >= dt and mx >= 0.1
    rate = multirank.aggregate_rate(100.0, world, mx)
    with open(os.path.join(result_dir, f"r{rank}.txt"), "w") as f:
        f.write(f"{mx} {rate}\n")
    multirank.shutdown()


def test_two_rank_gloo_plumbing(tmp_path):
    port = _free_port()
    mp.spawn(_worker, args=(2, port, str(tmp_path)), nprocs=2, join=True)
    vals = [open(tmp_path / f"r{r}.txt").read().split() for r in range(2)]
    assert vals[0] == vals[1], "ranks disagree on the reduced time"
    mx, rate = map(float, vals[0])
    assert abs(rate - 200.0 / mx) < 1e-9
