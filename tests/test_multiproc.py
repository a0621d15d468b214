"""The multi-rank host logic on CPU: two gloo ranks, each with its own seeded batch; the timed
interval is reduced to the slowest rank and the job rate counts every rank's steps."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        from sparse_kv_cache_kmin_b200 import replicas
        from sparse_kv_cache_kmin_b200.workloads import make
        r, w, lr = replicas.rank_info()
        wl = make("tiny", device="cpu", seed=replicas.workload_seed("tiny", r))
        local_time = 1.0 + r  # rank 1 is the slower one
        slowest = replicas.max_over_ranks(local_time)
        rate = replicas.job_rate(10, w, slowest)
        q = wl.q.flatten()[:4].tolist()
        dist.barrier()
        qout = [None] * w
        dist.all_gather_object(qout, q)
        if r == 0:
            q_ret = {"slowest": slowest, "rate": rate, "world": w, "queries": qout}
            qput(q_ret)
    finally:
        dist.destroy_process_group()


def qput(obj):
    path = os.environ["EKV_TEST_OUT"]
    torch.save(obj, path)


@pytest.mark.timeout(300)
def test_two_gloo_ranks(tmp_path):
    out = tmp_path / "res.pt"
    os.environ["EKV_TEST_OUT"] = str(out)
    mp.start_processes(_worker, args=(2, _free_port(), None), nprocs=2, join=True,
                       start_method="spawn")
    res = torch.load(out)
    assert res["world"] == 2
    assert res["slowest"] == 2.0
    assert res["rate"] == pytest.approx(2 * 10 / 2.0)
    # the two ranks decode different seeded batches
    assert res["queries"][0] != res["queries"][1]


def test_single_process_defaults():
    from sparse_kv_cache_kmin_b200 import replicas
    assert replicas.max_over_ranks(3.5) == 3.5
    assert replicas.workload_seed("needle128k", 0) == 3
    assert replicas.workload_seed("needle128k", 2) == 2003
