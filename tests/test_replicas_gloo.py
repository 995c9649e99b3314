"""Multi-rank bookkeeping of the verify-step replicas on CPU (gloo, world size 2)."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(world), RANK=str(rank),
                      LOCAL_RANK=str(rank))
    from speculative_decoding_rl_b200 import replicas as R
    import torch.distributed as dist
    R.init("gloo", timeout_s=60)
    w, r, _ = R.env_ranks()
    # rank r did 10*(r+1) steps in (r+1) seconds
    thr = R.job_throughput(10.0 * (r + 1), 1.0 + r, w)
    mx = R.max_over_ranks(3.0 + r, w)
    sm = R.sum_over_ranks(1.0, w)
    R.barrier(w)
    out[r] = (thr, mx, sm)
    dist.destroy_process_group()


def test_two_rank_throughput_uses_slowest_rank_and_total_work():
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    with ctx.Manager() as m:
        out = m.dict()
        procs = [ctx.Process(target=_worker, args=(r, world, port, out)) for r in range(world)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(120)
            assert p.exitcode == 0
        res = dict(out)
    for r in range(world):
        thr, mx, sm = res[r]
        assert thr == pytest.approx((10.0 + 20.0) / 2.0)  # 30 steps over the slowest rank's 2 s
        assert mx == 4.0
        assert sm == 2.0


def test_single_rank_is_identity():
    from speculative_decoding_rl_b200 import replicas as R
    assert R.job_throughput(5.0, 2.0, 1) == 2.5
    assert R.max_over_ranks(7.0, 1) == 7.0
