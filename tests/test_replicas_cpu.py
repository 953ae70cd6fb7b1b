"""The multi-replica host logic of bench.py over gloo on CPU, world size 2:
every rank reports the slowest rank's time, the whole-job throughput counts
all ranks' tokens, and a rank that dies before the timing reduction makes the
others fail within the process-group timeout instead of hanging."""
import datetime
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, mode, q):
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=10))
    try:
        if mode == "die" and rank == 1:
            os._exit(3)  # leaves without joining the reduction
        t = bench.max_over_ranks(1.0 + 0.25 * rank, world, "cpu")
        q.put((rank, "ok", t))
    except Exception as e:  # noqa: BLE001  (the failure is the expected outcome for mode "die")
        q.put((rank, "error", type(e).__name__))
    finally:
        if mode != "die":
            dist.destroy_process_group()


def _run(mode, world=2):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    ps = [ctx.Process(target=_rank_main, args=(r, world, port, mode, q)) for r in range(world)]
    for p in ps:
        p.start()
    for p in ps:
        p.join(timeout=60)
    alive = [p for p in ps if p.is_alive()]
    for p in alive:
        p.kill()
    assert not alive, "a rank hung"
    out = {}
    while not q.empty():
        r, status, v = q.get()
        out[r] = (status, v)
    return out


def test_max_over_ranks_and_aggregate():
    import bench
    out = _run("ok")
    assert out == {0: ("ok", 1.25), 1: ("ok", 1.25)}
    # 2 replicas x 131072 tokens through each of 4 blocks in 1 step of 1.25 s
    v = bench.replica_throughput(131072, 2, 1.25, 1, 4)
    assert v == pytest.approx(2 * 131072 * 4 / 1.25)


def test_dead_rank_fails_the_reduction_not_hangs():
    out = _run("die")
    assert 1 not in out  # it left
    assert out[0][0] == "error"
