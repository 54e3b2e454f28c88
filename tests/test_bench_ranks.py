"""The multi-GPU leg of bench.py runs independent replicas: ranks meet at a barrier around the timed
region and the job's time is the largest rank's. These two steps are host logic, checked here with two
`gloo` ranks on the CPU (the GPU run uses NCCL and CUDA tensors for the same calls)."""
import datetime
import multiprocessing as mp
import os
import socket


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, port, root, q):
    import sys
    sys.path.insert(0, root)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE="2")
    import torch.distributed as dist
    dist.init_process_group("gloo", rank=rank, world_size=2, timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        bench.barrier(2, cuda=False)
        slowest = bench.max_over_ranks(2, 10.0 + 5.0 * rank, device="cpu")  # rank 1 is the slow one
        alone = bench.max_over_ranks(1, 3.0 + rank)                        # one rank: its own value
        bench.barrier(2, cuda=False)
        q.put((rank, slowest, alone))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_meet_and_take_the_slowest_time():
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    port = _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank, args=(r, port, root, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    for p in procs:
        if p.is_alive():
            p.kill()
    assert [p.exitcode for p in procs] == [0, 0]
    got = sorted(q.get(timeout=10) for _ in range(2))
    assert got == [(0, 15.0, 3.0), (1, 15.0, 4.0)]
