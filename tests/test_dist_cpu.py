"""The replica path of the benchmark on two CPU ranks (gloo, world size 2).

bench.py --gpus N under torchrun runs N independent replicas of the layer, each routing
its own batch, and reports the whole job's tokens over the slowest rank's time. The host
logic of that path runs here without a GPU: the max-over-ranks reduction, the per-rank
seeds, the job throughput, and the reference arm's rank rule (only rank 0 works)."""
import datetime
import os
import socket
import sys

import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import bench
    from mixture_experts_layer_29_b200 import workloads as wl
    torch.distributed.init_process_group("gloo", rank=rank, world_size=world,
                                         timeout=datetime.timedelta(seconds=60))
    try:
        slowest = bench.max_over_ranks(1.5 * (rank + 1), True)
        cfg = wl.CONFIGS["prefill_bf16"]
        seed = bench.replica_seed(cfg, rank)
        value = bench.job_throughput(cfg.T, 10, world, slowest)
        # the reference arm: ranks other than 0 return at once with nothing printed
        ref_rc = bench.run_reference(bench.parser().parse_args(["--impl", "reference"])) \
            if rank != 0 else None
        torch.distributed.barrier()
        q.put((rank, slowest, seed, value, ref_rc))
    finally:
        torch.distributed.destroy_process_group()


def test_two_replicas_on_gloo():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=180)
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    res = sorted(q.get(timeout=10) for _ in range(2))
    (r0, slow0, seed0, val0, _), (r1, slow1, seed1, val1, ref1) = res
    assert slow0 == slow1 == 3.0                     # both ranks see the slowest time
    assert seed0 != seed1                            # each replica draws its own batch
    assert val0 == val1 == pytest.approx(8192 * 10 * 2 / 3.0e-3)
    assert ref1 == 0
