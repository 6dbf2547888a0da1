"""Host-side logic of the multi-GPU (data-parallel) benchmark path, run as two
gloo ranks on the CPU: the adapter-gradient exchange sums dA and dB over
ranks, and the step time reported is the maximum over ranks."""
import os
import socket

import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    import bench
    dA = torch.full((64, 8), float(rank + 1))
    dB = torch.arange(8 * 32, dtype=torch.float32).view(8, 32) * (rank + 1)
    bench.allreduce_adapter_grads(dA, dB, world)
    t = bench.max_over_ranks(10.0 + rank, world)
    out[rank] = (float(dA[0, 0]), float(dB[1, 3]), t)
    dist.barrier()
    dist.destroy_process_group()


def test_two_rank_gradient_exchange():
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    out = mgr.dict()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    for r in range(2):
        dA00, dB13, t = out[r]
        assert dA00 == 1.0 + 2.0                 # sum of the two ranks' gradients
        assert dB13 == (1 * 32 + 3) * (1 + 2)
        assert t == 11.0                         # max over ranks
