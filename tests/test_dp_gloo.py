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


def _worker_grads(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    import bench
    import oracle
    import synth_inputs as si
    wl = si.workload("tiny")
    L = wl.layers[0]
    inp = si.layer_inputs(wl, 0)
    f64 = lambda t: t.to(torch.float64).numpy()
    Wh = oracle.bf16_bits_to_f32(oracle.dequant(oracle.quantize(inp["W"].numpy()))).reshape(L.d_out, L.d_in)
    X, dY = bench.rank_batch(wl, 0, rank, "cpu")
    _, dA, dB = oracle.linear_bwd(f64(X), f64(dY), Wh.astype("float64"), f64(inp["A"]), f64(inp["B"]), L.s)
    dA, dB = torch.from_numpy(dA), torch.from_numpy(dB)
    bench.allreduce_adapter_grads(dA, dB, world)
    out[rank] = (dA.numpy().copy(), dB.numpy().copy())
    dist.barrier()
    dist.destroy_process_group()


def test_data_parallel_adapter_grads_equal_full_batch():
    """Each rank computes the oracle's adapter gradients on its own token batch (the
    partition bench.py trains with), the exchange sums them, and the sum must equal the
    oracle's gradients of the whole global batch: dA = s X^T (dY B^T) and
    dB = s (XA)^T dY are sums over tokens, so splitting the tokens changes only the
    order of fp64 additions."""
    import numpy as np
    import bench
    import oracle
    import synth_inputs as si
    world = 2
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    out = mgr.dict()
    port = _free_port()
    procs = [ctx.Process(target=_worker_grads, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(300)
        assert p.exitcode == 0

    wl = si.workload("tiny")
    L = wl.layers[0]
    inp = si.layer_inputs(wl, 0)
    batches = [bench.rank_batch(wl, 0, r, "cpu") for r in range(world)]
    assert not torch.equal(batches[0][0], batches[1][0])          # the ranks see different tokens
    assert torch.equal(batches[0][0], inp["X"])                    # rank 0 = the single-GPU batch
    X = torch.cat([b[0] for b in batches]).to(torch.float64).numpy()
    dY = torch.cat([b[1] for b in batches]).to(torch.float64).numpy()
    Wh = oracle.bf16_bits_to_f32(oracle.dequant(oracle.quantize(inp["W"].numpy()))).reshape(L.d_out, L.d_in)
    f64 = lambda t: t.to(torch.float64).numpy()
    _, dA_full, dB_full = oracle.linear_bwd(X, dY, Wh.astype("float64"), f64(inp["A"]), f64(inp["B"]), L.s)
    for r in range(world):
        dA, dB = out[r]
        assert np.allclose(dA, dA_full, rtol=1e-12, atol=1e-12 * np.abs(dA_full).max())
        assert np.allclose(dB, dB_full, rtol=1e-12, atol=1e-12 * np.abs(dB_full).max())
    # without the exchange a rank would hold only its own batch's gradient, which is far
    # from the global one (so the comparison above can tell the two apart)
    X0, dY0 = batches[0]
    _, dA0, _ = oracle.linear_bwd(f64(X0), f64(dY0), Wh.astype("float64"), f64(inp["A"]), f64(inp["B"]), L.s)
    assert not np.allclose(dA0, dA_full, rtol=1e-3, atol=1e-3 * np.abs(dA_full).max())
