"""Data-parallel decomposition on 2 CPU ranks (gloo): per-rank adapter
gradients on each rank's token shard, summed by allreduce_adapter_grads,
equal the full-batch gradients.  The per-rank compute here is the oracle;
the code under test is the sharding and the exchange that bench.py uses."""
import os
import socket

import numpy as np
import torch
import torch.multiprocessing as mp

from bit_nf4_quantized_22_b200 import synth
from bit_nf4_quantized_22_b200.dp import allreduce_adapter_grads, shard_rows
from bit_nf4_quantized_22_b200.synth import LinearSpec

SPEC = LinearSpec("dp", 128, 72, 4, 8.0, True)
M = 37


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, out):
    import datetime
    import torch.distributed as dist
    import oracle
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        a = synth.draw(SPEC, M, 31)
        sl = shard_rows(M, rank, world)
        dA, dB = oracle.backward_dadb(a["x"][sl], a["dY"][sl], a["A"], a["B"], SPEC.r, SPEC.alpha)
        tA, tB = torch.from_numpy(dA), torch.from_numpy(dB)
        allreduce_adapter_grads(tA, tB)
        out[rank] = (tA.numpy().copy(), tB.numpy().copy())
    finally:
        dist.destroy_process_group()


def test_shard_rows_cover_once():
    for m in (1, 7, 37, 4096):
        for w in (1, 2, 3, 8):
            idx = np.concatenate([np.arange(m)[shard_rows(m, r, w)] for r in range(w)])
            assert np.array_equal(idx, np.arange(m))


def test_two_rank_adapter_grad_allreduce():
    import oracle
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        out = mgr.dict()
        port = _free_port()
        procs = [ctx.Process(target=_worker, args=(r, 2, port, out)) for r in range(2)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(120)
            assert p.exitcode == 0
        res = dict(out)
    a = synth.draw(SPEC, M, 31)
    dA, dB = oracle.backward_dadb(a["x"], a["dY"], a["A"], a["B"], SPEC.r, SPEC.alpha)
    for r in range(2):
        np.testing.assert_allclose(res[r][0], dA, rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(res[r][1], dB, rtol=1e-12, atol=1e-12)


def _leaving_worker(rank, world, port, out):
    """Rank 1 completes one exchange, then leaves between steps without its
    second collective; rank 0's second exchange must end in an error within the
    process group's short timeout rather than wait for ever."""
    import datetime
    import time
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=5))
    dA, dB = torch.ones(4, 2, dtype=torch.float64), torch.ones(2, 3, dtype=torch.float64)
    allreduce_adapter_grads(dA, dB)
    out[f"step1_{rank}"] = float(dA.sum())
    if rank == 1:
        os._exit(0)                              # leaves between steps, nothing in flight
    t0 = time.monotonic()
    try:
        allreduce_adapter_grads(dA, dB)
        out["error"] = None
    except Exception as e:                       # the backend's timeout or connection error
        out["error"] = type(e).__name__
    out["waited_s"] = time.monotonic() - t0
    os._exit(0)


def test_rank_leaving_surfaces_as_error():
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        out = mgr.dict()
        port = _free_port()
        procs = [ctx.Process(target=_leaving_worker, args=(r, 2, port, out)) for r in range(2)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(120)
            assert p.exitcode == 0
        res = dict(out)
    assert res["step1_0"] == res["step1_1"] == 16.0      # the first exchange summed both ranks
    assert res["error"] is not None, "the surviving rank's collective returned without its peer"
    assert res["waited_s"] < 60
