"""Multi-process host logic on CPU with the gloo backend (world_size 2)."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from group_circulant_gemm_b200.parallel import allreduce_grad_buffer, max_over_ranks, row_shard


@pytest.mark.parametrize("N,world", [(0, 2), (1, 2), (7, 2), (12608, 2), (8224, 8), (5, 8)])
def test_row_shards_cover_rows_once(N, world):
    seen = np.zeros(N, dtype=int)
    last = 0
    for r in range(world):
        a, b = row_shard(N, world, r)
        assert a == last and b >= a
        seen[a:b] += 1
        last = b
    assert last == N and (seen == 1).all()


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import oracle
        from group_circulant_gemm_b200.synth import Workload, make_inputs
        w = Workload("dp", 4, 37, 6, 5, "f32", True, 77)
        inp = make_inputs(w, need_dy=True)
        a, b = row_shard(w.N, world, rank)
        # each rank's partial gradient over its rows, laid out as the flat FP32
        # buffer [dW (padded to 8) | dbias] (computed by the oracle here; on GPUs
        # it comes from eqlinear_backward_weight_f32)
        dW, db = oracle.backward_weight(4, inp["X"][a:b], inp["dY"][a:b], w.D)
        n_w = w.D * w.C * 4
        off = (n_w + 7) // 8 * 8
        buf = torch.zeros(off + w.D, dtype=torch.float32)
        buf[:n_w] = torch.tensor(dW.reshape(-1), dtype=torch.float32)
        buf[off:] = torch.tensor(db, dtype=torch.float32)
        handle = allreduce_grad_buffer(buf, async_op=True)
        handle.wait()
        dW_t, db_t = buf[:n_w].view(w.D, w.C, 4), buf[off:]
        slowest = max_over_ranks(1.0 + rank)
        if rank == 0:
            ref_dW, ref_db = oracle.backward_weight(4, inp["X"], inp["dY"], w.D)
            q.put((float(np.max(np.abs(dW_t.numpy() - ref_dW))),
                   float(np.max(np.abs(db_t.numpy() - ref_db))), slowest))
    finally:
        dist.destroy_process_group()


def test_data_parallel_weight_grad_allreduce_gloo():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    assert all(p.exitcode == 0 for p in procs)
    err_w, err_b, slowest = q.get(timeout=5)
    assert err_w < 1e-4 and err_b < 1e-4  # FP32 sum of two partials vs float64 full sum
    assert slowest == 2.0


def test_grad_buffer_reduction_single_rank_and_dtype():
    assert not dist.is_initialized()
    buf = torch.arange(12, dtype=torch.float32)
    assert allreduce_grad_buffer(buf) is None  # one rank: nothing to reduce
    assert torch.equal(buf, torch.arange(12, dtype=torch.float32))
    with pytest.raises(ValueError):
        allreduce_grad_buffer(buf.half())
