"""Multi-rank host logic on CPU (gloo, world size 2): row sharding and the
global NVFP4 tensor scale, checked against the oracle on the whole tensor."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as tdist
import torch.multiprocessing as mp

from fp4_micro_block_b200.dist import global_tensor_scale, row_range


def test_row_range_partitions_rows():
    for M in [0, 1, 127, 128, 129, 1000, 4096, 8192 + 17]:
        for world in [1, 2, 3, 4, 8]:
            spans = [row_range(M, r, world) for r in range(world)]
            assert spans[0][0] == 0 and spans[-1][1] == M
            for (a, b), (c, d) in zip(spans, spans[1:]):
                assert b == c and a <= b
            for a, b in spans[:-1]:
                assert a % 128 == 0 and b % 128 == 0 or b == M


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, M, K, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    tdist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import oracle
        import workloads
        x = workloads.nvfp4_outliers(M, K, seed=11)
        a, b = row_range(M, rank, world)
        local = oracle.tensor_scale(oracle.amax(oracle.bf16_to_f32(x[a:b])))
        t = torch.tensor([local], dtype=torch.float32)
        global_tensor_scale(t)
        out[rank] = float(t.item())
        tdist.barrier()
    finally:
        tdist.destroy_process_group()


@pytest.mark.parametrize("world", [2])
def test_global_tensor_scale_matches_whole_tensor(world):
    import oracle
    import workloads
    M, K = 600, 256
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    out = mgr.dict()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, M, K, out)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    x = workloads.nvfp4_outliers(M, K, seed=11)
    want = np.float32(oracle.tensor_scale(oracle.amax(oracle.bf16_to_f32(x))))
    for r in range(world):
        assert np.float32(out[r]) == want
