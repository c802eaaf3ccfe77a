"""The N>1 path of bench.py on CPU: two gloo ranks each own an independent
batch (no data exchange), prepare it through the host block manager, and
agree on the job time as the maximum over ranks."""
import os
import socket

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        from paged_kv_cache_400_b200.scenario import prepare_decode_step
        case = bench.rank_case(0, rank, 32)
        prep = prepare_decode_step(case)
        t = bench.max_over_ranks(float(rank + 1) * 10.0, dist, "cpu")
        out[rank] = (prep.seq_lens.tolist(), prep.slot_mapping.tolist(), t)
    finally:
        dist.destroy_process_group()


def test_two_ranks_own_independent_batches_and_take_max_time():
    ctx = mp.get_context("spawn")
    with ctx.Manager() as m:
        out = m.dict()
        port = _free_port()
        mp.start_processes(_worker, args=(2, port, out), nprocs=2, join=True, start_method="spawn")
        r0, r1 = out[0], out[1]
    assert r0[2] == r1[2] == 20.0
    assert r0[0] != r1[0]                      # different sequence lengths per rank
    assert len(r0[0]) == len(r1[0]) == 32
