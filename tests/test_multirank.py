"""The N > 1 host path of bench.py on CPU: world-size-2 gloo ranks agree on the
max-over-ranks timing and the aggregate throughput, and the per-rank inputs are
independent batches (weak scaling, no collective on the data path)."""
import os
import socket

import pytest
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
    try:
        import bench

        local_ms = 10.0 + 5.0 * rank  # rank 1 is the slow one
        ms_max = bench.max_over_ranks(local_ms, world, "cpu")
        value = bench.aggregate_tflops(world, 3.0e12, 4, ms_max)
        # each rank draws its own batch (seed 1000 + rank), as bench.run_ours does
        from trainable_block_sparse_sas_b200 import synthetic as syn

        inp = syn.train_inputs(syn.TINY_FP32, device="cpu", seed=1000 + rank)
        gathered = [torch.zeros(4) for _ in range(world)]
        dist.all_gather(gathered, inp["q"].flatten()[:4].contiguous())
        out[rank] = (ms_max, value, bool(torch.equal(gathered[0], gathered[1])))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_agree_on_max_timing():
    world, port = 2, _free_port()
    out = mp.get_context("spawn").Manager().dict()  # no fork of this multi-threaded process
    mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
    for rank in range(world):
        ms_max, value, same_batch = out[rank]
        assert ms_max == 15.0
        assert value == pytest.approx(2 * 3.0e12 * 4 / 15.0e-3 / 1e12)
        assert not same_batch


def test_single_rank_is_identity():
    import bench

    assert bench.max_over_ranks(7.5, 1) == 7.5
    assert bench.aggregate_tflops(1, 1e12, 2, 1.0) == pytest.approx(2000.0)
