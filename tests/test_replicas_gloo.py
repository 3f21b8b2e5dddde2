"""The N > 1 path of bench.py on CPU: two gloo ranks, each timing one replica,
agree on the max-over-ranks time and on the whole-job aggregate (the path
shards into independent replicas: no data-path collective exists)."""
import os
import socket

import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        local_ms = [120.0, 150.0][rank]
        bench.barrier(world)                              # the bench's barrier on a non-NCCL group
        ms = bench.max_over_ranks(local_ms, world, device="cpu")
        out[rank] = (ms, bench.aggregate_tflops(1e12, 10, world, ms))
    finally:
        dist.destroy_process_group()


def test_two_replicas_agree_on_max_time_and_aggregate():
    world, port = 2, _free_port()
    with mp.get_context("spawn").Manager() as m:
        out = m.dict()
        mp.spawn(_rank, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    assert res[0] == res[1]
    ms, tflops = res[0]
    assert ms == 150.0                                   # the slower rank sets the time
    assert abs(tflops - 2 * 1e12 * 10 / 0.150 / 1e12) < 1e-9   # both replicas' work counted


def test_single_rank_needs_no_process_group():
    assert bench.max_over_ranks(7.5, 1) == 7.5
    assert bench.dist_setup(1) == (0, 1, 0) or "RANK" in os.environ


def test_physical_gpu_index_follows_visible_devices(monkeypatch):
    import bench
    monkeypatch.setenv("CUDA_VISIBLE_DEVICES", "4,5,6,7")
    assert bench.physical_gpu(0) == 4 and bench.physical_gpu(3) == 7
    monkeypatch.setenv("CUDA_VISIBLE_DEVICES", "")
    assert bench.physical_gpu(2) == 2
    monkeypatch.setenv("CUDA_VISIBLE_DEVICES", "GPU-1234abcd")
    assert bench.physical_gpu(0) == 0
