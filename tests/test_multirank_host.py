"""The multi-GPU path of bench.py is replicas only (the layer has no exchange
step): each rank times its own replica, the job time is the slowest rank's,
and throughput counts every rank's work.  This host logic runs here as two
gloo ranks on the CPU."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    import bench
    ms = 100.0 + 50.0 * rank               # rank 1 is the slow one
    t_max = bench.max_over_ranks(ms, world, "cpu")
    thr = bench.job_throughput(1e12, ms, world, "cpu")
    bench.barrier(world)
    out[rank] = (t_max, thr)
    dist.destroy_process_group()


def test_two_gloo_ranks_take_the_slowest_rank():
    world = 2
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_worker, args=(world, _free_port(), out), nprocs=world, start_method="spawn")
    for r in range(world):
        t_max, thr = out[r]
        assert t_max == 150.0
        assert thr == pytest.approx(2 * 1e12 / 0.150)


def test_single_rank_is_identity():
    import bench
    assert bench.max_over_ranks(12.5, 1) == 12.5
    assert bench.job_throughput(3.0, 1000.0, 1) == pytest.approx(3.0)


def test_traffic_record_matches_the_attention_source():
    # bench.py reports the ncu-measured DRAM traffic only while the attention
    # kernels' sources are the ones it was captured from; a kernel edit must
    # come with a new capture
    import json
    import os
    import bench
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    rec = json.load(open(os.path.join(root, "profiles", "attn_traffic.json")))
    assert bench.attention_source_sha() == rec["kernel_source_sha256"]
    assert 0 < rec["dram_bytes_per_row"] < 4096
