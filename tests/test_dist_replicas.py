"""The multi-GPU bench path on CPU: two gloo ranks run the replica timing
logic of bench.py (the slowest rank's time, whole-job throughput) and draw
per-rank activations from the shared input recipe."""
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
        from mixture_experts_ffn_sigmoid_b200.inputs import CONFIGS, make_inputs
        ms = [3.0, 5.0][rank]
        slowest = bench.reduce_max(ms, torch.device("cpu"), world)
        rate = bench.whole_job_rate(4096, world, slowest)
        cfg = CONFIGS["tiny_fp32"]
        x = make_inputs(cfg, "cpu", seed=rank, x_only=True)["x"]
        xs = [torch.empty_like(x) for _ in range(world)]
        dist.all_gather(xs, x)
        out[rank] = (slowest, rate, bool(torch.equal(xs[0], xs[1])))
    finally:
        dist.destroy_process_group()


def test_two_rank_replica_timing():
    world = 2
    port = _free_port()
    # The result dict's server process is started with spawn too: the test
    # process may already run threads (torch's pools), and a forked child
    # would inherit any lock one of them held.
    with mp.get_context("spawn").Manager() as mgr:
        out = mgr.dict()
        mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    for rank in range(world):
        slowest, rate, same_x = res[rank]
        assert slowest == 5.0                      # max over ranks, seen by every rank
        assert rate == pytest.approx(2 * 4096 / 5e-3)
        assert not same_x                          # each replica routes its own tokens


def test_single_rank_helpers():
    import bench
    assert bench.reduce_max(7.5, torch.device("cpu"), 1) == 7.5
    assert bench.whole_job_rate(4096, 1, 5.0) == pytest.approx(4096 / 5e-3)
