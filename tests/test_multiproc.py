"""The multi-GPU plumbing of bench.py on CPU: two gloo ranks (no GPU).

The convolution partitions by batch (each output image depends only on its own input
image), so ranks exchange nothing on the data path; what needs testing is the host
logic around it: rank discovery from the launcher's environment, per-rank batches,
the barrier, the max-over-ranks timing and the weak-scaling aggregate."""
import multiprocessing as mp
import os
import socket

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, times, queue):
    import sys
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import datetime

    import torch
    import torch.distributed as dist

    import bench
    from cnn_convolution_conv2d_b200 import workloads
    dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
    try:
        r, w, local = bench.dist_env()
        bench.barrier(w)
        slowest = bench.max_over_ranks(times[rank], w, torch.device("cpu"))
        cfg = workloads.CONFIGS["tiny_f32_nchw"]
        x = workloads.make_inputs(cfg, seed=bench.rank_seed(cfg, r))["x"]
        queue.put((rank, r, w, local, slowest, float(x.sum())))
    finally:
        dist.destroy_process_group()


def test_two_ranks_gloo():
    world, port = 2, _free_port()
    times = [12.5, 17.25]  # ms of each rank's timed region
    ctx = mp.get_context("spawn")
    queue = ctx.Queue()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, times, queue)) for r in range(world)]
    for p in procs:
        p.start()
    results = sorted(queue.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [r[1] for r in results] == [0, 1] and all(r[2] == world for r in results)
    assert [r[3] for r in results] == [0, 1]
    assert all(r[4] == max(times) for r in results)        # every rank sees the slowest time
    assert results[0][5] != results[1][5]                    # different batches per rank


def test_weak_scaling_value():
    import sys
    sys.path.insert(0, ROOT)
    import bench
    from cnn_convolution_conv2d_b200 import workloads
    cfg = workloads.CONFIGS["stem_bf16"]
    f = bench.flops(cfg)
    assert f == pytest.approx(7552892928.0)                  # 2*N*C_out*Ho*Wo*C_in*Kh*Kw
    one = bench.weak_scaling_value(1, f, 100, 5.0)
    assert bench.weak_scaling_value(4, f, 100, 5.0) == pytest.approx(4 * one)
    assert one == pytest.approx(f * 100 / 5e-3 / 1e12)


def test_flop_formula_matches_the_page_example():
    # pwwt §3.3: N=8, C_in=64, C_out=128, 3x3, 32x32 output -> about 1.2e9
    import sys
    sys.path.insert(0, ROOT)
    import bench
    from cnn_convolution_conv2d_b200.workloads import ConvConfig
    cfg = ConvConfig("pwwt33", 8, 64, 32, 32, 128, 3, 3, 1, 1)
    assert bench.flops(cfg) == 2 * 8 * 128 * 32 * 32 * 64 * 9
    assert abs(bench.flops(cfg) - 1.2e9) / 1.2e9 < 0.01


def test_env_defaults_to_one_rank(monkeypatch):
    import sys
    sys.path.insert(0, ROOT)
    import bench
    for k in ("RANK", "WORLD_SIZE", "LOCAL_RANK"):
        monkeypatch.delenv(k, raising=False)
    assert bench.dist_env() == (0, 1, 0)
