"""Host-side multi-rank logic of bench.py (replicas, max-over-ranks time, summed
work) on two gloo ranks on the CPU."""
import os
import socket

import pytest

torch = pytest.importorskip("torch")
import torch.distributed as dist  # noqa: E402
import torch.multiprocessing as mp  # noqa: E402


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    import bench
    w, r, _ = bench.dist_setup()
    ms, units, flops, launches = bench.reduce_timing(10.0 + 5.0 * rank, 64, 1e12 * (rank + 1),
                                                     100 + rank, w)
    bench.barrier(w)
    q.put((r, ms, units, flops, launches))
    dist.destroy_process_group()


def test_two_rank_aggregation():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
    assert all(p.exitcode == 0 for p in procs)
    out = sorted(q.get(timeout=10) for _ in range(world))
    for r, ms, units, flops, launches in out:
        assert ms == 15.0            # max over ranks
        assert units == 128          # summed work
        assert flops == 3e12
        assert launches == 201


def test_replicas_draw_disjoint_blocks():
    # each rank seeds its 64 blocks by global block index
    import numpy as np

    from second_order_optimizer_shampoo_b200 import synth
    a0 = synth.spd_block(16, 1e-2, 1.0, 103, 0)
    a64 = synth.spd_block(16, 1e-2, 1.0, 103, 64)
    assert not np.array_equal(a0, a64)
    np.testing.assert_array_equal(a0, synth.spd_batch(16, 1, 1e-2, 1.0, 103, indices=[0])[0])


def test_reference_arm_prints_one_line(tmp_path):
    """bench.py --impl reference on rank > 0 exits without work."""
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(root, "bench.py"), "--impl", "reference",
                        "--steps", "1", "--warmup", "0"], capture_output=True, text=True,
                       env=env, timeout=120)
    assert r.returncode == 0 and r.stdout.strip() == ""
