"""Host-side logic of bench.py that the multi-GPU run depends on, on CPU:
the max-over-ranks aggregation with two gloo ranks, and the reference arm's
rule that only rank 0 works."""
import os
import socket
import subprocess
import sys

import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _rank_main(rank, world, port, out):
    import datetime

    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        out[rank] = bench.aggregate(dist, 10.0 + 5 * rank)
    finally:
        dist.destroy_process_group()


def test_aggregate_is_max_over_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    out = mgr.dict()
    mp.start_processes(_rank_main, args=(2, _free_port(), out), nprocs=2, start_method="spawn", join=True)
    assert out[0] == out[1] == 15.0


def test_aggregate_identity_without_process_group():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.aggregate(None, 3.5) == 3.5


def test_reference_arm_nonzero_rank_exits_without_work():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2"],
                       env=env, capture_output=True, text=True, timeout=120)
    assert r.returncode == 0 and r.stdout.strip() == ""


def test_stack_schedule_closed_form():
    # the 32-layer stack's linear schedule: 2048 -> 102 active rows per sequence over 256 steps,
    # 35,241,856 active-token-layers per run at B = 4, 32 layers
    import numpy as np

    import synth
    sched = synth.linear_schedule(2048, 256)
    assert sched[0] == 2048 and sched[-1] == 102 and np.all(np.diff(sched) <= 0)
    assert int(sched.sum()) * 4 * 32 == 35_241_856
    t = np.arange(256)
    assert np.array_equal(sched, 2048 - (t * (2048 - 2048 // 20)) // 255)


def test_long_context_block_draws():
    # M = 32 + min(G, 480), G ~ Geometric(1/64) on {0, 1, ...}: the eight block sizes the
    # long-context measurement uses, and the earlier positions each block recomputes
    import numpy as np

    import synth
    Ms = synth.geometric_block_m(8)
    assert np.all((Ms >= 32) & (Ms <= 512))
    assert Ms.tolist() == synth.geometric_block_m(8).tolist()  # seeded
    for blk, M in enumerate(Ms):
        b0 = 7936 + 32 * blk
        extra = synth.uniform_positions(0, b0, int(M) - 32, tag=100 + blk)
        assert extra.size == M - 32 and np.all(np.diff(extra) > 0) and (extra.size == 0 or extra[-1] < b0)


def test_bench_kernel_modes_are_listed():
    src = open(os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "bench.py")).read()
    for mode in ("step", "kl_lock", "slowfast", "configs", "stack", "long"):
        assert f'"{mode}"' in src
