"""Host side of the multi-GPU path ("replicas only"), on CPU with gloo ranks.

bench.py under torchrun runs one independent body pass per rank; the job's
time is the slowest rank's (an all-reduce MAX) and its rate counts the passes
of every rank.  Two gloo ranks with different local times check both.  The
reference arm under torchrun prints only on rank 0.
"""
import os
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _rank(rank, world, port, out):
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    local = [10.0, 25.0, 17.5, 3.0][rank]
    m = bench.max_over_ranks(local, world)
    out.put((rank, m, bench.job_rate(m, 4, world)))
    dist.barrier()
    dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_max_over_ranks_and_job_rate(world):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = 29500 + os.getpid() % 1000 + world
    procs = [ctx.Process(target=_rank, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    want = max([10.0, 25.0, 17.5][:world])
    for _, m, rate in res:
        assert m == want
        assert rate == want * 1e3 / (4 * world)


def test_world_one_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(12.5, 1) == 12.5
    assert bench.job_rate(12.5, 5, 1) == 2500.0


def test_reference_arm_prints_on_rank_zero_only():
    """Under torchrun the reference arm runs and prints on rank 0; rank 1 exits 0 silently."""
    env = dict(os.environ, RANK="1", LOCAL_RANK="1", WORLD_SIZE="2")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2",
                        "--steps", "1", "--warmup", "0"], env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0 and r.stdout.strip() == ""
