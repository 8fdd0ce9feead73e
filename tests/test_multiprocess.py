"""The N > 1 host logic of bench.py on CPU: world-size-2 gloo ranks reduce
their device times with a max (the slowest rank sets the job's time); with
replicas the job's per-layer time is that max over the rank count, with head
sharding it is the max itself, the ranks' head slices partition the layer and
their kept-tile counts add up; the reference arm's non-zero ranks leave
without work."""
import importlib.util
import os
import socket
import subprocess
import sys

import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    spec = importlib.util.spec_from_file_location("bench_mod", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, out):
    import datetime
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        b = _bench()
        ms, e2e = b.reduce_over_ranks([1.0 + rank, 10.0 * (rank + 1)], "cpu")
        # head sharding: each rank's slice of a 40-head layer, gathered
        h0, h1 = b.head_slice(40, rank, world)
        slices = [None] * world
        dist.all_gather_object(slices, (h0, h1))
        kept = b.sum_over_ranks([100.0 * (h1 - h0)], "cpu")[0]
        dist.barrier()
        out[rank] = (ms, e2e, b.job_ms_per_layer(ms, world),
                     b.job_ms_per_layer(ms, world, "heads"), slices, kept)
    finally:
        dist.destroy_process_group()


def test_timings_reduce_to_the_slowest_rank():
    world = 2
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_rank, args=(world, _free_port(), out), nprocs=world, join=True)
        res = dict(out)
    for rank in range(world):
        ms, e2e, per_layer, per_layer_heads, slices, kept = res[rank]
        assert ms == 2.0 and e2e == 20.0
        assert per_layer == 1.0
        assert per_layer_heads == 2.0          # one layer, done when the slowest rank is
        # the ranks' head slices cover the layer once, in order
        assert [tuple(x) for x in slices] == [(0, 20), (20, 40)]
        assert kept == 100.0 * 40               # the layer's work, summed over the slices


def test_reference_arm_other_ranks_exit_without_work():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--workload", "tiny", "--steps", "1", "--warmup", "1"],
                       env=env, capture_output=True, text=True, timeout=120)
    assert r.returncode == 0
    assert r.stdout.strip() == ""
