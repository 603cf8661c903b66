"""bench.py's multi-GPU mode is independent replicas: each rank decodes its
own sequence, with no collective on the decode path; the ranks meet only
for the barrier and the max-over-ranks time.  These tests run that host
logic as two gloo ranks on the CPU (no GPU needed)."""
import json
import os
import socket
import subprocess
import sys
import tempfile

import numpy as np
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, outdir):
    from datetime import timedelta

    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        import bench
        from kv_cache_decode_dualcache_b200 import synth
        ms = 100.0 + 50.0 * rank          # this rank's device time
        ms_max = bench.max_over_ranks(ms, world, "cpu")
        value = bench.job_tokens_per_s(world, 3, 256, ms_max)
        prompt = bench.replica_prompt(synth.TINY, 16, rank)
        prompts = [None] * world
        dist.all_gather_object(prompts, prompt.tolist())
        with open(os.path.join(outdir, f"rank{rank}.json"), "w") as f:
            json.dump({"ms_max": ms_max, "value": value, "prompts": prompts}, f)
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_agree_on_the_slowest_time_and_decode_distinct_prompts():
    from kv_cache_decode_dualcache_b200 import synth
    world = 2
    with tempfile.TemporaryDirectory() as d:
        mp.start_processes(_rank, args=(world, _free_port(), d), nprocs=world, join=True,
                           start_method="spawn")
        res = [json.load(open(os.path.join(d, f"rank{r}.json"))) for r in range(world)]
    for r in res:
        # every rank reports the slowest rank's time, and the whole-job rate
        # counts every rank's tokens over that time
        assert r["ms_max"] == 150.0
        assert abs(r["value"] - world * 3 * 256 / 0.150) < 1e-6
    p0, p1 = (np.array(p) for p in res[0]["prompts"])
    assert not np.array_equal(p0, p1)                       # independent sequences
    assert np.array_equal(p0, synth.make_prompt(synth.TINY, 16).numpy())  # rank 0 = 1-GPU prompt
    for p in (p0, p1):
        assert p.min() >= 0 and p.max() <= synth.TINY.vocab - 2   # never the mask id


def test_single_rank_time_is_its_own():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(123.5, 1, "cpu") == 123.5
    assert bench.job_tokens_per_s(1, 5, 256, 1000.0) == 5 * 256


def test_reference_arm_runs_on_rank_0_only():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--gpus", "2", "--steps", "1", "--warmup", "0"],
                       env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0
    assert r.stdout.strip() == ""


def test_bench_launches_its_own_replica_ranks():
    # bench.launch_replicas is what `bench.py --gpus N` runs when no launcher
    # started it: N ranks under torch.distributed.run on 127.0.0.1
    sys.path.insert(0, ROOT)
    import bench
    with tempfile.TemporaryDirectory() as d:
        out = os.path.join(d, "rank0.json")
        rc = bench.launch_replicas(2, [out], script=os.path.join(ROOT, "tests",
                                                                   "replica_rank_cpu.py"),
                                   timeout_s=240)
        assert rc == 0
        r = json.load(open(out))
    assert r["world"] == 2 and r["ms_max"] == 150.0 and r["local_rank"] == 0
    assert abs(r["value"] - 2 * 3 * 256 / 0.150) < 1e-6


def test_bench_rejects_a_world_size_that_disagrees_with_gpus():
    env = dict(os.environ, RANK="0", WORLD_SIZE="3", LOCAL_RANK="0")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--gpus", "2",
                        "--steps", "1", "--warmup", "0"],
                       env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 2 and "WORLD_SIZE" in r.stderr
