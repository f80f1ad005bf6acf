"""The multi-rank path of bench.py on CPU: two `gloo` ranks (world size 2, spawned processes) run the
same host logic the GPU job runs under torchrun -- per-rank workloads (weak scaling), the max-over-ranks
reduction of the timings, the whole-job throughput -- and the reference arm's rank-0-only rule."""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    import datetime

    import bench
    from parameter_space_moe_b200 import configs
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    r, wsz, local = bench.rank_env()
    w = bench.rank_workload(configs.BASE, r)
    # each rank's own "timings": rank 1 is slower on the first entry, rank 0 on the second
    mine = [10.0 + 5.0 * r, 7.0 - 3.0 * r, float(r)]
    got = bench.max_over_ranks(mine, dist, torch.device("cpu"))
    dist.barrier()
    with open(os.path.join(out_dir, f"rank{r}.json"), "w") as f:
        json.dump({"rank": r, "world": wsz, "local": local, "seed": w.seed, "shape": [w.batch, w.seqlen, w.d_model],
                   "max": got, "value": bench.job_throughput(w.M, wsz, 4, got[0])}, f)
    dist.destroy_process_group()


def test_two_gloo_ranks_reduce_and_weak_scaling(tmp_path):
    world, port = 2, _free_port()
    mp.start_processes(_rank_main, args=(world, port, str(tmp_path)), nprocs=world, start_method="spawn", join=True)
    res = [json.load(open(tmp_path / f"rank{r}.json")) for r in range(world)]
    for r, x in enumerate(res):
        assert x["rank"] == r and x["world"] == world and x["local"] == r
        assert x["max"] == [15.0, 7.0, 1.0]                # the same maxima on every rank
    assert res[0]["shape"] == res[1]["shape"]              # weak scaling: same shapes per rank ...
    assert res[0]["seed"] != res[1]["seed"]                # ... on each rank's own batch
    M = res[0]["shape"][0] * res[0]["shape"][1]
    assert res[0]["value"] == pytest.approx(M * world * 4 / (15.0 / 1e3))   # all ranks' tokens / slowest time


def test_reference_arm_prints_on_rank0_only(tmp_path):
    """Under torchrun the non-zero ranks of the reference arm exit 0 without output."""
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                        "--warmup", "3", "--workload", "tiny_f32"], env=env, capture_output=True, text=True,
                       timeout=300)
    assert r.returncode == 0 and r.stdout.strip() == ""
