"""The benchmark's multi-rank plumbing on CPU: two gloo ranks, as torchrun launches
them (RANK / WORLD_SIZE / LOCAL_RANK / MASTER_* from the environment).

The path shards by independent (sequence, head) problems, so N GPUs run N
replicas with no collective on the data path.  What ranks share is the timing
protocol: barriers around the timed region, the step time as the max over ranks,
and a distinct seeded sequence per rank.  The reference arm runs on rank 0 alone.
"""
import json
import os
import socket
import subprocess
import sys

import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(world), RANK=str(rank),
                      LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import torch
    import bench

    ranks = bench.Ranks("gloo", torch.device("cpu"), timeout_s=60)
    res = {"world": ranks.world, "rank": ranks.rank, "seed": ranks.seed(7)}
    ranks.barrier()
    res["max"] = ranks.max_over_ranks(1.5 + rank)  # each rank's "step time"
    res["max_again"] = ranks.max_over_ranks(10.0 - rank)
    ranks.barrier()
    ranks.close()
    with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
        json.dump(res, f)


def test_two_gloo_ranks_agree_on_the_max_and_draw_distinct_sequences(tmp_path):
    world = 2
    mp.spawn(_rank_main, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True)
    res = [json.load(open(tmp_path / f"rank{r}.json")) for r in range(world)]
    assert [r["rank"] for r in res] == [0, 1] and all(r["world"] == world for r in res)
    assert all(r["max"] == 2.5 for r in res)  # the slowest rank sets the step time, on every rank
    assert all(r["max_again"] == 10.0 for r in res)
    assert len({r["seed"] for r in res}) == world  # weak scaling: each rank its own sequence


def _bench(env_extra, *args):
    env = dict(os.environ, **env_extra)
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *args], cwd=ROOT, env=env,
                          capture_output=True, text=True, timeout=600)


def test_reference_arm_other_ranks_exit_without_work():
    r = _bench({"RANK": "1", "WORLD_SIZE": "2", "LOCAL_RANK": "1"}, "--impl", "reference", "--gpus", "2",
               "--steps", "1", "--warmup", "3")
    assert r.returncode == 0, r.stderr
    assert r.stdout.strip() == ""


def test_reference_arm_rank0_prints_one_contract_line():
    r = _bench({"RANK": "0", "WORLD_SIZE": "2", "LOCAL_RANK": "0"}, "--impl", "reference", "--gpus", "2",
               "--steps", "1", "--warmup", "3")
    assert r.returncode == 0, r.stderr
    lines = [ln for ln in r.stdout.splitlines() if ln.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2 and d["steps"] == 1 and d["warmup"] == 3
    assert d["value"] > 0 and d["higher_is_better"] is True and d["unit"] == "tokens/s"
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["value"] == d["value"]
    assert d["e2e"] == {"value": d["value"], "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}
