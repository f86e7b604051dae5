"""Data-parallel plumbing on CPU: two gloo ranks in separate processes run the
same helpers the multi-GPU bench uses (max over ranks, whole-job rate,
barriers) on per-rank data shards with replicated weights."""
import json
import os
import socket

import pytest
import torch

from mot_flow_matching_b200 import dp, synth


def _free_port() -> int:
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir):
    os.environ.update({"MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port), "WORLD_SIZE": str(world),
                       "RANK": str(rank), "LOCAL_RANK": str(rank)})
    w, r, local = dp.world_info()
    dp.init_group(w, "gloo", timeout_s=60)
    wl = synth.tiny_workload()
    t = synth.make_inputs(wl, 77, shard=r)
    # a rank-dependent "device time": rank 1 is the slow one
    ms = 10.0 + 5.0 * r
    slowest = dp.max_over_ranks(ms, w)
    rate = dp.aggregate_rate(wl.batch * wl.img_tokens, 4, slowest * 4, w)
    # each rank's checksum of its own shard, gathered to compare across ranks
    sums = torch.tensor([float(t["x"].float().sum()), float(t["w_q"].float().sum())], dtype=torch.float64)
    gathered = [torch.zeros_like(sums) for _ in range(w)]
    torch.distributed.all_gather(gathered, sums)
    dp.barrier(w)
    with open(os.path.join(out_dir, f"rank{r}.json"), "w") as f:
        json.dump({"world": w, "rank": r, "local": local, "slowest": slowest, "rate": rate,
                   "sums": [g.tolist() for g in gathered]}, f)
    dp.finish(w)


def test_two_gloo_ranks(tmp_path):
    import torch.multiprocessing as mp
    world = 2
    mp.start_processes(_rank_main, args=(world, _free_port(), str(tmp_path)), nprocs=world, start_method="spawn",
                       join=True)
    res = [json.loads((tmp_path / f"rank{r}.json").read_text()) for r in range(world)]
    wl = synth.tiny_workload()
    for r, d in enumerate(res):
        assert (d["world"], d["rank"], d["local"]) == (world, r, r)
        assert d["slowest"] == 15.0  # the max over ranks reaches every rank
        # two ranks x B*N units per step, 4 steps, over the slowest rank's 60 ms
        assert d["rate"] == pytest.approx(world * wl.batch * wl.img_tokens * 4 / 0.060)
    sums = res[0]["sums"]
    assert res[1]["sums"] == sums
    assert sums[0][1] == sums[1][1]  # replicated weights
    assert sums[0][0] != sums[1][0]  # independent data shards


def test_world_info_from_env():
    assert dp.world_info({}) == (1, 0, 0)
    assert dp.world_info({"WORLD_SIZE": "4", "RANK": "3", "LOCAL_RANK": "1"}) == (4, 3, 1)
    with pytest.raises(ValueError):
        dp.world_info({"WORLD_SIZE": "2", "RANK": "2"})


def test_single_rank_helpers_need_no_group():
    assert dp.max_over_ranks(3.5, 1) == 3.5
    assert dp.aggregate_rate(100, 10, 500.0, 1) == pytest.approx(2000.0)
    with pytest.raises(ValueError):
        dp.aggregate_rate(1, 1, 0.0, 1)
    dp.barrier(1)
    dp.finish(1)


def test_shards_share_weights_and_split_data():
    wl = synth.tiny_workload()
    base = synth.make_inputs(wl, 5)
    s0 = synth.make_inputs(wl, 5, shard=0)
    s1 = synth.make_inputs(wl, 5, shard=1)
    for k in base:
        assert torch.equal(base[k], s0[k]), k  # shard 0 is the unsharded call
    for k in ("x", "k_cache", "v_cache", "dy"):
        assert not torch.equal(s0[k], s1[k]), k
    for k in ("w_q", "w_k", "w_v", "w_o", "q_norm", "k_norm", "a_q", "b_o"):
        assert torch.equal(s0[k], s1[k]), k


def _bench(args, env_extra=None, timeout=240):
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    env = {k: v for k, v in os.environ.items() if k not in ("WORLD_SIZE", "RANK", "LOCAL_RANK", "MASTER_PORT")}
    env.update(env_extra or {})
    return subprocess.run([sys.executable, os.path.join(root, "bench.py")] + args, env=env, capture_output=True,
                          text=True, timeout=timeout)


def test_bench_gpus_two_spawns_two_ranks():
    # no launcher: bench.py --gpus 2 starts two ranks itself (gloo on CPU here)
    res = _bench(["--gpus", "2", "--steps", "3", "--check-ranks"])
    assert res.returncode == 0, res.stderr[-2000:]
    lines = [json.loads(l) for l in res.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1  # rank 0 alone prints
    line = lines[0]
    assert line["n_gpus"] == 2 and line["local_rank"] == 0
    s0, s1 = line["shard_sums"]
    assert s0 != s1  # each rank ran its own data shard
    assert line["value"] > 0


def test_bench_rejects_a_launcher_world_size_that_differs():
    res = _bench(["--gpus", "2", "--steps", "3", "--check-ranks"],
                 {"WORLD_SIZE": "1", "RANK": "0", "LOCAL_RANK": "0"})
    assert res.returncode == 2
    assert "WORLD_SIZE=1" in res.stderr


def test_check_world():
    assert dp.check_world(1, {}) == "run"
    assert dp.check_world(4, {}) == "spawn"
    assert dp.check_world(2, {"WORLD_SIZE": "2", "RANK": "1"}) == "run"
    with pytest.raises(ValueError):
        dp.check_world(8, {"WORLD_SIZE": "1", "RANK": "0"})
