"""CPU tests (gloo, world size 2) of the multi-process plumbing bench.py uses:
each rank draws its own batch (weak scaling, no collective on the data path)
and the reported time is the maximum over ranks."""
import os
import socket

import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
import synth


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        r, w, local = bench.dist_env()
        assert (r, w, local) == (rank, world, rank)
        # per-rank batches differ
        wl = synth.WORKLOADS["tiny_mha"]
        x = synth.make_inputs(wl.with_(seed=bench.rank_seed(wl.seed, rank)), dout=False)
        qs = [torch.empty_like(x["q"]) for _ in range(world)]
        dist.all_gather(qs, x["q"])
        distinct = not torch.equal(qs[0], qs[1])
        # max over ranks of a per-rank time
        t = bench.max_over_ranks(10.0 + rank, world)
        bench.barrier(world)
        out[rank] = (distinct, t)
    finally:
        dist.destroy_process_group()


def test_two_ranks_gloo():
    world = 2
    mgr = mp.Manager()
    out = mgr.dict()
    mp.spawn(_worker, args=(world, _free_port(), out), nprocs=world, join=True)
    assert out[0] == (True, 11.0) and out[1] == (True, 11.0)


def test_single_rank_helpers():
    assert bench.max_over_ranks(3.5, 1) == 3.5
    assert bench.rank_seed(1004, 0) == 1004 and bench.rank_seed(1004, 1) != 1004


def test_gpus_flag_starts_the_ranks_itself(tmp_path):
    """Without torchrun's environment, bench.py --gpus 2 starts two ranks
    through its replica launcher; each joins the process group (gloo here, in
    place of the GPU arm) and sees world == 2 on 127.0.0.1."""
    env_keys = ("RANK", "WORLD_SIZE", "LOCAL_RANK", "MASTER_ADDR", "MASTER_PORT")
    saved = {k: os.environ.pop(k) for k in env_keys if k in os.environ}
    try:
        probe = os.path.join(os.path.dirname(os.path.abspath(__file__)), "rank_probe.py")
        assert bench.spawn_replicas(2, [str(tmp_path)], script=probe) == 0
    finally:
        os.environ.update(saved)
    import json
    seen = [json.load(open(tmp_path / f"rank{r}.json")) for r in range(2)]
    for r, s in enumerate(seen):
        assert (s["rank"], s["world"], s["local"], s["group_world"]) == (r, 2, r, 2)
        assert s["rank_sum"] == 1.0 and s["master"] == "127.0.0.1" and s["max_over_ranks"] == 11.0


def test_main_spawns_only_outside_torchrun(monkeypatch):
    calls = []
    monkeypatch.setattr(bench, "spawn_replicas", lambda n, argv, script=None: calls.append((n, argv)) or 0)
    for k in ("RANK", "WORLD_SIZE", "LOCAL_RANK"):
        monkeypatch.delenv(k, raising=False)
    assert bench.main(["--gpus", "2", "--steps", "5"]) == 0
    assert calls == [(2, ["--gpus", "2", "--steps", "5"])]
    cmd = bench.replica_command(4, ["--steps", "5"], port=29555)
    assert cmd[1:3] == ["-m", "torch.distributed.run"] and "--nproc-per-node=4" in cmd
    assert cmd[cmd.index("--master-addr") + 1] == "127.0.0.1" and cmd[-2:] == ["--steps", "5"]
