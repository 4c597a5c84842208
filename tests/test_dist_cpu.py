"""Multi-rank host logic of bench.py on CPU (gloo, world size 2): the max-over-ranks timing reduction
and the per-rank workload replicas (weak scaling, no data-path collective)."""
import os
import socket

import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        m = bench.reduce_max(10.0 + 5.0 * rank, world)
        w = bench.rank_workload("tiny", rank)
        out[rank] = (m, w.seed, tuple(w.ctx_lens), w.num_q_heads)
    finally:
        dist.destroy_process_group()


def test_reduce_max_and_rank_replicas_gloo():
    world, port = 2, _free_port()
    with mp.Manager() as mgr:
        out = mgr.dict()
        mp.start_processes(_worker, args=(world, port, out), nprocs=world, start_method="spawn")
        res = dict(out)
    assert res[0][0] == res[1][0] == 15.0               # every rank sees the slowest rank's time
    assert res[0][1] != res[1][1]                       # independent replicas: different seeds
    assert res[0][2:] == res[1][2:]                     # same shapes on every rank (weak scaling)


def _report_rank(argv):
    """Stand-in for bench.main in a spawned rank: joins the job over gloo with the environment the launcher set,
    takes the max over ranks the way bench.py reports time, and records what it saw in the folder argv[0]."""
    import json
    dist.init_process_group("gloo")
    try:
        rank, world = dist.get_rank(), dist.get_world_size()
        m = bench.reduce_max(float(rank), world)
        env = {k: os.environ[k] for k in ("RANK", "LOCAL_RANK", "WORLD_SIZE", "MASTER_ADDR")}
        with open(os.path.join(argv[0], f"rank{rank}.json"), "w") as f:
            json.dump({"rank": rank, "world": world, "max": m, "env": env}, f)
    finally:
        dist.destroy_process_group()
    return 0


def test_launcher_starts_one_rank_per_gpu(tmp_path):
    """bench.py --gpus N started without torchrun spawns N ranks with torchrun's environment (checked here with the
    gloo backend on CPU: each rank joins, the max-over-ranks reduction spans both)."""
    import json
    rc = bench.spawn_ranks(2, _report_rank, [str(tmp_path)])
    assert rc == 0
    got = [json.load(open(tmp_path / f"rank{r}.json")) for r in range(2)]
    assert [g["rank"] for g in got] == [0, 1] and all(g["world"] == 2 for g in got)
    assert all(g["max"] == 1.0 for g in got)
    assert [g["env"]["LOCAL_RANK"] for g in got] == ["0", "1"]
    assert all(g["env"]["MASTER_ADDR"] == "127.0.0.1" for g in got)


def test_world_size_must_match_gpus(monkeypatch):
    """A job whose rank count differs from --gpus exits non-zero before doing any work."""
    monkeypatch.setenv("WORLD_SIZE", "1")
    monkeypatch.setenv("RANK", "0")
    assert bench.main(["--gpus", "2"]) == 2
    monkeypatch.setenv("WORLD_SIZE", "4")
    assert bench.main(["--gpus", "2", "--impl", "reference"]) == 2


def test_oracle_arm_loads_no_product_library():
    """bench.py --impl reference times the oracle alone: its process maps liboracle.so and never libsegpaged.so,
    and its config object has the same keys as the GPU arm's."""
    import json
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    code = ("import bench, json; bench.main(['--impl', 'reference', '--workload', 'tiny', '--steps', '1', "
            "'--warmup', '0', '--cpu-seconds', '0.3']); maps = open('/proc/self/maps').read(); "
            "print(json.dumps({'segpaged': 'libsegpaged.so' in maps, 'oracle': 'liboracle.so' in maps}))")
    out = subprocess.run([sys.executable, "-c", code], cwd=root, capture_output=True, text=True, timeout=240,
                         env={k: v for k, v in os.environ.items() if k not in ("RANK", "WORLD_SIZE")})
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [json.loads(x) for x in out.stdout.strip().splitlines()]
    line, maps = lines[0], lines[-1]
    assert maps == {"segpaged": False, "oracle": True}
    assert line["impl"] == "reference" and line["cpu_baseline"]["kind"] == "oracle"
    w = bench.rank_workload("tiny", 0)
    assert set(line["config"]) == set(bench.workload_config(w, 1, 0))
