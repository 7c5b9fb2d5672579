"""The multi-GPU host path of the benchmark, on CPU with two gloo ranks.

Tiles are independent, so N GPUs split one workload into tile shards with no
collective on the step: rank r owns tiles [r T / N, (r + 1) T / N).  The only
cross-rank operations are the barrier around the timed region and the max
over ranks of the timings.  These tests run the shard map (each rank
computes its shard with the oracle; together the shards must be the
one-rank result bit for bit, every tile covered once), the barrier and max,
and the reference arm's rank-0-only rule, as two processes."""
import json
import os
import socket
import subprocess
import sys
import textwrap

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


WORKER = textwrap.dedent("""
    import json, os, sys
    sys.path.insert(0, {root!r})
    import bench
    ws, rank, local = bench.dist_env()
    dist = bench.dist_init(ws, "gloo")
    # per-rank timings (ms): the reported figure is the max over ranks
    mine = [1.0 + rank, 5.0 - rank, 2.5]
    got = bench.max_over_ranks(dist, mine, "cpu")
    dist.barrier()
    # the value: whole-workload steps over the slowest rank's time
    K = 100
    value = K / (sum(got) / 1e3)
    print(json.dumps({{"rank": rank, "ws": ws, "max": got, "value": value}}), flush=True)
    dist.destroy_process_group()
""")


def test_two_gloo_ranks_max_and_barrier(tmp_path):
    port = _free_port()
    procs = []
    for rank in range(2):
        env = dict(os.environ, MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE="2",
                   RANK=str(rank), LOCAL_RANK=str(rank))
        procs.append(subprocess.Popen([sys.executable, "-c", WORKER.format(root=ROOT)], env=env,
                                      stdout=subprocess.PIPE, stderr=subprocess.PIPE, text=True))
    outs = []
    for p in procs:
        out, err = p.communicate(timeout=180)
        assert p.returncode == 0, err
        outs.append(json.loads(out.strip().splitlines()[-1]))
    for o in outs:
        assert o["ws"] == 2
        assert o["max"] == [2.0, 5.0, 2.5]
        assert abs(o["value"] - 100 / (9.5 / 1e3)) < 1e-6


SHARD_WORKER = textwrap.dedent("""
    import json, os, sys
    import numpy as np
    sys.path.insert(0, {root!r})
    import bench
    from ssm_decode_step_b200 import workloads as W
    from oracle import oracle as O
    ws, rank, local = bench.dist_env()
    dist = bench.dist_init(ws, "gloo")
    # a small stack with per-layer seeds: 3 layers x 5 tiles, split 7 / 8
    w = W.scaled_down(W.get("stack24"), tiles_per_layer=5, layers=3)
    mine = W.shard(w, rank, ws)

    def run(view):
        S0 = W.initial_state(view)
        out = {{"ids": list(view.tile_ids) if view.tile_ids else list(range(view.tiles))}}
        for arm in view.arms:
            cfg = O.OracleConfig(view.tiles, view.dk, view.dv, arm.bits, arm.group, view.delta,
                                 view.decay, arm.policy, arm.rounding)
            st = O.init(cfg, S0)
            os_ = []
            for t in range(3):
                os_.append(O.step(st, *W.slot(view, t)))
            out[arm.name] = (st.codes, st.scales, np.stack(os_))
        return out

    part = run(mine)
    gathered = [None] * ws
    dist.all_gather_object(gathered, part)
    ok = True
    if rank == 0:
        whole = run(w)
        ids = sum((g["ids"] for g in gathered), [])
        ok = ids == list(range(w.tiles))
        for arm in w.arms:
            for i in range(3):
                cat = np.concatenate([g[arm.name][i] for g in gathered], axis=1 if i == 2 else 0)
                ok = ok and np.array_equal(cat, whole[arm.name][i])
    dist.barrier()
    print(json.dumps({{"rank": rank, "tiles": mine.tiles, "ok": bool(ok)}}), flush=True)
    dist.destroy_process_group()
""")


def test_two_gloo_ranks_tile_shards_equal_one_rank():
    """Two ranks each run their tile shard of one workload (the oracle on the
    CPU, three steps, both arms of a small layer-seeded stack); gathered, the
    shards' codes, scales and readouts equal the one-rank run bit for bit,
    and the shards cover every tile exactly once, in order."""
    port = _free_port()
    procs = []
    for rank in range(2):
        env = dict(os.environ, MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE="2",
                   RANK=str(rank), LOCAL_RANK=str(rank))
        procs.append(subprocess.Popen([sys.executable, "-c", SHARD_WORKER.format(root=ROOT)], env=env,
                                      stdout=subprocess.PIPE, stderr=subprocess.PIPE, text=True))
    outs = []
    for p in procs:
        out, err = p.communicate(timeout=300)
        assert p.returncode == 0, err
        outs.append(json.loads(out.strip().splitlines()[-1]))
    assert sorted(o["tiles"] for o in outs) == [7, 8]
    assert all(o["ok"] for o in outs)


def test_reference_arm_runs_on_rank_zero_only():
    env = dict(os.environ, WORLD_SIZE="2", RANK="1", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--steps", "3", "--warmup", "3"], env=env, capture_output=True, text=True,
                       timeout=300)
    assert r.returncode == 0, r.stderr
    assert r.stdout.strip() == ""


def test_reference_arm_line_on_rank_zero():
    env = dict(os.environ, WORLD_SIZE="1", RANK="0", LOCAL_RANK="0")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--workload", "tiny-gdn", "--steps", "8", "--warmup", "3",
                        "--ref-budget", "2"], env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr
    line = json.loads(r.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] >= 1
    assert line["e2e"]["h2d_bytes_per_step"] == 0
