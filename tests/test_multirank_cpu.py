"""Multi-rank host logic of the bench on CPU (gloo, world size 2).

The scan shards into independent (batch, head, direction) chains, so the
multi-GPU bench gives every rank its own batch of sequences (weak scaling)
and exchanges nothing but the timing: a barrier and a MAX all-reduce.  These
tests run that logic with two gloo ranks on the host.
"""
import os
import socket

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    import sys
    sys.path.insert(0, ROOT)
    from datetime import timedelta

    import torch.distributed as dist

    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    plan = bench.shard_plan(rank, world, bench.DEFAULT_WORKLOAD)
    t = bench.max_over_ranks(1.5 + rank, dist)          # rank 1 is the slow one
    dist.barrier()
    dist.destroy_process_group()
    q.put((rank, plan["seed"], plan["tokens"], tuple(vars(plan["shape"]).values()), t))


def test_two_ranks_shard_and_max():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    res.sort()
    (r0, s0, n0, sh0, t0), (r1, s1, n1, sh1, t1) = res
    assert s0 != s1                      # independent sequences per rank
    assert sh0 == sh1 and n0 == n1       # same per-rank work: weak scaling
    assert t0 == t1 == 2.5               # everyone reports the slowest rank


def test_single_process_max_is_identity():
    import sys
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.25, None) == 3.25


def test_algorithmic_bytes_per_token():
    import sys
    sys.path.insert(0, ROOT)
    import bench
    import ssd_inputs as si
    shape = si.WORKLOADS[bench.DEFAULT_WORKLOAD]["shape"]
    # per direction: x 64*64*2 + dt 64*2 + B,C 2*128*2; y 64*64*2 written once
    assert bench.algorithmic_bytes_per_token(shape) == 2 * (8192 + 128 + 512) + 8192 == 25856


def test_traffic_record_survives_comment_edits_only():
    """The ncu traffic record is keyed on the kernel's code: comments and layout do not change
    the key, any code change does."""
    import sys
    sys.path.insert(0, ROOT)
    import bench
    src = "int f(int a) { // doubles\n  return 2 * a; /* the\n  result */ }\n"
    assert bench._code_only(src) == bench._code_only("int f(int a) {\n\n    return 2 * a;   }  // other words")
    assert bench._code_only(src) != bench._code_only(src.replace("2 * a", "3 * a"))


def test_traffic_record_is_keyed_on_the_current_kernel(tmp_path):
    """A record whose key is the current sources' hash is found; one with another key is not."""
    import sys
    sys.path.insert(0, ROOT)
    import bench
    key = bench._kernel_source_hash()
    (tmp_path / "a.md").write_text(
        f"traffic-record: kernel=k workload=w source={key} bytes_per_launch=123\n")
    (tmp_path / "b.md").write_text("traffic-record: kernel=k2 workload=w source=0000000000000000 bytes_per_launch=9\n")
    assert bench.profiled_traffic("k", "w", str(tmp_path)) == 123
    assert bench.profiled_traffic("k2", "w", str(tmp_path)) is None
    assert bench.profiled_traffic("k", "other", str(tmp_path)) is None


def test_bench_gpus_flag_spawns_ranks():
    """``bench.py --gpus 2`` outside torchrun starts two rank processes itself.  The dry run goes
    through the same spawn path and process-group setup on gloo: two ranks, their own seeds,
    the same per-rank work, and the slowest rank's time in the line."""
    import json
    import subprocess
    import sys
    env = {k: v for k, v in os.environ.items() if k not in ("WORLD_SIZE", "RANK", "LOCAL_RANK")}
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--gpus", "2", "--dry-run",
                        "--warmup", "3"], capture_output=True, text=True, timeout=300, env=env, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, r.stdout                     # rank 0 alone prints
    out = json.loads(lines[0])
    assert out["n_ranks"] == 2
    ranks = sorted(tuple(x) for x in out["ranks"])
    assert [x[0] for x in ranks] == [0, 1]
    assert ranks[0][1] != ranks[1][1]                    # independent sequences per rank
    assert ranks[0][2] == ranks[1][2]                    # the same work per rank: weak scaling
    assert out["max_time"] == 2.0                        # rank 1 reports 2.0, the slowest
    assert out["tokens_all"] == 2 * ranks[0][2]
