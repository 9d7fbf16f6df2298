"""bench.py's multi-rank plumbing on CPU: world_size 2 over gloo (127.0.0.1). Each rank runs
an independent replica (the workload has no cross-GPU exchange). The step time is the
maximum over ranks, and only rank 0 prints the JSON line."""
import io
import json
import os
import socket
import sys
from contextlib import redirect_stdout

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _env(rank, world, port):
    os.environ.update({"RANK": str(rank), "LOCAL_RANK": str(rank), "WORLD_SIZE": str(world),
                       "MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port)})


def _max_worker(rank, world, port, q):
    sys.path.insert(0, ROOT)
    _env(rank, world, port)
    import bench
    r, w, _ = bench.dist_init(bench.parse_args([]))
    bench.barrier(w)
    got = bench.max_over_ranks(10.0 + 5.0 * r, w)
    bench.dist_done(w)
    q.put((r, w, got))


def _reference_worker(rank, world, port, q):
    sys.path.insert(0, ROOT)
    _env(rank, world, port)
    import bench
    buf = io.StringIO()
    with redirect_stdout(buf):
        bench.main(["--impl", "reference", "--workload", "tiny", "--steps", "1"])
    q.put((rank, buf.getvalue()))


def _run(target, world=2):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=target, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    out = [q.get(timeout=240) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    return out


def test_max_over_ranks_gloo():
    out = _run(_max_worker)
    assert sorted(o[0] for o in out) == [0, 1]
    assert all(o[1] == 2 and o[2] == 15.0 for o in out)


def test_reference_arm_prints_on_rank0_only():
    out = dict(_run(_reference_worker))
    assert out[1].strip() == ""
    line = json.loads(out[0].strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["n_gpus"] == 2
    assert line["cpu_baseline"]["kind"] == "oracle" and line["value"] > 0
    assert line["e2e"]["h2d_bytes_per_step"] == 0
    # the JSON contract of the line
    for k in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better", "scaling",
              "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert k in line, k
    assert line["higher_is_better"] is True and line["vs_baseline"] is None and "workload" in line["config"]
    assert {"value", "unit", "cores", "kind", "sample"} <= set(line["cpu_baseline"])
    assert line["e2e"]["value"] == line["value"] and line["e2e"]["d2h_bytes_per_step"] == 0
