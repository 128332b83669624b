"""Multi-rank host logic on CPU: gloo process groups of world size 2.

The decode step shards by sequence (each attends only over its own K cache), so
ranks run disjoint batches; the only collectives time the job. These tests run
that logic as real processes on the host, without a GPU.
"""
from __future__ import annotations

import json
import os
import socket
import subprocess
import sys
import tempfile

import numpy as np
import pytest
import torch.multiprocessing as mp

from only_cache_exact_b200 import replicas

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, batch, out_dir):
    import datetime

    import torch.distributed as dist

    from only_cache_exact_b200 import replicas as R, synth

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        ids = R.global_sequence_ids(rank, world, batch)
        blocks = [None] * world
        dist.all_gather_object(blocks, ids)
        # this rank's first decode token row, drawn from its own stream
        row = synth.make_tokens(1, 8, 0, ids[0], "bf16", part=2)[0].tolist()
        rows = [None] * world
        dist.all_gather_object(rows, row)
        # a per-rank "duration": the slowest rank decides the job time
        dist.barrier()
        t_max = R.max_over_ranks(10.0 + 5.0 * rank, dist)
        rate = R.whole_job_rate(1, world, t_max)
        with open(os.path.join(out_dir, f"r{rank}.json"), "w") as f:
            json.dump({"blocks": blocks, "rows": rows, "t_max": t_max, "rate": rate}, f)
    finally:
        dist.destroy_process_group()


def test_two_ranks_disjoint_sequences_and_max_time():
    world, batch = 2, 3
    with tempfile.TemporaryDirectory(dir=ROOT) as tmp:
        ctx = mp.get_context("spawn")
        port = _free_port()
        procs = [ctx.Process(target=_worker, args=(r, world, port, batch, tmp)) for r in range(world)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(120)
        assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
        res = [json.load(open(os.path.join(tmp, f"r{r}.json"))) for r in range(world)]
    for r in res:
        assert r["blocks"] == [[0, 1, 2], [3, 4, 5]]
        assert replicas.check_disjoint(r["blocks"])
        assert r["t_max"] == 15.0  # both ranks see the slower rank's time
        assert r["rate"] == pytest.approx(2 * 1e3 / 15.0)
        assert not np.allclose(r["rows"][0], r["rows"][1])  # ranks draw different tokens
    assert res[0] == res[1]


def test_sequence_blocks_cover_the_job():
    world, batch = 4, 5
    blocks = [replicas.global_sequence_ids(r, world, batch) for r in range(world)]
    assert replicas.check_disjoint(blocks)
    assert sorted(g for b in blocks for g in b) == list(range(world * batch))
    assert not replicas.check_disjoint([[0, 1], [1, 2]])
    with pytest.raises(ValueError):
        replicas.global_sequence_ids(4, 4, 2)
    assert replicas.max_over_ranks(3.5) == 3.5  # no process group: identity
    with pytest.raises(ValueError):
        replicas.whole_job_rate(1, 2, 0.0)


def test_reference_arm_under_two_ranks_prints_one_line():
    """bench.py --impl reference under torchrun: rank 0 prints the oracle line, rank 1 exits 0."""
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node=2",
           "--master-addr=127.0.0.1", f"--master-port={_free_port()}", "bench.py",
           "--impl", "reference", "--gpus", "2", "--steps", "3", "--warmup", "3", "--ref-seconds", "0.5"]
    env = dict(os.environ, OMP_NUM_THREADS="2")
    r = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=300, env=env)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [json.loads(x) for x in r.stdout.splitlines() if x.startswith("{")]
    assert len(lines) == 1
    line = lines[0]
    assert line["impl"] == "reference" and line["n_gpus"] == 2
    assert line["cpu_baseline"]["kind"] == "oracle" and line["value"] > 0
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["d2h_bytes_per_step"] == 0
