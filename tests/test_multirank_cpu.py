"""bench.py's multi-rank plumbing on CPU: two gloo ranks (world size 2, one
process each, rendezvous on 127.0.0.1).  The GPU path uses the same helpers
over NCCL; the layer is replicated per rank with no data-path collective, so
what there is to test is the host logic: the max over ranks of a timing, the
barrier, and the reference arm printing its JSON line on rank 0 alone."""
import contextlib
import datetime
import io
import json
import os
import socket
import sys
import types

import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, outdir):
    sys.path.insert(0, ROOT)
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import torch.distributed as dist
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        t_max = bench.max_over_ranks(world, 1.5 + rank)
        bench.barrier(world)
        args = types.SimpleNamespace(workload="tiny_16x256x256_r32", steps=1, warmup=3, ref_rows=16)
        buf = io.StringIO()
        with contextlib.redirect_stdout(buf):
            bench.run_reference(args, world, rank)
        with open(os.path.join(outdir, f"rank{rank}.json"), "w") as f:
            json.dump({"t_max": t_max, "stdout": buf.getvalue()}, f)
        bench.barrier(world)
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks(tmp_path):
    mp.spawn(_worker, args=(2, _free_port(), str(tmp_path)), nprocs=2, join=True)
    r0 = json.loads((tmp_path / "rank0.json").read_text())
    r1 = json.loads((tmp_path / "rank1.json").read_text())
    # Every rank sees the slowest rank's time.
    assert r0["t_max"] == r1["t_max"] == 2.5
    # The reference arm: rank 0 prints exactly one JSON line, the others nothing.
    lines = [ln for ln in r0["stdout"].splitlines() if ln.strip()]
    assert len(lines) == 1
    line = json.loads(lines[0])
    assert line["impl"] == "reference" and line["n_gpus"] == 2 and line["value"] > 0
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["cpu_baseline"]["kind"] == "oracle"
    assert r1["stdout"].strip() == ""
