"""bench.py's multi-process host logic on CPU with the gloo backend, world size 2:
rank discovery from the launcher's environment, the max-over-ranks step time,
the barrier, the whole-job (weak scaling) throughput, and the reference arm's
rank-0-only output.  The GPU data path is not involved."""
import json
import multiprocessing as mp
import os
import socket
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q, run_reference):
    try:
        os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank),
                          MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
        sys.path.insert(0, ROOT)
        import datetime

        import torch
        import torch.distributed as dist

        import bench

        dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
        out = {"dist": bench._dist()}
        out["max"] = bench._max_over_ranks(1.5 + rank, world, torch.device("cpu"))
        bench._barrier(world)
        out["job"] = bench._job_tokens_per_s(world, 8192, 0.5)
        if run_reference:
            import contextlib
            import io

            buf = io.StringIO()
            with contextlib.redirect_stdout(buf):
                rc = bench.main(["--impl", "reference", "--gpus", str(world), "--steps", "1", "--warmup", "0"])
            out["ref_rc"] = rc
            out["ref_out"] = buf.getvalue()
        dist.barrier()
        dist.destroy_process_group()
        q.put((rank, out))
    except Exception as e:   # reported to the parent
        q.put((rank, {"error": repr(e)}))


def _run(world, run_reference=False, timeout=300):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q, run_reference)) for r in range(world)]
    for p in procs:
        p.start()
    res = {}
    for _ in range(world):
        r, out = q.get(timeout=timeout)
        res[r] = out
    for p in procs:
        p.join(timeout=60)
        if p.is_alive():
            p.kill()
    return res


def test_two_ranks_host_logic():
    res = _run(2)
    for r in (0, 1):
        assert "error" not in res[r], res[r]
        assert res[r]["dist"] == (2, r, r)
        assert res[r]["max"] == 2.5                   # max over ranks, seen by every rank
        assert res[r]["job"] == pytest.approx(2 * 8192 / 0.5e-3)


def test_reference_arm_prints_on_rank_zero_only():
    res = _run(2, run_reference=True)
    assert "error" not in res[0] and "error" not in res[1], res
    assert res[0]["ref_rc"] == 0 and res[1]["ref_rc"] == 0
    assert res[1]["ref_out"] == ""
    line = json.loads(res[0]["ref_out"].strip())
    assert line["impl"] == "reference" and line["n_gpus"] == 2 and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle"
    assert line["e2e"]["h2d_bytes_per_step"] == 0
