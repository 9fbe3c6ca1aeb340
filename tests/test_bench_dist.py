"""The benchmark's multi-process plumbing on CPU: two gloo ranks take the same
collective steps as a `torchrun --nproc-per-node 2 bench.py` run (process
group set-up from the environment, barrier, max over ranks of the step time),
and the reference arm runs on rank 0 only."""

import os
import socket
import sys
import types

import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ.update({"MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port), "WORLD_SIZE": str(world),
                       "RANK": str(rank), "LOCAL_RANK": str(rank)})
    sys.path.insert(0, ROOT)
    import torch

    import bench

    w, r, local = bench.dist_setup()
    assert (w, r, local) == (world, rank, rank)
    assert torch.distributed.get_backend() == "gloo"
    bench.barrier(w)
    step_ms = bench.max_over_ranks(1.5 + rank, w, "cpu")
    args = types.SimpleNamespace(workload="tiny_n256", steps=1, warmup=3)
    line = bench.run_reference(args, w, r)
    bench.barrier(w)
    torch.distributed.destroy_process_group()
    out.put((rank, step_ms, None if line is None else (line["impl"], line["n_gpus"], line["value"] > 0)))


def test_two_gloo_ranks_agree_on_max_and_reference_runs_on_rank0():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(out.get(timeout=300) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [r[1] for r in res] == [2.5, 2.5]  # max over ranks, seen by both
    assert res[0][2] == ("reference", 2, True)
    assert res[1][2] is None


def test_reference_line_keeps_the_contract():
    """The reference arm's JSON line (one process, the tiny workload): the base
    keys, the oracle as its own CPU baseline, and an end-to-end figure equal to
    its value with no host-device copies."""
    sys.path.insert(0, ROOT)
    import bench

    args = types.SimpleNamespace(workload="tiny_n256", steps=1, warmup=3)
    line = bench.run_reference(args, 1, 0)
    for key in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in line, key
    assert line["impl"] == "reference" and line["n_gpus"] == 1 and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["value"] == line["value"]
    assert line["cpu_baseline"]["cores"] >= 1 and line["cpu_baseline"]["sample"]
    assert line["e2e"]["value"] == line["value"] and line["e2e"]["unit"] == line["unit"]
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["d2h_bytes_per_step"] == 0
