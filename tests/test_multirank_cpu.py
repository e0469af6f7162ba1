"""The N > 1 path of bench.py on CPU: two ranks over gloo (world size 2).

With several GPUs every rank runs its own replica of the workload (no
collective in the data path): each rank draws its own seeded batch, the
timed region ends in a barrier, the job time is the maximum over ranks and
the work is summed over ranks.  The reference arm runs on rank 0 only and
the other ranks exit quietly.  These tests exercise exactly that host logic
with two gloo ranks (no GPU)."""
import json
import os
import socket
import types

import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, port, out_dir):
    # host-only ranks: gloo even where a GPU is visible
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE="2",
                      RANK=str(rank), LOCAL_RANK=str(rank), CUDA_VISIBLE_DEVICES="")
    import torch.distributed as dist

    import bench
    from attention_mqa_gqa_b200 import workloads as wl

    world, r, _ = bench.dist_setup(2)
    assert (world, r) == (2, rank)
    # each replica its own batch: the lengths differ between ranks
    w = wl.WORKLOADS["mqa_decode"]
    if r:
        w = w.scaled(seed=w.seed + 1000 * r)
    inp = wl.make_inputs(w)
    work = bench.kv_bytes(w, inp["skv"])
    t_ms = 10.0 + 5.0 * rank  # stand-in for the device-timed region of this rank
    bench.barrier(world)
    t_max = bench.allreduce(t_ms, dist.ReduceOp.MAX, world, "cpu")
    work_all = bench.allreduce(work, dist.ReduceOp.SUM, world, "cpu")
    # the reference arm: rank 0 prints one line, rank 1 returns without work
    args = types.SimpleNamespace(workload="mqa_prefill_tiny", steps=1, warmup=0,
                                 ref_step_budget=0.2, gpus=2)
    import contextlib
    import io

    buf = io.StringIO()
    with contextlib.redirect_stdout(buf):
        rc = bench.reference_arm(args, world, r)
    with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
        json.dump({"work": work, "t_max": t_max, "work_all": work_all, "rc": rc,
                   "ref_out": buf.getvalue()}, f)
    dist.barrier()
    dist.destroy_process_group()


def test_two_gloo_ranks(tmp_path):
    ctx = mp.get_context("spawn")
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, port, str(tmp_path))) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=240)
    for p in procs:
        if p.is_alive():
            p.kill()
        assert p.exitcode == 0
    res = [json.load(open(tmp_path / f"rank{r}.json")) for r in range(2)]
    assert res[0]["work"] != res[1]["work"]  # different seeded batches
    for r in res:
        assert r["t_max"] == 15.0  # max over ranks
        assert r["work_all"] == res[0]["work"] + res[1]["work"]
        assert r["rc"] == 0
    line = json.loads(res[0]["ref_out"].strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["n_gpus"] == 2
    assert res[1]["ref_out"] == ""
