"""The N > 1 replica path of bench.py on CPU: two gloo ranks, one process each.

On GPUs the same helpers run over NCCL, one process per GPU; every (batch, head) is independent, so
the replicas exchange nothing on the data path and only the timing scalar is reduced (max over
ranks).  These tests exercise that host logic without a GPU: the process group with its short
timeout, the max over ranks, the weak-scaling aggregate, disjoint per-rank inputs, the library's
host-side entry points in every rank, and a rank that leaves early.
"""
import json
import os
import socket

import pytest
import torch.multiprocessing as mp

import bench

WORLD = 2


def _free_port():
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, port, outdir, scenario):
    os.environ.update({"MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port),
                       "RANK": str(rank), "WORLD_SIZE": str(WORLD)})
    import torch.distributed as dist
    import bench as b
    res = {"rank": rank}
    if scenario == "replicas":
        b.init_ranks(WORLD, "gloo", timeout_s=30)
        # per-rank step times: the job's step time is the slowest rank's
        ms = [0.25, 0.40][rank]
        res["ms_max"] = b.max_over_ranks(ms, "cpu", WORLD)
        res["value"] = b.weak_scaling_mtok_s(4096, WORLD, res["ms_max"])
        res["seeds"] = [b.input_seed(rank, i) for i in range(b.N_ROTATE)]
        # the library's host-side entry points answer the same in every rank
        import gated_delta_rule_82_b200 as ck
        import torch
        res["ws"] = ck.workspace_bytes(2, 2048, 16, 128, 128, 64, torch.bfloat16, "tc")
        dist.barrier()
        dist.destroy_process_group()
    elif scenario == "early_exit":
        b.init_ranks(WORLD, "gloo", timeout_s=5)
        dist.barrier()
        if rank == 1:
            os._exit(0)   # leaves between steps, with nothing in flight
        try:
            b.max_over_ranks(1.0, "cpu", WORLD)
            res["error"] = None
        except Exception as e:  # the peer is gone: the collective must fail, not hang
            res["error"] = type(e).__name__
    with open(os.path.join(outdir, f"rank{rank}.json"), "w") as f:
        json.dump(res, f)


def _run(tmp_path, scenario):
    port = _free_port()
    ctx = mp.get_context("spawn")
    procs = [ctx.Process(target=_rank_main, args=(r, port, str(tmp_path), scenario))
             for r in range(WORLD)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    for p in procs:
        if p.is_alive():
            p.kill()
            pytest.fail(f"{scenario}: a rank did not finish")
    out = {}
    for r in range(WORLD):
        path = tmp_path / f"rank{r}.json"
        if path.exists():
            out[r] = json.loads(path.read_text())
    return out


def test_weak_scaling_value():
    # 2 ranks x 4096 tokens in 0.5 ms = 16.384 Mtok/s
    assert bench.weak_scaling_mtok_s(4096, 2, 0.5) == pytest.approx(16.384)
    assert bench.max_over_ranks(0.3, "cpu", 1) == 0.3


def test_replicas_reduce_max_and_use_disjoint_inputs(tmp_path):
    out = _run(tmp_path, "replicas")
    assert sorted(out) == [0, 1]
    for r in (0, 1):
        assert out[r]["ms_max"] == pytest.approx(0.40)
        assert out[r]["value"] == pytest.approx(4096 * 2 / 0.40e-3 / 1e6)
        assert out[r]["ws"] == 2 * 16 * 32 * 90112 + 2 * 16 * 32 * 4
    assert not set(out[0]["seeds"]) & set(out[1]["seeds"])


def test_rank_leaving_early_fails_the_next_collective(tmp_path):
    out = _run(tmp_path, "early_exit")
    assert 0 in out and out[0]["error"] is not None
