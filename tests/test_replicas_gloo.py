"""Host logic of the multi-process path of bench.py on CPU: two ranks over the gloo
backend (world size 2, rendezvous on 127.0.0.1).

The draft step has no exchange step (requests are independent), so N GPUs run N
replicas, each with its own batch.  What crosses ranks is timing only: the step time
is the max over ranks, and the whole-job throughput is all ranks' tokens over that
time.  These tests run that aggregation, the per-rank batches and the reference-arm
rule (rank 0 alone runs the oracle) in real processes.
"""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    from datetime import timedelta
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        import bench
        from hybrid_mamba_attention_b200 import inputs as I
        out = {}
        # max over ranks: rank r reports 10 + 5 r ms
        out["max"] = bench.max_over_ranks(10.0 + 5.0 * rank, world)
        # whole-job throughput: C*K tokens per rank over the slowest rank's time
        out["thr"] = bench.replica_throughput(64, 10.0 + 5.0 * rank, world)
        # per-rank batches: same shapes and range, different requests
        wl = bench.replica_workload(I, I.WORKLOADS["llama_c32"], rank)
        out["seed"] = wl.seed
        out["lens"] = I.make_ctx_lens(wl).tolist()
        out["shape"] = (wl.C, wl.K, wl.ctx_lo, wl.ctx_hi)
        bench.barrier(world)
        q.put((rank, out))
    finally:
        dist.destroy_process_group()


def _run(world=2):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = dict(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    return res


@pytest.fixture(scope="module")
def two_ranks():
    return _run(2)


def test_step_time_is_the_max_over_ranks(two_ranks):
    assert two_ranks[0]["max"] == two_ranks[1]["max"] == 15.0


def test_throughput_counts_every_rank_over_the_slowest(two_ranks):
    for r in (0, 1):
        ms, value = two_ranks[r]["thr"]
        assert ms == 15.0
        assert value == pytest.approx(2 * 64 / 15e-3)


def test_replicas_draw_different_requests_of_the_same_shape(two_ranks):
    a, b = two_ranks[0], two_ranks[1]
    assert a["shape"] == b["shape"]
    assert a["seed"] != b["seed"]
    assert a["lens"] != b["lens"]
    lo, hi = a["shape"][2], a["shape"][3]
    assert all(lo <= v <= hi for v in a["lens"] + b["lens"])


def test_reference_arm_runs_on_rank_zero_only(monkeypatch, capsys):
    # ranks other than 0 leave the reference arm without work and without output
    import bench

    class Args:
        steps, warmup, C, K = 1, 3, 4, 4

    called = []
    monkeypatch.setattr(bench, "oracle_one_request", lambda *a, **k: called.append(1))
    bench.run_reference(Args(), rank=1, world=2)
    assert called == [] and capsys.readouterr().out == ""
