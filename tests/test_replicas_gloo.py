"""The multi-rank replica path on CPU: two gloo ranks, as ``bench.py --gpus 2``
runs them (one process per rank, rendezvous on 127.0.0.1).

Covers the host logic of the replicas: each rank's own seeded batch, the
maximum of the ranks' durations, whole-job throughput, the barrier, and a rank
that leaves before a collective (the other rank gets an error, not a hang).
"""
import multiprocessing as mp
import os
import socket

import numpy as np
import pytest

WORLD = 2


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, port, mode, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(WORLD), LOCAL_RANK=str(rank))
    try:
        from expert_routing_dispatch_router_b200 import replicas
        info = replicas.init("gloo", timeout_s=10.0 if mode == "leave" else 60.0)
        if mode == "leave":
            if rank == 1:
                os._exit(0)  # gone before the collective, without saying so
            try:
                replicas.barrier(info)
                q.put((rank, "no error"))
            except Exception as e:  # noqa: BLE001 - any collective error counts
                q.put((rank, "error: " + type(e).__name__))
            return
        import oracle
        from moe_synth import get_config, make_inputs
        sh = get_config("tiny_fp32")
        inp = make_inputs(sh, replicas.batch_seed(11, info))
        out, idx, _ = oracle.layer(inp.x, inp.w_router, inp.bias, inp.w_gate, inp.w_up,
                                   inp.w_down, sh.n_routed, sh.top_k,
                                   tokens=np.arange(4, dtype=np.int32))
        own_ms = 10.0 * (rank + 1)  # rank 1 is the slow one
        slowest = replicas.max_over_ranks(own_ms, info)
        rate = replicas.job_throughput(sh.T, 5, info, slowest)
        replicas.barrier(info)
        q.put((rank, {"slowest": slowest, "rate": rate, "T": sh.T,
                      "x0": inp.x[0, :8].tolist(), "out_sum": float(out.sum()),
                      "idx": idx.tolist()}))
        replicas.finalize(info)
    except Exception as e:  # noqa: BLE001 - reported to the parent
        q.put((rank, "exception: " + repr(e)))


def _run(mode, timeout=120):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, port, mode, q)) for r in range(WORLD)]
    for p in procs:
        p.start()
    results = {}
    expected = 1 if mode == "leave" else WORLD
    try:
        for _ in range(expected):
            rank, val = q.get(timeout=timeout)
            results[rank] = val
    finally:
        for p in procs:
            p.join(timeout=30)
            if p.is_alive():
                p.kill()
                p.join()
    return results


def test_replicas_two_ranks():
    res = _run("ok")
    assert set(res) == {0, 1}, res
    for r in (0, 1):
        assert isinstance(res[r], dict), res[r]
    a, b = res[0], res[1]
    # both ranks agree on the slowest rank's time and on the job's rate
    assert a["slowest"] == b["slowest"] == 20.0
    assert a["rate"] == b["rate"] == pytest.approx(WORLD * 5 * a["T"] / 0.020)
    # each replica has its own batch, and so its own routing and output
    assert a["x0"] != b["x0"]
    assert a["out_sum"] != b["out_sum"]


def test_rank_leaving_before_a_collective():
    res = _run("leave", timeout=90)
    assert 0 in res, res
    assert res[0].startswith("error"), res[0]


def test_single_process_defaults(monkeypatch):
    for k in ("RANK", "WORLD_SIZE", "LOCAL_RANK"):
        monkeypatch.delenv(k, raising=False)
    from expert_routing_dispatch_router_b200 import replicas
    info = replicas.rank_info()
    assert (info.rank, info.world, info.local, info.distributed) == (0, 1, 0, False)
    assert replicas.batch_seed(5, info) == 5
    assert replicas.max_over_ranks(3.5, info) == 3.5
    assert replicas.job_throughput(64, 10, info, 5.0) == pytest.approx(64 * 10 / 0.005)
    with pytest.raises(ValueError):
        replicas.job_throughput(64, 10, info, 0.0)
