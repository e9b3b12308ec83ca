"""Expert parallelism across ranks, on the CPU: two gloo ranks run the
exchange plan of ``expert_parallel.ep_layer_step`` with the oracle as the
compute steps, so only the plan and the two all-to-all-v exchanges are under
test.

Checks, on each rank:
  * the split sizes are the row counts of the destination's experts, and no
    zero-expert slot is sent;
  * the rows a rank regroups for its experts, expert-major, are exactly the
    rows the oracle's dispatch gives for those experts over the whole job's
    tokens (both ranks' batches, rank 0's first): same counts, same offsets,
    same (expert, token) order;
  * the layer output equals the oracle's per-token layer on the rank's own
    batch.
Plus host-only checks of the plan arithmetic (uneven splits, empty blocks).
"""
import multiprocessing as mp
import os
import socket

import numpy as np
import pytest
import torch

from expert_routing_dispatch_router_b200 import expert_parallel as ep

WORLD = 2


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _shape():
    from moe_synth import MoEShape
    # 7 routed experts: rank 0 owns 4, rank 1 owns 3
    return MoEShape("ep_tiny", T=48, d=64, n_routed=7, n_zero=3, top_k=3, ffn=96,
                    act_dtype="f32")


def _worker(rank, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(WORLD), LOCAL_RANK=str(rank))
    try:
        import torch.distributed as dist
        from datetime import timedelta

        import oracle
        from moe_synth import make_inputs
        dist.init_process_group("gloo", timeout=timedelta(seconds=60))
        sh = _shape()
        N, E, k = sh.n_routed, sh.E, sh.top_k
        # one model (router and expert weights of seed 31), and every rank
        # has its own batch of tokens
        inp = make_inputs(sh, 31)
        inp.x = make_inputs(sh, 31 + rank, with_experts=False).x
        bounds = ep.expert_bounds(N, WORLD)

        def route(x):
            _, idx, gate, _ = oracle.route(x, inp.w_router, inp.bias, k)
            return torch.from_numpy(idx), torch.from_numpy(gate).float()

        def dispatch(x, idx):
            c, o, rt, sr = oracle.dispatch(idx.numpy(), N, E)
            R = int(o[N])
            xp = torch.zeros(sh.T * k, sh.d, dtype=x.dtype)
            xp[:R] = x[torch.from_numpy(rt[:R]).long()]
            return (torch.from_numpy(c), torch.from_numpy(o), torch.from_numpy(rt),
                    torch.from_numpy(sr), xp)

        def expert_ffn(rows, local_offsets, lo, hi):
            n = np.diff(local_offsets.numpy())
            row_expert = (lo + np.repeat(np.arange(hi - lo), n)).astype(np.int32)
            if rows.shape[0] == 0:
                return torch.zeros(0, sh.d, dtype=torch.float64)
            return torch.from_numpy(oracle.expert_rows(inp.w_gate, inp.w_up, inp.w_down,
                                                       row_expert, rows))

        def combine(x, y_perm, idx, gate, slot_row):
            return torch.from_numpy(oracle.combine(x, y_perm, idx.numpy(), gate,
                                                   slot_row.numpy(), N, sh.routed_scale))

        out, plan = ep.ep_layer_step(rank, bounds, inp.x, route, dispatch, expert_ffn,
                                     combine, dist.all_to_all_single)
        ref, _, _ = oracle.layer(inp.x, inp.w_router, inp.bias, inp.w_gate, inp.w_up,
                                 inp.w_down, N, k, sh.routed_scale)
        # the token ids behind this rank's regrouped rows, as global ids
        # (source * T + token): what the rank received, in expert-major order
        row_tok = plan["row_token"]
        R = int(plan["offsets"][-1])
        send_tok = [row_tok[int(plan["offsets"][bounds[r]]):int(plan["offsets"][bounds[r + 1]])]
                    + rank * sh.T for r in range(WORLD)]
        got_tok = ep.exchange_rows(torch.cat(send_tok).to(torch.int64).unsqueeze(1),
                                   plan["send"], plan["recv"],
                                   dist.all_to_all_single).squeeze(1)
        regrouped = got_tok[plan["perm"]]
        q.put((rank, {"err": float(np.max(np.abs(out.numpy() - ref))),
                      "scale": float(np.max(np.abs(ref))),
                      "send": plan["send"], "recv": plan["recv"],
                      "R": R, "T": sh.T, "k": k,
                      "regrouped": regrouped.tolist(),
                      "local_offsets": plan["local_offsets"].tolist(),
                      "idx": route(inp.x)[0].numpy().tolist()}))
        dist.barrier()
        dist.destroy_process_group()
    except Exception as e:  # noqa: BLE001 - reported to the parent
        import traceback
        q.put((rank, "exception: " + repr(e) + traceback.format_exc()))


def test_two_rank_exchange_matches_the_oracle():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    ps = [ctx.Process(target=_worker, args=(r, port, q)) for r in range(WORLD)]
    for p in ps:
        p.start()
    res = {}
    for _ in range(WORLD):
        rank, val = q.get(timeout=240)
        res[rank] = val
    for p in ps:
        p.join(timeout=60)
    for r in range(WORLD):
        assert isinstance(res[r], dict), res[r]
    import oracle
    sh = _shape()
    N, E = sh.n_routed, sh.E
    bounds = ep.expert_bounds(N, WORLD)
    # the whole job's dispatch: both batches, rank 0's tokens first
    idx_all = np.concatenate([np.array(res[r]["idx"], np.int32) for r in range(WORLD)])
    c, o, rt, _ = oracle.dispatch(idx_all, N, E)
    for r in range(WORLD):
        v = res[r]
        # the gates cross to combine in fp32, as the library passes them
        assert v["err"] <= 1e-6 * max(v["scale"], 1.0)
        # what rank r sends is what each destination receives from it
        for s in range(WORLD):
            assert res[s]["recv"][r] == v["send"][s]
        # sends hold routed rows only: zero-expert slots stay home
        own_idx = np.array(v["idx"])
        assert sum(v["send"]) == int((own_idx < N).sum()) == v["R"]
        # rank r's regrouped rows are the global dispatch's rows of its experts
        lo, hi = bounds[r], bounds[r + 1]
        np.testing.assert_array_equal(np.array(v["regrouped"]), rt[o[lo]:o[hi]])
        np.testing.assert_array_equal(np.array(v["local_offsets"]), o[lo:hi + 1] - o[lo])
        np.testing.assert_array_equal(np.diff(v["local_offsets"]), c[lo:hi])


def test_plan_arithmetic_on_the_host():
    assert ep.expert_bounds(7, 2) == [0, 4, 7]
    assert ep.expert_bounds(8, 3) == [0, 3, 6, 8]
    assert ep.expert_bounds(2, 4) == [0, 1, 2, 2, 2]  # ranks with no experts
    assert [ep.owner_of(e, [0, 3, 6, 8]) for e in range(8)] == [0, 0, 0, 1, 1, 1, 2, 2]
    with pytest.raises(ValueError):
        ep.owner_of(8, [0, 3, 6, 8])  # a zero expert has no owner
    offsets = torch.tensor([0, 2, 2, 5, 9, 9, 12, 12, 15], dtype=torch.int32)
    assert ep.send_splits(offsets, [0, 3, 6, 8]) == [5, 7, 3]
    counts = torch.tensor([2, 0, 3, 4, 0, 3, 0, 3, 5, 5], dtype=torch.int32)
    sc = ep.send_counts(counts, [0, 3, 6, 8])
    assert sc.tolist() == [[2, 0, 3], [4, 0, 3], [0, 3, 0]]
    # received blocks of 2 sources for 3 local experts, empty blocks included
    rc = torch.tensor([[1, 0, 2], [2, 1, 0]])
    perm, loc = ep.regroup_plan(rc, 3)
    # received order: s0e0 [0], s0e2 [1, 2], s1e0 [3, 4], s1e1 [5]
    assert perm.tolist() == [0, 3, 4, 5, 1, 2]
    assert loc.tolist() == [0, 3, 4, 6]
    assert ep.inverse(perm)[perm].tolist() == list(range(6))
    perm, loc = ep.regroup_plan(torch.zeros(2, 3, dtype=torch.int64), 3)
    assert perm.numel() == 0 and loc.tolist() == [0, 0, 0, 0]
