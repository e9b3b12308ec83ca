"""Expert parallelism across GPUs: the exchange plan of the layer when the
routed experts are split over G ranks, one process per GPU.

The pages' decode deployment shards the experts over 128 cards (Ascend
deployment article, "Decode节点：EP128超大专家并行"), with data parallelism over
tokens beside it (same article, "多场景模型分层切分优化", DP128 + EP128), and
zero-expert-aware Dispatch/Combine operators that move token rows between
cards (same article, "底层定制算子深度优化"). This module holds the host side of
that exchange; the layer's arithmetic stays in the CUDA library (route,
dispatch, expert FFN and combine are its entry points), and the exchange is two
all-to-all-v collectives (NCCL over NVLink on GPUs, gloo on the CPU tests).

Ownership: rank r owns the routed experts [bounds[r], bounds[r + 1]), an even
split of the N routed ids (the first N % G ranks take one more). Zero experts
belong to no rank: their slots never leave the token's own rank, and the
identity term is added by that rank's combine.

One step on rank s (every rank runs the same steps in the same order):
 1. route and dispatch its own T tokens locally: x_perm holds the routed rows
    in (expert, token) order and offsets[e] is where expert e's rows start.
    Because each rank's experts form one contiguous id range, the rows bound
    for rank r are the single block x_perm[offsets[bounds[r]] :
    offsets[bounds[r + 1]]]; zero-expert slots are in no block.
 2. exchange the per-expert counts of each block (an all-to-all of
    G x n_local integers), so every rank knows how many rows of each of its
    experts each source sends;
 3. all-to-all-v of the row blocks: rank r receives, source by source, the
    rows of its experts in (source, expert, token) order;
 4. regroup the received rows expert-major, (expert, source, token), and run
    the grouped expert FFN on them with the local offsets;
 5. put the outputs back in received order and send each block home with the
    reverse all-to-all-v (split sizes swapped);
 6. each source now holds y_perm in its own dispatch order and combines it
    with its gates, slot rows and the identity term, as on one GPU.

The functions below compute the plan (split sizes, the regrouping permutation
and local offsets) from the counts the dispatch step already returns, so the
plan costs no extra pass over the token rows.

The library's device calls (moe_ep_plan, moe_ep_dispatch, moe_ep_return) do
the same exchange without the all-to-all and without the regrouping pass:
once every rank's per-expert counts and offsets are gathered (G x E and
G x (N + 1) integers), each rank knows where each of its rows lands in its
owner's receive buffer, already expert-major, and writes it there (peer
stores on one node); the owners send the expert outputs back the same way.
`run_ranks_on_one_device` runs that sequence for G ranks on one GPU.
"""
from __future__ import annotations

from typing import Callable, List, Sequence

import torch


def expert_bounds(n_routed: int, world: int) -> List[int]:
    """bounds[r] .. bounds[r + 1] are rank r's routed expert ids."""
    if world <= 0 or n_routed < 0:
        raise ValueError("world must be positive and n_routed non-negative")
    base, extra = divmod(n_routed, world)
    b = [0]
    for r in range(world):
        b.append(b[-1] + base + (1 if r < extra else 0))
    return b


def owner_of(expert: int, bounds: Sequence[int]) -> int:
    """Rank owning routed expert `expert` (bounds from expert_bounds)."""
    for r in range(len(bounds) - 1):
        if bounds[r] <= expert < bounds[r + 1]:
            return r
    raise ValueError(f"expert {expert} is not a routed expert")


def send_splits(offsets: torch.Tensor, bounds: Sequence[int]) -> List[int]:
    """Rows of x_perm bound for each rank: the routed rows of its experts.

    offsets [N + 1] int32 as returned by the dispatch (host copy)."""
    o = offsets.tolist()
    return [int(o[bounds[r + 1]] - o[bounds[r]]) for r in range(len(bounds) - 1)]


def send_counts(counts: torch.Tensor, bounds: Sequence[int]) -> torch.Tensor:
    """Per-expert counts of every block, laid out for an all-to-all: entry
    [r, j] is the number of rows this rank sends to rank r for r's j-th local
    expert (j < n_local_max; padded with zeros where rank r owns fewer)."""
    G = len(bounds) - 1
    n_max = max(bounds[r + 1] - bounds[r] for r in range(G))
    out = torch.zeros(G, n_max, dtype=torch.int64)
    for r in range(G):
        n = bounds[r + 1] - bounds[r]
        out[r, :n] = counts[bounds[r]:bounds[r + 1]].to(torch.int64)
    return out


def regroup_plan(recv_counts: torch.Tensor, n_local: int):
    """Plan of the received rows of one rank.

    recv_counts [G, n_max]: rows each source sent for each local expert, the
    blocks arriving source by source, each in (expert, token) order. Returns
    (perm, local_offsets): perm[i] is the received row that becomes row i of
    the expert-major order (expert, source, token), and local_offsets
    [n_local + 1] are the expert segments of that order (the offsets the
    grouped expert FFN takes)."""
    rc = recv_counts[:, :n_local].to(torch.int64)
    G = rc.shape[0]
    # start of block (s, e) in the received buffer
    src_start = torch.zeros(G, dtype=torch.int64)
    if G > 1:
        src_start[1:] = torch.cumsum(rc.sum(dim=1), 0)[:-1]
    within = torch.zeros_like(rc)
    if n_local > 1:
        within[:, 1:] = torch.cumsum(rc, dim=1)[:, :-1]
    perm_parts = []
    for e in range(n_local):
        for s in range(G):
            n = int(rc[s, e])
            if n:
                a = int(src_start[s] + within[s, e])
                perm_parts.append(torch.arange(a, a + n, dtype=torch.int64))
    total = int(rc.sum())
    perm = torch.cat(perm_parts) if perm_parts else torch.zeros(0, dtype=torch.int64)
    assert perm.numel() == total
    local_offsets = torch.zeros(n_local + 1, dtype=torch.int32)
    if n_local:
        local_offsets[1:] = torch.cumsum(rc.sum(dim=0), 0).to(torch.int32)
    return perm, local_offsets


def inverse(perm: torch.Tensor) -> torch.Tensor:
    inv = torch.empty_like(perm)
    inv[perm] = torch.arange(perm.numel(), dtype=perm.dtype)
    return inv


def exchange_rows(rows: torch.Tensor, send: Sequence[int], recv: Sequence[int],
                  all_to_all_single: Callable) -> torch.Tensor:
    """all-to-all-v of row blocks: send[r] rows go to rank r, recv[r] rows come
    from rank r (the collective is passed in: torch.distributed's, on NCCL or
    gloo)."""
    out = torch.empty((int(sum(recv)),) + tuple(rows.shape[1:]), dtype=rows.dtype,
                      device=rows.device)
    all_to_all_single(out, rows.contiguous(), list(recv), list(send))
    return out


def exchange_counts(cnt: torch.Tensor, all_to_all_single: Callable) -> torch.Tensor:
    """all-to-all of the [G, n_max] per-expert counts: row r goes to rank r,
    and row s of the result came from rank s."""
    out = torch.empty_like(cnt)
    all_to_all_single(out, cnt.contiguous())
    return out


def ep_layer_step(rank: int, bounds: Sequence[int], x: torch.Tensor,
                  route: Callable, dispatch: Callable, expert_ffn: Callable,
                  combine: Callable, all_to_all_single: Callable):
    """One expert-parallel layer step on this rank, with the compute steps
    passed in (on GPUs: the library's moe_route, moe_dispatch, moe_expert_ffn
    over this rank's experts, moe_combine).

      route(x) -> (idx [T, k] int32, gate [T, k] float32)
      dispatch(x, idx) -> (counts [E], offsets [N + 1], row_token, slot_row,
                           x_perm [T*k, d]) with rows in (expert, token) order
      expert_ffn(rows [n, d], local_offsets [n_local + 1], lo, hi) -> y [n, d]
        over experts lo..hi-1 (local expert j is global expert lo + j)
      combine(x, y_perm [T*k, d], idx, gate, slot_row) -> out [T, d]

    Returns (out, plan) where plan holds the split sizes and counts, for
    checks."""
    G = len(bounds) - 1
    idx, gate = route(x)
    counts, offsets, row_token, slot_row, x_perm = dispatch(x, idx)
    offs = offsets.to("cpu")
    send = send_splits(offs, bounds)
    cnt = send_counts(counts.to("cpu"), bounds)
    recv_cnt = exchange_counts(cnt.to(x.device), all_to_all_single).to("cpu")
    lo, hi = bounds[rank], bounds[rank + 1]
    n_local = hi - lo
    recv = [int(recv_cnt[s, :n_local].sum()) for s in range(G)]
    R = int(offs[-1])
    start = int(offs[bounds[0]])
    sent_rows = x_perm[start:start + R]
    got = exchange_rows(sent_rows, send, recv, all_to_all_single)
    perm, local_offsets = regroup_plan(recv_cnt, n_local)
    p = perm.to(x.device)
    y_local = expert_ffn(got.index_select(0, p), local_offsets.to(x.device), lo, hi)
    y_recv = torch.empty_like(y_local)
    y_recv.index_copy_(0, p, y_local)
    y_home = exchange_rows(y_recv, recv, send, all_to_all_single)
    y_perm = torch.zeros((x_perm.shape[0],) + tuple(y_home.shape[1:]), dtype=y_home.dtype,
                         device=y_home.device)
    y_perm[start:start + R] = y_home
    out = combine(x, y_perm, idx, gate, slot_row)
    plan = {"send": send, "recv": recv, "send_counts": cnt, "recv_counts": recv_cnt,
            "perm": perm, "local_offsets": local_offsets, "counts": counts.to("cpu"),
            "offsets": offs, "row_token": row_token.to("cpu")}
    return out, plan


def run_ranks_on_one_device(shape, xs, w_router, bias, w_gate, w_up, w_down):
    """Every rank's expert-parallel step with the library's device calls, the
    ranks run one after another on the current device, each phase one call per
    rank (so no kernel waits on another). On a node of G GPUs the same calls
    run one rank per GPU, with the gathers of counts and offsets as
    collectives, the receive buffers and y_perm as peer memory, and a barrier
    between the phases.

    shape: the per-rank layer (T tokens per rank); xs: G token batches.
    Returns (outs, info): every rank's layer output, and the plan and the
    receive buffers for checks."""
    import expert_routing_dispatch_router_b200 as moe

    G = len(xs)
    T, k, d, N, F = shape.T, shape.top_k, shape.d, shape.n_routed, shape.ffn
    dev = xs[0].device
    # 1. route and dispatch locally
    local = []
    for s in range(G):
        ws = moe.alloc_workspace(shape, dev)
        idx, gate = moe.route(shape, xs[s], w_router, bias, ws)
        counts, offsets, row_token, slot_row, _ = moe.dispatch(shape, xs[s], idx, ws)
        local.append({"idx": idx, "gate": gate, "counts": counts, "offsets": offsets,
                      "row_token": row_token, "slot_row": slot_row})
    # 2. the gathers (a collective on several GPUs)
    counts_all = torch.stack([p["counts"] for p in local]).contiguous()
    offsets_all = torch.stack([p["offsets"] for p in local]).contiguous()
    # 3. plans and the dispatch into the owners' receive buffers
    cap = G * T * k
    recv = [torch.zeros(cap, d, dtype=shape.act_dtype, device=dev) for _ in range(G)]
    recv_offsets, keep = [], []
    for s in range(G):
        dest_row, roff = moe.ep_plan(shape, s, G, counts_all)
        recv_offsets.append(roff)
        keep.append(moe.ep_dispatch(shape, G, xs[s], local[s]["offsets"],
                                    local[s]["row_token"], dest_row, recv))
    # 4. each owner's expert FFN over its receive buffer and its experts
    y_recv = []
    lo = 0
    for r in range(G):
        n_r = moe.ep_local_experts(shape, r, G)
        if n_r == 0:
            y_recv.append(torch.zeros(cap, d, dtype=shape.act_dtype, device=dev))
            continue
        sh_r = moe.LayerShape(G * T, d, n_r, shape.n_zero, k, F, shape.act_dtype,
                              shape.routed_scale)
        ws_r = moe.alloc_workspace(sh_r, dev)
        y_recv.append(moe.expert_ffn(sh_r, recv[r], recv_offsets[r], w_gate[lo:lo + n_r],
                                     w_up[lo:lo + n_r], w_down[lo:lo + n_r], ws_r))
        lo += n_r
    # 5. the outputs back to their sources, 6. combine as on one GPU
    y_perm = [torch.zeros(T * k, d, dtype=shape.act_dtype, device=dev) for _ in range(G)]
    for r in range(G):
        keep.append(moe.ep_return(shape, r, G, y_recv[r], recv_offsets[r], counts_all,
                                  offsets_all, y_perm))
    outs = [moe.combine(shape, xs[s], y_perm[s], local[s]["idx"], local[s]["gate"],
                        local[s]["slot_row"]) for s in range(G)]
    torch.cuda.synchronize(dev)
    return outs, {"local": local, "counts_all": counts_all, "offsets_all": offsets_all,
                  "recv": recv, "recv_offsets": recv_offsets, "y_perm": y_perm}
