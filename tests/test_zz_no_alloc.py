"""moe_route_noalloc, the router call for callers that cannot allocate device
memory (for instance code running inside a pool or allocator that owns the
whole device). It takes only inputs and outputs and keeps its scratch in a
fixed array inside the library, so it is compared here with moe_route, the
workspace-based call, on two calls in a row (the second call reuses the
array as the first left it). Its refusal of problems beyond the array is a
host-side check and is tested without a GPU in test_api_cpu.py.

This file is collected last so that a stop at the first failure has already
run every other test; it also passes on its own in a fresh process.
"""
import numpy as np
import pytest
import torch

import expert_routing_dispatch_router_b200 as moe
from moe_synth import MoEShape, make_inputs
from parity_helpers import GATE_ATOL, LOGIT_RTOL

pytestmark = pytest.mark.gpu
DEV = "cuda"

CASES = [
    MoEShape("noalloc_decode", T=64, d=4096, n_routed=128, n_zero=32, top_k=8, ffn=1024),
    MoEShape("noalloc_big", T=1536, d=1024, n_routed=40, n_zero=8, top_k=6, ffn=256),
    # T * E = 2,621,440: the partial sums fill most of the 16 MiB array
    MoEShape("noalloc_one_split", T=16384, d=1024, n_routed=128, n_zero=32, top_k=8,
             ffn=256),
]


@pytest.mark.parametrize("sh", CASES, ids=lambda s: s.name)
def test_route_noalloc_matches_route_twice(sh):
    inp = make_inputs(sh, 21, with_experts=False)
    ls = moe.LayerShape(sh.T, sh.d, sh.n_routed, sh.n_zero, sh.top_k, sh.ffn)
    d = inp.to(DEV)
    ws = moe.alloc_workspace(ls)
    ref_logits = torch.empty(sh.T, sh.E, dtype=torch.float32, device=DEV)
    ref_flags = torch.empty(sh.T, dtype=torch.uint8, device=DEV)
    ref_idx, ref_gate = moe.route(ls, d.x, d.w_router, d.bias, ws, logits=ref_logits,
                                  flags=ref_flags)
    torch.cuda.synchronize()
    rl = ref_logits.double().cpu().numpy()
    clear = ref_flags.cpu().numpy() == 0
    for _ in range(2):
        idx = torch.full((sh.T, sh.top_k), -1, dtype=torch.int32, device=DEV)
        gate = torch.zeros(sh.T, sh.top_k, dtype=torch.float32, device=DEV)
        logits = torch.zeros(sh.T, sh.E, dtype=torch.float32, device=DEV)
        moe.route_noalloc(ls, d.x, d.w_router, d.bias, idx, gate, logits=logits)
        torch.cuda.synchronize()
        gl = logits.double().cpu().numpy()
        assert np.all(np.abs(gl - rl) <= LOGIT_RTOL * np.maximum(np.abs(rl), 1.0))
        a = np.sort(idx.cpu().numpy()[clear], axis=1)
        b = np.sort(ref_idx.cpu().numpy()[clear], axis=1)
        np.testing.assert_array_equal(a, b)
        ga = np.take_along_axis(gate.cpu().numpy()[clear],
                                np.argsort(idx.cpu().numpy()[clear], axis=1), axis=1)
        gb = np.take_along_axis(ref_gate.cpu().numpy()[clear],
                                np.argsort(ref_idx.cpu().numpy()[clear], axis=1), axis=1)
        assert np.max(np.abs(ga - gb)) <= GATE_ATOL
