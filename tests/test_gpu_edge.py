"""GPU edge cases of the layer, each against the oracle or an exact property:
T = 0 and T = 1, every slot on zero experts (R = 0: the expert GEMMs launch no work),
every token on one expert, segment sizes around the 128-row token tile,
only zero experts (N = 0), no zero experts (Z = 0), k = E, the largest
supported E and k, and the device-side wait limit (a wait that nothing
completes reports error 1 and leaves the context usable)."""
import time

import numpy as np
import pytest
import torch

import expert_routing_dispatch_router_b200 as moe
import oracle
from moe_synth import MoEShape, make_inputs
from parity_helpers import OUT_RTOL_RMS, out_err

pytestmark = pytest.mark.gpu
DEV = "cuda"


def shape_of(sh, dtype=torch.bfloat16, s=1.0):
    return moe.LayerShape(sh.T, sh.d, sh.n_routed, sh.n_zero, sh.top_k, sh.ffn, dtype, s)


def fused(sh, inp, s=1.0):
    ls = shape_of(sh, inp.x.dtype, s)
    d = inp.to(DEV)
    ws = moe.alloc_workspace(ls)
    counts = torch.empty(sh.E, dtype=torch.int32, device=DEV)
    out = moe.layer_forward(ls, d.x, d.w_router, d.bias, d.w_gate, d.w_up, d.w_down,
                            ws, counts=counts)
    torch.cuda.synchronize()
    assert moe.read_device_error(ws) == 0
    return out.cpu(), counts.cpu().numpy()


def check_layer(sh, inp, s=1.0):
    out, counts = fused(sh, inp, s)
    ref, idx, _ = oracle.layer(inp.x, inp.w_router, inp.bias, inp.w_gate, inp.w_up,
                               inp.w_down, sh.n_routed, sh.top_k, s)
    assert counts.sum() == sh.T * sh.top_k
    np.testing.assert_array_equal(counts, np.bincount(idx.ravel(), minlength=sh.E))
    assert out_err(out.double().numpy(), ref, inp.x.dtype) <= OUT_RTOL_RMS
    return out, counts


BASE = MoEShape("edge", T=200, d=256, n_routed=16, n_zero=4, top_k=4, ffn=256)


def test_single_token():
    sh = MoEShape("t1", T=1, d=256, n_routed=16, n_zero=4, top_k=4, ffn=256)
    check_layer(sh, make_inputs(sh, 3))


def test_all_slots_to_zero_experts_returns_input():
    sh = BASE
    inp = make_inputs(sh, 4)
    inp.bias[sh.n_routed:] += 1e3
    out, counts = fused(sh, inp, s=9.0)
    assert counts[: sh.n_routed].sum() == 0
    # out = sum_j g_j x with sum_j g_j = 1 (fp32), rounded once: x itself, up to
    # one bf16 rounding step
    diff = (out.float() - inp.x.float()).abs()
    assert float((diff / inp.x.float().abs().clamp_min(1e-30)).max()) <= 2 ** -8


def test_all_tokens_to_one_expert_multiple_tiles():
    sh = MoEShape("one", T=300, d=256, n_routed=4, n_zero=2, top_k=1, ffn=256)
    inp = make_inputs(sh, 5)
    inp.bias[2] += 1e3
    out, counts = check_layer(sh, inp)
    assert counts[2] == 300


PAIRS = MoEShape("pairs_edge", T=1100, d=512, n_routed=6, n_zero=2, top_k=2, ffn=512)


def test_pairs_all_tokens_to_one_expert():
    # T > 1024: CTA pairs; one expert gets every token (9 token tiles x 2
    # weight tiles, all taken from the unit counter by whichever pair is free)
    inp = make_inputs(PAIRS, 12)
    inp.bias[3] += 1e3
    out, counts = check_layer(PAIRS, inp)
    assert counts[3] == PAIRS.T


def test_pairs_no_routed_slots():
    # CTA pairs with no work at all: the first unit handed out is the end mark
    inp = make_inputs(PAIRS, 13)
    inp.bias[PAIRS.n_routed:] += 1e3
    out, counts = fused(PAIRS, inp)
    assert counts[: PAIRS.n_routed].sum() == 0
    diff = (out.float() - inp.x.float()).abs()
    assert float((diff / inp.x.float().abs().clamp_min(1e-30)).max()) <= 2 ** -8


@pytest.mark.parametrize("sizes,F", [((1, 127, 128, 129, 0, 256, 3), 384),
                                     ((255, 0, 0, 1, 17, 384, 64), 384),
                                     # T > 1024: both GEMMs run on CTA pairs
                                     ((1, 31, 32, 33, 255, 256, 257, 300), 512),
                                     ((0, 600, 0, 1, 520), 512),
                                     # T > 1024 with F = 384 (not a multiple of
                                     # 256): single-CTA GEMMs with 256-token
                                     # tiles, segments around 1 and 2 tiles and
                                     # one expert cut into 33 tiles
                                     ((287, 288, 289, 511, 512, 513, 1025), 384),
                                     ((8200, 3, 0, 700), 384)])
def test_expert_segments_around_tile_size(sizes, F):
    """moe_expert_ffn on crafted segments: offsets give exactly these rows per
    expert; rows are random bf16; checked row by row against the oracle."""
    N, d = len(sizes), 256
    sh = MoEShape("seg", T=sum(sizes), d=d, n_routed=N, n_zero=1, top_k=1, ffn=F)
    inp = make_inputs(sh, 6)
    ls = shape_of(sh)
    R = sum(sizes)
    g = torch.Generator().manual_seed(11)
    x_perm = torch.randn(R, d, generator=g).to(torch.bfloat16)
    offsets = torch.tensor(np.concatenate([[0], np.cumsum(sizes)]), dtype=torch.int32)
    ws = moe.alloc_workspace(ls)
    y = moe.expert_ffn(ls, x_perm.to(DEV), offsets.to(DEV), inp.w_gate.to(DEV),
                       inp.w_up.to(DEV), inp.w_down.to(DEV), ws)
    torch.cuda.synchronize()
    assert moe.read_device_error(ws) == 0
    row_expert = np.repeat(np.arange(N), sizes).astype(np.int32)
    ref = oracle.expert_rows(inp.w_gate, inp.w_up, inp.w_down, row_expert, x_perm)
    assert out_err(y.double().cpu().numpy(), ref, torch.bfloat16) <= OUT_RTOL_RMS  # y in bf16


def test_only_zero_experts():
    sh = MoEShape("z", T=50, d=128, n_routed=0, n_zero=6, top_k=3, ffn=128)
    inp = make_inputs(sh, 7, with_experts=False)
    ls = shape_of(sh)
    d = inp.to(DEV)
    ws = moe.alloc_workspace(ls)
    out = moe.layer_forward(ls, d.x, d.w_router, d.bias, None, None, None, ws)
    torch.cuda.synchronize()
    diff = (out.cpu().float() - inp.x.float()).abs()
    assert float((diff / inp.x.float().abs().clamp_min(1e-30)).max()) <= 2 ** -8


def test_no_zero_experts():
    sh = MoEShape("nz", T=150, d=256, n_routed=8, n_zero=0, top_k=2, ffn=128)
    check_layer(sh, make_inputs(sh, 8))


def test_k_equals_E():
    sh = MoEShape("kE", T=40, d=128, n_routed=5, n_zero=3, top_k=8, ffn=128)
    check_layer(sh, make_inputs(sh, 9))


def test_max_experts_and_topk():
    sh = MoEShape("maxE", T=70, d=128, n_routed=1000, n_zero=24, top_k=32, ffn=128)
    inp = make_inputs(sh, 10)
    check_layer(sh, inp)


def test_host_entry_point_matches_device_entry_point():
    sh = BASE
    inp = make_inputs(sh, 12)
    ls = shape_of(sh)
    d = inp.to(DEV)
    ws = moe.alloc_workspace(ls)
    out_dev = moe.layer_forward(ls, d.x, d.w_router, d.bias, d.w_gate, d.w_up,
                                d.w_down, ws)
    x_host = inp.x.clone().pin_memory()
    out_host = torch.empty(sh.T, sh.d, dtype=torch.bfloat16).pin_memory()
    counts_host = torch.empty(sh.E, dtype=torch.int32).pin_memory()
    moe.layer_forward_host(ls, x_host, d.w_router, d.bias, d.w_gate, d.w_up, d.w_down,
                           ws, out_host, counts_host)
    torch.cuda.synchronize()
    assert torch.equal(out_host, out_dev.cpu())
    assert int(counts_host.sum()) == sh.T * sh.top_k


def test_bad_expert_id_is_reported_not_written():
    sh = BASE
    inp = make_inputs(sh, 13, with_experts=False)
    ls = shape_of(sh)
    ws = moe.alloc_workspace(ls)
    idx = torch.stack([torch.arange(4)] * sh.T).int()
    idx[5, 2] = sh.E + 7  # out of range
    idx[9, 1] = idx[9, 0]  # repeated inside one token
    counts, offsets, row_token, slot_row, _ = moe.dispatch(ls, inp.x.to(DEV), idx.to(DEV), ws)
    torch.cuda.synchronize()
    assert moe.read_device_error(ws) == 2
    assert moe.read_device_error(ws) == 0  # cleared by the read
    assert int(slot_row.view(sh.T, 4)[5, 2]) == -1


def test_router_exact_ties_go_to_lower_id():
    """Experts 3..12 share one router row and one bias, so their keys tie
    exactly (the same dot product in the same order on both sides): the
    selection must take the lowest ids among them, in id order."""
    sh = MoEShape("ties", T=96, d=256, n_routed=12, n_zero=4, top_k=6, ffn=128)
    inp = make_inputs(sh, 14, with_experts=False)
    inp.w_router[3:13] = inp.w_router[3]
    inp.bias[3:13] = 50.0  # the tied group is always selected first
    ls = shape_of(sh)
    d = inp.to(DEV)
    ws = moe.alloc_workspace(ls)
    idx, gate = moe.route(ls, d.x, d.w_router, d.bias, ws)
    torch.cuda.synchronize()
    _, ref_idx, ref_gate, _ = oracle.route(inp.x, inp.w_router, inp.bias, sh.top_k)
    np.testing.assert_array_equal(idx.cpu().numpy(), ref_idx)
    np.testing.assert_array_equal(ref_idx, np.tile(np.arange(3, 9), (sh.T, 1)))
    np.testing.assert_allclose(gate.cpu().numpy(), 1.0 / 6, rtol=1e-6)


def test_empty_batch():
    # T = 0 through every binding call: empty outputs, no launch, no device
    # error; the same workspace then serves a real batch of the same layer
    sh = MoEShape("empty", T=0, d=256, n_routed=8, n_zero=2, top_k=2, ffn=256)
    inp = make_inputs(sh, 15)
    ls = shape_of(sh)
    d = inp.to(DEV)
    ws = moe.alloc_workspace(ls)
    idx, gate = moe.route(ls, d.x, d.w_router, d.bias, ws)
    assert idx.shape == (0, 2) and gate.shape == (0, 2)
    counts, offsets, row_token, slot_row, x_perm = moe.dispatch(ls, d.x, idx, ws)
    y = moe.expert_ffn(ls, x_perm, offsets, d.w_gate, d.w_up, d.w_down, ws)
    out = moe.combine(ls, d.x, y, idx, gate, slot_row)
    assert out.shape == (0, sh.d)
    out = moe.layer_forward(ls, d.x, d.w_router, d.bias, d.w_gate, d.w_up, d.w_down, ws)
    assert out.shape == (0, sh.d)
    torch.cuda.synchronize()
    assert moe.read_device_error(ws) == 0
    full = MoEShape("after_empty", T=24, d=256, n_routed=8, n_zero=2, top_k=2, ffn=256)
    check_layer(full, make_inputs(full, 16))


def test_wait_limit_reports_and_context_stays_usable():
    # a wait that nothing completes runs out after its limit: error 1 in the
    # workspace, read on the host; then the same context runs a layer cleanly
    sh = MoEShape("after_timeout", T=40, d=256, n_routed=4, n_zero=2, top_k=2, ffn=256)
    ls = moe.LayerShape(sh.T, sh.d, sh.n_routed, sh.n_zero, sh.top_k, sh.ffn)
    ws = moe.alloc_workspace(ls)
    t0 = time.time()
    moe.selftest_wait_limit(ws)
    assert moe.read_device_error(ws) == 1
    assert 1.5 < time.time() - t0 < 30.0
    assert moe.read_device_error(ws) == 0  # read clears it
    inp = make_inputs(sh, 3)
    d = inp.to("cuda")
    out = moe.layer_forward(ls, d.x, d.w_router, d.bias, d.w_gate, d.w_up, d.w_down, ws)
    torch.cuda.synchronize()
    assert moe.read_device_error(ws) == 0
    ref, _, _ = oracle.layer(inp.x, inp.w_router, inp.bias, inp.w_gate, inp.w_up, inp.w_down,
                             sh.n_routed, sh.top_k)
    assert out_err(out.double().cpu().numpy(), ref, inp.x.dtype) <= OUT_RTOL_RMS
