"""GPU parity: every stage of the CUDA library against the CPU oracle on the
same seeded inputs, through the C ABI (Python binding = marshalling only).

Staged calls are fed the ORACLE's outputs of the previous stage (never the
GPU's), so each stage is compared on identical inputs. The fused layer is
compared end to end. Small cases span several tiles and ragged tails; the
named workloads run at full size, with the expert FFN checked on a seeded
sample of tokens/rows that the oracle computes one by one.
"""
import numpy as np
import pytest
import torch

import expert_routing_dispatch_router_b200 as moe
import oracle
from moe_synth import CONFIGS, MoEShape, get_config, make_inputs, torch_dtype
from parity_helpers import (OUT_RTOL_RMS, alternative_selection, assert_logits_close,
                            compare_selection, out_err)

pytestmark = pytest.mark.gpu

DEV = "cuda"


def layer_shape(sh: MoEShape, s=None) -> moe.LayerShape:
    return moe.LayerShape(sh.T, sh.d, sh.n_routed, sh.n_zero, sh.top_k, sh.ffn,
                          torch_dtype(sh.act_dtype),
                          sh.routed_scale if s is None else s)


SMALL = [
    # several 128-row token tiles and ragged tails; F, d multiples of 128 -> tcgen05
    MoEShape("small_bf16", T=300, d=256, n_routed=6, n_zero=2, top_k=3, ffn=384),
    # skewed: one expert gets most tokens (multiple token tiles per expert)
    MoEShape("skew_bf16", T=517, d=384, n_routed=5, n_zero=3, top_k=2, ffn=256,
             routing="zipf"),
    # T > 1024 with d, F multiples of 256 -> the expert GEMMs run on CTA pairs
    MoEShape("pairs_bf16", T=1100, d=512, n_routed=8, n_zero=2, top_k=4, ffn=512,
             routing="zipf"),
    # d, F not multiples of 128 -> CUDA-core path in bf16
    MoEShape("odd_bf16", T=77, d=200, n_routed=4, n_zero=1, top_k=2, ffn=136),
    CONFIGS["tiny_fp32"],
]


def stratified_rows(r_counts, r_offsets, N, seed, n_sub=48, n_full=2):
    """Rows of y_perm (dispatch order) to check at sizes where the oracle
    cannot compute them all. The expert GEMMs cut an expert's segment into
    token tiles of 64, 128 or 256 rows (the batch size decides), and a CTA pair
    splits each tile in halves. The sample holds:
      * for every touched expert, the first and last row of its segment and
        its last partial 256-row tile (whole up to 16 rows, else its first and
        last 8);
      * for n_sub seeded experts, the first and last row of every 128- and
        256-row tile and the last partial 128-row tile (same rule);
      * every row of the first and last 256-row tiles of the most loaded
        expert (the Zipf-hot one under skewed routing) and of n_full seeded
        others.
    """
    rows = set()
    touched = np.nonzero(r_counts[:N])[0]
    rng = np.random.default_rng(seed)
    sub = {int(e) for e in rng.choice(touched, size=min(n_sub, touched.size), replace=False)}

    def tail_of(o, n, tile):
        t = list(range(o + ((n - 1) // tile) * tile, o + n))
        return t if len(t) <= 16 else t[:8] + t[-8:]

    for e in touched:
        o, n = int(r_offsets[e]), int(r_counts[e])
        rows.update((o, o + n - 1))
        rows.update(tail_of(o, n, 256))
        if int(e) in sub:
            for tile in (128, 256):
                for t in range((n + tile - 1) // tile):
                    rows.update((o + t * tile, min(o + n, o + (t + 1) * tile) - 1))
            rows.update(tail_of(o, n, 128))
    hot = int(touched[np.argmax(r_counts[touched])])
    full = {hot} | {int(e) for e in rng.choice(touched, size=min(n_full, touched.size),
                                               replace=False)}
    for e in sorted(full):
        o, n = int(r_offsets[e]), int(r_counts[e])
        rows.update(range(o, o + min(n, 256)))
        rows.update(range(o + ((n - 1) // 256) * 256, o + n))
    return np.array(sorted(rows), dtype=np.int64)


def stratified_tokens(rows, r_row_token, ref_idx, N, T, seed, n_tok=48):
    """Tokens whose whole layer output is checked: up to n_tok of the tokens
    behind the stratified rows, 8 seeded others, and up to 8 tokens that send
    a slot to a zero expert (the identity term)."""
    rng = np.random.default_rng(seed + 7)
    behind = np.unique(r_row_token[rows])
    pick = set(rng.choice(behind, size=min(n_tok, behind.size), replace=False).tolist())
    pick |= set(rng.choice(T, size=min(8, T), replace=False).tolist())
    zero_tok = np.nonzero((ref_idx >= N).any(axis=1))[0]
    if zero_tok.size:
        pick |= set(rng.choice(zero_tok, size=min(8, zero_tok.size), replace=False).tolist())
    return np.array(sorted(pick), dtype=np.int64)


def run_staged_and_fused(sh: MoEShape, seed: int, sample=None, s=None):
    """sample=None checks every row and token; sample="strat" checks the
    stratified rows and tokens above."""
    inp = make_inputs(sh, seed)
    ls = layer_shape(sh, s)
    scale = ls.routed_scale
    d_inp = inp.to(DEV)
    ws = moe.alloc_workspace(ls)
    T, k, N, E = sh.T, sh.top_k, sh.n_routed, sh.E

    # ---- router
    ref_logits, ref_idx, ref_gate, ref_margin = oracle.route(inp.x, inp.w_router,
                                                             inp.bias, k)
    logits = torch.empty(T, E, dtype=torch.float32, device=DEV)
    flags = torch.empty(T, dtype=torch.uint8, device=DEV)
    g_idx, g_gate = moe.route(ls, d_inp.x, d_inp.w_router, d_inp.bias, ws,
                              logits=logits, flags=flags)
    torch.cuda.synchronize()
    assert_logits_close(logits, ref_logits)
    flagged = compare_selection(g_idx, g_gate, ref_idx, ref_gate, ref_margin,
                                ref_logits, inp.bias, k)
    fl = flags.cpu().numpy().astype(bool)
    assert not np.any(fl & (ref_margin >= 2 * 1e-4)), "GPU flags a clear margin"
    assert np.all(fl[ref_margin < 5e-5]), "GPU misses a near tie"

    # ---- dispatch, fed the oracle's selection
    r_counts, r_offsets, r_row_token, r_slot_row = oracle.dispatch(ref_idx, N, E)
    R = int(r_offsets[N])
    counts, offsets, row_token, slot_row, x_perm = moe.dispatch(
        ls, d_inp.x, torch.from_numpy(ref_idx).to(DEV), ws)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(counts.cpu().numpy(), r_counts)
    np.testing.assert_array_equal(offsets.cpu().numpy(), r_offsets)
    np.testing.assert_array_equal(row_token.cpu().numpy(), r_row_token)
    np.testing.assert_array_equal(slot_row.cpu().numpy(), r_slot_row)
    assert torch.equal(x_perm[:R].cpu(), inp.x[torch.from_numpy(r_row_token[:R]).long()])

    # ---- expert FFN, fed the oracle's dispatch
    x_perm_ref = torch.zeros(T * k, sh.d, dtype=inp.x.dtype)
    x_perm_ref[:R] = inp.x[torch.from_numpy(r_row_token[:R]).long()]
    y_perm = moe.expert_ffn(ls, x_perm_ref.to(DEV), torch.from_numpy(r_offsets).to(DEV),
                            d_inp.w_gate, d_inp.w_up, d_inp.w_down, ws)
    torch.cuda.synchronize()
    row_expert = np.repeat(np.arange(N), r_counts[:N]).astype(np.int32)
    rows = np.arange(R) if sample is None else stratified_rows(r_counts, r_offsets, N, seed)
    if R > 0:
        y_ref = oracle.expert_rows(inp.w_gate, inp.w_up, inp.w_down, row_expert[rows],
                                   x_perm_ref[torch.from_numpy(rows).long()])
        got = y_perm[torch.from_numpy(rows).long().to(DEV)].double().cpu().numpy()
        # y_perm is stored in the activation dtype, like the layer output
        err = out_err(got, y_ref, inp.x.dtype)
        assert err <= OUT_RTOL_RMS, f"expert rows: max err {err:.3e} x rms beyond half an ulp"

    # ---- combine, fed the oracle's gates and expert outputs (rounded to the
    # activation dtype, as y_perm is stored)
    tok = np.arange(T) if sample is None else stratified_tokens(rows, r_row_token, ref_idx,
                                                                N, T, seed)
    if sample is None and R > 0:
        y_all = oracle.expert_rows(inp.w_gate, inp.w_up, inp.w_down, row_expert,
                                   x_perm_ref[:R])
        y_in = torch.zeros(T * k, sh.d, dtype=inp.x.dtype)
        y_in[:R] = torch.from_numpy(y_all).to(inp.x.dtype)
        gate32 = torch.from_numpy(ref_gate).float()
        out_c = moe.combine(ls, d_inp.x, y_in.to(DEV), torch.from_numpy(ref_idx).to(DEV),
                            gate32.to(DEV), torch.from_numpy(r_slot_row).to(DEV))
        torch.cuda.synchronize()
        ref_c = oracle.combine(inp.x, y_in, ref_idx, gate32, r_slot_row, N, scale)
        # fp32 sums of exact inputs, rounded once: only the output rounding
        err = out_err(out_c.double().cpu().numpy(), ref_c, inp.x.dtype)
        assert err <= 1e-4, f"combine: max err {err:.3e} x rms beyond half an ulp"

    # ---- fused layer
    out = torch.empty(T, sh.d, dtype=inp.x.dtype, device=DEV)
    g_counts = torch.empty(E, dtype=torch.int32, device=DEV)
    moe.layer_forward(ls, d_inp.x, d_inp.w_router, d_inp.bias, d_inp.w_gate,
                      d_inp.w_up, d_inp.w_down, ws, out=out, counts=g_counts)
    torch.cuda.synchronize()
    assert moe.read_device_error(ws) == 0
    gc = g_counts.cpu().numpy()
    assert gc.sum() == T * k
    if not flagged.any():
        np.testing.assert_array_equal(gc, r_counts)
    else:
        assert np.abs(gc - r_counts).sum() <= 2 * int(flagged.sum())
    out_ref, _, _ = oracle.layer(inp.x, inp.w_router, inp.bias, inp.w_gate, inp.w_up,
                                 inp.w_down, N, k, scale, tokens=tok.astype(np.int32))
    got = out[torch.from_numpy(tok).long().to(DEV)].double().cpu().numpy()
    keep = ~flagged[tok]
    err = out_err(got[keep], out_ref[keep], inp.x.dtype)
    assert err <= OUT_RTOL_RMS, f"layer: max err {err:.3e} x rms beyond half an ulp"
    # near-tied tokens must match one of the valid answers
    for n in np.nonzero(~keep)[0]:
        t = int(tok[n])
        alt = ref_idx.copy()
        alt[t] = alternative_selection(ref_logits[t], inp.bias, k)
        alt_out, _, _ = oracle.layer(inp.x, inp.w_router, inp.bias, inp.w_gate,
                                     inp.w_up, inp.w_down, N, k, scale,
                                     tokens=np.array([t], np.int32), force_idx=alt)
        e1 = out_err(got[n:n + 1], out_ref[n:n + 1], inp.x.dtype)
        e2 = out_err(got[n:n + 1], alt_out, inp.x.dtype)
        assert min(e1, e2) <= OUT_RTOL_RMS
    # deterministic: a second run is bit-identical
    out2 = torch.empty_like(out)
    moe.layer_forward(ls, d_inp.x, d_inp.w_router, d_inp.bias, d_inp.w_gate,
                      d_inp.w_up, d_inp.w_down, ws, out=out2)
    torch.cuda.synchronize()
    assert torch.equal(out, out2)
    # the fused layer equals the staged calls on the GPU's own intermediates,
    # bit for bit; where the gate/up GEMM gathers token rows from x itself
    # (tensor cores, T <= 1024), this pins the gather against x_perm
    s_idx, s_gate = moe.route(ls, d_inp.x, d_inp.w_router, d_inp.bias, ws)
    _, s_offs, _, s_slot, s_xp = moe.dispatch(ls, d_inp.x, s_idx, ws)
    s_y = moe.expert_ffn(ls, s_xp, s_offs, d_inp.w_gate, d_inp.w_up, d_inp.w_down, ws)
    s_out = moe.combine(ls, d_inp.x, s_y, s_idx, s_gate, s_slot)
    torch.cuda.synchronize()
    assert torch.equal(s_out, out), "fused layer differs from the staged calls"
    return {"flagged": int(flagged.sum()), "R": R}


@pytest.mark.parametrize("sh", SMALL, ids=lambda s: s.name)
@pytest.mark.parametrize("seed", [0, 1])
def test_small_configs(sh, seed):
    run_staged_and_fused(sh, seed)


def test_routed_scale_nine():
    run_staged_and_fused(SMALL[0], 2, s=9.0)


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_decode_full(seed):
    run_staged_and_fused(CONFIGS["decode"], seed)


def test_prefill_full_sampled():
    run_staged_and_fused(CONFIGS["prefill"], 0, sample="strat")


# the large-expert layer and the sweep share one set of expert weights (d=6144,
# 256 experts of width 2048), drawn once while these tests run back to back
def test_large_e_full_sampled():
    info = run_staged_and_fused(CONFIGS["large_e"], 0, sample="strat")
    sh = CONFIGS["large_e"]
    zero_share = 1.0 - info["R"] / (sh.T * sh.top_k)
    assert 0.29 <= zero_share <= 0.31


@pytest.mark.parametrize("routing", ["uniform", "zipf"])
@pytest.mark.parametrize("T", [1, 8, 64])
def test_sweep_small_T(T, routing):
    run_staged_and_fused(get_config(f"sweep_{routing}_T{T}"), 0)


@pytest.mark.parametrize("routing", ["uniform", "zipf"])
@pytest.mark.parametrize("T", [512, 4096, 32768])
def test_sweep_large_T_sampled(T, routing):
    run_staged_and_fused(get_config(f"sweep_{routing}_T{T}"), 0, sample="strat")
