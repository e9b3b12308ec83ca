"""Pins of the CPU oracle against things other than itself.

Each test ties one oracle function to a library routine (torch fp64 matmul,
sort, softmax, numpy bincount/lexsort), to a closed form worked by hand, or to
an invariant the pages fix (identity zero experts, gates summing to 1, counts
summing to T*k). Together they are chosen so that a dropped term, a wrong sign,
a wrong index or a transposed operand anywhere in the oracle fails one of them.
"""
import math

import numpy as np
import pytest
import torch
import torch.nn.functional as Fn

import oracle
from moe_synth import MoEShape, make_inputs

pytestmark = pytest.mark.filterwarnings("ignore")


def _rand_layer(T=12, d=24, N=5, Z=3, k=3, F=16, seed=0, dtype=torch.float32,
                bias_scale=0.1):
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(T, d, generator=g).to(dtype)
    wr = torch.randn(N + Z, d, generator=g) / math.sqrt(d)
    b = (torch.rand(N + Z, generator=g) * 2 - 1) * bias_scale
    wg = (torch.randn(N, F, d, generator=g) / math.sqrt(d)).to(dtype)
    wu = (torch.randn(N, F, d, generator=g) / math.sqrt(d)).to(dtype)
    wd = (torch.randn(N, d, F, generator=g) / math.sqrt(d)).to(dtype)
    return x, wr, b, wg, wu, wd


# --------------------------------------------------------------- router --

@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_logits_match_torch_fp64_matmul(dtype):
    """Router classifier [E, d] (model card, Mixture of experts): x W_r^T."""
    x, wr, *_ = _rand_layer(T=33, d=70, N=9, Z=4, dtype=dtype)
    got = oracle.router_logits(x, wr)
    ref = (x.double() @ wr.double().T).numpy()
    np.testing.assert_allclose(got, ref, rtol=0, atol=1e-12)


def test_selection_matches_stable_sort_with_ties():
    """Top-k set = the k largest keys, ties to the lower id, descending order."""
    g = torch.Generator().manual_seed(3)
    T, E, k = 200, 17, 5
    # integer-valued logits and bias create many exact ties
    logits = torch.randint(-3, 4, (T, E), generator=g).double()
    bias = torch.randint(-1, 2, (E,), generator=g).float()
    idx, gate, margin = oracle.select(logits, bias, k)
    keys = logits + bias.double()
    order = torch.sort(-keys, dim=1, stable=True).indices  # ties: lower id first
    np.testing.assert_array_equal(idx, order[:, :k].numpy())
    sk = torch.gather(keys, 1, order)
    np.testing.assert_array_equal(margin, (sk[:, k - 1] - sk[:, k]).numpy())


def test_margin_is_inf_when_k_equals_E():
    logits = torch.randn(4, 6, dtype=torch.float64)
    _, _, margin = oracle.select(logits, torch.zeros(6), 6)
    assert np.all(np.isinf(margin))


def test_gates_with_k_equal_E_are_plain_softmax():
    """k = E reduces the renormalised gates to a softmax over all experts."""
    g = torch.Generator().manual_seed(4)
    logits = torch.randn(50, 9, generator=g, dtype=torch.float64) * 3
    bias = torch.rand(9, generator=g) * 0.2 - 0.1
    idx, gate, _ = oracle.select(logits, bias, 9)
    sm = torch.softmax(logits, dim=1).numpy()
    ref = np.take_along_axis(sm, idx.astype(np.int64), axis=1)
    np.testing.assert_allclose(gate, ref, rtol=1e-14, atol=1e-15)


def test_gates_sum_to_one_and_use_raw_logits():
    """Reading R2/R4: the bias steers selection only; gates use raw logits."""
    x, wr, b, *_ = _rand_layer(T=64, d=32, N=10, Z=4, k=4)
    logits, idx, gate, _ = oracle.route(x, wr, b, 4)
    np.testing.assert_allclose(gate.sum(1), 1.0, rtol=0, atol=1e-14)
    sel = np.take_along_axis(logits, idx.astype(np.int64), axis=1)
    ref = torch.softmax(torch.from_numpy(sel), dim=1).numpy()
    np.testing.assert_allclose(gate, ref, rtol=1e-13, atol=1e-15)
    # a constant shift of every bias changes neither the selection nor gates
    _, idx2, gate2, _ = oracle.route(x, wr, b + 0.37, 4)
    np.testing.assert_array_equal(idx, idx2)
    np.testing.assert_allclose(gate, gate2, rtol=1e-14, atol=0)


# -------------------------------------------------------------- dispatch --

def test_dispatch_matches_bincount_and_lexsort():
    g = torch.Generator().manual_seed(5)
    T, k, N, Z = 301, 4, 11, 3
    E = N + Z
    idx = torch.stack([torch.randperm(E, generator=g)[:k] for _ in range(T)]).int()
    counts, offsets, row_token, slot_row = oracle.dispatch(idx, N, E)
    ix = idx.numpy()
    np.testing.assert_array_equal(counts, np.bincount(ix.ravel(), minlength=E))
    assert counts.sum() == T * k
    np.testing.assert_array_equal(offsets, np.concatenate([[0], np.cumsum(counts[:N])]))
    R = int(offsets[N])
    tok = np.repeat(np.arange(T), k)
    ex = ix.ravel()
    routed = np.nonzero(ex < N)[0]
    order = routed[np.lexsort((tok[routed], ex[routed]))]  # by expert, then token
    np.testing.assert_array_equal(row_token[:R], tok[order])
    assert np.all(row_token[R:] == -1)
    ref_slot = np.full(T * k, -1)
    ref_slot[order] = np.arange(R)
    np.testing.assert_array_equal(slot_row, ref_slot)


# ------------------------------------------------------------ expert FFN --

@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_expert_rows_match_torch_swiglu(dtype):
    """Reading R5: y = W_d (silu(W_g x) * W_u x), with non-square F != d so a
    transposed operand cannot pass."""
    x, _, _, wg, wu, wd = _rand_layer(T=7, d=24, N=3, F=40, dtype=dtype)
    rows = torch.tensor([0, 2, 1, 1, 0, 2, 2], dtype=torch.int32)
    y, h = oracle.expert_rows(wg, wu, wd, rows, x, want_h=True)
    X = x.double()
    for r in range(7):
        e = int(rows[r])
        a = X[r] @ wg[e].double().T
        u = X[r] @ wu[e].double().T
        hh = Fn.silu(a) * u
        np.testing.assert_allclose(h[r], hh.numpy(), rtol=1e-12, atol=1e-13)
        np.testing.assert_allclose(y[r], (hh @ wd[e].double().T).numpy(),
                                   rtol=1e-12, atol=1e-13)


def test_silu_closed_form_points():
    """silu(z) = z / (1 + e^-z) at z = 0, 1, -2 through a 1x1 expert."""
    for z in (0.0, 1.0, -2.0):
        wg = torch.tensor([[[1.0]]])
        wu = torch.tensor([[[1.0]]])
        wd = torch.tensor([[[1.0]]])
        y = oracle.expert_rows(wg, wu, wd, torch.tensor([0], dtype=torch.int32),
                               torch.tensor([[z]]))
        assert y[0, 0] == pytest.approx(z * z / (1 + math.exp(-z)), rel=1e-15, abs=1e-300)


# --------------------------------------------------------------- combine --

def test_combine_matches_torch_gather_sum():
    g = torch.Generator().manual_seed(6)
    T, d, N, Z, k = 20, 8, 4, 2, 3
    E = N + Z
    idx = torch.stack([torch.randperm(E, generator=g)[:k] for _ in range(T)]).int()
    gate = torch.rand(T, k, generator=g, dtype=torch.float64)
    x = torch.randn(T, d, generator=g, dtype=torch.float64)
    _, _, row_token, slot_row = oracle.dispatch(idx, N, E)
    R = int((idx < N).sum())
    y = torch.randn(T * k, d, generator=g, dtype=torch.float64)
    s = 9.0
    out = oracle.combine(x, y, idx, gate, slot_row, N, s)
    ref = torch.zeros(T, d, dtype=torch.float64)
    for t in range(T):
        for j in range(k):
            e = int(idx[t, j])
            if e < N:
                ref[t] += s * gate[t, j] * y[int(slot_row[t * k + j])]
            else:
                ref[t] += gate[t, j] * x[t]
    np.testing.assert_allclose(out, ref.numpy(), rtol=1e-14, atol=1e-14)
    assert R == int((slot_row >= 0).sum())


# ---------------------------------------------------------- whole layer --

def test_worked_example_closed_form():
    """Hand-worked layer: T=2, d=2, 2 routed experts (F=1) + 1 zero expert, k=2.

    logits t0 = [1, 0, .5], t1 = [0, 2, 1]; bias [0, 0, .25] gives keys
    t0 = [1, 0, .75] -> {0, 2}, t1 = [0, 2, 1.25] -> {1, 2}. Gates are the
    softmax of the raw logits of the chosen pair. Expert 0 on x=[1,0]:
    a=1, u=2, h=2 silu(1), y=[h,-h]. Expert 1 on x=[0,2]: a=2, u=2,
    h=2 silu(2), y=[0,h]. The zero expert returns x."""
    x = torch.tensor([[1.0, 0.0], [0.0, 2.0]])
    wr = torch.tensor([[1.0, 0.0], [0.0, 1.0], [0.5, 0.5]])
    b = torch.tensor([0.0, 0.0, 0.25])
    wg = torch.tensor([[[1.0, 0.0]], [[0.0, 1.0]]])
    wu = torch.tensor([[[2.0, 0.0]], [[0.0, 1.0]]])
    wd = torch.tensor([[[1.0], [-1.0]], [[0.0], [1.0]]])
    silu = lambda z: z / (1 + math.exp(-z))
    for s in (1.0, 9.0):
        out, idx, gate = oracle.layer(x, wr, b, wg, wu, wd, n_routed=2, top_k=2,
                                      routed_scale=s)
        np.testing.assert_array_equal(idx, [[0, 2], [1, 2]])
        g00 = 1 / (1 + math.exp(-0.5))
        g11 = 1 / (1 + math.exp(-1.0))
        np.testing.assert_allclose(gate, [[g00, 1 - g00], [g11, 1 - g11]], rtol=1e-15)
        h0 = 2 * silu(1.0)
        h1 = 2 * silu(2.0)
        ref = [[s * g00 * h0 + (1 - g00) * 1.0, -s * g00 * h0],
               [0.0, s * g11 * h1 + (1 - g11) * 2.0]]
        np.testing.assert_allclose(out, ref, rtol=1e-14, atol=1e-15)


def test_all_zero_routing_returns_input():
    """Identity zero experts: a large bias on every zero expert routes every
    slot there, so out = sum_j g_j x = x whatever the routed scale."""
    x, wr, b, wg, wu, wd = _rand_layer(T=16, d=20, N=6, Z=4, k=3)
    bb = b.clone()
    bb[6:] += 1e3
    for s in (1.0, 9.0):
        out, idx, _ = oracle.layer(x, wr, bb, wg, wu, wd, 6, 3, s)
        assert np.all(idx >= 6)
        np.testing.assert_allclose(out, x.double().numpy(), rtol=0, atol=1e-14)


def test_zero_experts_pushed_out_gives_standard_topk_moe():
    """A -1e3 bias on every zero expert makes the layer a standard top-k MoE
    over the routed experts; checked against torch.topk + softmax + SwiGLU."""
    x, wr, b, wg, wu, wd = _rand_layer(T=10, d=16, N=6, Z=3, k=2, F=12)
    bb = b.clone()
    bb[6:] -= 1e3
    out, idx, _ = oracle.layer(x, wr, bb, wg, wu, wd, 6, 2, 1.0)
    X = x.double()
    logits = X @ wr.double().T
    keys = logits + bb.double()
    ref = torch.zeros_like(X)
    for t in range(10):
        top = torch.topk(keys[t], 2).indices
        g = torch.softmax(logits[t, top], 0)
        for j in range(2):
            e = int(top[j])
            h = Fn.silu(X[t] @ wg[e].double().T) * (X[t] @ wu[e].double().T)
            ref[t] += g[j] * (h @ wd[e].double().T)
    np.testing.assert_allclose(out, ref.numpy(), rtol=1e-12, atol=1e-12)


def test_single_expert_is_dense_swiglu_ffn():
    """N=1, Z=0, k=1: the layer is one dense SwiGLU FFN (gate = 1)."""
    x, wr, b, wg, wu, wd = _rand_layer(T=9, d=24, N=1, Z=0, k=1, F=36)
    out, idx, gate = oracle.layer(x, wr, b, wg, wu, wd, 1, 1, 1.0)
    assert np.all(idx == 0) and np.all(gate == 1.0)
    X = x.double()
    ref = (Fn.silu(X @ wg[0].double().T) * (X @ wu[0].double().T)) @ wd[0].double().T
    np.testing.assert_allclose(out, ref.numpy(), rtol=1e-12, atol=1e-12)


def test_routed_scale_multiplies_routed_part_only():
    """Reading R7: out(s) - out(1) = (s - 1) * routed part."""
    x, wr, b, wg, wu, wd = _rand_layer(T=30, d=16, N=4, Z=4, k=3, bias_scale=0.5)
    o1, idx, gate = oracle.layer(x, wr, b, wg, wu, wd, 4, 3, 1.0)
    o9, _, _ = oracle.layer(x, wr, b, wg, wu, wd, 4, 3, 9.0)
    zero_part = np.zeros_like(o1)
    for t in range(30):
        for j in range(3):
            if idx[t, j] >= 4:
                zero_part[t] += gate[t, j] * x[t].double().numpy()
    np.testing.assert_allclose(o9 - zero_part, 9.0 * (o1 - zero_part), rtol=1e-12, atol=1e-12)
    assert np.any(idx >= 4) and np.any(idx < 4)


def test_layer_equals_route_dispatch_ffn_combine():
    """The per-token definition equals the staged pipeline (route -> dispatch
    -> expert rows -> combine), which goes through the permutation."""
    x, wr, b, wg, wu, wd = _rand_layer(T=40, d=16, N=5, Z=3, k=3, F=20)
    out, idx_l, gate_l = oracle.layer(x, wr, b, wg, wu, wd, 5, 3, 9.0)
    logits, idx, gate, _ = oracle.route(x, wr, b, 3)
    np.testing.assert_array_equal(idx, idx_l)
    np.testing.assert_allclose(gate, gate_l, rtol=1e-15)
    counts, offsets, row_token, slot_row = oracle.dispatch(idx, 5, 8)
    R = int(offsets[5])
    row_expert = np.repeat(np.arange(5), counts[:5]).astype(np.int32)
    y = oracle.expert_rows(wg, wu, wd, row_expert, x.double()[row_token[:R]])
    yp = np.zeros((40 * 3, 16))
    yp[:R] = y
    staged = oracle.combine(x, yp, idx, gate, slot_row, 5, 9.0)
    np.testing.assert_allclose(staged, out, rtol=1e-13, atol=1e-13)


def test_force_idx_reproduces_own_selection_and_subset_tokens():
    x, wr, b, wg, wu, wd = _rand_layer(T=25, d=16, N=5, Z=3, k=2)
    out, idx, gate = oracle.layer(x, wr, b, wg, wu, wd, 5, 2, 1.0)
    toks = np.array([3, 17, 0], np.int32)
    out2, idx2, gate2 = oracle.layer(x, wr, b, wg, wu, wd, 5, 2, 1.0, tokens=toks,
                                     force_idx=idx)
    np.testing.assert_array_equal(idx2, idx[toks])
    np.testing.assert_allclose(out2, out[toks], rtol=1e-15)


def test_synthetic_recipe_shapes_and_stats():
    sh = MoEShape("t", T=64, d=128, n_routed=6, n_zero=2, top_k=2, ffn=32)
    inp = make_inputs(sh, seed=1)
    assert inp.x.dtype == torch.bfloat16 and inp.x.shape == (64, 128)
    assert inp.w_router.dtype == torch.float32 and inp.w_router.shape == (8, 128)
    assert inp.w_gate.shape == (6, 32, 128) and inp.w_down.shape == (6, 128, 32)
    assert float(inp.bias.abs().max()) <= 0.1
    assert abs(float(inp.w_gate.float().std()) - 128 ** -0.5) < 0.01
    again = make_inputs(sh, seed=1)
    assert torch.equal(inp.x, again.x) and torch.equal(inp.w_down, again.w_down)
