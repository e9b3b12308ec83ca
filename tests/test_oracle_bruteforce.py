"""Pure-Python brute force of the whole layer on tiny inputs, against the C
oracle. The brute force selects by fully sorting (key, id) pairs and evaluates
every expert with Python floats, so it shares neither the selection method nor
the language with the oracle. Constructed exact ties and near-ties check the
tie rule (lower expert id first)."""
import math
import random

import numpy as np
import pytest
import torch

import oracle


def brute_layer(x, wr, b, wg, wu, wd, N, k, s):
    T, d = len(x), len(x[0])
    E = len(wr)
    F = len(wg[0]) if N else 0
    outs, sels = [], []
    for t in range(T):
        logit = [sum(x[t][i] * wr[e][i] for i in range(d)) for e in range(E)]
        order = sorted(range(E), key=lambda e: (-(logit[e] + b[e]), e))
        sel = order[:k]
        m = max(logit[e] for e in sel)
        z = sum(math.exp(logit[e] - m) for e in sel)
        out = [0.0] * d
        for e in sel:
            g = math.exp(logit[e] - m) / z
            if e < N:
                a = [sum(wg[e][f][i] * x[t][i] for i in range(d)) for f in range(F)]
                u = [sum(wu[e][f][i] * x[t][i] for i in range(d)) for f in range(F)]
                h = [a[f] / (1.0 + math.exp(-a[f])) * u[f] for f in range(F)]
                for n in range(d):
                    out[n] += s * g * sum(wd[e][n][f] * h[f] for f in range(F))
            else:
                for n in range(d):
                    out[n] += g * x[t][n]
        outs.append(out)
        sels.append(sel)
    return outs, sels


def _lists(t):
    return t.double().tolist()


@pytest.mark.parametrize("seed", range(6))
def test_oracle_matches_brute_force(seed):
    rnd = random.Random(seed)
    T = rnd.randint(1, 16)
    d = rnd.choice([3, 8, 17, 32])
    N = rnd.randint(1, 7)
    Z = rnd.randint(0, 3)
    k = rnd.randint(1, N + Z)
    F = rnd.choice([1, 5, 12])
    s = rnd.choice([1.0, 9.0, 0.5])
    dtype = rnd.choice([torch.float32, torch.bfloat16])
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(T, d, generator=g).to(dtype)
    wr = torch.randn(N + Z, d, generator=g) / math.sqrt(d)
    b = torch.rand(N + Z, generator=g) * 0.2 - 0.1
    wg = (torch.randn(N, F, d, generator=g) / math.sqrt(d)).to(dtype)
    wu = (torch.randn(N, F, d, generator=g) / math.sqrt(d)).to(dtype)
    wd = (torch.randn(N, d, F, generator=g) / math.sqrt(d)).to(dtype)
    out, idx, _ = oracle.layer(x, wr, b, wg, wu, wd, N, k, s)
    ref, sel = brute_layer(_lists(x), _lists(wr), _lists(b), _lists(wg), _lists(wu),
                           _lists(wd), N, k, s)
    np.testing.assert_array_equal(idx, np.array(sel))
    np.testing.assert_allclose(out, np.array(ref), rtol=1e-11, atol=1e-12)


def test_exact_ties_go_to_lower_id():
    # three experts with identical rows and bias: every key ties
    d, N, Z, k = 4, 2, 1, 2
    x = torch.tensor([[1.0, -2.0, 0.5, 3.0], [0.0, 1.0, 1.0, 0.0]])
    wr = torch.tensor([[0.25, 0.5, -1.0, 0.125]] * 3)
    b = torch.zeros(3)
    wg = torch.ones(N, 2, d) * 0.1
    wu = torch.ones(N, 2, d) * 0.2
    wd = torch.ones(N, d, 2) * 0.3
    out, idx, gate = oracle.layer(x, wr, b, wg, wu, wd, N, k, 1.0)
    np.testing.assert_array_equal(idx, [[0, 1], [0, 1]])
    np.testing.assert_allclose(gate, 0.5, rtol=1e-15)
    ref, sel = brute_layer(_lists(x), _lists(wr), _lists(b), _lists(wg), _lists(wu),
                           _lists(wd), N, k, 1.0)
    np.testing.assert_allclose(out, np.array(ref), rtol=1e-12)


def test_near_tie_margin_is_reported():
    logits = torch.tensor([[1.0, 1.0 + 5e-5, 0.2, 0.3]], dtype=torch.float64)
    idx, gate, margin = oracle.select(logits, torch.zeros(4), 1)
    assert idx[0, 0] == 1
    assert margin[0] == pytest.approx(5e-5, rel=1e-9)


def test_card_arithmetic_pins_three_matrix_experts_and_zero_skip():
    """The card's numbers (tests/golden/longcat2_moe_card.txt) fix the spread
    of activated parameters: 12 slots x 3 matrices x d x F x 38 layers is the
    whole 33-56B range, so a zero-expert slot skips all three matrices
    (reading R5/R6). A two-matrix expert would give only 15.3B."""
    vals = {}
    with open(__file__.replace("test_oracle_bruteforce.py", "golden/longcat2_moe_card.txt")) as f:
        for line in f:
            line = line.split("#")[0].split()
            if len(line) == 2:
                vals[line[0]] = float(line[1])
    assert vals["router_rows"] == vals["n_routed_experts"] + vals["zero_expert_num"]
    assert vals["router_cols"] == vals["hidden_size"]
    per_slot = 3 * vals["hidden_size"] * vals["expert_ffn_hidden_size"] * vals["num_layers"]
    spread = vals["moe_topk"] * per_slot / 1e9
    assert abs(spread - (vals["active_high_b"] - vals["active_low_b"])) < 0.5
    two_matrix = vals["moe_topk"] * 2 / 3 * per_slot / 1e9
    assert abs(two_matrix - 23) > 5
    # average 48B: about (48 - 33) / 22.9 of the slots are routed
    routed_share = (vals["active_avg_b"] - vals["active_low_b"]) / spread
    assert 0.6 < routed_share < 0.7
