"""PID controller on the zero experts' router bias (the pages' bias
controller, with gains and set-point as parameters).

CPU: the oracle's update against closed forms. GPU: moe_bias_pid_update
against the oracle step by step (bit-exact: both sides do the same IEEE double
operations), and a closed loop in which the layer's own counts drive the
routed share to the set-point on the GPU as in the oracle."""
import numpy as np
import pytest
import torch

import expert_routing_dispatch_router_b200 as moe
import oracle
from moe_synth import MoEShape, make_router_inputs

f32 = lambda v: float(np.float32(v))


def test_p_only_step_is_kp_times_error():
    counts = np.array([5, 0, 3, 2, 6], np.int32)  # N=3 routed: 8 of 16 slots
    bias = np.array([0.1, -0.2, 0.3, 0.5, -0.5], np.float32)
    b, st = oracle.pid_update(counts, bias, np.zeros(2), T=4, k=4, n_routed=3,
                              target=0.25, kp=2.0, ki=0.0, kd=0.0, max_step=10.0)
    u = 2.0 * (8 / 16 - 0.25)
    np.testing.assert_array_equal(b[:3], bias[:3])  # routed experts untouched
    np.testing.assert_array_equal(b[3:], (bias[3:].astype(np.float64) + u).astype(np.float32))
    np.testing.assert_allclose(st, [0.25, 0.25], rtol=0, atol=0)


def test_integral_and_derivative_terms_and_clamp():
    counts = np.array([2, 2, 0, 0], np.int32)  # share 4/8 = 0.5
    b, st = oracle.pid_update(counts, np.zeros(4, np.float32), np.array([0.1, 0.3]), T=2,
                              k=4, n_routed=2, target=0.4, kp=0.0, ki=1.0, kd=0.0,
                              max_step=10.0)
    np.testing.assert_allclose(b[2:], np.float32(0.1 + 0.1), rtol=1e-7)  # ki (I + err)
    np.testing.assert_allclose(st, [0.2, 0.1], rtol=1e-12)
    b, _ = oracle.pid_update(counts, np.zeros(4, np.float32), np.array([0.0, 0.3]), T=2,
                             k=4, n_routed=2, target=0.4, kp=0.0, ki=0.0, kd=1.0,
                             max_step=10.0)
    np.testing.assert_allclose(b[2:], np.float32(0.1 - 0.3), rtol=1e-7)  # kd (err - prev)
    b, _ = oracle.pid_update(counts, np.zeros(4, np.float32), np.zeros(2), T=2, k=4,
                             n_routed=2, target=0.0, kp=100.0, ki=0.0, kd=0.0, max_step=0.05)
    np.testing.assert_array_equal(b[2:], np.float32(0.05))  # clamped


@pytest.mark.gpu
def test_gpu_update_matches_oracle_bit_for_bit():
    g = torch.Generator().manual_seed(0)
    sh = moe.LayerShape(T=100, d=64, n_routed=40, n_zero=10, top_k=6, ffn=64)
    params = dict(target=f32(0.7), kp=f32(0.8), ki=f32(0.05), kd=f32(0.3), max_step=f32(0.5))
    bias = (torch.rand(50, generator=g) - 0.5).float()
    state = torch.zeros(2, dtype=torch.float64)
    b_dev, s_dev = bias.cuda(), state.cuda()
    b_ref, s_ref = bias.numpy().copy(), state.numpy().copy()
    for step in range(6):
        counts = torch.randint(0, 25, (50,), generator=g, dtype=torch.int32)
        counts[-1] = 600 - int(counts[:-1].sum()) if int(counts[:-1].sum()) < 600 else 0
        moe.bias_pid_update(sh, counts.cuda(), b_dev, s_dev, **params)
        b_ref, s_ref = oracle.pid_update(counts, b_ref, s_ref, T=100, k=6, n_routed=40,
                                         **params)
        torch.cuda.synchronize()
        np.testing.assert_array_equal(b_dev.cpu().numpy(), b_ref)
        np.testing.assert_array_equal(s_dev.cpu().numpy(), s_ref)


@pytest.mark.gpu
def test_closed_loop_reaches_the_set_point():
    """Layer counts -> controller -> bias, 25 times. The routed share starts
    near N/E = 0.8 and must settle at 0.6 on the GPU; the oracle's own loop on
    the same inputs settles there too."""
    shape = MoEShape("pid", T=512, d=256, n_routed=32, n_zero=8, top_k=4, ffn=256)
    x, w_r, b0 = make_router_inputs(shape, 5)
    ls = moe.LayerShape(shape.T, shape.d, shape.n_routed, shape.n_zero, shape.top_k,
                        shape.ffn)
    params = dict(target=f32(0.6), kp=f32(2.0), ki=f32(0.5), kd=f32(0.0), max_step=f32(0.5))
    ws = moe.alloc_workspace(ls)
    xd, wd = x.cuda(), w_r.cuda()
    bias, state = b0.clone().cuda(), torch.zeros(2, dtype=torch.float64, device="cuda")
    idx = torch.empty(shape.T, shape.top_k, dtype=torch.int32, device="cuda")
    shares = []
    for _ in range(25):
        idx, _ = moe.route(ls, xd, wd, bias, ws)
        counts = torch.bincount(idx.view(-1).long(), minlength=shape.E).int()
        shares.append(float(counts[: shape.n_routed].sum()) / (shape.T * shape.top_k))
        moe.bias_pid_update(ls, counts, bias, state, **params)
    torch.cuda.synchronize()
    assert abs(shares[0] - 0.8) < 0.1
    assert all(abs(s - 0.6) < 0.03 for s in shares[-5:]), shares
    # the oracle's loop
    logits = oracle.router_logits(x, w_r)
    b_ref, s_ref = b0.numpy().copy(), np.zeros(2)
    ref_shares = []
    for _ in range(25):
        ridx, _, _ = oracle.select(logits, b_ref, shape.top_k)
        c = np.bincount(ridx.ravel(), minlength=shape.E).astype(np.int32)
        ref_shares.append(c[: shape.n_routed].sum() / (shape.T * shape.top_k))
        b_ref, s_ref = oracle.pid_update(c, b_ref, s_ref, T=shape.T, k=shape.top_k,
                                         n_routed=shape.n_routed, **params)
    assert all(abs(s - 0.6) < 0.03 for s in ref_shares[-5:]), ref_shares
