"""Every binding function reaches the library with the right arguments: with
an empty batch (T = 0) the library returns before it reads any pointer, so the
calls run here without a GPU. Host tensors stand in for device ones (the
binding's device checks are relaxed for this test only), and a stand-in
stream handle replaces torch's current stream."""
import types

import pytest
import torch

import expert_routing_dispatch_router_b200 as moe


@pytest.fixture
def relaxed(monkeypatch):
    real_need = moe._need

    def need(t, name, dtype, shape=None, on_device=True):
        real_need(t, name, dtype, shape, on_device=False)

    def ws_of(ws):
        return moe.ctypes.c_void_p(ws.data_ptr()), ws.numel() * ws.element_size()

    monkeypatch.setattr(moe, "_need", need)
    monkeypatch.setattr(moe, "_ws", ws_of)
    return types.SimpleNamespace(cuda_stream=0)


def test_every_call_with_an_empty_batch(relaxed):
    st = relaxed
    sh = moe.LayerShape(T=0, d=64, n_routed=2, n_zero=1, top_k=2, ffn=64)
    bf = torch.bfloat16
    x = torch.zeros(0, 64, dtype=bf)
    w_r, b = torch.zeros(3, 64), torch.zeros(3)
    wg, wd = torch.zeros(2, 64, 64, dtype=bf), torch.zeros(2, 64, 64, dtype=bf)
    ws = torch.zeros(moe.workspace_size(sh), dtype=torch.uint8)
    idx, gate = moe.route(sh, x, w_r, b, ws, stream=st)
    assert idx.shape == (0, 2) and gate.shape == (0, 2)
    moe.route_noalloc(sh, x, w_r, b, idx, gate, stream=st)
    counts, offsets, row_token, slot_row, x_perm = moe.dispatch(sh, x, idx, ws, stream=st)
    y = moe.expert_ffn(sh, x_perm, offsets, wg, wg, wd, ws, stream=st)
    out = moe.combine(sh, x, y, idx, gate, slot_row, stream=st)
    assert out.shape == (0, 64)
    out = moe.layer_forward(sh, x, w_r, b, wg, wg, wd, ws, stream=st)
    assert out.shape == (0, 64)
    moe.layer_forward_host(sh, x, w_r, b, wg, wg, wd, ws, torch.zeros(0, 64, dtype=bf),
                           stream=st)
