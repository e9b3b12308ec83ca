"""Host-side tests of the C ABI: the library builds for sm_100a, loads, exports
every function the header declares, sizes its workspace, and rejects bad
arguments on the host before anything would be launched (so these run without
a GPU: no call here reaches a kernel launch)."""
import ctypes

import pytest

import expert_routing_dispatch_router_b200 as moe
from expert_routing_dispatch_router_b200 import build as moe_build

P = ctypes.c_void_p


@pytest.fixture(scope="module")
def L():
    moe_build.build()
    return moe.lib()


def cfg(T=64, d=256, N=8, Z=2, k=2, F=512, dt=moe.MOE_BF16, s=1.0):
    return moe.MoEConfig(T, d, N, Z, k, F, dt, s)


def test_every_declared_function_is_exported(L):
    names = moe.declared_functions()
    assert {"moe_route", "moe_dispatch", "moe_expert_ffn", "moe_combine",
            "moe_layer_forward", "moe_workspace_size", "moe_status_string",
            "moe_layer_forward_host", "moe_read_device_error",
            "moe_layer_launch_count"} <= set(names)
    for n in names:
        assert hasattr(L, n), n


def test_status_strings(L):
    for code in range(6):
        assert L.moe_status_string(code)
    assert L.moe_status_string(0) == b"ok"


def test_workspace_size_valid_and_invalid(L):
    c = cfg()
    n = L.moe_workspace_size(ctypes.byref(c))
    assert n > 0 and n % 1024 == 0
    big = cfg(T=16384, d=4096, N=128, Z=32, k=8, F=1024)
    nb = L.moe_workspace_size(ctypes.byref(big))
    # holds at least x_perm, h and y_perm for T*k rows
    assert nb >= 16384 * 8 * (4096 * 2 + 1024) * 2
    # an empty batch has a (small) workspace too
    assert 0 < L.moe_workspace_size(ctypes.byref(cfg(T=0))) < n
    for bad in (cfg(k=0), cfg(k=11), cfg(d=0), cfg(T=-1), cfg(N=0, Z=0),
                cfg(dt=7), cfg(k=33, N=40), cfg(N=1020, Z=10), cfg(d=260),
                cfg(F=100), cfg(s=float("inf"))):
        assert L.moe_workspace_size(ctypes.byref(bad)) == 0
    assert L.moe_workspace_size(None) == 0


def test_host_sizing_defined_across_the_limits(L):
    # workspace size and launch count for every d the limits allow up to 1024,
    # at batch sizes on both sides of each path threshold: each is defined
    # (no division by an empty count) and the config is accepted
    for d in range(8, 1025, 8):
        for T in (0, 1, 63, 257, 512, 1025, 4097):
            for dt in (moe.MOE_BF16, moe.MOE_F32):
                for N, Z, k, F in ((6, 2, 2, 8), (1, 0, 1, 256), (0, 3, 2, 128)):
                    c = cfg(T=T, d=d, N=N, Z=Z, k=k, F=F, dt=dt)
                    assert L.moe_workspace_size(ctypes.byref(c)) > 0, (d, T, dt, N, F)
                    assert L.moe_layer_launch_count(ctypes.byref(c)) >= 0


def test_cuda_core_router_token_limit(L):
    # the CUDA-core router (f32, or d not a multiple of 128) takes at most
    # 65535 tiles of 64 tokens; beyond that the config is refused up front
    for dt, d in ((moe.MOE_F32, 128), (moe.MOE_BF16, 64)):
        ok = cfg(T=65535 * 64, d=d, N=2, Z=1, k=1, F=8, dt=dt)
        over = cfg(T=65535 * 64 + 1, d=d, N=2, Z=1, k=1, F=8, dt=dt)
        assert L.moe_workspace_size(ctypes.byref(ok)) > 0
        assert L.moe_workspace_size(ctypes.byref(over)) == 0
    # the tensor-core router (bf16, d a multiple of 128) has no such limit
    big = cfg(T=65535 * 64 + 1, d=128, N=2, Z=1, k=1, F=8)
    assert L.moe_workspace_size(ctypes.byref(big)) > 0


def test_launch_count(L):
    # router 1 (T <= 256), 2 (CUDA cores) or 3 (split + tensor-core GEMM +
    # top-k); dispatch 1 (one block for T <= 4096) or 3, + gather unless the
    # single-CTA gate/up GEMM gathers (tensor cores, T <= 1024) or the
    # one-block dispatch gathers in its own launch (T * k <= 2048); FFN 2
    # (tcgen05, plans written by the one-block dispatch), 3 (tcgen05 + plan)
    # or 2 (CUDA cores), + 1 SwiGLU fixup when a tiny batch splits the gate/up
    # contraction; combine 1
    decode = cfg(T=64, d=4096, N=128, Z=32, k=8, F=1024)
    assert L.moe_layer_launch_count(ctypes.byref(decode)) == 1 + 1 + 2 + 1
    # 8 experts at T=64 make 32 gate/up units: split
    assert L.moe_layer_launch_count(ctypes.byref(cfg())) == 1 + 1 + 3 + 1
    single = cfg(T=1, d=6144, N=256, Z=64, k=12, F=2048)
    assert L.moe_layer_launch_count(ctypes.byref(single)) == 1 + 1 + 3 + 1
    assert L.moe_layer_launch_count(ctypes.byref(cfg(dt=moe.MOE_F32))) == 1 + 1 + 2 + 1
    f32_wide = cfg(T=1100, k=2, dt=moe.MOE_F32)  # 2200 slots: a separate gather
    assert L.moe_layer_launch_count(ctypes.byref(f32_wide)) == 2 + 2 + 2 + 1
    assert L.moe_layer_launch_count(ctypes.byref(cfg(T=300))) == 2 + 1 + 2 + 1
    assert L.moe_layer_launch_count(ctypes.byref(cfg(T=1100))) == 3 + 2 + 2 + 1
    big = cfg(T=16384, d=4096, N=128, Z=32, k=8, F=1024)
    assert L.moe_layer_launch_count(ctypes.byref(big)) == 3 + 4 + 3 + 1
    assert L.moe_layer_launch_count(ctypes.byref(cfg(T=0))) == 0


def _fake(addr=0x10000):
    return P(addr)


def test_config_errors_before_launch(L):
    st = P(0)
    bad = [(cfg(k=11), 1), (cfg(k=33, N=40), 2), (cfg(N=1100, Z=0), 2),
           (cfg(d=12), 2), (cfg(F=20), 2), (cfg(T=-5), 1), (cfg(dt=3), 1),
           (cfg(N=0, Z=0), 1), (cfg(s=float("nan")), 1)]
    for c, want in bad:
        r = L.moe_route(ctypes.byref(c), _fake(), _fake(), _fake(), None, _fake(),
                        _fake(), None, _fake(), 1 << 40, st)
        assert r == want, (c.T, c.d, c.top_k, r)
        r = L.moe_layer_forward(ctypes.byref(c), _fake(), _fake(), _fake(), _fake(),
                                _fake(), _fake(), _fake(), None, _fake(), 1 << 40, st)
        assert r == want
    assert L.moe_route(None, _fake(), _fake(), _fake(), None, _fake(), _fake(), None,
                       _fake(), 1 << 40, st) == 1


def test_pointer_errors_before_launch(L):
    c = cfg()
    st = P(0)
    ws_n = L.moe_workspace_size(ctypes.byref(c))
    ok = [_fake(0x10000 + 0x100 * i) for i in range(12)]
    # null required pointer
    r = L.moe_layer_forward(ctypes.byref(c), None, *ok[1:7], None, ok[8], ws_n, st)
    assert r == 1
    # misaligned pointer
    r = L.moe_layer_forward(ctypes.byref(c), _fake(0x10008), *ok[1:7], None, ok[8],
                            ws_n, st)
    assert r == 1
    # misaligned optional pointer
    r = L.moe_layer_forward(ctypes.byref(c), *ok[0:7], _fake(0x10004), ok[8], ws_n, st)
    assert r == 1
    # workspace missing / too small / misaligned base
    r = L.moe_layer_forward(ctypes.byref(c), *ok[0:7], None, None, ws_n, st)
    assert r == 3
    r = L.moe_layer_forward(ctypes.byref(c), *ok[0:7], None, ok[8], ws_n - 1, st)
    assert r == 3
    r = L.moe_layer_forward(ctypes.byref(c), *ok[0:7], None, _fake(0x10010), ws_n, st)
    assert r == 1
    # staged calls
    assert L.moe_dispatch(ctypes.byref(c), ok[0], None, *ok[2:7], ok[8], ws_n, st) == 1
    assert L.moe_expert_ffn(ctypes.byref(c), ok[0], ok[1], None, ok[3], ok[4], ok[5],
                            ok[8], ws_n, st) == 1
    assert L.moe_combine(ctypes.byref(c), *ok[0:5], _fake(0x10001), ok[6], st) == 1
    assert L.moe_expert_ffn(ctypes.byref(c), *ok[0:6], ok[8], 16, st) == 3
    # host entry point: host pointers may be null-checked only
    assert L.moe_layer_forward_host(ctypes.byref(c), None, *ok[1:6], ok[6], None,
                                    ok[8], ws_n, st) == 1
    assert L.moe_read_device_error(None, None, st) == 3


def test_route_noalloc_refuses_problems_beyond_its_limits(L):
    # moe_route_noalloc checks its limits on the host before it looks up its
    # scratch array or launches anything, so fake device addresses never reach
    # a kernel (runs without a GPU)
    st = P(0)
    # T * E beyond the 16 MiB scratch array
    c = cfg(T=32768, d=256, N=121, Z=8, k=4, F=128)
    assert L.moe_route_noalloc(ctypes.byref(c), _fake(), _fake(), _fake(), None, _fake(),
                               _fake(), None, st) == 2
    # T * E within the array, but more token tiles than the CUDA-core router's
    # grid takes (moe_route would run this shape on the tensor cores)
    c = cfg(T=65536 * 64, d=128, N=1, Z=0, k=1, F=8)
    assert L.moe_workspace_size(ctypes.byref(c)) > 0
    assert L.moe_route_noalloc(ctypes.byref(c), _fake(), _fake(), _fake(), None, _fake(),
                               _fake(), None, st) == 2


def test_expert_parallel_calls_check_ranks_on_the_host(L):
    # moe_ep_*: the even split of the routed experts, and refusals of a bad
    # rank, world or pointer before anything is launched (runs without a GPU)
    st = P(0)
    c = cfg(N=7, Z=3, k=3)
    assert [L.moe_ep_local_experts(ctypes.byref(c), r, 2) for r in range(2)] == [4, 3]
    assert [L.moe_ep_local_experts(ctypes.byref(c), r, 4) for r in range(4)] == [2, 2, 2, 1]
    assert [L.moe_ep_local_experts(ctypes.byref(c), r, 9) for r in range(9)] == [1] * 7 + [0] * 2
    assert L.moe_ep_local_experts(ctypes.byref(c), 2, 2) == -1
    assert L.moe_ep_local_experts(ctypes.byref(c), 0, 0) == -1
    f = _fake
    assert L.moe_ep_plan(ctypes.byref(c), 2, 2, f(), f(), f(), st) == 1  # rank >= world
    assert L.moe_ep_plan(ctypes.byref(c), -1, 2, f(), f(), f(), st) == 1
    assert L.moe_ep_plan(ctypes.byref(c), 0, 2, None, f(), f(), st) == 1
    assert L.moe_ep_dispatch(ctypes.byref(c), 0, f(), f(), f(), f(), f(), st) == 1
    assert L.moe_ep_dispatch(ctypes.byref(c), 2, f(), f(), f(), f(0x10004), f(), st) == 1
    assert L.moe_ep_return(ctypes.byref(c), 0, 2, f(), f(), f(), None, f(), st) == 1
    assert L.moe_ep_return(ctypes.byref(c), 3, 2, f(), f(), f(), f(), f(), st) == 1
    no_routed = cfg(N=0, Z=4, k=2)
    assert L.moe_ep_plan(ctypes.byref(no_routed), 0, 2, f(), f(), f(), st) == 1
    # the split agrees with the host plan's
    from expert_routing_dispatch_router_b200 import expert_parallel as ep
    for N, G in ((7, 2), (18, 4), (3, 4), (256, 8), (1, 1)):
        b = ep.expert_bounds(N, G)
        cc = cfg(N=N, Z=4, k=2)
        assert [L.moe_ep_local_experts(ctypes.byref(cc), r, G) for r in range(G)] == \
            [b[r + 1] - b[r] for r in range(G)]


def test_empty_batch_is_a_no_op_before_any_pointer_check(L):
    # T == 0: every entry point returns MOE_OK with all pointers null (empty
    # buffers have no address) and no workspace; nothing is launched, so this
    # runs without a GPU. A bad config is still an error.
    c = cfg(T=0)
    st = P(0)
    assert L.moe_route(ctypes.byref(c), *[None] * 8, 0, st) == 0
    assert L.moe_route_noalloc(ctypes.byref(c), *[None] * 7, st) == 0
    assert L.moe_dispatch(ctypes.byref(c), *[None] * 8, 0, st) == 0
    assert L.moe_expert_ffn(ctypes.byref(c), *[None] * 7, 0, st) == 0
    assert L.moe_combine(ctypes.byref(c), *[None] * 6, st) == 0
    assert L.moe_layer_forward(ctypes.byref(c), *[None] * 9, 0, st) == 0
    assert L.moe_layer_forward_host(ctypes.byref(c), *[None] * 9, 0, st) == 0
    bad = cfg(T=0, k=11)
    assert L.moe_layer_forward(ctypes.byref(bad), *[None] * 9, 0, st) == 1


def test_binding_refuses_host_tensors_for_device_arguments():
    # a host tensor's address handed to a kernel would fault the GPU: the
    # binding refuses it before the library is called (runs without a GPU)
    import torch
    sh = moe.LayerShape(T=4, d=64, n_routed=2, n_zero=1, top_k=2, ffn=64)
    x = torch.zeros(4, 64, dtype=torch.bfloat16)
    w_r, b = torch.zeros(3, 64), torch.zeros(3)
    wg, wd = torch.zeros(2, 64, 64, dtype=torch.bfloat16), torch.zeros(2, 64, 64,
                                                                        dtype=torch.bfloat16)
    ws = torch.zeros(1 << 20, dtype=torch.uint8)
    with pytest.raises(ValueError, match="CUDA tensor"):
        moe.layer_forward(sh, x, w_r, b, wg, wg, wd, ws)
    with pytest.raises(ValueError, match="CUDA tensor"):
        moe.route(sh, x, w_r, b, ws)
    with pytest.raises(ValueError, match="CUDA tensor"):
        moe.read_device_error(ws)
    # the host entry point checks its device weights as well as its host buffers
    with pytest.raises(ValueError, match="CUDA tensor"):
        moe.layer_forward_host(sh, x, w_r, b, wg, wg, wd, ws, torch.zeros_like(x))


def test_python_binding_marshalling_checks():
    import torch
    sh = moe.LayerShape(T=4, d=64, n_routed=2, n_zero=1, top_k=2, ffn=64)
    x = torch.zeros(4, 64, dtype=torch.float32)
    with pytest.raises(ValueError):
        moe.route(sh, x, torch.zeros(3, 64), torch.zeros(3), ws=torch.zeros(1))
