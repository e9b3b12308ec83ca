"""B200 (sm_100a) library for the forward pass of a mixture-of-experts FFN
layer with zero-computation (identity) experts: Python binding.

Every step of the layer runs in the CUDA library ``_lib/libmoe.so`` behind the
C ABI declared in ``include/moe_api.h``. This module only marshals torch CUDA
tensors into that ABI (pointers, sizes, the current stream); it computes
nothing itself and has no fallback: if the library is missing, importing the
binding's functions raises.

All CUDA tensors of a call must live on the current device
(``torch.cuda.set_device``): the library launches its kernels there, on the
given stream or that device's current stream, and they read the tensors
directly.

Build the library with ``python -m expert_routing_dispatch_router_b200.build``.
"""
from __future__ import annotations

import ctypes
import os
import re
from dataclasses import dataclass
from typing import Optional

import torch

from . import build as _build

LIB_PATH = _build.LIB
HEADER = os.path.join(_build.ROOT, "include", "moe_api.h")

MOE_F32, MOE_BF16 = 0, 1
STATUS = {0: "MOE_OK", 1: "MOE_ERR_INVALID_ARG", 2: "MOE_ERR_UNSUPPORTED",
          3: "MOE_ERR_WORKSPACE", 4: "MOE_ERR_CUDA", 5: "MOE_ERR_DEVICE_CHECK"}


class MoEError(RuntimeError):
    def __init__(self, fn: str, status: int, msg: str):
        super().__init__(f"{fn}: {STATUS.get(status, status)} ({msg})")
        self.status = status


class MoEConfig(ctypes.Structure):
    _fields_ = [("T", ctypes.c_int32), ("d", ctypes.c_int32),
                ("n_routed", ctypes.c_int32), ("n_zero", ctypes.c_int32),
                ("top_k", ctypes.c_int32), ("ffn", ctypes.c_int32),
                ("act_dtype", ctypes.c_int32), ("routed_scale", ctypes.c_float)]


class MoEPIDParams(ctypes.Structure):
    _fields_ = [("target_routed_share", ctypes.c_float), ("kp", ctypes.c_float),
                ("ki", ctypes.c_float), ("kd", ctypes.c_float),
                ("max_step", ctypes.c_float)]


@dataclass(frozen=True)
class LayerShape:
    """Sizes of one layer call (mirrors moe_config_t)."""
    T: int
    d: int
    n_routed: int
    n_zero: int
    top_k: int
    ffn: int
    act_dtype: torch.dtype = torch.bfloat16
    routed_scale: float = 1.0

    @property
    def E(self) -> int:
        return self.n_routed + self.n_zero

    def c(self) -> MoEConfig:
        code = {torch.float32: MOE_F32, torch.bfloat16: MOE_BF16}[self.act_dtype]
        return MoEConfig(self.T, self.d, self.n_routed, self.n_zero, self.top_k,
                         self.ffn, code, float(self.routed_scale))


_lib = None
P = ctypes.c_void_p


def declared_functions():
    """Names of the functions ``include/moe_api.h`` declares."""
    with open(HEADER) as f:
        text = f.read()
    return sorted(set(re.findall(r"^\s*(?:[\w]+\s*\*?\s+)+\*?(moe_\w+)\(", text, re.M)))


def lib():
    """The loaded CUDA library (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(
                f"CUDA library {LIB_PATH} is missing; build it with "
                "`python -m expert_routing_dispatch_router_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        C = ctypes.POINTER(MoEConfig)
        i32 = ctypes.c_int
        sz = ctypes.c_size_t
        sig = {
            "moe_workspace_size": ([C], sz),
            "moe_route": ([C, P, P, P, P, P, P, P, P, sz, P], i32),
            "moe_dispatch": ([C, P, P, P, P, P, P, P, P, sz, P], i32),
            "moe_expert_ffn": ([C, P, P, P, P, P, P, P, sz, P], i32),
            "moe_combine": ([C, P, P, P, P, P, P, P], i32),
            "moe_layer_forward": ([C, P, P, P, P, P, P, P, P, P, sz, P], i32),
            "moe_layer_forward_host": ([C, P, P, P, P, P, P, P, P, P, sz, P], i32),
            "moe_read_device_error": ([P, P, P], i32),
            "moe_selftest_wait_limit": ([P, ctypes.c_size_t, P], i32),
            "moe_route_noalloc": ([C, P, P, P, P, P, P, P, P], i32),
            "moe_bias_pid_update": ([C, P, P, P, ctypes.POINTER(MoEPIDParams), P], i32),
            "moe_layer_launch_count": ([C], ctypes.c_int32),
            "moe_ep_local_experts": ([C, ctypes.c_int32, ctypes.c_int32], ctypes.c_int32),
            "moe_ep_plan": ([C, ctypes.c_int32, ctypes.c_int32, P, P, P, P], i32),
            "moe_ep_dispatch": ([C, ctypes.c_int32, P, P, P, P, P, P], i32),
            "moe_ep_return": ([C, ctypes.c_int32, ctypes.c_int32, P, P, P, P, P, P], i32),
            "moe_status_string": ([i32], ctypes.c_char_p),
        }
        for name, (args, res) in sig.items():
            fn = getattr(L, name)
            fn.argtypes = args
            fn.restype = res
        _lib = L
    return _lib


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _check(fn: str, status: int):
    if status != 0:
        raise MoEError(fn, status, lib().moe_status_string(status).decode())


def _need(t: torch.Tensor, name: str, dtype, shape=None, on_device=True):
    """Checks one tensor argument before its address goes to the library. A
    host tensor where device memory is expected (or the reverse) would be
    dereferenced by a kernel or a copy on the wrong side, so it is refused."""
    if t.dtype != dtype:
        raise ValueError(f"{name}: dtype {t.dtype}, expected {dtype}")
    if on_device and not t.is_cuda:
        raise ValueError(f"{name}: must be a CUDA tensor")
    if not on_device and t.is_cuda:
        raise ValueError(f"{name}: must be a host tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name}: must be contiguous")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name}: shape {tuple(t.shape)}, expected {tuple(shape)}")


def _ws(ws: torch.Tensor):
    """(address, size in bytes) of a workspace tensor, which must be device
    memory (alloc_workspace gives one)."""
    if not ws.is_cuda or not ws.is_contiguous():
        raise ValueError("ws: must be a contiguous CUDA tensor (use alloc_workspace)")
    return ctypes.c_void_p(ws.data_ptr()), ws.numel() * ws.element_size()


def workspace_size(shape: LayerShape) -> int:
    return int(lib().moe_workspace_size(ctypes.byref(shape.c())))


def alloc_workspace(shape: LayerShape, device="cuda") -> torch.Tensor:
    """Zeroed workspace (the error word must start at zero)."""
    n = workspace_size(shape)
    if n == 0:
        raise ValueError(f"invalid or unsupported shape {shape}")
    return torch.zeros(n, dtype=torch.uint8, device=device)


def launch_count(shape: LayerShape) -> int:
    return int(lib().moe_layer_launch_count(ctypes.byref(shape.c())))


def route(shape: LayerShape, x, w_router, bias, ws, logits=None, flags=None,
          stream=None):
    """Router + top-k + gates -> (topk_idx [T,k] int32, topk_gate [T,k] f32)."""
    T, E, k = shape.T, shape.E, shape.top_k
    _need(x, "x", shape.act_dtype, (T, shape.d))
    _need(w_router, "w_router", torch.float32, (E, shape.d))
    _need(bias, "bias", torch.float32, (E,))
    idx = torch.empty(T, k, dtype=torch.int32, device=x.device)
    gate = torch.empty(T, k, dtype=torch.float32, device=x.device)
    if logits is not None:
        _need(logits, "logits", torch.float32, (T, E))
    if flags is not None:
        _need(flags, "flags", torch.uint8, (T,))
    st = lib().moe_route(ctypes.byref(shape.c()), _ptr(x), _ptr(w_router), _ptr(bias),
                         _ptr(logits), _ptr(idx), _ptr(gate), _ptr(flags), *_ws(ws),
                         _stream(stream))
    _check("moe_route", st)
    return idx, gate


def route_noalloc(shape: LayerShape, x, w_router, bias, topk_idx, topk_gate,
                  logits=None, flags=None, stream=None):
    """moe_route without a workspace, for callers that cannot allocate device
    memory: every output is caller-provided and the library's own fixed
    scratch array is used (T * E <= 4194304). Calls sharing a device must not
    overlap on the GPU."""
    T, E, k = shape.T, shape.E, shape.top_k
    _need(x, "x", shape.act_dtype, (T, shape.d))
    _need(w_router, "w_router", torch.float32, (E, shape.d))
    _need(bias, "bias", torch.float32, (E,))
    _need(topk_idx, "topk_idx", torch.int32, (T, k))
    _need(topk_gate, "topk_gate", torch.float32, (T, k))
    if logits is not None:
        _need(logits, "logits", torch.float32, (T, E))
    if flags is not None:
        _need(flags, "flags", torch.uint8, (T,))
    st = lib().moe_route_noalloc(ctypes.byref(shape.c()), _ptr(x), _ptr(w_router),
                                 _ptr(bias), _ptr(logits), _ptr(topk_idx),
                                 _ptr(topk_gate), _ptr(flags), _stream(stream))
    _check("moe_route_noalloc", st)
    return topk_idx, topk_gate


def dispatch(shape: LayerShape, x, topk_idx, ws, stream=None):
    """-> (counts [E], offsets [N+1], row_token [T*k], slot_row [T*k], x_perm [T*k, d])."""
    T, k = shape.T, shape.top_k
    _need(x, "x", shape.act_dtype, (T, shape.d))
    _need(topk_idx, "topk_idx", torch.int32, (T, k))
    dev = x.device
    counts = torch.empty(shape.E, dtype=torch.int32, device=dev)
    offsets = torch.empty(shape.n_routed + 1, dtype=torch.int32, device=dev)
    row_token = torch.empty(T * k, dtype=torch.int32, device=dev)
    slot_row = torch.empty(T * k, dtype=torch.int32, device=dev)
    x_perm = torch.empty(T * k, shape.d, dtype=shape.act_dtype, device=dev)
    st = lib().moe_dispatch(ctypes.byref(shape.c()), _ptr(x), _ptr(topk_idx),
                            _ptr(counts), _ptr(offsets), _ptr(row_token),
                            _ptr(slot_row), _ptr(x_perm), *_ws(ws),
                            _stream(stream))
    _check("moe_dispatch", st)
    return counts, offsets, row_token, slot_row, x_perm


def expert_ffn(shape: LayerShape, x_perm, offsets, w_gate, w_up, w_down, ws,
               y_perm=None, stream=None):
    """-> y_perm [T*k, d] in the activation dtype (rows >= R untouched)."""
    T, k, d, F, N = shape.T, shape.top_k, shape.d, shape.ffn, shape.n_routed
    _need(x_perm, "x_perm", shape.act_dtype, (T * k, d))
    _need(offsets, "offsets", torch.int32, (N + 1,))
    for name, w, shp in (("w_gate", w_gate, (N, F, d)), ("w_up", w_up, (N, F, d)),
                         ("w_down", w_down, (N, d, F))):
        _need(w, name, shape.act_dtype, shp)
    if y_perm is None:
        y_perm = torch.empty(T * k, d, dtype=shape.act_dtype, device=x_perm.device)
    _need(y_perm, "y_perm", shape.act_dtype, (T * k, d))
    st = lib().moe_expert_ffn(ctypes.byref(shape.c()), _ptr(x_perm), _ptr(offsets),
                              _ptr(w_gate), _ptr(w_up), _ptr(w_down), _ptr(y_perm),
                              *_ws(ws), _stream(stream))
    _check("moe_expert_ffn", st)
    return y_perm


def combine(shape: LayerShape, x, y_perm, topk_idx, topk_gate, slot_row, out=None,
            stream=None):
    T, k, d = shape.T, shape.top_k, shape.d
    _need(x, "x", shape.act_dtype, (T, d))
    _need(y_perm, "y_perm", shape.act_dtype, (T * k, d))
    _need(topk_idx, "topk_idx", torch.int32, (T, k))
    _need(topk_gate, "topk_gate", torch.float32, (T, k))
    _need(slot_row, "slot_row", torch.int32, (T * k,))
    if out is None:
        out = torch.empty(T, d, dtype=shape.act_dtype, device=x.device)
    _need(out, "out", shape.act_dtype, (T, d))
    st = lib().moe_combine(ctypes.byref(shape.c()), _ptr(x), _ptr(y_perm),
                           _ptr(topk_idx), _ptr(topk_gate), _ptr(slot_row), _ptr(out),
                           _stream(stream))
    _check("moe_combine", st)
    return out


def ep_local_experts(shape: LayerShape, rank: int, world: int) -> int:
    """Routed experts rank `rank` owns when the N routed ids are split evenly
    over `world` ranks (the first N % world ranks take one more)."""
    n = int(lib().moe_ep_local_experts(ctypes.byref(shape.c()), rank, world))
    if n < 0:
        raise ValueError(f"invalid rank {rank} of {world} or shape {shape}")
    return n


def _pointer_array(tensors, dtype, rows_min, d, device):
    """Device array of the data addresses of `tensors` (one per rank)."""
    for r, t in enumerate(tensors):
        _need(t, f"buffer of rank {r}", dtype)
        if t.dim() != 2 or t.shape[1] != d or t.shape[0] < rows_min:
            raise ValueError(f"buffer of rank {r}: shape {tuple(t.shape)}, expected "
                             f"[>= {rows_min}, {d}]")
    return torch.tensor([t.data_ptr() for t in tensors], dtype=torch.int64, device=device)


def ep_plan(shape: LayerShape, rank: int, world: int, counts_all, stream=None):
    """-> (dest_row [N], recv_offsets [n_rank + 1]) from every rank's counts
    (counts_all [world, E] int32, on the device)."""
    N, E = shape.n_routed, shape.E
    _need(counts_all, "counts_all", torch.int32, (world, E))
    dev = counts_all.device
    dest_row = torch.empty(N, dtype=torch.int32, device=dev)
    recv_offsets = torch.empty(ep_local_experts(shape, rank, world) + 1, dtype=torch.int32,
                               device=dev)
    st = lib().moe_ep_plan(ctypes.byref(shape.c()), rank, world, _ptr(counts_all),
                           _ptr(dest_row), _ptr(recv_offsets), _stream(stream))
    _check("moe_ep_plan", st)
    return dest_row, recv_offsets


def ep_dispatch(shape: LayerShape, world: int, x, offsets, row_token, dest_row, recv_bufs,
                stream=None):
    """Sends this rank's routed rows into the owners' receive buffers
    (recv_bufs: one [rows, d] tensor per rank, each with room for every row
    its experts get)."""
    T, k, d, N = shape.T, shape.top_k, shape.d, shape.n_routed
    _need(x, "x", shape.act_dtype, (T, d))
    _need(offsets, "offsets", torch.int32, (N + 1,))
    _need(row_token, "row_token", torch.int32, (T * k,))
    _need(dest_row, "dest_row", torch.int32, (N,))
    if len(recv_bufs) != world:
        raise ValueError("one receive buffer per rank")
    ptrs = _pointer_array(recv_bufs, shape.act_dtype, 0, d, x.device)
    st = lib().moe_ep_dispatch(ctypes.byref(shape.c()), world, _ptr(x), _ptr(offsets),
                               _ptr(row_token), _ptr(dest_row), _ptr(ptrs), _stream(stream))
    _check("moe_ep_dispatch", st)
    return ptrs  # kept alive by the caller until the stream has run the kernel


def ep_return(shape: LayerShape, rank: int, world: int, y_recv, recv_offsets, counts_all,
              offsets_all, y_homes, stream=None):
    """Sends this rank's expert output rows back into every source rank's
    y_perm (y_homes: one [T*k, d] tensor per rank)."""
    T, k, d, N, E = shape.T, shape.top_k, shape.d, shape.n_routed, shape.E
    _need(y_recv, "y_recv", shape.act_dtype)
    _need(recv_offsets, "recv_offsets", torch.int32,
          (ep_local_experts(shape, rank, world) + 1,))
    _need(counts_all, "counts_all", torch.int32, (world, E))
    _need(offsets_all, "offsets_all", torch.int32, (world, N + 1))
    if len(y_homes) != world:
        raise ValueError("one y_perm per rank")
    ptrs = _pointer_array(y_homes, shape.act_dtype, T * k, d, y_recv.device)
    st = lib().moe_ep_return(ctypes.byref(shape.c()), rank, world, _ptr(y_recv),
                             _ptr(recv_offsets), _ptr(counts_all), _ptr(offsets_all),
                             _ptr(ptrs), _stream(stream))
    _check("moe_ep_return", st)
    return ptrs


def layer_forward(shape: LayerShape, x, w_router, bias, w_gate, w_up, w_down, ws,
                  out=None, counts=None, stream=None):
    """The whole layer -> out [T, d]; counts [E] (optional) gets slots per expert."""
    T, d, F, N, E = shape.T, shape.d, shape.ffn, shape.n_routed, shape.E
    _need(x, "x", shape.act_dtype, (T, d))
    _need(w_router, "w_router", torch.float32, (E, d))
    _need(bias, "bias", torch.float32, (E,))
    if N > 0:
        for name, w, shp in (("w_gate", w_gate, (N, F, d)), ("w_up", w_up, (N, F, d)),
                             ("w_down", w_down, (N, d, F))):
            _need(w, name, shape.act_dtype, shp)
    if out is None:
        out = torch.empty(T, d, dtype=shape.act_dtype, device=x.device)
    _need(out, "out", shape.act_dtype, (T, d))
    if counts is not None:
        _need(counts, "counts", torch.int32, (E,))
    st = lib().moe_layer_forward(ctypes.byref(shape.c()), _ptr(x), _ptr(w_router),
                                 _ptr(bias), _ptr(w_gate), _ptr(w_up), _ptr(w_down),
                                 _ptr(out), _ptr(counts), *_ws(ws),
                                 _stream(stream))
    _check("moe_layer_forward", st)
    return out


def layer_forward_host(shape: LayerShape, x_host, w_router, bias, w_gate, w_up,
                       w_down, ws, out_host, counts_host=None, stream=None):
    """The whole layer with x and out in (pinned) host memory; asynchronous:
    synchronise the stream before reading out_host."""
    T, d, E = shape.T, shape.d, shape.E
    F, N = shape.ffn, shape.n_routed
    _need(x_host, "x_host", shape.act_dtype, (T, d), on_device=False)
    _need(out_host, "out_host", shape.act_dtype, (T, d), on_device=False)
    if counts_host is not None:
        _need(counts_host, "counts_host", torch.int32, (E,), on_device=False)
    _need(w_router, "w_router", torch.float32, (E, d))
    _need(bias, "bias", torch.float32, (E,))
    if N > 0:
        for name, w, shp in (("w_gate", w_gate, (N, F, d)), ("w_up", w_up, (N, F, d)),
                             ("w_down", w_down, (N, d, F))):
            _need(w, name, shape.act_dtype, shp)
    st = lib().moe_layer_forward_host(ctypes.byref(shape.c()), _ptr(x_host),
                                      _ptr(w_router), _ptr(bias), _ptr(w_gate),
                                      _ptr(w_up), _ptr(w_down), _ptr(out_host),
                                      _ptr(counts_host), *_ws(ws),
                                      _stream(stream))
    _check("moe_layer_forward_host", st)
    return out_host


def read_device_error(ws, stream=None) -> int:
    """Waits for the stream; returns (and clears) the workspace error word."""
    code = ctypes.c_int32(0)
    lib().moe_read_device_error(_ws(ws)[0], ctypes.byref(code), _stream(stream))
    return int(code.value)


def selftest_wait_limit(ws, stream=None) -> None:
    """Runs the device-side wait-limit self-test: after ~2 s the workspace
    error word holds 1 (read it with read_device_error)."""
    _check("moe_selftest_wait_limit",
           lib().moe_selftest_wait_limit(*_ws(ws),
                                         _stream(stream)))


def bias_pid_update(shape: LayerShape, counts, bias, state, target: float, kp: float,
                    ki: float = 0.0, kd: float = 0.0, max_step: float = 1.0,
                    stream=None):
    """One PID step on the zero experts' router bias (in place on `bias` and
    `state`), from the per-expert counts of the last layer call."""
    _need(counts, "counts", torch.int32, (shape.E,))
    _need(bias, "bias", torch.float32, (shape.E,))
    _need(state, "state", torch.float64, (2,))
    prm = MoEPIDParams(target, kp, ki, kd, max_step)
    st = lib().moe_bias_pid_update(ctypes.byref(shape.c()), _ptr(counts), _ptr(bias),
                                   _ptr(state), ctypes.byref(prm), _stream(stream))
    _check("moe_bias_pid_update", st)
    return bias, state
