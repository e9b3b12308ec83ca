"""CPU oracle for the MoE layer with zero-computation experts (test infrastructure).

Only the tests, ``__graft_entry__.smoke()`` and the bench's CPU-baseline leg may
import this package. It is the plain fp64 definition of the layer
(``moe_oracle.c``) behind a ctypes wrapper; it shares no code with the CUDA
library and is never fed anything the CUDA library computed.

Every function takes CPU torch tensors (or numpy arrays) in their stored types
and returns float64 / int32 numpy arrays. bf16 tensors are passed as their raw
16-bit patterns and widened exactly inside the C code.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "moe_oracle.c")
_BUILD = os.path.join(_HERE, "_build")
_SO = os.path.join(_BUILD, "libmoe_oracle.so")
_lock = threading.Lock()
_lib = None

F32, BF16 = 0, 1


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (plain -O2, OpenMP, no fast-math)."""
    os.makedirs(_BUILD, exist_ok=True)
    if (not force and os.path.exists(_SO)
            and os.path.getmtime(_SO) >= os.path.getmtime(_SRC)):
        return _SO
    tmp = _SO + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11",
           "-fno-fast-math", "-o", tmp, _SRC, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _SO)
    return _SO


def _load():
    """The compiled oracle. MOE_ORACLE_LIB, when set, names a compiled variant
    of moe_oracle.c to load instead: the test that plants mistakes in the
    oracle uses it to check that the pins catch each one."""
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(os.environ.get("MOE_ORACLE_LIB") or build())
            P, I64, I, D = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_double
            sig = {
                "oracle_num_threads": ([], I),
                "oracle_set_num_threads": ([I], None),
                "oracle_router_logits": ([I64, I64, I64, I, P, P, P], None),
                "oracle_select": ([I64, I64, I64, P, P, P, P, P], None),
                "oracle_gates_of": ([I64, I64, I64, P, P, P], None),
                "oracle_route": ([I64, I64, I64, I64, I, P, P, P, P, P, P, P], None),
                "oracle_dispatch": ([I64, I64, I64, I64, P, P, P, P, P], None),
                "oracle_expert_rows": ([I64, I64, I, P, P, P, I64, P, P, P, P], None),
                "oracle_combine": ([I64, I64, I64, I64, D, P, P, P, P, P, P], None),
                "oracle_layer": ([I64, P, I64, I64, I64, I64, I64, I64, D, I, P, P,
                                  P, P, P, P, P, P, P, P], None),
                "oracle_pid_update": ([I64, I64, I64, I64, P, P, P, D, D, D, D, D], None),
            }
            for name, (args, res) in sig.items():
                fn = getattr(lib, name)
                fn.argtypes = args
                fn.restype = res
            _lib = lib
    return _lib


# ----------------------------------------------------------------- helpers --

def _raw(t):
    """(numpy array holding the stored bits, dtype code) of a CPU tensor."""
    if isinstance(t, np.ndarray):
        if t.dtype == np.float32:
            return np.ascontiguousarray(t), F32
        raise TypeError(t.dtype)
    t = t.detach().cpu().contiguous()
    if t.dtype == torch.float32:
        return t.numpy(), F32
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy(), BF16
    raise TypeError(t.dtype)


def _f32(t) -> np.ndarray:
    if isinstance(t, torch.Tensor):
        t = t.detach().cpu().to(torch.float32).numpy()
    return np.ascontiguousarray(t, dtype=np.float32)


def _f64(t) -> np.ndarray:
    if isinstance(t, torch.Tensor):
        t = t.detach().cpu().to(torch.float64).numpy()
    return np.ascontiguousarray(t, dtype=np.float64)


def _i32(t) -> np.ndarray:
    if isinstance(t, torch.Tensor):
        t = t.detach().cpu().to(torch.int32).numpy()
    return np.ascontiguousarray(t, dtype=np.int32)


def _p(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def num_threads() -> int:
    return _load().oracle_num_threads()


def set_num_threads(n: int) -> None:
    _load().oracle_set_num_threads(int(n))


# --------------------------------------------------------------- functions --

def router_logits(x, w_router) -> np.ndarray:
    """logits [T, E] in fp64."""
    xr, xdt = _raw(x)
    w = _f32(w_router)
    T, d = xr.shape
    E = w.shape[0]
    out = np.empty((T, E), np.float64)
    _load().oracle_router_logits(T, d, E, xdt, _p(xr), _p(w), _p(out))
    return out


def select(logits, bias, k: int):
    """(idx [T,k] int32, gate [T,k] fp64, margin [T] fp64) from fp64 logits."""
    lg = _f64(logits)
    b = _f32(bias)
    T, E = lg.shape
    idx = np.empty((T, k), np.int32)
    gate = np.empty((T, k), np.float64)
    margin = np.empty((T,), np.float64)
    _load().oracle_select(T, E, k, _p(lg), _p(b), _p(idx), _p(gate), _p(margin))
    return idx, gate, margin


def gates_of(logits, idx) -> np.ndarray:
    lg = _f64(logits)
    ix = _i32(idx)
    T, E = lg.shape
    k = ix.shape[1]
    gate = np.empty((T, k), np.float64)
    _load().oracle_gates_of(T, E, k, _p(lg), _p(ix), _p(gate))
    return gate


def route(x, w_router, bias, k: int):
    """(logits [T,E], idx [T,k], gate [T,k], margin [T])."""
    xr, xdt = _raw(x)
    w = _f32(w_router)
    b = _f32(bias)
    T, d = xr.shape
    E = w.shape[0]
    logits = np.empty((T, E), np.float64)
    idx = np.empty((T, k), np.int32)
    gate = np.empty((T, k), np.float64)
    margin = np.empty((T,), np.float64)
    _load().oracle_route(T, d, E, k, xdt, _p(xr), _p(w), _p(b), _p(logits),
                         _p(idx), _p(gate), _p(margin))
    return logits, idx, gate, margin


def dispatch(idx, n_routed: int, n_experts: int):
    """(counts [E], offsets [N+1], row_token [T*k], slot_row [T*k])."""
    ix = _i32(idx)
    T, k = ix.shape
    counts = np.empty((n_experts,), np.int32)
    offsets = np.empty((n_routed + 1,), np.int32)
    row_token = np.empty((T * k,), np.int32)
    slot_row = np.empty((T * k,), np.int32)
    _load().oracle_dispatch(T, k, n_routed, n_experts, _p(ix), _p(counts),
                            _p(offsets), _p(row_token), _p(slot_row))
    return counts, offsets, row_token, slot_row


def expert_rows(w_gate, w_up, w_down, row_expert, x_rows, want_h: bool = False):
    """y [n, d] (and h [n, F]) of each row through its expert, in fp64."""
    wg, wdt = _raw(w_gate)
    wu, wdt2 = _raw(w_up)
    wd, wdt3 = _raw(w_down)
    assert wdt == wdt2 == wdt3
    N, F, d = wg.shape
    re = _i32(row_expert)
    xr = _f64(x_rows)
    n = re.shape[0]
    y = np.empty((n, d), np.float64)
    h = np.empty((n, F), np.float64) if want_h else None
    _load().oracle_expert_rows(d, F, wdt, _p(wg), _p(wu), _p(wd), n, _p(re),
                               _p(xr), _p(y), _p(h) if want_h else None)
    return (y, h) if want_h else y


def combine(x, y_perm, idx, gate, slot_row, n_routed: int, routed_scale: float):
    """out [T, d] fp64 from dispatched expert outputs (reading R7)."""
    xx = _f64(x)
    yy = _f64(y_perm)
    ix = _i32(idx)
    g = _f64(gate)
    sr = _i32(slot_row)
    T, d = xx.shape
    k = ix.shape[1]
    out = np.empty((T, d), np.float64)
    _load().oracle_combine(T, d, n_routed, k, float(routed_scale), _p(xx),
                           _p(yy), _p(ix), _p(g), _p(sr), _p(out))
    return out


def layer(x, w_router, bias, w_gate, w_up, w_down, n_routed: int, top_k: int,
          routed_scale: float = 1.0, tokens=None, force_idx=None):
    """Per-token definition of the whole layer.

    Returns (out [n_tok, d] fp64, idx [n_tok, k], gate [n_tok, k]) for the
    tokens listed in ``tokens`` (all tokens when None)."""
    xr, xdt = _raw(x)
    wr = _f32(w_router)
    b = _f32(bias)
    T, d = xr.shape
    E = wr.shape[0]
    Z = E - n_routed
    if n_routed > 0:
        wg, wdt = _raw(w_gate)
        wu, _ = _raw(w_up)
        wd, _ = _raw(w_down)
        F = wg.shape[1]
        assert wdt == xdt, "expert weights and activations share one dtype"
    else:
        wg = wu = wd = np.zeros(1, np.float32)
        F = 1
    tok = np.arange(T, dtype=np.int32) if tokens is None else _i32(tokens)
    n = tok.shape[0]
    fi = None if force_idx is None else _i32(force_idx)
    out = np.empty((n, d), np.float64)
    idx = np.empty((n, top_k), np.int32)
    gate = np.empty((n, top_k), np.float64)
    _load().oracle_layer(n, _p(tok), T, d, n_routed, Z, top_k, F,
                         float(routed_scale), xdt, _p(xr), _p(wr), _p(b),
                         _p(wg), _p(wu), _p(wd),
                         None if fi is None else _p(fi), _p(out), _p(idx),
                         _p(gate))
    return out, idx, gate


def pid_update(counts, bias, state, T: int, k: int, n_routed: int, target: float,
               kp: float, ki: float, kd: float, max_step: float):
    """One controller step on copies of bias (fp32 [E]) and state (fp64 [2]).
    Returns (new_bias, new_state)."""
    c = _i32(counts)
    b = np.array(_f32(bias), copy=True)
    st = np.array(_f64(state), copy=True)
    E = b.shape[0]
    _load().oracle_pid_update(T, k, n_routed, E, _p(c), _p(b), _p(st), float(target),
                              float(kp), float(ki), float(kd), float(max_step))
    return b, st
