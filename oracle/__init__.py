"""CPU oracle for the routed int4 expert layer -- TEST INFRASTRUCTURE ONLY.

A ctypes front end over ``oracle.cpp`` (plain single-threaded C++).  Only the
tests, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline leg may
import this package; the CUDA library and its Python binding never do.

Every function here is pinned by ``tests/test_oracle_pins.py`` against things
other than itself: a naive fp64 brute-force path (dense dequantisation, all
experts for every token, top-k by enumerating expert subsets), the dense
softmax mixture that top_k = n_experts reduces to, a plain SwiGLU FFN for one
expert with weight 1 (torch fp64), closed forms (all-equal weights, one-hot
activations, tied router rows) and the paged-vs-resident invariant under slot
permutation and routed-only binding.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.cpp")
_LIB = os.path.join(_HERE, "liboracle.so")

OK, BAD_ARG, NOT_BOUND, SLOT_CONFLICT = 0, 1, 2, 3
FORMATS = {"int4": 0, "nvfp4": 1}   # weight formats of an expert blob

_lib = None


def build(force: bool = False) -> str:
    """Compile oracle.cpp into liboracle.so (plain g++, no GPU)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + ".tmp%d" % os.getpid()
        subprocess.check_call(["g++", "-O2", "-std=c++17", "-ffp-contract=off",
                               "-fno-fast-math", "-shared", "-fPIC", _SRC, "-o", tmp])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB)
        P = ctypes.c_void_p
        i = ctypes.c_int
        lib.oracle_expert_bytes.restype = ctypes.c_size_t
        lib.oracle_expert_bytes.argtypes = [i, i]
        lib.oracle_route.restype = i
        lib.oracle_route.argtypes = [P, i, i, P, P, i, i, P, P, P]
        lib.oracle_route_sigmoid.restype = i
        lib.oracle_route_sigmoid.argtypes = [P, i, i, P, P, P, ctypes.c_float, i, i, P, P, P]
        lib.oracle_expert_ffn.restype = i
        lib.oracle_expert_ffn.argtypes = [P, i, i, P, i, P, P, P, P]
        lib.oracle_expert_bytes_fmt.restype = ctypes.c_size_t
        lib.oracle_expert_bytes_fmt.argtypes = [i, i, i]
        lib.oracle_expert_ffn_fmt.restype = i
        lib.oracle_expert_ffn_fmt.argtypes = [P, i, i, i, P, i, P, P, P, P]
        lib.oracle_forward_routed_fmt.restype = i
        lib.oracle_forward_routed_fmt.argtypes = [P, i, i, i, i, i, i, P, P, i, P, P, P, P, i]
        lib.oracle_forward_routed.restype = i
        lib.oracle_forward_routed.argtypes = [P, i, i, i, i, i, i, P, P, i, P, P, P, P]
        lib.oracle_forward.restype = i
        lib.oracle_forward.argtypes = [P, i, i, i, i, i, i, P, P, P, P, i, P, P, P, P, P]
        _lib = lib
    return _lib


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    return None if a is None else np.ascontiguousarray(a, dtype=dtype)


def _ptr_array(blobs):
    arr = (ctypes.c_void_p * max(1, len(blobs)))()
    for n, b in enumerate(blobs):
        arr[n] = None if b is None else b.ctypes.data
    return arr


def expert_bytes(hidden: int, inter: int, fmt: str = "int4") -> int:
    return int(_load().oracle_expert_bytes_fmt(hidden, inter, FORMATS[fmt]))


def route(x_bf16: np.ndarray, W: np.ndarray, bias, top_k: int):
    """Router.  x_bf16: u16 bf16 bits [T][H]; W: fp32 [E][H]; bias fp32 [E] or None.

    Returns (logits fp32 [T][E], idx int32 [T][k], w fp32 [T][k]).
    """
    x = _c(x_bf16, np.uint16)
    W = _c(W, np.float32)
    b = _c(bias, np.float32)
    T, H = x.shape
    E = W.shape[0]
    logits = np.zeros((T, E), np.float32)
    idx = np.zeros((T, top_k), np.int32)
    w = np.zeros((T, top_k), np.float32)
    st = _load().oracle_route(_ptr(x), T, H, _ptr(W), _ptr(b), E, top_k,
                              _ptr(logits), _ptr(idx), _ptr(w))
    if st != OK:
        raise ValueError("oracle_route status %d" % st)
    return logits, idx, w


def route_sigmoid(x_bf16: np.ndarray, W: np.ndarray, bias, corr, scale: float, top_k: int):
    """Sigmoid router with correction bias `corr` (fp32 [E] or None) and routed
    scale.  Returns (logits fp32 [T][E], idx int32 [T][k], w fp32 [T][k])."""
    x = _c(x_bf16, np.uint16)
    W = _c(W, np.float32)
    b = _c(bias, np.float32)
    c = _c(corr, np.float32)
    T, H = x.shape
    E = W.shape[0]
    logits = np.zeros((T, E), np.float32)
    idx = np.zeros((T, top_k), np.int32)
    w = np.zeros((T, top_k), np.float32)
    st = _load().oracle_route_sigmoid(_ptr(x), T, H, _ptr(W), _ptr(b), _ptr(c), float(scale), E,
                                      top_k, _ptr(logits), _ptr(idx), _ptr(w))
    if st != OK:
        raise ValueError("oracle_route_sigmoid status %d" % st)
    return logits, idx, w


def expert_ffn(blob: np.ndarray, hidden: int, inter: int, x: np.ndarray, fmt: str = "int4"):
    """One expert on fp32 activations x [n][H].  Returns (g, u, h, y)."""
    blob = _c(blob, np.uint8)
    x = _c(x, np.float32)
    n = x.shape[0]
    g = np.zeros((n, inter), np.float32)
    u = np.zeros((n, inter), np.float32)
    h = np.zeros((n, inter), np.float32)
    y = np.zeros((n, hidden), np.float32)
    st = _load().oracle_expert_ffn_fmt(_ptr(blob), hidden, inter, FORMATS[fmt], _ptr(x), n,
                                       _ptr(g), _ptr(u), _ptr(h), _ptr(y))
    if st != OK:
        raise ValueError("oracle_expert_ffn status %d" % st)
    return g, u, h, y


def forward_routed(x_bf16, hidden, inter, n_experts, top_k, slot_expert, slot_blobs,
                   shared_blobs, idx, w, fmt: str = "int4"):
    """Layer output (fp32 [T][H]) for given routing; returns (status, out).

    slot_expert: int [n_slots] expert id per slot (-1 = empty); slot_blobs:
    list of u8 arrays (or None) per slot; shared_blobs: list of S u8 arrays.
    """
    x = _c(x_bf16, np.uint16)
    T = x.shape[0]
    S = len(shared_blobs)
    se = _c(slot_expert, np.int32)
    slot_blobs = [None if b is None else _c(b, np.uint8) for b in slot_blobs]
    shared_blobs = [_c(b, np.uint8) for b in shared_blobs]
    idx = _c(idx, np.int32)
    w = _c(w, np.float32)
    out = np.zeros((T, hidden), np.float32)
    st = _load().oracle_forward_routed_fmt(
        _ptr(x), T, hidden, inter, n_experts, top_k, S, _ptr(se), _ptr_array(slot_blobs),
        len(se), _ptr_array(shared_blobs), _ptr(idx), _ptr(w), _ptr(out), FORMATS[fmt])
    return st, out


def forward(x_bf16, hidden, inter, W, bias, top_k, slot_expert, slot_blobs, shared_blobs):
    """Router + layer.  Returns (status, out fp32 [T][H], logits, idx, w)."""
    x = _c(x_bf16, np.uint16)
    T = x.shape[0]
    W = _c(W, np.float32)
    b = _c(bias, np.float32)
    E = W.shape[0]
    S = len(shared_blobs)
    se = _c(slot_expert, np.int32)
    slot_blobs = [None if bb is None else _c(bb, np.uint8) for bb in slot_blobs]
    shared_blobs = [_c(bb, np.uint8) for bb in shared_blobs]
    logits = np.zeros((T, E), np.float32)
    idx = np.zeros((T, top_k), np.int32)
    w = np.zeros((T, top_k), np.float32)
    out = np.zeros((T, hidden), np.float32)
    st = _load().oracle_forward(
        _ptr(x), T, hidden, inter, E, top_k, S, _ptr(W), _ptr(b), _ptr(se),
        _ptr_array(slot_blobs), len(se), _ptr_array(shared_blobs), _ptr(logits),
        _ptr(idx), _ptr(w), _ptr(out))
    return st, out, logits, idx, w
