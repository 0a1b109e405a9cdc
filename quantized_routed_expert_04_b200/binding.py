"""Thin ctypes binding of libstrata_moe.so (include/strata_moe.h).

Argument marshalling only: every step of the layer runs in the library's CUDA
kernels.  Functions take the C names; device buffers may be torch tensors
(their data_ptr is passed) or integer device addresses; streams may be
torch.cuda.Stream objects, raw handles, or None for the current torch stream.
The library must have been built (quantized_routed_expert_04_b200.build);
there is no fallback: a missing library raises.
"""
from __future__ import annotations

import ctypes
import enum
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libstrata_moe.so")

_lib = None


class Status(enum.IntEnum):
    OK = 0
    INVALID_ARG = 1
    UNSUPPORTED = 2
    NOT_BOUND = 3
    SLOT_CONFLICT = 4
    TOO_MANY_EXPERTS = 5
    OOM = 6
    CUDA = 7
    DEVICE_STATUS = 8
    SCRATCH_LIMIT = 9
    RANGE = 10


class ArenaStats(ctypes.Structure):
    _fields_ = [("hits", ctypes.c_int), ("misses", ctypes.c_int), ("bytes", ctypes.c_size_t)]


class PrefillStats(ctypes.Structure):
    _fields_ = [("chunks", ctypes.c_int), ("passes", ctypes.c_int), ("hits", ctypes.c_int),
                ("misses", ctypes.c_int), ("bytes", ctypes.c_size_t)]


class StrataError(RuntimeError):
    def __init__(self, status, where=""):
        self.status = Status(status)
        super().__init__("%s: %s" % (where, _load().strata_status_str(int(status)).decode()))


def load_library():
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError("libstrata_moe.so is not built (run python -m "
                               "quantized_routed_expert_04_b200.build)")
        lib = ctypes.CDLL(LIB_PATH)
        P, I, Z = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
        sig = {
            "strata_moe_create": (I, [I, I, I, I, I, I, ctypes.POINTER(P)]),
            "strata_moe_destroy": (None, [P]),
            "strata_moe_expert_bytes": (Z, [I, I]),
            "strata_moe_expert_bytes_fmt": (Z, [I, I, I]),
            "strata_moe_set_format": (I, [P, I]),
            "strata_moe_set_router": (I, [P, P, P]),
            "strata_moe_bind_shared": (I, [P, I, P]),
            "strata_moe_set_routing": (I, [P, I, P, ctypes.c_float]),
            "strata_moe_bind_slot": (I, [P, I, I, P]),
            "strata_moe_slot_expert": (I, [P, I]),
            "strata_moe_reserve": (I, [P, I]),
            "strata_moe_route": (I, [P, P, I, P, P, P, P]),
            "strata_moe_forward": (I, [P, P, I, P, P]),
            "strata_moe_forward_routed": (I, [P, P, I, P, P, P, P]),
            "strata_moe_forward_noalloc": (I, [P, P, I, P, P]),
            "strata_moe_get_status": (I, [P, P]),
            "strata_moe_last_device_bits": (I, [P]),
            "strata_moe_profile": (I, [P, I]),
            "strata_moe_set_wait_limit": (I, [P, ctypes.c_ulonglong]),
            "strata_moe_profile_read": (I, [P, I, P, P]),
            "strata_status_str": (ctypes.c_char_p, [I]),
            "strata_arena_create": (I, [P, P, P, ctypes.POINTER(P)]),
            "strata_arena_destroy": (None, [P]),
            "strata_arena_ensure": (I, [P, P, I, P, P, ctypes.POINTER(ArenaStats)]),
            "strata_arena_copy_ms": (I, [P, ctypes.POINTER(ctypes.c_float)]),
            "strata_arena_slot_of": (I, [P, I]),
            "strata_arena_prefill": (I, [P, P, I, I, P, P, P, ctypes.POINTER(PrefillStats)]),
        }
        for name, (res, args) in sig.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _lib = lib
    return _lib


_load = load_library


def _addr(buf):
    if buf is None:
        return None
    if isinstance(buf, int):
        return buf
    return buf.data_ptr()


def _stream(stream):
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(st, where):
    if st != 0:
        raise StrataError(st, where)


def strata_moe_create(hidden, inter, n_experts, top_k, n_shared, n_slots):
    h = ctypes.c_void_p()
    _check(_load().strata_moe_create(hidden, inter, n_experts, top_k, n_shared, n_slots,
                                     ctypes.byref(h)), "strata_moe_create")
    return h.value


def strata_moe_destroy(h):
    _load().strata_moe_destroy(h)


def strata_moe_expert_bytes(hidden, inter):
    return int(_load().strata_moe_expert_bytes(hidden, inter))


FORMAT_INT4, FORMAT_NVFP4 = 0, 1


def strata_moe_expert_bytes_fmt(hidden, inter, fmt):
    return int(_load().strata_moe_expert_bytes_fmt(hidden, inter, fmt))


def strata_moe_set_format(h, fmt):
    _check(_load().strata_moe_set_format(h, int(fmt)), "strata_moe_set_format")


def strata_moe_set_router(h, W, bias=None):
    _check(_load().strata_moe_set_router(h, _addr(W), _addr(bias)), "strata_moe_set_router")


ROUTE_SOFTMAX, ROUTE_SIGMOID = 0, 1


def strata_moe_set_routing(h, mode, corr=None, routed_scale=1.0):
    _check(_load().strata_moe_set_routing(h, int(mode), _addr(corr), float(routed_scale)),
           "strata_moe_set_routing")


def strata_moe_bind_shared(h, i, blob):
    _check(_load().strata_moe_bind_shared(h, i, _addr(blob)), "strata_moe_bind_shared")


def strata_moe_bind_slot(h, slot, expert_id, blob):
    _check(_load().strata_moe_bind_slot(h, slot, expert_id, _addr(blob)), "strata_moe_bind_slot")


def strata_moe_slot_expert(h, slot):
    return int(_load().strata_moe_slot_expert(h, slot))


def strata_moe_reserve(h, max_tokens):
    _check(_load().strata_moe_reserve(h, max_tokens), "strata_moe_reserve")


def strata_moe_route(h, x, n_tokens, logits, idx, w, stream=None):
    _check(_load().strata_moe_route(h, _addr(x), n_tokens, _addr(logits), _addr(idx), _addr(w),
                                    _stream(stream)), "strata_moe_route")


def strata_moe_forward(h, x, n_tokens, out, stream=None):
    _check(_load().strata_moe_forward(h, _addr(x), n_tokens, _addr(out), _stream(stream)),
           "strata_moe_forward")


def strata_moe_forward_routed(h, x, n_tokens, idx, w, out, stream=None):
    _check(_load().strata_moe_forward_routed(h, _addr(x), n_tokens, _addr(idx), _addr(w),
                                             _addr(out), _stream(stream)),
           "strata_moe_forward_routed")


def strata_moe_forward_noalloc(h, x, n_tokens, out, stream=None):
    _check(_load().strata_moe_forward_noalloc(h, _addr(x), n_tokens, _addr(out), _stream(stream)),
           "strata_moe_forward_noalloc")


NOALLOC_SCRATCH_BYTES = 16 << 20
NOALLOC_MAX_TOKENS = 64


def strata_moe_get_status(h, stream=None):
    """Synchronise and return (Status, raw device bits); does not raise."""
    st = _load().strata_moe_get_status(h, _stream(stream))
    return Status(st), int(_load().strata_moe_last_device_bits(h))


DEFAULT_WAIT_NS = 2_000_000_000


def strata_moe_set_wait_limit(h, ns):
    _check(_load().strata_moe_set_wait_limit(h, int(ns)), "strata_moe_set_wait_limit")


def strata_moe_profile(h, enable):
    _check(_load().strata_moe_profile(h, 1 if enable else 0), "strata_moe_profile")


PHASES = ("router", "topk", "bucket", "pack", "gate_up", "down", "combine", "gather", "fused")


def strata_moe_profile_read(h):
    """{phase: (launches, total ms)} since the last read."""
    n = len(PHASES)
    launches = (ctypes.c_int * n)()
    ms = (ctypes.c_double * n)()
    _check(_load().strata_moe_profile_read(h, n, launches, ms), "strata_moe_profile_read")
    return {PHASES[i]: (launches[i], ms[i]) for i in range(n)}


def strata_status_str(st):
    return _load().strata_status_str(int(st)).decode()


def strata_arena_create(layer_h, host_pool, arena_dev):
    a = ctypes.c_void_p()
    _check(_load().strata_arena_create(layer_h, _addr(host_pool), _addr(arena_dev),
                                       ctypes.byref(a)), "strata_arena_create")
    return a.value


def strata_arena_destroy(a):
    _load().strata_arena_destroy(a)


def strata_arena_ensure(a, ids, stream=None, copy_stream=None):
    """ids: a sequence of expert ids (host).  Returns (hits, misses, bytes)."""
    import numpy as np
    arr = np.ascontiguousarray(np.asarray(ids, dtype=np.int32).reshape(-1))
    st = ArenaStats()
    _check(_load().strata_arena_ensure(a, arr.ctypes.data, int(arr.size), _stream(stream),
                                       _stream(copy_stream), ctypes.byref(st)),
           "strata_arena_ensure")
    return st.hits, st.misses, int(st.bytes)


def strata_arena_copy_ms(a):
    ms = ctypes.c_float()
    _check(_load().strata_arena_copy_ms(a, ctypes.byref(ms)), "strata_arena_copy_ms")
    return ms.value


def strata_arena_slot_of(a, expert_id):
    return int(_load().strata_arena_slot_of(a, expert_id))


def strata_arena_prefill(a, x, n_tokens, chunk_tokens, out, stream=None, copy_stream=None):
    """Chunked prefill through the arena; returns its stats as a dict."""
    st = PrefillStats()
    _check(_load().strata_arena_prefill(a, _addr(x), n_tokens, chunk_tokens, _addr(out),
                                        _stream(stream), _stream(copy_stream), ctypes.byref(st)),
           "strata_arena_prefill")
    return {"chunks": st.chunks, "passes": st.passes, "hits": st.hits, "misses": st.misses,
            "bytes": int(st.bytes)}


class Arena:
    """Owning wrapper of an expert arena over a StrataMoE layer."""

    def __init__(self, layer, host_pool, arena_dev):
        self.layer, self.host_pool, self.arena_dev = layer, host_pool, arena_dev
        self.a = strata_arena_create(layer.h, host_pool, arena_dev)

    def ensure(self, ids, stream=None, copy_stream=None):
        return strata_arena_ensure(self.a, ids, stream, copy_stream)

    def copy_ms(self):
        return strata_arena_copy_ms(self.a)

    def slot_of(self, expert_id):
        return strata_arena_slot_of(self.a, expert_id)

    def prefill(self, x, chunk_tokens, out, stream=None, copy_stream=None):
        return strata_arena_prefill(self.a, x, x.shape[0], chunk_tokens, out, stream, copy_stream)

    def close(self):
        if self.a:
            strata_arena_destroy(self.a)
            self.a = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


class StrataMoE:
    """Owning wrapper: a layer handle plus convenience methods (same calls)."""

    def __init__(self, hidden, inter, n_experts, top_k, n_shared, n_slots):
        self.hidden, self.inter, self.n_experts = hidden, inter, n_experts
        self.top_k, self.n_shared, self.n_slots = top_k, n_shared, n_slots
        self.h = strata_moe_create(hidden, inter, n_experts, top_k, n_shared, n_slots)

    def close(self):
        if self.h:
            strata_moe_destroy(self.h)
            self.h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def set_router(self, W, bias=None):
        strata_moe_set_router(self.h, W, bias)

    def set_format(self, fmt):
        strata_moe_set_format(self.h, fmt)

    def set_routing(self, mode, corr=None, routed_scale=1.0):
        strata_moe_set_routing(self.h, mode, corr, routed_scale)

    def bind_shared(self, i, blob):
        strata_moe_bind_shared(self.h, i, blob)

    def bind_slot(self, slot, expert_id, blob):
        strata_moe_bind_slot(self.h, slot, expert_id, blob)

    def reserve(self, max_tokens):
        strata_moe_reserve(self.h, max_tokens)

    def route(self, x, logits, idx, w, stream=None):
        strata_moe_route(self.h, x, x.shape[0], logits, idx, w, stream)

    def forward(self, x, out, stream=None):
        strata_moe_forward(self.h, x, x.shape[0], out, stream)

    def forward_routed(self, x, idx, w, out, stream=None):
        strata_moe_forward_routed(self.h, x, x.shape[0], idx, w, out, stream)

    def forward_noalloc(self, x, out, stream=None):
        strata_moe_forward_noalloc(self.h, x, x.shape[0], out, stream)

    def status(self, stream=None):
        return strata_moe_get_status(self.h, stream)

    def set_wait_limit(self, ns):
        strata_moe_set_wait_limit(self.h, ns)
