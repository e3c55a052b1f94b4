"""Thin ctypes binding of libmoe.so (include/moe.h), same function names.

Argument marshalling only: every step of the layer runs in the CUDA library.
Arrays may be passed as torch tensors (device or host), numpy arrays (host)
or raw integer addresses.  A status other than MOE_OK raises MoeError.  The
library must have been built (``python -m sparse_moe_expert_gemv_b200.build``);
importing this module without it raises ImportError -- there is no fallback.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

_PKG = os.path.dirname(os.path.abspath(__file__))
SO_PATH = os.path.join(_PKG, "libmoe.so")

MOE_OK = 0
STATUS_NAMES = {0: "MOE_OK", 1: "MOE_ERR_INVALID_ARG", 2: "MOE_ERR_OOM", 3: "MOE_ERR_CUDA",
                4: "MOE_ERR_STATE", 5: "MOE_ERR_BAD_SLOT", 6: "MOE_ERR_DEVICE",
                7: "MOE_ERR_TIMEOUT", 8: "MOE_ERR_NOT_SUPPORTED"}
(MOE_ERR_INVALID_ARG, MOE_ERR_OOM, MOE_ERR_CUDA, MOE_ERR_STATE, MOE_ERR_BAD_SLOT,
 MOE_ERR_DEVICE, MOE_ERR_TIMEOUT, MOE_ERR_NOT_SUPPORTED) = range(1, 9)
MOE_Q4_SYM_G32_F16 = 1
MOE_Q2_ASYM_G64_F16 = 2

# every symbol include/moe.h declares
EXPORTS = ("moe_create", "moe_configure", "moe_destroy", "moe_load_experts",
           "moe_load_shared", "moe_set_router", "moe_set_norm", "moe_set_slots",
           "moe_route", "moe_bucket", "moe_forward", "moe_forward_delta",
           "moe_forward_stack", "moe_prefill", "moe_sync", "moe_get_stats",
           "moe_last_error", "moe_status_string", "moe_expert_bytes",
           "moe_debug_poke_slot", "moe_set_profiling", "moe_read_profile",
           "moe_set_trace", "moe_read_trace", "moe_route_static", "moe_prefill_delta",
           "moe_prefill_route", "moe_route_static_status", "moe_debug_last_h",
           "moe_debug_stall_next_decode", "moe_set_host_tier", "moe_tier_prepare",
           "moe_tier_prefetch", "moe_forward_tiered", "moe_tier_stats", "moe_tier_dump_trace",
           "moe_tier_sim_create", "moe_tier_sim_request", "moe_tier_sim_counts",
           "moe_tier_sim_destroy", "moe_rmsnorm", "moe_experts_given", "moe_ep_dispatch",
           "moe_ep_combine", "moe_experts_rows")


class MoeError(RuntimeError):
    def __init__(self, status, msg):
        super().__init__(f"{STATUS_NAMES.get(status, status)}: {msg}")
        self.status = status


class MoeStats(ctypes.Structure):
    _fields_ = [("calls", ctypes.c_int64), ("tokens", ctypes.c_int64),
                ("hits", ctypes.c_int64), ("misses", ctypes.c_int64),
                ("near_ties", ctypes.c_int64), ("last_T", ctypes.c_int32),
                ("last_active", ctypes.c_int32), ("last_layer", ctypes.c_int32),
                ("E", ctypes.c_int32), ("expert_count", ctypes.POINTER(ctypes.c_int32))]


def _load():
    if not os.path.exists(SO_PATH):
        raise ImportError(f"{SO_PATH} is missing: build it with "
                          "`python -m sparse_moe_expert_gemv_b200.build`")
    L = ctypes.CDLL(SO_PATH)
    P, I, F = ctypes.c_void_p, ctypes.c_int, ctypes.c_float
    sig = {
        "moe_create": [I, I, I, I, I, ctypes.POINTER(P)],
        "moe_configure": [P, I, I, I, I],
        "moe_destroy": [P],
        "moe_load_experts": [P, I, I, I, P, P, P, I],
        "moe_load_shared": [P, I, P, P, P, I],
        "moe_set_router": [P, I, P, P, I],
        "moe_set_norm": [P, I, P, F],
        "moe_set_slots": [P, P],
        "moe_route": [P, I, P, I, P, P, P, P, P],
        "moe_bucket": [P, P, I, P, P, P],
        "moe_forward": [P, I, P, I, P],
        "moe_forward_delta": [P, I, P, I, P, P],
        "moe_forward_stack": [P, P, I, P],
        "moe_prefill": [P, I, P, I, P],
        "moe_prefill_delta": [P, I, P, I, P, P],
        "moe_prefill_route": [P, I, P, I, P, P, P, P, P],
        "moe_route_static_status": [ctypes.POINTER(I), P],
        "moe_debug_last_h": [P, P, I, P],
        "moe_debug_stall_next_decode": [P, ctypes.c_uint32],
        "moe_sync": [P, I],
        "moe_get_stats": [P, ctypes.POINTER(MoeStats)],
        "moe_debug_poke_slot": [P, I, I, ctypes.c_int32],
        "moe_set_profiling": [P, I],
        "moe_set_trace": [P, I],
        "moe_route_static": [P, I, I, I, I, P, P, P, P, P, P, P],
        "moe_read_trace": [P, ctypes.POINTER(ctypes.c_int64), I],
        "moe_read_profile": [P, ctypes.POINTER(ctypes.c_double), ctypes.POINTER(ctypes.c_int64)],
        "moe_set_host_tier": [P, I, I, ctypes.c_double],
        "moe_tier_prepare": [P, I, P, I, P],
        "moe_tier_prefetch": [P, I, P, I, P],
        "moe_forward_tiered": [P, I, P, I, P],
        "moe_tier_stats": [P, ctypes.POINTER(ctypes.c_int64)],
        "moe_tier_dump_trace": [P, ctypes.c_char_p],
        "moe_tier_sim_request": [P, ctypes.POINTER(ctypes.c_int64), I, I, ctypes.POINTER(I)],
        "moe_rmsnorm": [P, I, P, I, P, P],
        "moe_experts_given": [P, I, P, I, I, P, P, I, P, P],
        "moe_ep_dispatch": [P, P, I, I, P, P, P, P, ctypes.POINTER(ctypes.c_int32), P],
        "moe_ep_combine": [P, I, P, P, P, P, P, P, P],
        "moe_experts_rows": [P, I, P, I, P, P, P],
    }
    for name, args in sig.items():
        fn = getattr(L, name)
        fn.argtypes = args
        fn.restype = I
    L.moe_last_error.argtypes = [P]
    L.moe_last_error.restype = ctypes.c_char_p
    L.moe_status_string.argtypes = [I]
    L.moe_status_string.restype = ctypes.c_char_p
    L.moe_expert_bytes.argtypes = [I, I, I]
    L.moe_expert_bytes.restype = ctypes.c_int64
    L.moe_tier_sim_create.argtypes = [I, I, ctypes.c_double, ctypes.c_int64]
    L.moe_tier_sim_create.restype = P
    L.moe_tier_sim_counts.argtypes = [P, ctypes.POINTER(ctypes.c_int64)]
    L.moe_tier_sim_counts.restype = None
    L.moe_tier_sim_destroy.argtypes = [P]
    L.moe_tier_sim_destroy.restype = None
    return L


_lib = _load()


def lib():
    return _lib


def _ptr(a):
    """Address of a tensor / ndarray / int / None."""
    if a is None:
        return None
    if isinstance(a, int):
        return a
    if isinstance(a, np.ndarray):
        if not a.flags["C_CONTIGUOUS"]:
            raise ValueError("array must be C-contiguous")
        return a.ctypes.data
    if hasattr(a, "data_ptr"):
        if not a.is_contiguous():
            raise ValueError("tensor must be contiguous")
        return a.data_ptr()
    raise TypeError(f"cannot pass {type(a)} as a pointer")


def _is_dev(a):
    return bool(hasattr(a, "is_cuda") and a.is_cuda)


def _stream(stream):
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(ctx, rc):
    if rc != MOE_OK:
        msg = _lib.moe_last_error(ctx).decode() if ctx else ""
        raise MoeError(rc, msg)


# ------------------------------------------------------------------ C ABI
def moe_create(d, f, E, k, quant_fmt):
    out = ctypes.c_void_p()
    _check(None, _lib.moe_create(d, f, E, k, quant_fmt, ctypes.byref(out)))
    return out.value


def moe_configure(ctx, n_layers, n_shared, n_slots, max_tokens):
    _check(ctx, _lib.moe_configure(ctx, n_layers, n_shared, n_slots, max_tokens))


def moe_destroy(ctx):
    _check(None, _lib.moe_destroy(ctx))


def moe_load_experts(ctx, layer, first_expert, n_experts, codes, scales, mins=None,
                     src_is_device=None):
    dev = _is_dev(codes) if src_is_device is None else bool(src_is_device)
    _check(ctx, _lib.moe_load_experts(ctx, layer, first_expert, n_experts, _ptr(codes),
                                      _ptr(scales), _ptr(mins), int(dev)))


def moe_load_shared(ctx, layer, codes, scales, mins=None, src_is_device=None):
    dev = _is_dev(codes) if src_is_device is None else bool(src_is_device)
    _check(ctx, _lib.moe_load_shared(ctx, layer, _ptr(codes), _ptr(scales), _ptr(mins), int(dev)))


def moe_set_router(ctx, layer, W, bias=None, src_is_device=None):
    dev = _is_dev(W) if src_is_device is None else bool(src_is_device)
    _check(ctx, _lib.moe_set_router(ctx, layer, _ptr(W), _ptr(bias), int(dev)))


def moe_set_norm(ctx, layer, gamma=None, eps=1e-6):
    _check(ctx, _lib.moe_set_norm(ctx, layer, _ptr(gamma), float(eps)))


def moe_set_slots(ctx, slot_of):
    a = np.ascontiguousarray(slot_of, dtype=np.int32)
    _check(ctx, _lib.moe_set_slots(ctx, _ptr(a)))


def moe_route(ctx, layer, h, T, idx, w, bucket_off=None, bucket_perm=None, stream=None):
    _check(ctx, _lib.moe_route(ctx, layer, _ptr(h), T, _ptr(idx), _ptr(w), _ptr(bucket_off),
                               _ptr(bucket_perm), _stream(stream)))


def moe_bucket(ctx, idx, T, bucket_off, bucket_perm, stream=None):
    _check(ctx, _lib.moe_bucket(ctx, _ptr(idx), T, _ptr(bucket_off), _ptr(bucket_perm),
                                _stream(stream)))


def moe_forward(ctx, layer, x, T, stream=None):
    _check(ctx, _lib.moe_forward(ctx, layer, _ptr(x), T, _stream(stream)))


def moe_forward_delta(ctx, layer, x, T, delta, stream=None):
    _check(ctx, _lib.moe_forward_delta(ctx, layer, _ptr(x), T, _ptr(delta), _stream(stream)))


def moe_forward_stack(ctx, x, T, stream=None):
    _check(ctx, _lib.moe_forward_stack(ctx, _ptr(x), T, _stream(stream)))


def moe_prefill(ctx, layer, x, N, stream=None):
    _check(ctx, _lib.moe_prefill(ctx, layer, _ptr(x), N, _stream(stream)))


def moe_prefill_delta(ctx, layer, x, N, delta, stream=None):
    _check(ctx, _lib.moe_prefill_delta(ctx, layer, _ptr(x), N, _ptr(delta), _stream(stream)))


def moe_prefill_route(ctx, layer, h, N, idx, w, bucket_off=None, bucket_perm=None, stream=None):
    _check(ctx, _lib.moe_prefill_route(ctx, layer, _ptr(h), N, _ptr(idx), _ptr(w),
                                       _ptr(bucket_off), _ptr(bucket_perm), _stream(stream)))


def moe_rmsnorm(ctx, layer, x, T, h, stream=None):
    _check(ctx, _lib.moe_rmsnorm(ctx, layer, _ptr(x), T, _ptr(h), _stream(stream)))


def moe_experts_given(ctx, layer, h, N, kk, idx, w, with_shared, delta, stream=None):
    _check(ctx, _lib.moe_experts_given(ctx, layer, _ptr(h), N, kk, _ptr(idx), _ptr(w),
                                       int(bool(with_shared)), _ptr(delta), _stream(stream)))


def moe_experts_rows(ctx, layer, h, M, e, y16, stream=None):
    _check(ctx, _lib.moe_experts_rows(ctx, layer, _ptr(h), M, _ptr(e), _ptr(y16), _stream(stream)))


def moe_ep_dispatch(ctx, idx, N, n_ranks, h, send_h, send_e, row_of, stream=None):
    """Returns the rows sent to each rank (a list of n_ranks ints)."""
    counts = (ctypes.c_int32 * n_ranks)()
    _check(ctx, _lib.moe_ep_dispatch(ctx, _ptr(idx), N, n_ranks, _ptr(h), _ptr(send_h),
                                     _ptr(send_e), _ptr(row_of), counts, _stream(stream)))
    return list(counts)


def moe_ep_combine(ctx, N, w, y, row_of, y_shared=None, x=None, delta=None, stream=None):
    _check(ctx, _lib.moe_ep_combine(ctx, N, _ptr(w), _ptr(y), _ptr(row_of), _ptr(y_shared),
                                    _ptr(x), _ptr(delta), _stream(stream)))


def moe_sync(ctx, timeout_ms=-1):
    _check(ctx, _lib.moe_sync(ctx, int(timeout_ms)))


def moe_get_stats(ctx):
    st = MoeStats()
    _check(ctx, _lib.moe_get_stats(ctx, ctypes.byref(st)))
    counts = np.ctypeslib.as_array(st.expert_count, shape=(st.E,)).copy() if st.E else None
    return dict(calls=st.calls, tokens=st.tokens, hits=st.hits, misses=st.misses,
                near_ties=st.near_ties, last_T=st.last_T, last_active=st.last_active,
                last_layer=st.last_layer, expert_count=counts)


def moe_last_error(ctx):
    return _lib.moe_last_error(ctx).decode()


def moe_status_string(status):
    return _lib.moe_status_string(status).decode()


def moe_expert_bytes(d, f, quant_fmt):
    return int(_lib.moe_expert_bytes(d, f, quant_fmt))


def moe_debug_poke_slot(ctx, layer, expert, slot):
    _check(ctx, _lib.moe_debug_poke_slot(ctx, layer, expert, slot))


def moe_debug_stall_next_decode(ctx, polls):
    _check(ctx, _lib.moe_debug_stall_next_decode(ctx, int(polls)))


def moe_debug_last_h(ctx, out, T, stream=None):
    _check(ctx, _lib.moe_debug_last_h(ctx, _ptr(out), T, _stream(stream)))


def moe_set_profiling(ctx, enable):
    _check(ctx, _lib.moe_set_profiling(ctx, int(enable)))


def moe_read_profile(ctx):
    """-> (route_ms, experts_ms, combine_ms, n_calls), summed over the calls."""
    ms = (ctypes.c_double * 3)(0.0, 0.0, 0.0)
    n = ctypes.c_int64(0)
    _check(ctx, _lib.moe_read_profile(ctx, ms, ctypes.byref(n)))
    return ms[0], ms[1], ms[2], n.value


TRACE_POINTS = ("route_start", "route_waited", "route_logits", "route_last_start", "route_topk",
                "route_bucket", "route_end", "gate_start", "gate_waited", "gate_first_item",
                "gate_end", "down_start", "down_waited", "down_end", "comb_start", "comb_end",
                "route_loaded", "route_selected")


def moe_set_trace(ctx, enable):
    _check(ctx, _lib.moe_set_trace(ctx, int(enable)))


def moe_read_trace(ctx):
    """-> {point: (earliest_ns, latest_ns)}; points no CTA reached are omitted."""
    n = 2 * len(TRACE_POINTS)
    buf = (ctypes.c_int64 * n)()
    _check(ctx, _lib.moe_read_trace(ctx, buf, n))
    k = len(TRACE_POINTS)
    return {name: (buf[i], buf[k + i]) for i, name in enumerate(TRACE_POINTS) if buf[i] != -1}


def moe_route_static(h, T, d, E, k, W, bias, idx, w, bucket_off, bucket_perm, stream=None):
    """Routing that allocates nothing (see include/moe.h)."""
    _check(None, _lib.moe_route_static(_ptr(h), T, d, E, k, _ptr(W), _ptr(bias), _ptr(idx),
                                       _ptr(w), _ptr(bucket_off), _ptr(bucket_perm),
                                       _stream(stream)))


def moe_route_static_status(stream=None):
    """Device status word of the last moe_route_static call on this device.
    Returns the word (0 = fine); raises MoeError when it is non-zero."""
    st = ctypes.c_int(0)
    rc = _lib.moe_route_static_status(ctypes.byref(st), _stream(stream))
    if rc not in (MOE_OK, 6):
        _check(None, rc)
    if rc == 6:
        raise MoeError(rc, f"moe_route_static device status 0x{st.value:x}")
    return st.value


# ------------------------------------------------------------- host tier
TIER_LRU, TIER_ADAPTIVE = 0, 1


def moe_set_host_tier(ctx, enable=1, policy=TIER_ADAPTIVE, half_life=64.0):
    """Backing copies in pinned host memory, the slot pool as an HBM cache
    (before moe_configure; see include/moe.h)."""
    _check(ctx, _lib.moe_set_host_tier(ctx, int(enable), int(policy), float(half_life)))


def moe_tier_prepare(ctx, layer, idx, T, stream=None):
    _check(ctx, _lib.moe_tier_prepare(ctx, layer, _ptr(idx), T, _stream(stream)))


def moe_tier_prefetch(ctx, layer, idx, T, stream=None):
    _check(ctx, _lib.moe_tier_prefetch(ctx, layer, _ptr(idx), T, _stream(stream)))


def moe_forward_tiered(ctx, layer, x, T, stream=None):
    _check(ctx, _lib.moe_forward_tiered(ctx, layer, _ptr(x), T, _stream(stream)))


def moe_tier_stats(ctx):
    """{"hits", "misses", "evictions", "bytes", "requests", "slots_used"}"""
    out = (ctypes.c_int64 * 6)()
    _check(ctx, _lib.moe_tier_stats(ctx, out))
    return dict(zip(("hits", "misses", "evictions", "bytes", "requests", "slots_used"), out))


def moe_tier_dump_trace(ctx, path):
    _check(ctx, _lib.moe_tier_dump_trace(ctx, os.fsencode(path)))


class TierSim:
    """Host-only model of the tier's replacement policy (moe_tier_sim_*)."""

    def __init__(self, n_slots, policy, half_life, n_keys):
        self.h = _lib.moe_tier_sim_create(n_slots, policy, float(half_life), n_keys)
        if not self.h:
            raise ValueError("moe_tier_sim_create: bad arguments")

    def request(self, keys, protect_prev=False):
        """(misses, slots) for one request of distinct keys; raises on -1 / -2."""
        n = len(keys)
        karr = (ctypes.c_int64 * max(n, 1))(*keys)
        sarr = (ctypes.c_int * max(n, 1))()
        r = _lib.moe_tier_sim_request(self.h, karr, n, int(protect_prev), sarr)
        if r == -1:
            raise ValueError("moe_tier_sim_request: bad arguments")
        if r == -2:
            raise MoeError(1, "the request needs more slots than may be taken")
        return r, list(sarr[:n])

    def counts(self):
        out = (ctypes.c_int64 * 3)()
        _lib.moe_tier_sim_counts(self.h, out)
        return dict(zip(("hits", "misses", "evictions"), out))

    def close(self):
        if self.h:
            _lib.moe_tier_sim_destroy(self.h)
            self.h = None

    def __del__(self):
        self.close()
