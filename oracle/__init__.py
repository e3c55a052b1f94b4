"""Scalar fp64 CPU oracle for the sparse MoE expert layer.

TEST INFRASTRUCTURE ONLY.  The product package never imports this module;
only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` use it.  It wraps ``moe_oracle.c`` (plain C, IEEE double) through
ctypes and shares no code with the CUDA path.

What it computes, and the passages it follows, is stated at the top of
``moe_oracle.c``.  Each Python function below marshals numpy arrays only.

Parity pins: every function here is pinned by ``tests/test_oracle_pins.py``
(closed forms, invariants, brute force and printed page numbers); none is
"parity unpinned".
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "moe_oracle.c")
_SO = os.path.join(_HERE, "liboracle.so")
# a test may point the wrapper at a separately built copy (planted mistakes)
_SO_OVERRIDE = os.environ.get("MOE_ORACLE_SO")
_lock = threading.Lock()
_lib = None

Q4 = 1
Q2 = 2
GROUP = {Q4: 32, Q2: 64}


def build(force: bool = False) -> str:
    """Compile moe_oracle.c with gcc (no fast-math, no FMA contraction)."""
    if force or not os.path.exists(_SO) or os.path.getmtime(_SO) < max(
        os.path.getmtime(_SRC), os.path.getmtime(os.path.join(_HERE, "moe_oracle.h"))
    ):
        tmp = _SO + f".tmp{os.getpid()}"
        subprocess.check_call(
            ["gcc", "-O2", "-std=c11", "-Wall", "-fPIC", "-shared",
             "-ffp-contract=off", "-fno-fast-math", "-o", tmp, _SRC, "-lm"]
        )
        os.replace(tmp, _SO)
    return _SO


def lib():
    global _lib
    with _lock:
        if _lib is None:
            if _SO_OVERRIDE:
                L = ctypes.CDLL(_SO_OVERRIDE)
            else:
                build()
                L = ctypes.CDLL(_SO)
            P = ctypes.c_void_p
            I = ctypes.c_int
            D = ctypes.c_double
            L.orc_f16_to_f64.argtypes = [ctypes.c_uint16]
            L.orc_f16_to_f64.restype = D
            L.orc_f64_to_f16.argtypes = [D]
            L.orc_f64_to_f16.restype = ctypes.c_uint16
            L.orc_bf16_to_f64.argtypes = [ctypes.c_uint16]
            L.orc_bf16_to_f64.restype = D
            L.orc_f64_to_bf16.argtypes = [D]
            L.orc_f64_to_bf16.restype = ctypes.c_uint16
            L.orc_dequant.argtypes = [I, P, P, P, I, I, P]
            L.orc_quantize.argtypes = [I, P, I, I, P, P, P]
            L.orc_rmsnorm.argtypes = [P, P, D, I, I, P]
            L.orc_rmsnorm.restype = None
            L.orc_router.argtypes = [P, P, P, I, I, I, P]
            L.orc_router.restype = None
            L.orc_topk.argtypes = [P, I, I, I, P, P, P]
            L.orc_bucket.argtypes = [P, I, I, I, P, P, P]
            L.orc_silu.argtypes = [D]
            L.orc_silu.restype = D
            L.orc_expert.argtypes = [P, P, P, I, I, P, I, P]
            L.orc_expert.restype = None
            L.orc_dequant_expert.argtypes = [I, I, I, P, P, P, P, P, P]
            L.orc_moe_layer.argtypes = [P, P]
            _lib = L
    return _lib


def _p(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


# --------------------------------------------------------------- encodings
def f16_to_f64(bits):
    return lib().orc_f16_to_f64(int(bits))


def f64_to_f16(v):
    return lib().orc_f64_to_f16(float(v))


def bf16_to_f64(bits):
    return lib().orc_bf16_to_f64(int(bits))


def f64_to_bf16(v):
    return lib().orc_f64_to_bf16(float(v))


def silu(z):
    return lib().orc_silu(float(z))


# ---------------------------------------------------------------- formats
def code_bytes(fmt, R, K):
    return R * K // 2 if fmt == Q4 else R * K // 4


def dequant(fmt, codes, scales, mins, R, K):
    """Packed [R,K] matrix -> float64 [R,K]."""
    codes = _c(codes, np.uint8)
    scales = _c(scales, np.uint16)
    mins = None if mins is None else _c(mins, np.uint16)
    W = np.empty((R, K), np.float64)
    rc = lib().orc_dequant(fmt, _p(codes), _p(scales), _p(mins), R, K, _p(W))
    if rc:
        raise ValueError(f"orc_dequant rc={rc}")
    return W


def quantize(fmt, W):
    """float64 [R,K] -> (codes uint8, scales uint16 bits, mins uint16 bits|None)."""
    W = _c(W, np.float64)
    R, K = W.shape
    G = GROUP[fmt]
    codes = np.empty(code_bytes(fmt, R, K), np.uint8)
    scales = np.empty(R * (K // G), np.uint16)
    mins = np.empty(R * (K // G), np.uint16) if fmt == Q2 else None
    rc = lib().orc_quantize(fmt, _p(W), R, K, _p(codes), _p(scales), _p(mins))
    if rc:
        raise ValueError(f"orc_quantize rc={rc}")
    return codes, scales, mins


def dequant_expert(fmt, d, f, codes, scales, mins):
    codes = _c(codes, np.uint8)
    scales = _c(scales, np.uint16)
    mins = None if mins is None else _c(mins, np.uint16)
    Wg = np.empty((f, d)); Wu = np.empty((f, d)); Wd = np.empty((d, f))
    rc = lib().orc_dequant_expert(fmt, d, f, _p(codes), _p(scales), _p(mins),
                                  _p(Wg), _p(Wu), _p(Wd))
    if rc:
        raise ValueError(f"orc_dequant_expert rc={rc}")
    return Wg, Wu, Wd


# ------------------------------------------------------------- layer steps
def rmsnorm(x_bf16_bits, gamma, eps):
    x = _c(x_bf16_bits, np.uint16)
    T, d = x.shape
    g = None if gamma is None else _c(gamma, np.float32)
    h = np.empty((T, d), np.uint16)
    lib().orc_rmsnorm(_p(x), _p(g), float(eps), T, d, _p(h))
    return h


def router(h_bf16_bits, W, bias=None):
    h = _c(h_bf16_bits, np.uint16)
    W = _c(W, np.float32)
    T, d = h.shape
    E = W.shape[0]
    b = None if bias is None else _c(bias, np.float32)
    out = np.empty((T, E), np.float64)
    lib().orc_router(_p(h), _p(W), _p(b), T, d, E, _p(out))
    return out


def topk(logits, k):
    lg = _c(logits, np.float64)
    T, E = lg.shape
    idx = np.empty((T, k), np.int32)
    w = np.empty((T, k), np.float64)
    margin = np.empty(T, np.float64)
    rc = lib().orc_topk(_p(lg), T, E, k, _p(idx), _p(w), _p(margin))
    if rc:
        raise ValueError(f"orc_topk rc={rc}")
    return idx, w, margin


def bucket(idx, E):
    idx = _c(idx, np.int32)
    T, k = idx.shape
    cnt = np.empty(E, np.int32)
    off = np.empty(E + 1, np.int32)
    perm = np.empty(T * k, np.int32)
    rc = lib().orc_bucket(_p(idx), T, k, E, _p(cnt), _p(off), _p(perm))
    if rc:
        raise ValueError(f"orc_bucket rc={rc}")
    return cnt, off, perm


def expert(Wg, Wu, Wd, h_bf16_bits):
    h = _c(h_bf16_bits, np.uint16)
    n, d = h.shape
    f = Wg.shape[0]
    Wg = _c(Wg, np.float64); Wu = _c(Wu, np.float64); Wd = _c(Wd, np.float64)
    y = np.empty((n, d), np.float64)
    lib().orc_expert(_p(Wg), _p(Wu), _p(Wd), d, f, _p(h), n, _p(y))
    return y


class _LayerIn(ctypes.Structure):
    _fields_ = [
        ("T", ctypes.c_int), ("d", ctypes.c_int), ("f", ctypes.c_int),
        ("E", ctypes.c_int), ("k", ctypes.c_int), ("fmt", ctypes.c_int),
        ("x", ctypes.c_void_p), ("use_norm", ctypes.c_int),
        ("gamma", ctypes.c_void_p), ("eps", ctypes.c_double),
        ("router_w", ctypes.c_void_p), ("router_bias", ctypes.c_void_p),
        ("codes_of", ctypes.c_void_p), ("scales_of", ctypes.c_void_p),
        ("mins_of", ctypes.c_void_p),
        ("shared_codes", ctypes.c_void_p), ("shared_scales", ctypes.c_void_p),
        ("shared_mins", ctypes.c_void_p),
    ]


class _LayerOut(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in
                ("h", "logits", "idx", "w", "margin", "cnt", "off", "perm",
                 "delta", "x_out")]


def moe_layer(x_bf16_bits, *, fmt, d, f, E, k, router_w, router_bias=None,
              experts, shared=None, norm=False, gamma=None, eps=1e-6):
    """One MoE layer over the rows of ``x`` (bf16 bits, [T, d]).

    ``experts`` maps expert id -> (codes, scales, mins|None) packed arrays;
    only ids that some token selects need to be present.  ``shared`` is the
    shared expert's (codes, scales, mins) or None.  Returns a dict with h,
    logits, idx, w, margin, cnt, off, perm, delta (fp64) and x_out (bf16 bits).
    """
    x = _c(x_bf16_bits, np.uint16)
    T = x.shape[0]
    assert x.shape[1] == d
    keep = []

    def arr(a, dt):
        if a is None:
            return None
        a = _c(a, dt)
        keep.append(a)
        return a

    codes_of = (ctypes.c_void_p * E)()
    scales_of = (ctypes.c_void_p * E)()
    mins_of = (ctypes.c_void_p * E)()
    for e, (c, s, m) in experts.items():
        codes_of[e] = _p(arr(c, np.uint8))
        scales_of[e] = _p(arr(s, np.uint16))
        mins_of[e] = _p(arr(m, np.uint16)) if m is not None else None
    W = arr(router_w, np.float32)
    b = arr(router_bias, np.float32)
    g = arr(gamma, np.float32)
    sc = ss = sm = None
    if shared is not None:
        sc = arr(shared[0], np.uint8)
        ss = arr(shared[1], np.uint16)
        sm = arr(shared[2], np.uint16) if shared[2] is not None else None
    li = _LayerIn(T, d, f, E, k, fmt, _p(x), int(bool(norm)), _p(g), float(eps),
                  _p(W), _p(b), ctypes.cast(codes_of, ctypes.c_void_p),
                  ctypes.cast(scales_of, ctypes.c_void_p),
                  ctypes.cast(mins_of, ctypes.c_void_p), _p(sc), _p(ss), _p(sm))
    out = dict(
        h=np.empty((T, d), np.uint16), logits=np.empty((T, E), np.float64),
        idx=np.empty((T, k), np.int32), w=np.empty((T, k), np.float64),
        margin=np.empty(T, np.float64), cnt=np.empty(E, np.int32),
        off=np.empty(E + 1, np.int32), perm=np.empty(T * k, np.int32),
        delta=np.empty((T, d), np.float64), x_out=np.empty((T, d), np.uint16),
    )
    lo = _LayerOut(*[_p(out[n]) for n in
                     ("h", "logits", "idx", "w", "margin", "cnt", "off", "perm",
                      "delta", "x_out")])
    rc = lib().orc_moe_layer(ctypes.byref(li), ctypes.byref(lo))
    if rc:
        raise ValueError(f"orc_moe_layer rc={rc}")
    return out
