"""Seeded synthetic inputs for the MoE expert layer.

This module holds no step of the MoE method: it only draws random numbers.
Both the CPU oracle (through the tests) and the CUDA library consume exactly
the bytes it produces.  Every value is a pure function of
``(seed, stream, counter)`` through a counter-based 32-bit hash, so any slice
(one expert of one layer, one token window) can be regenerated on its own,
and the numpy (CPU) and torch (GPU) implementations give identical bits.

Hash: two rounds of a 32-bit xor-shift-multiply finaliser (the "lowbias32"
constants 0x7feb352d / 0x846ca68b), keyed per stream.

Distributions (the pages print no weight values; these mirror a Gaussian
N(0, 0.02) weight matrix after quantisation in each format):

* Q4 (4-bit symmetric, group 32): integer level q = nibble - 8 in [-7, 7],
  drawn from a normal of std 2.8 levels rounded to the nearest level; the
  fp16 scale is uniform over the fp16 values in [0.0055, 0.0090], so the
  weights s*q have a standard deviation of about 0.02.
* Q2 (2-bit asymmetric, group 64): code q in {0,1,2,3} with probabilities
  (0.06, 0.44, 0.44, 0.06); fp16 scale uniform in [0.028, 0.036] and fp16
  min uniform in [-0.052, -0.040] (weights s*q + m, std about 0.02).
* router weights: fp32 N(0, 0.02) (Box-Muller in float64, then fp32);
* hidden states: bf16 N(0, 1) (float64 -> fp32 -> bf16, round to nearest even);
* Zipf router bias: b[e] = ln p_rank(e), p_r proportional to r^-s, with a
  seeded per-layer permutation mapping rank to expert.

Two more expert sources serve the parity tests: ``expert_weights_np`` draws
an expert's unquantised matrices from N(0, 0.02) (float64), for a quantiser
to encode; ``expert_uniform_codes_np`` draws every code value with equal
probability (all 16 Q4 nibbles, level -8 included; all four Q2 codes).
"""
from __future__ import annotations

import math

import numpy as np

M32 = 0xFFFFFFFF
_C1 = 0x7FEB352D
_C2 = 0x846CA68B
_GOLD = 0x9E3779B9

# stream kinds
K_CODES, K_SCALES, K_MINS, K_ROUTER, K_ZIPF, K_HIDDEN, K_IDX, K_GAMMA = range(1, 9)
K_WEIGHTS, K_UCODES = 9, 10
SHARED_INDEX = 4095  # expert index used for the shared expert's streams

Q4, Q2 = 1, 2
GROUP = {Q4: 32, Q2: 64}


# ------------------------------------------------------------------ hashing
def _mix_int(x: int) -> int:
    x &= M32
    x ^= x >> 16
    x = (x * _C1) & M32
    x ^= x >> 15
    x = (x * _C2) & M32
    x ^= x >> 16
    return x


def stream_id(kind: int, layer: int = 0, index: int = 0) -> int:
    """32-bit stream id of (kind, layer, index), each a non-negative int < 2^32."""
    assert 0 <= kind < 256 and 0 <= layer <= M32 and 0 <= index <= M32
    return _mix_int(_mix_int(_mix_int(kind) ^ layer) + 0x632BE5AB ^ index)


def stream_keys(seed: int, stream: int):
    k1 = _mix_int(_mix_int(seed ^ 0xA5A5A5A5) + ((stream * _GOLD) & M32))
    k2 = _mix_int(k1 ^ 0x68E31DA4)
    return k1, k2


def _mix_np(x):
    x = x.astype(np.uint32, copy=True)
    x ^= x >> np.uint32(16)
    x *= np.uint32(_C1)
    x ^= x >> np.uint32(15)
    x *= np.uint32(_C2)
    x ^= x >> np.uint32(16)
    return x


def u32_np(seed: int, stream: int, counters) -> np.ndarray:
    """uint32 draws for the given counters (numpy, CPU)."""
    k1, k2 = stream_keys(seed, stream)
    c = np.asarray(counters, dtype=np.uint64)
    x = ((c + np.uint64(k1)) & np.uint64(M32)).astype(np.uint32)
    return _mix_np(_mix_np(x) ^ np.uint32(k2))


def _mul32_t(x, c):
    # (x * c) mod 2^32 without int64 overflow: split c into 16-bit halves
    lo = x * (c & 0xFFFF)
    hi = ((x * (c >> 16)) & 0xFFFF) << 16
    return (lo + hi) & M32


def _mix_t(x):
    x = x ^ (x >> 16)
    x = _mul32_t(x, _C1)
    x = x ^ (x >> 15)
    x = _mul32_t(x, _C2)
    x = x ^ (x >> 16)
    return x


def u32_torch(key1, key2, counters):
    """uint32 draws as int64 tensors; key1/key2 broadcast against counters."""
    x = (counters + key1) & M32
    return _mix_t(_mix_t(x) ^ key2)


# ------------------------------------------------------------ distributions
def _normal_cdf(x):
    return 0.5 * (1.0 + math.erf(x / math.sqrt(2.0)))


def _q4_thresholds():
    # levels -7..7, normal with std 2.8 levels, tails folded into +-7
    std = 2.8
    cuts = []
    for q in range(-7, 7):  # boundary between q and q+1
        cuts.append(int(round(65536.0 * _normal_cdf((q + 0.5) / std))))
    return np.array(cuts, np.int64)  # 14 thresholds -> 15 levels


Q4_THRESH = _q4_thresholds()
Q2_THRESH = np.array([3932, 32768, 61604], np.int64)  # P = .06 .44 .44 .06


def _f16_bits(v: float) -> int:
    return int(np.array([v], np.float16).view(np.uint16)[0])


Q4_SCALE_BITS = (_f16_bits(0.0055), _f16_bits(0.0090))
Q2_SCALE_BITS = (_f16_bits(0.028), _f16_bits(0.036))
Q2_MIN_MAG_BITS = (_f16_bits(0.040), _f16_bits(0.052))


def expert_sizes(fmt: int, d: int, f: int):
    """(code bytes, scale count) of one expert: Wg [f,d], Wu [f,d], Wd [d,f]."""
    G = GROUP[fmt]
    per = 2 if fmt == Q4 else 4
    return 3 * f * d // per, 3 * f * d // G


# ------------------------------------------------------- numpy generators
def expert_np(seed: int, fmt: int, d: int, f: int, layer: int, e: int):
    """One packed expert (codes uint8, scales uint16, mins uint16|None)."""
    nb, ns = expert_sizes(fmt, d, f)
    sc = stream_id(K_CODES, layer, e)
    if fmt == Q4:
        u = u32_np(seed, sc, np.arange(nb, dtype=np.uint64)).astype(np.int64)
        lo = 1 + np.searchsorted(Q4_THRESH, u & 0xFFFF, side="right")
        hi = 1 + np.searchsorted(Q4_THRESH, u >> 16, side="right")
        codes = (lo | (hi << 4)).astype(np.uint8)
    else:
        u = u32_np(seed, sc, np.arange(2 * nb, dtype=np.uint64)).astype(np.int64)
        u = u.reshape(nb, 2)
        q = [np.searchsorted(Q2_THRESH, (u[:, i // 2] >> (16 * (i % 2))) & 0xFFFF,
                             side="right") for i in range(4)]
        codes = (q[0] | (q[1] << 2) | (q[2] << 4) | (q[3] << 6)).astype(np.uint8)
    lo_b, hi_b = Q4_SCALE_BITS if fmt == Q4 else Q2_SCALE_BITS
    us = u32_np(seed, stream_id(K_SCALES, layer, e), np.arange(ns, dtype=np.uint64))
    scales = (lo_b + us.astype(np.int64) % (hi_b - lo_b + 1)).astype(np.uint16)
    mins = None
    if fmt == Q2:
        um = u32_np(seed, stream_id(K_MINS, layer, e), np.arange(ns, dtype=np.uint64))
        lo_m, hi_m = Q2_MIN_MAG_BITS
        mins = (0x8000 | (lo_m + um.astype(np.int64) % (hi_m - lo_m + 1))).astype(np.uint16)
    return codes, scales, mins


def shared_np(seed: int, fmt: int, d: int, f: int, layer: int):
    return expert_np(seed, fmt, d, f, layer, SHARED_INDEX)


def expert_uniform_codes_np(seed: int, fmt: int, d: int, f: int, layer: int, e: int):
    """One packed expert whose code bytes are uniform (every nibble / 2-bit
    code equally likely); scales (and mins) as in ``expert_np``."""
    nb, _ = expert_sizes(fmt, d, f)
    u = u32_np(seed, stream_id(K_UCODES, layer, e), np.arange(nb, dtype=np.uint64))
    _, scales, mins = expert_np(seed, fmt, d, f, layer, e)
    return (u & 0xFF).astype(np.uint8), scales, mins


def _normal_np(seed, stream, n):
    u = u32_np(seed, stream, np.arange(2 * n, dtype=np.uint64)).astype(np.float64)
    u1 = (u[0::2] + 0.5) / 4294967296.0
    u2 = (u[1::2] + 0.5) / 4294967296.0
    return np.sqrt(-2.0 * np.log(u1)) * np.cos(2.0 * np.pi * u2)


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """float32 -> bf16 bits, round to nearest even (input generation only)."""
    b = np.ascontiguousarray(a, np.float32).view(np.uint32).astype(np.uint64)
    b = (b + 0x7FFF + ((b >> 16) & 1)) >> 16
    return b.astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, np.uint16).astype(np.uint32) << 16).view(np.float32)


def hidden_np(seed: int, T: int, d: int, window: int = 0, layer: int = 0):
    """bf16 bits [T, d], N(0,1)."""
    z = _normal_np(seed, stream_id(K_HIDDEN, layer, window), T * d)
    return f32_to_bf16_bits(z.astype(np.float32)).reshape(T, d)


def expert_weights_np(seed: int, d: int, f: int, layer: int, e: int, std: float = 0.02):
    """Unquantised matrices of one expert, N(0, std) in float64:
    (Wg [f, d], Wu [f, d], Wd [d, f])."""
    z = _normal_np(seed, stream_id(K_WEIGHTS, layer, e), 3 * f * d) * std
    return (z[:f * d].reshape(f, d), z[f * d:2 * f * d].reshape(f, d),
            z[2 * f * d:].reshape(d, f))


def router_np(seed: int, E: int, d: int, layer: int = 0, std: float = 0.02):
    z = _normal_np(seed, stream_id(K_ROUTER, layer, 0), E * d)
    return (z * std).astype(np.float32).reshape(E, d)


def zipf_bias_np(seed: int, E: int, layer: int = 0, s: float = 1.1):
    """b[e] = ln p_rank(e); returns (bias fp32 [E], rank_of_expert int [E], p [E])."""
    r = np.arange(1, E + 1, dtype=np.float64)
    p = r ** (-s)
    p /= p.sum()
    u = u32_np(seed, stream_id(K_ZIPF, layer, 0), np.arange(E, dtype=np.uint64))
    order = np.argsort(u, kind="stable")  # order[rank-1] = expert
    rank_of = np.empty(E, np.int64)
    rank_of[order] = np.arange(1, E + 1)
    bias = np.log(p[rank_of - 1]).astype(np.float32)
    return bias, rank_of, p


def routing_idx_np(seed: int, T: int, k: int, E: int, window: int = 0):
    """Random distinct expert ids per token [T, k] (for stand-alone bucketing)."""
    u = u32_np(seed, stream_id(K_IDX, 0, window), np.arange(T * E, dtype=np.uint64))
    u = u.reshape(T, E)
    return np.argsort(u, axis=1, kind="stable")[:, :k].astype(np.int32)


def slot_table_np(E: int, L: int, n_slots: int, ranks):
    """Residency table [L*E]: the n_slots (layer, expert) pairs of highest
    Zipf probability (ties to lower (layer, expert)) get slots 0..n_slots-1
    in that order; every other pair gets -1.  ranks: [L, E] Zipf ranks."""
    ranks = np.asarray(ranks).reshape(L, E)
    keys = ranks.reshape(-1) * (L * E) + np.arange(L * E)  # rank, then (l,e)
    order = np.argsort(keys, kind="stable")[:n_slots]
    table = np.full(L * E, -1, np.int32)
    table[order] = np.arange(len(order), dtype=np.int32)
    return table


# ------------------------------------------------------- torch generators
def experts_torch(seed: int, fmt: int, d: int, f: int, layer: int, first: int,
                  count: int, device, chunk: int = 16):
    """Packed experts [first, first+count) of one layer on ``device``:
    (codes uint8 [count, nb], scales int16 [count, ns], mins int16|None).
    Bit-identical to ``expert_np`` for each expert."""
    import torch

    nb, ns = expert_sizes(fmt, d, f)
    codes = torch.empty((count, nb), dtype=torch.uint8, device=device)
    scales = torch.empty((count, ns), dtype=torch.int16, device=device)
    mins = torch.empty((count, ns), dtype=torch.int16, device=device) if fmt == Q2 else None
    q4t = torch.tensor(Q4_THRESH, dtype=torch.int64, device=device)
    q2t = torch.tensor(Q2_THRESH, dtype=torch.int64, device=device)

    def keys(kind, es):
        k1 = [stream_keys(seed, stream_id(kind, layer, e))[0] for e in es]
        k2 = [stream_keys(seed, stream_id(kind, layer, e))[1] for e in es]
        return (torch.tensor(k1, dtype=torch.int64, device=device)[:, None],
                torch.tensor(k2, dtype=torch.int64, device=device)[:, None])

    for c0 in range(0, count, chunk):
        es = list(range(first + c0, first + min(count, c0 + chunk)))
        n = len(es)
        k1, k2 = keys(K_CODES, es)
        if fmt == Q4:
            cnt = torch.arange(nb, dtype=torch.int64, device=device)[None, :]
            u = u32_torch(k1, k2, cnt)
            lo = 1 + torch.bucketize(u & 0xFFFF, q4t, right=True)
            hi = 1 + torch.bucketize(u >> 16, q4t, right=True)
            codes[c0:c0 + n] = (lo | (hi << 4)).to(torch.uint8)
            del u, lo, hi
        else:
            out = torch.zeros((n, nb), dtype=torch.int64, device=device)
            for half in range(2):
                cnt = 2 * torch.arange(nb, dtype=torch.int64, device=device)[None, :] + half
                u = u32_torch(k1, k2, cnt)
                for j in range(2):
                    q = torch.bucketize((u >> (16 * j)) & 0xFFFF, q2t, right=True)
                    out |= q << (2 * (2 * half + j))
                del u
            codes[c0:c0 + n] = out.to(torch.uint8)
            del out
        cnt = torch.arange(ns, dtype=torch.int64, device=device)[None, :]
        k1, k2 = keys(K_SCALES, es)
        lo_b, hi_b = Q4_SCALE_BITS if fmt == Q4 else Q2_SCALE_BITS
        us = u32_torch(k1, k2, cnt)
        scales[c0:c0 + n] = (lo_b + us % (hi_b - lo_b + 1)).to(torch.int16)
        if fmt == Q2:
            k1, k2 = keys(K_MINS, es)
            um = u32_torch(k1, k2, cnt)
            lo_m, hi_m = Q2_MIN_MAG_BITS
            v = 0x8000 | (lo_m + um % (hi_m - lo_m + 1))
            mins[c0:c0 + n] = (v - 65536).to(torch.int16)  # same 16 bits
    return codes, scales, mins
