"""Seeded, counter-based synthetic inputs shared by the CUDA path's tests/bench and
by the oracle's callers.

This module holds NO attention arithmetic: it only turns (seed, tensor id, flat
element index) into a BF16 value, and picks sampled query rows.  Because the
generator is counter based, any subset of a tensor (one head, a few query rows)
can be produced without generating the rest, which is how the oracle is fed at
sizes where the full tensors would not fit its time budget.

Definition (fixed here, used by every consumer):

  gamma      = 0x9E3779B97F4A7C15                (SplitMix64 increment)
  mix(z)     = SplitMix64 finaliser: z ^= z>>30; z *= 0xBF58476D1CE4E5B9;
                                     z ^= z>>27; z *= 0x94D049BB133111EB; z ^= z>>31
  key        = mix(mix(seed + gamma) + tensor_id)  tensor_id: Q=0, K=1, V=2
  bits(i)    = mix(key + (i + 1) * gamma)          (all arithmetic mod 2^64)
  normal     : u1 = (hi32 + 0.5) / 2^32, u2 = lo32 / 2^32,
               z = sqrt(-2 ln u1) * cos(2 pi u2)   (Box-Muller, cosine branch, fp64)
  uniform    : u = (bits >> 40) / 2^24,  z = 2u - 1  in [-1, 1)
  value      = bf16_rne(fp32_rne(mult * z))
  unit draw  : (bits >> 11) / 2^53 in [0, 1), fp64 (sequence lengths, id 3;
               column-interval masks, id 4)

(SplitMix64: Steele, Lea & Flood, "Fast splittable pseudorandom number
generators", OOPSLA 2014.)
"""
from __future__ import annotations

import concurrent.futures
import os

import numpy as np

GAMMA = np.uint64(0x9E3779B97F4A7C15)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)

# "len": sequence / document lengths; "mask": column-interval stress masks
TENSOR_ID = {"q": 0, "k": 1, "v": 2, "len": 3, "mask": 4}

_CHUNK = 1 << 22


def _mix(z: np.ndarray) -> np.ndarray:
    z = z ^ (z >> np.uint64(30))
    z = z * _M1
    z = z ^ (z >> np.uint64(27))
    z = z * _M2
    return z ^ (z >> np.uint64(31))


def _key(seed: int, tensor_id: int) -> np.uint64:
    with np.errstate(over="ignore"):
        s = np.array([seed], dtype=np.uint64) + GAMMA
        k = _mix(s) + np.uint64(tensor_id)
        return _mix(k)[0]


def _bits(key: np.uint64, idx: np.ndarray) -> np.ndarray:
    with np.errstate(over="ignore"):
        ctr = key + (idx.astype(np.uint64) + np.uint64(1)) * GAMMA
        return _mix(ctr)


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round fp32 to BF16 (round to nearest, ties to even); returns uint16 bits."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    rounding = ((u >> np.uint32(16)) & np.uint32(1)) + np.uint32(0x7FFF)
    return ((u + rounding) >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def bf16_bits_to_f64(b: np.ndarray) -> np.ndarray:
    """Exact widening of BF16 bit patterns to fp64."""
    return bf16_bits_to_f32(b).astype(np.float64)


def _draw(key: np.uint64, idx: np.ndarray, dist: str) -> np.ndarray:
    """fp64 draws z (before the multiplier and rounding)."""
    bits = _bits(key, idx)
    if dist == "normal":
        hi = (bits >> np.uint64(32)).astype(np.float64)
        lo = (bits & np.uint64(0xFFFFFFFF)).astype(np.float64)
        u1 = (hi + 0.5) * (1.0 / 4294967296.0)
        u2 = lo * (1.0 / 4294967296.0)
        z = np.sqrt(-2.0 * np.log(u1)) * np.cos(2.0 * np.pi * u2)
    elif dist == "uniform":
        u = (bits >> np.uint64(40)).astype(np.float64) * (1.0 / 16777216.0)
        z = 2.0 * u - 1.0
    else:
        raise ValueError(f"unknown distribution {dist!r}")
    return z


def _values(key: np.uint64, idx: np.ndarray, dist: str, mult: float) -> np.ndarray:
    return f32_to_bf16_bits((mult * _draw(key, idx, dist)).astype(np.float32))


def gen_bf16_at(seed: int, tensor: str, flat_idx: np.ndarray, dist: str = "normal",
                mult: float = 1.0) -> np.ndarray:
    """BF16 bits of the elements with the given flat indices (any shape)."""
    key = _key(seed, TENSOR_ID[tensor])
    idx = np.asarray(flat_idx, dtype=np.int64)
    flat = idx.reshape(-1)
    out = np.empty(flat.shape, dtype=np.uint16)
    for s in range(0, flat.size, _CHUNK):
        out[s:s + _CHUNK] = _values(key, flat[s:s + _CHUNK], dist, mult)
    return out.reshape(idx.shape)


def uniform_at(seed: int, tensor: str, idx: np.ndarray) -> np.ndarray:
    """fp64 draws in [0, 1) at the given counter indices of stream ``tensor``."""
    bits = _bits(_key(seed, TENSOR_ID[tensor]), np.asarray(idx, dtype=np.int64))
    return (bits >> np.uint64(11)).astype(np.float64) * (1.0 / 9007199254740992.0)


def gen_bf16(seed: int, tensor: str, shape, dist: str = "normal", mult: float = 1.0,
             out: np.ndarray | None = None) -> np.ndarray:
    """BF16 bits of a whole contiguous tensor of ``shape`` (flat index = C order).

    Chunks are independent (counter based), so they are filled by a thread pool;
    numpy releases the GIL inside its element-wise kernels.
    """
    n = int(np.prod(shape))
    key = _key(seed, TENSOR_ID[tensor])
    if out is None:
        out = np.empty(n, dtype=np.uint16)
    flat = out.reshape(-1)
    assert flat.size == n

    def fill(s):
        e = min(n, s + _CHUNK)
        flat[s:e] = _values(key, np.arange(s, e, dtype=np.int64), dist, mult)

    starts = range(0, n, _CHUNK)
    if n > 2 * _CHUNK:
        with concurrent.futures.ThreadPoolExecutor(max_workers=min(16, os.cpu_count() or 1)) as ex:
            list(ex.map(fill, starts))
    else:
        for s in starts:
            fill(s)
    return out.reshape(shape)


# ---------------------------------------------------------------------------
# FP8 E4M3 (the OCP "E4M3FN" format): 1 sign bit, 4 exponent bits (bias 7),
# 3 mantissa bits; exponent field 0 holds the subnormals m/8 * 2^-6; code
# S.1111.111 is NaN and there is no infinity, so the largest finite value is
# 1.75 * 2^8 = 448.
# ---------------------------------------------------------------------------
def e4m3_decode_table() -> np.ndarray:
    """fp64 value of each of the 256 codes (NaN for the two NaN codes)."""
    vals = np.empty(256, dtype=np.float64)
    for code in range(256):
        sign = -1.0 if code & 0x80 else 1.0
        e, m = (code >> 3) & 0xF, code & 0x7
        if e == 0xF and m == 0x7:
            vals[code] = np.nan
        elif e == 0:
            vals[code] = sign * (m / 8.0) * 2.0 ** -6
        else:
            vals[code] = sign * (1.0 + m / 8.0) * 2.0 ** (e - 7)
    return vals


_E4M3 = e4m3_decode_table()
_E4M3_POS = _E4M3[:127]  # codes 0 .. 126: +0 .. 448, increasing


def e4m3_from_f32(x: np.ndarray) -> np.ndarray:
    """Round fp32 values to the nearest E4M3 code (ties to the even code),
    saturating at +-448.  Returns uint8 codes."""
    x = np.asarray(x, dtype=np.float32).astype(np.float64)
    a = np.minimum(np.abs(x), 448.0)
    hi = np.searchsorted(_E4M3_POS, a, side="left")      # first code with value >= a
    hi = np.minimum(hi, 126)
    lo = np.maximum(hi - 1, 0)
    d_lo = a - _E4M3_POS[lo]
    d_hi = _E4M3_POS[hi] - a
    pick_hi = (d_hi < d_lo) | ((d_hi == d_lo) & (hi % 2 == 0))
    code = np.where(pick_hi, hi, lo).astype(np.uint8)
    return np.where(np.signbit(x), code | np.uint8(0x80), code).astype(np.uint8)


def e4m3_to_f64(codes: np.ndarray) -> np.ndarray:
    return _E4M3[np.asarray(codes, dtype=np.uint8)]


def gen_e4m3(seed: int, tensor: str, shape, dist: str = "normal", mult: float = 1.0) -> np.ndarray:
    """E4M3 codes of a whole tensor: the BF16 generator's fp32 draw (mult * z)
    rounded to E4M3 instead of BF16."""
    n = int(np.prod(shape))
    key = _key(seed, TENSOR_ID[tensor])
    out = np.empty(n, dtype=np.uint8)
    for s in range(0, n, _CHUNK):
        e = min(n, s + _CHUNK)
        out[s:e] = e4m3_from_f32((mult * _draw(key, np.arange(s, e, dtype=np.int64), dist))
                                 .astype(np.float32))
    return out.reshape(shape)


def e4m3_at(seed: int, tensor: str, flat_idx: np.ndarray, dist: str = "normal",
            mult: float = 1.0) -> np.ndarray:
    """E4M3 codes of the elements with the given flat indices (any shape)."""
    key = _key(seed, TENSOR_ID[tensor])
    idx = np.asarray(flat_idx, dtype=np.int64)
    z = _draw(key, idx.reshape(-1), dist)
    return e4m3_from_f32((mult * z).astype(np.float32)).reshape(idx.shape)


def sample_rows(seed: int, bh: int, n: int, count: int) -> np.ndarray:
    """``count`` distinct query rows of head ``bh`` (sorted), always with 0 and n-1.

    Drawn with the same counter generator (tensor id 16 + bh), so they are fixed
    by (seed, bh, n, count) alone.
    """
    if count >= n:
        return np.arange(n, dtype=np.int64)
    key = _key(seed, 16 + bh)
    chosen = {0, n - 1}
    ctr = 0
    while len(chosen) < count:
        bits = _bits(key, np.arange(ctr, ctr + 4 * count, dtype=np.int64))
        ctr += 4 * count
        for b in (bits % np.uint64(n)).tolist():
            chosen.add(int(b))
            if len(chosen) == count:
                break
    return np.array(sorted(chosen), dtype=np.int64)
