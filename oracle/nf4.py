"""Oracle: 4-bit NormalFloat storage with double-quantised block constants.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__``).

Follows [P1] section "What QLoRA freezes, and in how many bits" (the
"4-bit NormalFloat" and "Double quantisation" paragraphs and the forward
equation with doubleDequant(c1 FP32, c2 k-bit, W NF4)), [P2] section
"QLoRA: shrink the frozen part too", and [P1] "What to choose and why"
(NF4, block size 64, double-quant block size 256).

Readings taken where the pages are silent:
  R1  outermost quantile probability p_max = 1 - (1/2)(1/(2*16) + 1/(2*15)).
  R2  blocks are consecutive runs of 64 elements of row-major W0.
  R3  an all-zero block encodes every element as the zero level.
  R4  nearest level with ties going to the lower code.
  R5  byte m holds element 2m in its low nibble, element 2m+1 in its high one.
  R6  one mean per tensor, summed in float64 by a pairwise tree over the
      block constants padded with zeros to a power of two; mu = fp32(S / n_b).
  R7  "FP8" is OCP E4M3 (round to nearest even, saturating to +-448); each
      256-group's absmax of the centred constants maps to 448:
      s1 = fp32(c1 / 448), c2 = E4M3(fp32(fp32(a - mu) / s1)).
  R8  dequant a' = fp32(fp32(E4M3(c2) * s1) + mu), w' = bf16(fp32(q[code] * a'))
      (single fp32 multiply, then one round-to-nearest-even to bf16).
"""
from __future__ import annotations

import math
from typing import Dict, Tuple

import numpy as np

BLOCK = 64      # weights per first-level constant ([P1] double-quant paragraph)
BLOCK2 = 256    # first-level constants per second-level constant (same paragraph)
E4M3_MAX = 448.0

# R1: the pages never print the outermost probability; Phi^-1(1) is infinite,
# so an offset is needed.  This is the average of the half-bin offsets for 16
# and 15 bins.
NF4_PMAX = 1.0 - 0.5 * (1.0 / 32.0 + 1.0 / 30.0)


# --------------------------------------------------------------------------
# O1 - NF4 levels from N(0,1) quantiles ([P1] 4-bit NormalFloat paragraph)
# --------------------------------------------------------------------------
def std_normal_cdf(x: float) -> float:
    return 0.5 * math.erfc(-x / math.sqrt(2.0))


def std_normal_quantile(p: float) -> float:
    """Phi^-1(p) by bisection on the CDF, run until the bracket stops shrinking."""
    if p == 0.5:
        return 0.0
    lo, hi = -40.0, 40.0
    while True:
        mid = 0.5 * (lo + hi)
        if mid == lo or mid == hi:
            break
        if std_normal_cdf(mid) < p:
            lo = mid
        else:
            hi = mid
    # pick whichever bracket end has the CDF closer to p
    return lo if abs(std_normal_cdf(lo) - p) <= abs(std_normal_cdf(hi) - p) else hi


def nf4_levels_f64() -> np.ndarray:
    """The 16 NF4 levels in float64, ascending, before rounding to fp32.

    k = 4 bits: 2^(k-1) = 8 quantile points on the negative side and
    2^(k-1)+1 = 9 on the positive side, each side spaced with equal probability
    from p_max down to 1/2 (whose quantile is 0).  The two zeros coincide and
    one is dropped, leaving 7 negative, 1 zero and 8 positive levels.  All are
    divided by the largest magnitude so the ends are exactly -1 and +1.
    """
    pos_p = [NF4_PMAX - i * (NF4_PMAX - 0.5) / 8.0 for i in range(9)]
    neg_p = [NF4_PMAX - i * (NF4_PMAX - 0.5) / 7.0 for i in range(8)]
    pos = [std_normal_quantile(p) if i < 8 else 0.0 for i, p in enumerate(pos_p)]
    neg = [-std_normal_quantile(p) if i < 7 else 0.0 for i, p in enumerate(neg_p)]
    levels = sorted(set(pos) | set(neg))          # the shared zero appears once
    assert len(levels) == 16
    top = max(abs(v) for v in levels)
    return np.array([v / top for v in levels], dtype=np.float64)


def nf4_levels() -> np.ndarray:
    """The fp32 table q[0..15] (parity unpinned beyond its structure, see R1)."""
    return nf4_levels_f64().astype(np.float32)


# --------------------------------------------------------------------------
# OCP E4M3 codec (R7), built by enumeration of the format's definition
# --------------------------------------------------------------------------
def e4m3_decode_table() -> np.ndarray:
    """float64 value of each of the 256 E4M3 codes (NaN for 0x7F and 0xFF)."""
    vals = np.empty(256, dtype=np.float64)
    for c in range(256):
        sign = -1.0 if (c >> 7) & 1 else 1.0
        e = (c >> 3) & 0xF
        m = c & 0x7
        if e == 0xF and m == 0x7:
            vals[c] = np.nan
        elif e == 0:
            vals[c] = sign * (m / 8.0) * 2.0 ** (-6)
        else:
            vals[c] = sign * (1.0 + m / 8.0) * 2.0 ** (e - 7)
    return vals


_E4M3 = e4m3_decode_table()
_E4M3_POS_CODES = np.arange(0, 0x7F)          # 0x00..0x7E: the 127 finite magnitudes
_E4M3_POS_VALS = _E4M3[_E4M3_POS_CODES]


def e4m3_encode(x: np.ndarray) -> np.ndarray:
    """Nearest finite E4M3 code, ties to the even code, saturating at 448.

    Brute force: distance to every non-negative finite magnitude.  The sign
    bit is copied from the input (a negative value that rounds to zero gives
    0x80).
    """
    x = np.asarray(x, dtype=np.float64)
    mag = np.abs(x).ravel()
    out = np.empty(mag.shape, dtype=np.uint8)
    chunk = 1 << 16
    for s in range(0, mag.size, chunk):
        m = mag[s:s + chunk]
        dist = np.abs(m[:, None] - _E4M3_POS_VALS[None, :])
        best = dist.min(axis=1, keepdims=True)
        cand = dist == best
        # among the (at most two) tied nearest codes prefer the even one
        even = (_E4M3_POS_CODES % 2 == 0)[None, :]
        pick_even = cand & even
        has_even = pick_even.any(axis=1)
        idx = np.where(has_even, pick_even.argmax(axis=1), cand.argmax(axis=1))
        code = _E4M3_POS_CODES[idx]
        code = np.where(m > E4M3_MAX, 0x7E, code)      # satfinite
        out[s:s + chunk] = code.astype(np.uint8)
    neg = np.signbit(x.ravel())
    out = np.where(neg, out | 0x80, out).astype(np.uint8)
    return out.reshape(x.shape)


def e4m3_value(codes: np.ndarray) -> np.ndarray:
    return _E4M3[np.asarray(codes, dtype=np.uint8)]


# --------------------------------------------------------------------------
# bf16 rounding (own definition: 8 significant bits, ties to even)
# --------------------------------------------------------------------------
BF16_MIN_NORMAL = 2.0 ** -126
BF16_SUBNORMAL_STEP = 2.0 ** -133     # 7 fraction bits below the smallest normal
BF16_MAX = (2.0 - 2.0 ** -7) * 2.0 ** 127


def to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float64 values to bf16 (nearest, ties to even); return uint16 bits.

    A bf16 number has an 8-bit significand and float32's exponent range.  With
    x = m * 2^e, 0.5 <= |m| < 1, a normal result is rint(m * 256) / 256 * 2^e
    (numpy's rint rounds half to even).  Below the smallest normal 2^-126 the
    representable values are the multiples of 2^-133 (exponent field 0, seven
    fraction bits), so the result is rint(x / 2^-133) * 2^-133; a value that
    rounds up to 2^-126 is the smallest normal.  Results beyond the largest
    finite bf16 are outside this oracle (asserted).
    """
    x = np.asarray(x, dtype=np.float64)
    m, e = np.frexp(x)
    r = np.ldexp(np.rint(m * 256.0), e - 8)
    sub = np.abs(x) < BF16_MIN_NORMAL
    r = np.where(sub, np.rint(x / BF16_SUBNORMAL_STEP) * BF16_SUBNORMAL_STEP, r)
    assert np.all(np.abs(r) <= BF16_MAX)
    f = r.astype(np.float32)                      # exact: at most 8 significant bits
    bits = (f.view(np.uint32) >> 16).astype(np.uint16)
    # zero keeps the sign of the input
    bits = np.where(r == 0, np.where(np.signbit(x), 0x8000, 0).astype(np.uint16), bits)
    return bits


def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16
    return b.view(np.float32).astype(np.float64)


def bf16_to_f32(bits: np.ndarray) -> np.ndarray:
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16
    return b.view(np.float32)


# --------------------------------------------------------------------------
# O2 - first-level blocks: absmax, normalise, nearest level, pack
# --------------------------------------------------------------------------
def block_absmax(W0: np.ndarray) -> np.ndarray:
    """a_b = max |w| over each consecutive 64-element block of row-major W0 (R2)."""
    w = np.ascontiguousarray(W0, dtype=np.float32).reshape(-1, BLOCK)
    return np.abs(w).max(axis=1)


def encode_blocks(wblocks: np.ndarray, absmax: np.ndarray) -> np.ndarray:
    """Codes (0..15, uint8) for blocks of 64 fp32 weights (n, 64).

    x = fp32(w / a_b) (one IEEE division), then the index of the nearest level
    measured exactly in float64; ties go to the lower index (R4).  An all-zero
    block gives the zero level (R3).
    """
    q = nf4_levels().astype(np.float64)
    wblocks = np.asarray(wblocks, dtype=np.float32)
    a = np.asarray(absmax, dtype=np.float32)[:, None]
    zero_block = (a == 0)
    with np.errstate(divide="ignore", invalid="ignore"):
        x = np.where(zero_block, np.float32(0), wblocks / a).astype(np.float32)
    xd = x.astype(np.float64)[..., None]
    dist = np.abs(xd - q)                       # exact: difference of two fp32
    codes = dist.argmin(axis=-1)                # argmin returns the first (lowest) index
    return codes.astype(np.uint8)


def pack_codes(codes: np.ndarray) -> np.ndarray:
    """Two 4-bit codes per byte: even element in the low nibble (R5)."""
    c = np.asarray(codes, dtype=np.uint8).reshape(-1, 2)
    return (c[:, 0] | (c[:, 1] << 4)).astype(np.uint8)


def unpack_codes(packed: np.ndarray) -> np.ndarray:
    p = np.asarray(packed, dtype=np.uint8)
    out = np.empty(p.size * 2, dtype=np.uint8)
    out[0::2] = p & 0xF
    out[1::2] = p >> 4
    return out


# --------------------------------------------------------------------------
# O3 - mean of the block constants (R6)
# --------------------------------------------------------------------------
def pairwise_sum_f64(v: np.ndarray) -> float:
    """float64 pairwise sum: pad with zeros to a power of two, add adjacent pairs."""
    x = np.asarray(v, dtype=np.float64).ravel()
    n = 1
    while n < x.size:
        n *= 2
    x = np.concatenate([x, np.zeros(n - x.size)])
    while x.size > 1:
        x = x[0::2] + x[1::2]
    return float(x[0])


def block_mean(absmax: np.ndarray) -> np.float32:
    n_b = absmax.size
    S = pairwise_sum_f64(absmax.astype(np.float64))
    return np.float32(S / float(n_b))


# --------------------------------------------------------------------------
# O4 - second-level quantisation of the constants (R7)
# --------------------------------------------------------------------------
def double_quant(absmax: np.ndarray, mu: np.float32) -> Tuple[np.ndarray, np.ndarray]:
    """Return (c2 codes uint8 per block, s1 fp32 per group of 256 blocks)."""
    a = np.asarray(absmax, dtype=np.float32)
    n_b = a.size
    n_g = (n_b + BLOCK2 - 1) // BLOCK2
    centred = (a - np.float32(mu)).astype(np.float32)          # fp32(a_b - mu)
    c2 = np.zeros(n_b, dtype=np.uint8)
    s1 = np.zeros(n_g, dtype=np.float32)
    for j in range(n_g):
        seg = centred[j * BLOCK2:(j + 1) * BLOCK2]
        c1 = np.float32(np.abs(seg).max())
        if c1 == 0:
            s1[j] = np.float32(0)
            c2[j * BLOCK2:(j + 1) * BLOCK2] = 0
            continue
        s = np.float32(c1 / np.float32(E4M3_MAX))
        s1[j] = s
        scaled = (seg / s).astype(np.float32)                   # fp32 division
        c2[j * BLOCK2:(j + 1) * BLOCK2] = e4m3_encode(scaled.astype(np.float64))
    return c2, s1


# --------------------------------------------------------------------------
# Full quantise and dequantise
# --------------------------------------------------------------------------
def quantize(W0: np.ndarray) -> Dict[str, np.ndarray]:
    """nf4_quantize(W0, block=64) with double quantisation (block 256)."""
    W0 = np.ascontiguousarray(W0, dtype=np.float32)
    d, k = W0.shape
    assert (d * k) % BLOCK == 0
    a = block_absmax(W0)
    codes = np.empty(W0.size, dtype=np.uint8)
    wb = W0.reshape(-1, BLOCK)
    step = 1 << 14
    for s in range(0, wb.shape[0], step):
        codes[s * BLOCK:(s + step) * BLOCK] = encode_blocks(wb[s:s + step], a[s:s + step]).ravel()
    mu = block_mean(a)
    c2, s1 = double_quant(a, mu)
    return {"codes": pack_codes(codes), "absmax": a, "absmax_q": c2, "scale2": s1,
            "mean": np.float32(mu), "d": d, "k": k}


def block_scale(c2: np.ndarray, s1: np.ndarray, mu: np.float32,
                blocks: np.ndarray = None) -> np.ndarray:
    """a'_b = fp32(fp32(E4M3(c2_b) * s1_j) + mu) for the given block indices (R8)."""
    c2 = np.asarray(c2, dtype=np.uint8)
    if blocks is None:
        blocks = np.arange(c2.size)
    v = e4m3_value(c2[blocks]).astype(np.float32)               # exact in fp32
    prod = (v * s1[blocks // BLOCK2]).astype(np.float32)
    return (prod + np.float32(mu)).astype(np.float32)


def dequantize_blocks(packed: np.ndarray, c2: np.ndarray, s1: np.ndarray, mu: np.float32,
                      blocks: np.ndarray) -> np.ndarray:
    """bf16 bits (len(blocks), 64) of w' = bf16(fp32(q[code] * a'_b)) (R8)."""
    q = nf4_levels()
    blocks = np.asarray(blocks, dtype=np.int64)
    byte_idx = blocks[:, None] * (BLOCK // 2) + np.arange(BLOCK // 2)[None, :]
    codes = unpack_codes(packed[byte_idx].ravel()).reshape(blocks.size, BLOCK)
    a = block_scale(c2, s1, mu, blocks)
    prod = (q[codes] * a[:, None]).astype(np.float32)           # one fp32 multiply
    return to_bf16_bits(prod.astype(np.float64))


def dequantize(qt: Dict[str, np.ndarray]) -> np.ndarray:
    """Full W' (d, k) as bf16 bits."""
    d, k = qt["d"], qt["k"]
    n_b = d * k // BLOCK
    out = np.empty((n_b, BLOCK), dtype=np.uint16)
    step = 1 << 14
    for s in range(0, n_b, step):
        blk = np.arange(s, min(n_b, s + step))
        out[s:s + blk.size] = dequantize_blocks(qt["codes"], qt["absmax_q"], qt["scale2"],
                                                qt["mean"], blk)
    return out.reshape(d, k)


# --------------------------------------------------------------------------
# Storage arithmetic ([P1] double-quant paragraph; [P2]; [P3] "Quick reference")
# --------------------------------------------------------------------------
def storage_bytes(d: int, k: int) -> int:
    """codes + one 8-bit constant per block + one fp32 per 256 blocks + the fp32 mean."""
    n_b = d * k // BLOCK
    n_g = (n_b + BLOCK2 - 1) // BLOCK2
    return d * k // 2 + n_b + 4 * n_g + 4


def constant_bits_per_param(double_quantised: bool) -> float:
    if not double_quantised:
        return 32.0 / BLOCK
    return 8.0 / BLOCK + 32.0 / (BLOCK * BLOCK2)
