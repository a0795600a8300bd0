"""Pins for the NF4 / double-quant oracle against what the pages and the
mathematics fix (no comparison of the oracle with itself)."""
import json
import math
import os
import statistics
from fractions import Fraction

import numpy as np
import pytest

from oracle import nf4
import synthetic


# ----------------------------------------------------------------- NF4 levels
def test_quantile_matches_library_routines():
    # special case that reduces to library routines: the N(0,1) inverse CDF
    from scipy.special import ndtri
    nd = statistics.NormalDist()
    for p in [0.5000001, 0.55, 0.6, 0.75, 0.9, 0.9677083, 0.99, 0.999]:
        x = nf4.std_normal_quantile(p)
        assert abs(x - nd.inv_cdf(p)) < 1e-12
        assert abs(x - float(ndtri(p))) < 1e-12


def test_nf4_structure(golden_dir):
    g = json.load(open(os.path.join(golden_dir, "pages_numbers.json")))["nf4_level_counts"]
    q = nf4.nf4_levels()
    assert q.dtype == np.float32 and q.size == g["total"]
    assert np.all(np.diff(q.astype(np.float64)) > 0)            # distinct, ascending
    assert q[0] == -1.0 and q[15] == 1.0                          # endpoints +-1
    assert q[7] == 0.0 and np.signbit(q[7]) == False              # exact zero
    assert int((q < 0).sum()) == g["negative"]
    assert int((q > 0).sum()) == g["positive"]
    assert int((q == 0).sum()) == g["zero"]


def test_nf4_equal_probability_spacing():
    # Each side's levels sit at equally spaced probabilities from p_max to 1/2:
    # undo the normalisation and map back through the CDF.
    q = nf4.nf4_levels_f64()
    scale = nf4.std_normal_quantile(nf4.NF4_PMAX)
    probs = np.array([nf4.std_normal_cdf(v * scale) for v in q])
    pos = probs[7:]                     # 0 .. +1  (9 points incl. zero)
    neg = 1.0 - probs[:8][::-1]         # 0 .. -1 mirrored (8 points incl. zero)
    dp = np.diff(pos)
    dn = np.diff(neg)
    assert np.allclose(dp, (nf4.NF4_PMAX - 0.5) / 8, rtol=0, atol=1e-12)
    assert np.allclose(dn, (nf4.NF4_PMAX - 0.5) / 7, rtol=0, atol=1e-12)
    # the asymmetry: the negative side is coarser, so |q_neg[i]| > q_pos[i]
    assert abs(q[6]) > q[8]


def test_nf4_levels_round_to_fp32_unambiguously():
    # every level lies far (relative) from an fp32 rounding midpoint, so any
    # float64-accurate construction rounds to the same fp32 table
    q64 = nf4.nf4_levels_f64()
    q32 = q64.astype(np.float32).astype(np.float64)
    for v, r in zip(q64, q32):
        if v == 0 or abs(v) == 1:
            continue
        ulp = np.spacing(np.float32(abs(r)))
        frac = abs(v - r) / ulp
        assert frac < 0.5 - 1e-6


# ------------------------------------------------------------------- encoder
def test_encoder_roundtrip_levels():
    q = nf4.nf4_levels()
    for a in [np.float32(0.02), np.float32(1.0), np.float32(3.5e-3), np.float32(7.25)]:
        block = np.tile(q * a, 4).astype(np.float32)       # 64 values, max = a
        codes = nf4.encode_blocks(block[None, :], np.array([a], np.float32))[0]
        assert list(codes) == list(range(16)) * 4


def test_encoder_nearest_and_ties_bruteforce():
    # brute force over a dense grid of fp32 x in [-1, 1]: the chosen level is
    # at minimal distance, and on an exact tie the lower code wins
    q = nf4.nf4_levels().astype(np.float64)
    xs = np.linspace(-1, 1, 200001).astype(np.float32)
    # add every fp32 value within 64 ulps of each exact midpoint
    extra = []
    for i in range(15):
        m = np.float32((q[i] + q[i + 1]) / 2)
        v = m
        for _ in range(64):
            v = np.nextafter(v, np.float32(-2))
        for _ in range(129):
            extra.append(v)
            v = np.nextafter(v, np.float32(2))
    xs = np.concatenate([xs, np.array(extra, np.float32)])
    blocks = xs[: (xs.size // 64) * 64].reshape(-1, 64)
    a = np.ones(blocks.shape[0], np.float32)                # x = w / 1 exactly
    codes = nf4.encode_blocks(blocks, a).ravel()
    x = blocks.ravel().astype(np.float64)
    for xi, ci in zip(x[::7], codes[::7]):
        d = [abs(xi - qq) for qq in q]
        best = min(d)
        assert d[ci] == best
        assert ci == d.index(best)                           # lowest tied index
    # monotone in x
    order = np.argsort(x, kind="stable")
    assert np.all(np.diff(codes[order].astype(int)) >= 0)


def test_encoder_exact_tie_goes_low():
    q = nf4.nf4_levels().astype(np.float64)
    found = 0
    for i in range(15):
        m = (q[i] + q[i + 1]) / 2
        if float(np.float32(m)) == m:                         # representable midpoint
            found += 1
            blk = np.full((1, 64), np.float32(m))
            blk[0, 0] = np.float32(1.0)
            c = nf4.encode_blocks(blk, np.array([1.0], np.float32))[0]
            assert c[1] == i
    # midpoints between levels -1 and the next one etc. are not all representable;
    # the brute-force test above covers the rest


def test_zero_block_and_pack_order():
    blk = np.zeros((1, 64), np.float32)
    c = nf4.encode_blocks(blk, np.zeros(1, np.float32))[0]
    assert np.all(c == 7)
    packed = nf4.pack_codes(np.array([1, 2, 3, 15], np.uint8))
    assert list(packed) == [0x21, 0xF3]
    assert list(nf4.unpack_codes(packed)) == [1, 2, 3, 15]


# ---------------------------------------------------------------------- E4M3
def test_e4m3_decode_matches_torch():
    torch = pytest.importorskip("torch")
    codes = torch.arange(256, dtype=torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    ours = nf4.e4m3_decode_table()
    finite = ~np.isnan(ref)
    assert np.array_equal(np.isnan(ours), ~finite)
    assert np.array_equal(ours[finite], ref[finite])
    assert ours[0x7E] == 448.0 and ours[0x08] == 2.0 ** -6 and ours[0x01] == 2.0 ** -9


def test_e4m3_encode_roundtrip_and_torch():
    torch = pytest.importorskip("torch")
    table = nf4.e4m3_decode_table()
    codes = np.array([c for c in range(256) if not np.isnan(table[c])])
    vals = table[codes]
    enc = nf4.e4m3_encode(vals)
    # +0 and -0 keep their codes; every finite code re-encodes to itself
    assert np.array_equal(enc, codes.astype(np.uint8))
    # random fp32 values inside the finite range: torch's RN-even cast agrees
    rng = np.random.Generator(np.random.Philox(key=7))
    x = (rng.standard_normal(200000) * np.exp(rng.uniform(-12, 6, 200000))).astype(np.float32)
    x = x[np.abs(x) <= 448]
    # include exact ties between neighbouring codes
    mids = ((vals[1:0x7E] + vals[2:0x7F]) / 2).astype(np.float32)
    x = np.concatenate([x, mids, -mids])
    ours = nf4.e4m3_encode(x.astype(np.float64))
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(ours, ref)
    # saturation beyond the largest finite value
    assert nf4.e4m3_encode(np.array([460.0, 1e6, -500.0])).tolist() == [0x7E, 0x7E, 0xFE]


# ---------------------------------------------------------------------- bf16
def test_bf16_rounding_matches_torch():
    torch = pytest.importorskip("torch")
    rng = np.random.Generator(np.random.Philox(key=11))
    x = (rng.standard_normal(100000) * np.exp(rng.uniform(-20, 20, 100000))).astype(np.float32)
    # ties: fp32 values exactly halfway between two bf16 numbers
    ties = ((rng.integers(0x3000, 0x4F00, 2000).astype(np.uint32) << 16) | 0x8000).view(np.float32)
    x = np.concatenate([x, ties, -ties])
    ours = nf4.to_bf16_bits(x.astype(np.float64))
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, ref)


def test_bf16_rounding_subnormal_range():
    # below 2^-126 the bf16 grid is the multiples of 2^-133; every fp32
    # subnormal pattern class (random bits, exact ties between grid points,
    # values rounding up into the normal range) against torch's conversion
    torch = pytest.importorskip("torch")
    rng = np.random.Generator(np.random.Philox(key=12))
    rand = rng.integers(1, 0x00800000, 50000).astype(np.uint32)
    ties = (rng.integers(0, 0x80, 2000).astype(np.uint32) << 16) | 0x8000
    edge = np.array([0x007F8000, 0x007FFFFF, 0x00008000, 0x00018000, 0x00000001], np.uint32)
    bits = np.concatenate([rand, ties, edge])
    x = np.concatenate([bits, bits | 0x80000000]).view(np.float32)
    ours = nf4.to_bf16_bits(x.astype(np.float64))
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, ref)
    # closed forms: half the smallest step rounds to (signed) zero, 1.5 steps to 2
    step = 2.0 ** -133
    assert nf4.to_bf16_bits(np.array([0.5 * step, -0.5 * step, 1.5 * step])).tolist() == [0x0000, 0x8000, 0x0002]
    # just below the smallest normal rounds up to it (exponent field 1)
    assert nf4.to_bf16_bits(np.array([2.0 ** -126 - 0.25 * step])).tolist() == [0x0080]


# ---------------------------------------------------------------------- mean
def test_pairwise_sum_exact_on_integers_and_close_to_fsum():
    v = np.arange(1, 1001, dtype=np.float64)
    assert nf4.pairwise_sum_f64(v) == 500500.0
    rng = np.random.Generator(np.random.Philox(key=3))
    a = np.abs(rng.standard_normal(70001)).astype(np.float32)
    s = nf4.pairwise_sum_f64(a)
    assert abs(s - math.fsum(a.astype(np.float64))) <= 1e-12 * s


def test_mean_is_rounded_exact_mean_on_seeded_weights():
    # property: mu equals the fp32 rounding of the exact rational mean of the
    # block constants (float64 summation error is far below fp32 resolution)
    for ci in (1, 2):
        cfg = synthetic.config(ci)
        lay = synthetic.make_layer(cfg, with_acts=False)
        a = nf4.block_absmax(lay.W0)
        mu = nf4.block_mean(a)
        exact = sum((Fraction(float(v)) for v in a), Fraction(0)) / a.size
        lo = np.float32(float(exact))
        cands = [np.nextafter(lo, np.float32(-1)), lo, np.nextafter(lo, np.float32(1))]
        best = min(cands, key=lambda c: abs(Fraction(float(c)) - exact))
        assert mu == best


# ----------------------------------------------------------- double quant
def test_double_quant_maps_group_absmax_to_448():
    rng = np.random.Generator(np.random.Philox(key=5))
    a = np.abs(rng.standard_normal(1000) * 0.02).astype(np.float32) + np.float32(0.01)
    mu = nf4.block_mean(a)
    c2, s1 = nf4.double_quant(a, mu)
    assert s1.size == 4 and c2.size == 1000
    cen = (a - mu).astype(np.float32)
    for j in range(4):
        seg = cen[j * 256:(j + 1) * 256]
        i = int(np.abs(seg).argmax())
        assert (c2[j * 256 + i] & 0x7F) == 0x7E                  # |value| 448
        assert s1[j] == np.float32(np.float32(np.abs(seg).max()) / np.float32(448))
    # reconstruction error of every constant within half an E4M3 step at its scale
    a2 = nf4.block_scale(c2, s1, mu)
    v = nf4.e4m3_value(c2)
    step = np.maximum(np.abs(v) * 2.0 ** -3, 2.0 ** -9) * s1[np.arange(1000) // 256]
    assert np.all(np.abs(a2.astype(np.float64) - a) <= step * 0.5 + 1e-7)


def test_double_quant_zero_group():
    a = np.full(256, 0.5, np.float32)
    mu = nf4.block_mean(a)
    assert mu == np.float32(0.5)
    c2, s1 = nf4.double_quant(a, mu)
    assert s1[0] == 0 and np.all(c2 == 0)
    assert np.all(nf4.block_scale(c2, s1, mu) == np.float32(0.5))


# ------------------------------------------------------------ storage pins
def test_storage_arithmetic_matches_pages(golden_dir):
    g = json.load(open(os.path.join(golden_dir, "pages_numbers.json")))
    single = nf4.constant_bits_per_param(False)
    double = nf4.constant_bits_per_param(True)
    assert single == g["constant_bits_single_quant"]["value"]
    assert round(double, 3) == g["constant_bits_double_quant"]["value"]
    assert round(single - double, 3) == g["double_quant_saving_bits"]["value"]
    gb = (single - double) * g["double_quant_saving_65B_GB"]["params"] / 8 / 1e9
    assert round(gb) == g["double_quant_saving_65B_GB"]["value"]
    assert round(16 / (4 + double)) == g["base_vram_reduction_approx"]["value"]
    # exact byte counts of the stored format
    assert nf4.storage_bytes(256, 256) == 33812
    assert nf4.storage_bytes(4096, 4096) == 8654852
    assert nf4.storage_bytes(11008, 4096) == 23259908
    assert nf4.storage_bytes(22016, 8192) == 93039620


# ------------------------------------------------------------------ dequant
def test_dequant_error_bound_and_blocks_roundtrip():
    lay = synthetic.make_layer(synthetic.config(1), with_acts=False)
    qt = nf4.quantize(lay.W0)
    assert qt["codes"].size == 256 * 256 // 2
    Wp = nf4.bf16_to_f64(nf4.dequantize(qt))
    W = lay.W0.astype(np.float64)
    q = nf4.nf4_levels().astype(np.float64)
    half_gap = np.max(np.diff(q)) / 2
    a = qt["absmax"].astype(np.float64)
    a2 = nf4.block_scale(qt["absmax_q"], qt["scale2"], qt["mean"]).astype(np.float64)
    assert np.all(a2 > 0)                                  # invariant on Gaussian weights
    err = np.abs(W - Wp).reshape(-1, 64)
    bound = half_gap * a + np.abs(a - a2) + np.abs(Wp).reshape(-1, 64).max(1) * 2.0 ** -8
    assert np.all(err.max(axis=1) <= bound * (1 + 1e-6) + 1e-8)
    # re-encoding the dequantised weights with the stored constants returns the codes
    x = (Wp.reshape(-1, 64) / a2[:, None])
    codes = np.abs(x[..., None] - q).argmin(-1).ravel()
    assert np.array_equal(codes.astype(np.uint8), nf4.unpack_codes(qt["codes"]))
