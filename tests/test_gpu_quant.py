"""GPU parity: nf4_quantize and doubleDequant are bit-exact with the oracle."""
import numpy as np
import pytest
import torch

import synthetic
from oracle import nf4
from tests.gpu_helpers import bf16_host_bits, f32_dev

pytestmark = pytest.mark.gpu

q4 = pytest.importorskip("parameter_efficient_fine_nf4_b200")


def _gpu_quant(W0: np.ndarray):
    qw = q4.qlora_nf4_quantize(f32_dev(W0))
    Wp = q4.qlora_nf4_dequantize(qw)
    torch.cuda.synchronize()
    assert q4.qlora_get_device_status() == 0
    return qw, Wp


def _check_full(W0: np.ndarray, qw, Wp):
    ref = nf4.quantize(W0)
    assert np.array_equal(qw.codes.cpu().numpy(), ref["codes"])
    assert np.array_equal(qw.absmax_q.cpu().numpy(), ref["absmax_q"])
    assert np.array_equal(qw.scale2.cpu().numpy().view(np.uint32), ref["scale2"].view(np.uint32))
    assert qw.mean.cpu().numpy().view(np.uint32)[0] == np.float32(ref["mean"]).view(np.uint32)
    assert np.array_equal(bf16_host_bits(Wp), nf4.dequantize(ref))


@pytest.mark.parametrize("ci", [1, 2, 3])
def test_quantize_dequantize_bit_exact_full(ci):
    cfg = synthetic.config(ci)
    lay = synthetic.make_layer(cfg, with_acts=False)
    qw, Wp = _gpu_quant(lay.W0)
    _check_full(lay.W0, qw, Wp)


@pytest.mark.parametrize("ci,li", [(4, 0), (4, 1), (5, 4), (5, 6)])
def test_quantize_bit_exact_large_sampled(ci, li):
    # full-size weights; constants and mean exact everywhere, codes and the
    # dequantised weights on a seeded sample of blocks
    cfg = synthetic.config(ci)
    lay = synthetic.make_layer(cfg, li, with_acts=False)
    qw, Wp = _gpu_quant(lay.W0)
    a = nf4.block_absmax(lay.W0)
    mu = nf4.block_mean(a)
    c2, s1 = nf4.double_quant(a, mu)
    assert qw.mean.cpu().numpy().view(np.uint32)[0] == np.float32(mu).view(np.uint32)
    assert np.array_equal(qw.absmax_q.cpu().numpy(), c2)
    assert np.array_equal(qw.scale2.cpu().numpy().view(np.uint32), s1.view(np.uint32))
    n_b = a.size
    blocks = synthetic.sample_rows(1000 + ci * 10 + li, n_b, 20000)
    ref_codes = nf4.pack_codes(nf4.encode_blocks(lay.W0.reshape(-1, 64)[blocks], a[blocks]).ravel())
    gpu_codes = qw.codes.cpu().numpy().reshape(n_b, 32)[blocks].ravel()
    assert np.array_equal(gpu_codes, ref_codes)
    # dequantised weights of the sampled blocks, from the oracle's own codes
    oracle_packed = np.zeros(n_b * 32, np.uint8)
    oracle_packed.reshape(n_b, 32)[blocks] = ref_codes.reshape(-1, 32)
    ref_w = nf4.dequantize_blocks(oracle_packed, c2, s1, mu, blocks)
    gpu_w = bf16_host_bits(Wp).reshape(n_b, 64)[blocks]
    assert np.array_equal(gpu_w, ref_w)


def _near(x: np.float32, n: int):
    """x and its n fp32 neighbours on each side."""
    out = [np.float32(x)]
    lo = hi = np.float32(x)
    for _ in range(n):
        lo = np.nextafter(lo, np.float32(-4))
        hi = np.nextafter(hi, np.float32(4))
        out += [lo, hi]
    return out


def _edge_weights():
    rng = np.random.Generator(np.random.Philox(key=4242))
    q = nf4.nf4_levels()
    _, thr = q4.qlora_nf4_levels()
    d, k = 37, 192            # n_b = 111: one partial group of 256
    W = (rng.standard_normal((d, k)) * 0.02).astype(np.float32)
    flat = W.reshape(-1, 64)
    flat[0] = 0.0                                  # all-zero block
    flat[1] = np.float32(-0.0)
    flat[2] = 0.013                                # constant block
    flat[3] = np.tile(q * np.float32(0.05), 4)     # exactly the levels
    # weights whose quotient by the block absmax lands next to a threshold
    a = np.float32(0.0371)
    xs = np.array([v for t in thr for v in _near(np.float32(t), 3)], np.float32)
    w = (xs * a).astype(np.float32)                # 105 values
    flat[4, :63] = w[:63]
    flat[4, 63] = a
    flat[5, :42] = w[63:]
    flat[5, 42:] = 0.0
    flat[5, 63] = -a                               # absmax from a negative weight
    flat[6] = -flat[4]
    return W


def test_quantize_edge_cases_bit_exact():
    W = _edge_weights()
    qw, Wp = _gpu_quant(W)
    _check_full(W, qw, Wp)


def test_quantize_threshold_sweep():
    # every fp32 quotient within 15 ulps of each threshold, for several block scales
    _, thr = q4.qlora_nf4_levels()
    blocks = []
    for a in (np.float32(1.0), np.float32(0.02), np.float32(3.3e-5), np.float32(7.0e3)):
        for t in thr:
            xs = np.array(_near(np.float32(t), 15), np.float32)      # 31 values
            blk = np.zeros(64, np.float32)
            blk[:31] = (xs * a).astype(np.float32)
            blk[31:62] = (-xs * a).astype(np.float32)
            blk[63] = a
            blocks.append(blk)
    W = np.ascontiguousarray(np.stack(blocks).reshape(-1, 128))    # 60 blocks -> 30 x 128
    qw, Wp = _gpu_quant(W)
    _check_full(W, qw, Wp)


@pytest.mark.parametrize("a", [np.float32(1e-39), np.float32(2.0 ** -126), np.float32(2.0 ** -125),
                               np.float32(2.0 ** 125), np.float32(2.0 ** 126), np.float32(3.0e38)],
                         ids=["subnormal", "min_normal", "fast_lo", "fast_hi", "huge", "near_max"])
def test_quantize_extreme_block_scales(a):
    # blocks whose absmax sits at and beyond both ends of the normal range:
    # quotients next to every threshold, plus one block of subnormal multiples
    _, thr = q4.qlora_nf4_levels()
    blocks = []
    for t in thr:
        xs = np.array(_near(np.float32(t), 3), np.float32)           # 7 values
        blk = np.zeros(64, np.float32)
        blk[:7] = (xs * a).astype(np.float32)
        blk[7:14] = (-xs * a).astype(np.float32)
        blk[14:20] = (a * (np.float32(0.3) / np.float32(7)
                           * np.arange(1, 7, dtype=np.float32))).astype(np.float32)
        blk[63] = a
        blocks.append(blk)
    tiny = (np.arange(64, dtype=np.float32) - np.float32(31)) * np.float32(2.0 ** -149)
    blocks.append(tiny.astype(np.float32))
    W = np.ascontiguousarray(np.stack(blocks).reshape(-1, 128))     # 16 blocks -> 8 x 128
    qw = q4.qlora_nf4_quantize(f32_dev(W))
    Wp = q4.qlora_nf4_dequantize(qw)
    torch.cuda.synchronize()
    assert q4.qlora_get_device_status() == 0
    ref = nf4.quantize(W)
    assert np.array_equal(qw.codes.cpu().numpy(), ref["codes"])
    assert np.array_equal(qw.absmax_q.cpu().numpy(), ref["absmax_q"])
    assert np.array_equal(qw.scale2.cpu().numpy().view(np.uint32), ref["scale2"].view(np.uint32))
    assert qw.mean.cpu().numpy().view(np.uint32)[0] == np.float32(ref["mean"]).view(np.uint32)
    # the dequantised weights too, subnormal results included (the oracle
    # rounds to bf16 over the whole finite range)
    assert np.array_equal(bf16_host_bits(Wp), nf4.dequantize(ref))


def test_quantize_is_deterministic():
    lay = synthetic.make_layer(synthetic.config(2), with_acts=False)
    W = f32_dev(lay.W0)
    a = q4.qlora_nf4_quantize(W)
    b = q4.qlora_nf4_quantize(W)
    torch.cuda.synchronize()
    for x, y in ((a.codes, b.codes), (a.absmax_q, b.absmax_q), (a.scale2, b.scale2), (a.mean, b.mean)):
        assert torch.equal(x, y)
