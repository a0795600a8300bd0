"""GPU parity of LoRA dropout on the adapter input ([P5] "LoRA vs QLoRA:
Parameter-Efficient Fine-Tuning Explained", run configuration: LoRA dropout
0.05-0.1) against the float64 oracle's forward_dropout / backward_dropout,
both sides given the same keep mask (drawn here from a seeded generator and
bit-packed for the library)."""
import numpy as np
import pytest
import torch

import synthetic
from oracle import lora, nf4
from tests.gpu_helpers import bf16_dev, bf16_host_f64, f32_dev, f32_host_f64, rows_within

pytestmark = pytest.mark.gpu

q4 = pytest.importorskip("parameter_efficient_fine_nf4_b200")


def _mask(seed, T, k, p):
    gen = np.random.Generator(np.random.Philox(key=seed))
    keep = (gen.random((T, k)) >= p).astype(np.uint8)
    packed = np.packbits(keep.reshape(-1), bitorder="little")
    return keep.astype(np.float64), torch.from_numpy(packed).cuda()


def _run(lay, alpha, p, seed, rows=None, keep=None):
    s = alpha / lay.r
    T, k = lay.T, lay.k
    if keep is None:
        keep_f, keep_dev = _mask(seed, T, k, p)
    else:
        keep_f = keep.astype(np.float64)
        keep_dev = torch.from_numpy(np.packbits(keep.reshape(-1), bitorder="little")).cuda()
    qw = q4.qlora_nf4_quantize(f32_dev(lay.W0))
    A, B, X, dY = bf16_dev(lay.A), bf16_dev(lay.B), bf16_dev(lay.X), bf16_dev(lay.dY)
    Y, U = q4.qlora_fwd_dropout(qw, A, B, alpha, X, keep_dev, p)
    dX, dA, dB = q4.qlora_bwd_dropout(qw, A, B, alpha, X, keep_dev, p, U, dY)
    torch.cuda.synchronize()
    assert q4.qlora_get_device_status() == 0
    Wp = nf4.bf16_to_f64(nf4.dequantize(nf4.quantize(lay.W0)))
    Xf, Af, Bf, dYf = (nf4.bf16_to_f64(v) for v in (lay.X, lay.A, lay.B, lay.dY))
    if rows is None:
        rows = np.arange(T)
    fw = lora.forward_dropout(Xf[rows], Wp, Af, Bf, s, keep_f[rows], p)
    rows_within(bf16_host_f64(Y)[rows], fw["Y"], what="Y")
    rows_within(f32_host_f64(U)[rows], fw["U"], what="U")
    bw = lora.backward_dropout(Xf, Wp, Af, Bf, s, dYf, keep_f, p)
    rows_within(bf16_host_f64(dX)[rows], bw["dX"][rows], what="dX")
    rows_within(f32_host_f64(dA), bw["dA"], what="dA")
    rows_within(f32_host_f64(dB), bw["dB"], what="dB")
    return Y, U, dX, dA, dB


@pytest.mark.parametrize("ci,p", [(1, 0.1), (2, 0.05), (2, 0.5)])
def test_dropout_configs(ci, p):
    cfg = synthetic.config(ci)
    _run(synthetic.make_layer(cfg), cfg.alpha, p, seed=700 + ci)


def test_dropout_config3_sampled_rows():
    cfg = synthetic.config(3)
    lay = synthetic.make_layer(cfg, T=2048)
    _run(lay, cfg.alpha, 0.1, seed=703, rows=synthetic.sample_rows(704, lay.T, 128))


@pytest.mark.parametrize("d,k,r,T", [
    (328, 192, 5, 17),        # few tokens (split-depth kernels), ragged tiles
    (264, 512, 100, 257),     # r > 64, T just past a 256-row unit
    (200, 64, 16, 1),         # one token
    (512, 384, 16, 300),
])
def test_dropout_ragged(d, k, r, T):
    lay = synthetic.custom_layer(seed=d + 3 * k + r + T, d=d, k=k, r=r, T=T, alpha=2.0 * r)
    _run(lay, 2.0 * r, 0.1, seed=d + T)


@pytest.mark.parametrize("T", [16, 300])
def test_dropout_p0_is_the_plain_layer(T):
    # p = 0 keeps every element: the same bits as qlora_fwd / qlora_bwd
    cfg = synthetic.config(1)
    lay = synthetic.make_layer(cfg, T=T)
    qw = q4.qlora_nf4_quantize(f32_dev(lay.W0))
    A, B, X, dY = bf16_dev(lay.A), bf16_dev(lay.B), bf16_dev(lay.X), bf16_dev(lay.dY)
    Y0, U0 = q4.qlora_fwd(qw, A, B, cfg.alpha, X)
    d0 = q4.qlora_bwd(qw, A, B, cfg.alpha, X, U0, dY)
    Y1, U1 = q4.qlora_fwd_dropout(qw, A, B, cfg.alpha, X, None, 0.0)
    d1 = q4.qlora_bwd_dropout(qw, A, B, cfg.alpha, X, None, 0.0, U1, dY)
    torch.cuda.synchronize()
    for a, b in zip((Y0, U0) + tuple(d0), (Y1, U1) + tuple(d1)):
        assert torch.equal(a, b)


@pytest.mark.parametrize("T", [16, 300])
def test_dropout_everything_dropped(T):
    # a mask of zeros removes the adapter: U = 0, dA = dB = 0 exactly, and Y,
    # dX are the base products
    cfg = synthetic.config(1)
    lay = synthetic.make_layer(cfg, T=T)
    Y, U, dX, dA, dB = _run(lay, cfg.alpha, 0.5, seed=0, keep=np.zeros((T, lay.k), np.uint8))
    assert torch.count_nonzero(U).item() == 0
    assert torch.count_nonzero(dA).item() == 0 and torch.count_nonzero(dB).item() == 0


def test_dropout_masks_differ_in_results():
    # two complementary masks give different adapter gradients whose
    # oracle values differ too: the mask really reaches the kernels
    cfg = synthetic.config(1)
    lay = synthetic.make_layer(cfg)
    keep = (np.arange(lay.T * lay.k).reshape(lay.T, lay.k) % 3 != 0).astype(np.uint8)
    r1 = _run(lay, cfg.alpha, 1.0 / 3.0, seed=0, keep=keep)
    r2 = _run(lay, cfg.alpha, 1.0 / 3.0, seed=0, keep=1 - keep)
    assert not torch.equal(r1[3], r2[3])
