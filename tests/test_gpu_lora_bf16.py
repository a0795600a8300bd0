"""GPU parity of plain LoRA on a bf16 base (lora_fwd / lora_bwd) against the
float64 oracle, and bit-for-bit agreement with the QLoRA entry points when
the bf16 base is the dequantised weight (both run the same GEMMs)."""
import numpy as np
import pytest
import torch

import synthetic
from oracle import lora, nf4
from tests.gpu_helpers import bf16_dev, bf16_host_f64, f32_dev, f32_host_f64, rows_within

pytestmark = pytest.mark.gpu

q4 = pytest.importorskip("parameter_efficient_fine_nf4_b200")


def _run(lay, alpha, rows=None, full_adapter_grads=True):
    """lora_fwd/lora_bwd on W = bf16(W0), checked against the oracle on that W."""
    W_bits = synthetic.f32_to_bf16_bits(lay.W0)
    W = bf16_dev(W_bits)
    A, B, X, dY = bf16_dev(lay.A), bf16_dev(lay.B), bf16_dev(lay.X), bf16_dev(lay.dY)
    Y, U = q4.lora_fwd(W, A, B, alpha, X)
    dX, dA, dB = q4.lora_bwd(W, A, B, alpha, X, U, dY)
    torch.cuda.synchronize()
    assert q4.qlora_get_device_status() == 0
    s = alpha / lay.r
    Wf, Xf, Af, Bf, dYf = (nf4.bf16_to_f64(v) for v in (W_bits, lay.X, lay.A, lay.B, lay.dY))
    if rows is None:
        rows = np.arange(lay.T)
    fw = lora.forward(Xf[rows], Wf, Af, Bf, s)
    rows_within(bf16_host_f64(Y)[rows], fw["Y"], what="Y")
    rows_within(f32_host_f64(U)[rows], fw["U"], what="U")
    gi = lora.grad_input(Wf, Af, Bf, s, dYf[rows])
    rows_within(bf16_host_f64(dX)[rows], gi["dX"], what="dX")
    if full_adapter_grads:
        ga = lora.grad_adapters(Xf, Af, Bf, s, dYf)
        rows_within(f32_host_f64(dA), ga["dA"], what="dA")
        rows_within(f32_host_f64(dB), ga["dB"], what="dB")


@pytest.mark.parametrize("ci", [1, 2])
def test_configs_full(ci):
    cfg = synthetic.config(ci)
    _run(synthetic.make_layer(cfg), cfg.alpha)


def test_config3_sampled_rows():
    cfg = synthetic.config(3)
    lay = synthetic.make_layer(cfg)
    _run(lay, cfg.alpha, rows=synthetic.sample_rows(903, lay.T, 192))


@pytest.mark.parametrize("d,k,r,T", [
    (320, 200, 5, 200),      # k a multiple of 8 but not of 64: ragged K step
    (136, 128, 3, 129),
    (256, 512, 100, 300),    # r > 64
    (64, 64, 1, 1),
])
def test_ragged_shapes(d, k, r, T):
    lay = synthetic.custom_layer(seed=d * 17 + k * 5 + r + T, d=d, k=k, r=r, T=T, alpha=2.0 * r)
    _run(lay, 2.0 * r)


def test_same_bits_as_qlora_on_the_dequantised_weight():
    cfg = synthetic.config(3)
    lay = synthetic.make_layer(cfg, T=1024)
    qw = q4.qlora_nf4_quantize(f32_dev(lay.W0))
    Wp = q4.qlora_nf4_dequantize(qw)
    A, B, X, dY = bf16_dev(lay.A), bf16_dev(lay.B), bf16_dev(lay.X), bf16_dev(lay.dY)
    Yq, Uq = q4.qlora_fwd(qw, A, B, cfg.alpha, X)
    dXq, dAq, dBq = q4.qlora_bwd(qw, A, B, cfg.alpha, X, Uq, dY)
    Yp, Up = q4.lora_fwd(Wp, A, B, cfg.alpha, X)
    dXp, dAp, dBp = q4.lora_bwd(Wp, A, B, cfg.alpha, X, Up, dY)
    torch.cuda.synchronize()
    for a, b in ((Yq, Yp), (Uq, Up), (dXq, dXp), (dAq, dAp), (dBq, dBp)):
        assert torch.equal(a, b)


def test_rejects_k_not_multiple_of_8():
    W = torch.zeros(64, 60, dtype=torch.bfloat16, device="cuda")
    A = torch.zeros(4, 60, dtype=torch.bfloat16, device="cuda")
    B = torch.zeros(64, 4, dtype=torch.bfloat16, device="cuda")
    X = torch.zeros(8, 60, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(q4.QloraError) as e:
        q4.lora_fwd(W, A, B, 8.0, X)
    assert e.value.status == 2
