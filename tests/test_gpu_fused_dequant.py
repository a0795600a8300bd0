"""The QLoRA forward and backward dequantise the NF4 weight inside the tensor-core
GEMM ([P1] "What QLoRA freezes, and in how many bits": W is dequantised to
BF16 for the multiply in the forward pass and again for the activation
gradient).  The dequantising warps write the weight tile in the same
shared-memory layout a TMA load of the dequantised weight produces, and the
MMA sequence is the same as the plain-LoRA GEMM's, so every output must be
bit-identical to lora_fwd / lora_bwd on qlora_nf4_dequantize's W' (itself
bit-exact against the oracle), on every tile shape the kernel meets."""
import numpy as np
import pytest
import torch

import synthetic
from tests.gpu_helpers import bf16_dev, f32_dev

pytestmark = pytest.mark.gpu

q4 = pytest.importorskip("parameter_efficient_fine_nf4_b200")


# Both builds of the NF4 GEMM: one CTA per 256 x 256 tile (mode 1), and CTA
# pairs that share the decode of each weight tile over 512-token units
# (mode 2).  Both must give the plain-LoRA GEMM's bits.
@pytest.fixture(params=[1, 2], ids=["one_cta", "cta_pair"])
def gemm_mode(request):
    q4.qlora_set_nf4_gemm_mode(request.param)
    yield request.param
    q4.qlora_set_nf4_gemm_mode(0)


def _same_bits(lay, alpha):
    qw = q4.qlora_nf4_quantize(f32_dev(lay.W0))
    Wp = q4.qlora_nf4_dequantize(qw)
    A, B, X, dY = bf16_dev(lay.A), bf16_dev(lay.B), bf16_dev(lay.X), bf16_dev(lay.dY)
    n0 = q4.qlora_launch_count()
    Yq, Uq = q4.qlora_fwd(qw, A, B, alpha, X)
    dXq, dAq, dBq = q4.qlora_bwd(qw, A, B, alpha, X, Uq, dY)
    torch.cuda.synchronize()
    Yp, Up = q4.lora_fwd(Wp, A, B, alpha, X)
    dXp, dAp, dBp = q4.lora_bwd(Wp, A, B, alpha, X, Up, dY)
    torch.cuda.synchronize()
    assert q4.qlora_get_device_status() == 0
    for name, a, b in (("Y", Yq, Yp), ("U", Uq, Up), ("dX", dXq, dXp), ("dA", dAq, dAp), ("dB", dBq, dBp)):
        assert torch.equal(a, b), f"{name} differs from the plain-LoRA GEMM on W'"


# (T > 64: the 256 x 256-tile kernel; fewer tokens take the split-depth
# kernel, whose fp32 sums run in another order: see test_gpu_small_tokens.py.
# In a pair, the second CTA's 256 rows start at token 256 of the unit: the
# shapes below leave it empty, one row, partial and full.)
@pytest.mark.parametrize("d,k,r,T", [
    (256, 256, 8, 100),       # one tile, T < 128: the second M tile is absent
    (512, 384, 16, 300),      # two N tiles in the forward, ragged N tile (k = 384) in dX
    (328, 192, 5, 200),       # ragged N tile (d = 328); d % 64 != 0 ends dX on a partial K-step
    (136, 128, 3, 129),       # T just past one 128-row tile
    (264, 512, 100, 257),     # r > 64: two rank-r steps; T just past a 256-row unit
    (384, 256, 256, 72),      # maximum rank (four rank-r steps)
    (1024, 1024, 64, 1000),   # several units per CTA
    (200, 64, 16, 65),        # K = 64: one main step
    (520, 320, 16, 513),      # one token past a 512-token unit
    (256, 640, 32, 1536),     # three full 512-token units, ragged dX tile (k = 640)
])
def test_fused_dequant_bit_identical(d, k, r, T, gemm_mode):
    lay = synthetic.custom_layer(seed=d * 31 + k * 3 + r + T, d=d, k=k, r=r, T=T, alpha=2.0 * r)
    _same_bits(lay, 2.0 * r)


@pytest.mark.parametrize("ci", [2, 3])
def test_fused_dequant_bit_identical_configs(ci, gemm_mode):
    cfg = synthetic.config(ci)
    _same_bits(synthetic.make_layer(cfg, T=512 if ci == 3 else None), cfg.alpha)


def test_fused_dequant_large_shape(gemm_mode):
    # the 8192 -> 22016 projection at 2048 tokens: long K loops, many units
    cfg = synthetic.config(4)
    lay = synthetic.make_layer(cfg, 0, T=2048)
    _same_bits(lay, cfg.alpha)


@pytest.mark.parametrize("T", [16, 300])
def test_qlora_launches_no_separate_dequantisation(T):
    cfg = synthetic.config(1)
    lay = synthetic.make_layer(cfg, T=T)
    qw = q4.qlora_nf4_quantize(f32_dev(lay.W0))
    A, B, X, dY = bf16_dev(lay.A), bf16_dev(lay.B), bf16_dev(lay.X), bf16_dev(lay.dY)
    torch.cuda.synchronize()
    q4.qlora_profile_begin()
    Y, U = q4.qlora_fwd(qw, A, B, cfg.alpha, X)
    q4.qlora_bwd(qw, A, B, cfg.alpha, X, U, dY)
    stats = q4.qlora_profile_end()
    names = {s["name"] for s in stats}
    assert "nf4_dequantize" not in names
    if T <= 64:
        assert {"gemm_nf4_small_fwd", "gemm_nf4_small_dx"} <= names
    else:
        assert {"gemm_nf4_fwd", "gemm_nf4_dx"} <= names
