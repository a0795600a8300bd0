"""Few tokens (T <= 64, the decode-like case of the seven-linear decoder
workload at 16 tokens): the QLoRA forward and backward take the split-depth
kernel with the dequantised weight as the 128-row MMA operand.  Checked
against the float64 oracle on the same seeded inputs ([P1] forward equation
and "The update LoRA is allowed to learn"), on ragged shapes, every token
bucket (16, 32, 64), ranks up to 256, repeated calls (deterministic split
order) and a shared workspace."""
import numpy as np
import pytest
import torch

import synthetic
from oracle import lora, nf4
from tests.gpu_helpers import bf16_dev, bf16_host_f64, f32_dev, f32_host_f64, rows_within

pytestmark = pytest.mark.gpu

q4 = pytest.importorskip("parameter_efficient_fine_nf4_b200")


def _check(lay, alpha, repeat=False):
    qw = q4.qlora_nf4_quantize(f32_dev(lay.W0))
    A, B, X, dY = bf16_dev(lay.A), bf16_dev(lay.B), bf16_dev(lay.X), bf16_dev(lay.dY)
    ws = q4.workspace(max(q4.qlora_fwd_workspace_bytes(lay.d, lay.k, lay.r, lay.T),
                          q4.qlora_bwd_workspace_bytes(lay.d, lay.k, lay.r, lay.T)))
    Y, U = q4.qlora_fwd(qw, A, B, alpha, X, ws=ws)
    dX, dA, dB = q4.qlora_bwd(qw, A, B, alpha, X, U, dY, ws=ws)
    torch.cuda.synchronize()
    assert q4.qlora_get_device_status() == 0
    s = alpha / lay.r
    Wp = nf4.bf16_to_f64(nf4.dequantize(nf4.quantize(lay.W0)))
    Xf, Af, Bf, dYf = (nf4.bf16_to_f64(v) for v in (lay.X, lay.A, lay.B, lay.dY))
    fw = lora.forward(Xf, Wp, Af, Bf, s)
    rows_within(bf16_host_f64(Y), fw["Y"], what="Y")
    rows_within(f32_host_f64(U), fw["U"], what="U")
    bw = lora.backward(Xf, Wp, Af, Bf, s, dYf)
    rows_within(bf16_host_f64(dX), bw["dX"], what="dX")
    rows_within(f32_host_f64(dA), bw["dA"], what="dA")
    rows_within(f32_host_f64(dB), bw["dB"], what="dB")
    if repeat:
        # the same workspace again (tickets re-armed every call), same bits
        Y2, U2 = q4.qlora_fwd(qw, A, B, alpha, X, ws=ws)
        dX2, dA2, dB2 = q4.qlora_bwd(qw, A, B, alpha, X, U2, dY, ws=ws)
        torch.cuda.synchronize()
        for a, b in ((Y, Y2), (U, U2), (dX, dX2), (dA, dA2), (dB, dB2)):
            assert torch.equal(a, b)


@pytest.mark.parametrize("d,k,r,T", [
    (256, 256, 8, 16),        # config-1 shape
    (4096, 4096, 64, 16),     # the decoder's q/k/v/o projection at 16 tokens
    (11008, 4096, 64, 5),     # gate/up projection, T not a multiple of 16
    (4096, 11008, 64, 16),    # down projection (k = 11008: ragged 128-row tile in dX)
    (328, 192, 5, 17),        # ragged tiles, T in the 32 bucket, d % 64 != 0 (partial dX K-step)
    (200, 64, 16, 1),         # one token, one K-step
    (384, 512, 256, 64),      # maximum rank, T at the top of the 64 bucket
    (520, 1024, 100, 33),     # r > 64, T in the 64 bucket, d just past a 128-row tile
])
def test_small_tokens_against_oracle(d, k, r, T):
    lay = synthetic.custom_layer(seed=d * 13 + k + r * 7 + T, d=d, k=k, r=r, T=T, alpha=2.0 * r)
    _check(lay, 2.0 * r, repeat=(T == 16))


def test_small_tokens_b_zero():
    # B = 0: the adapter term vanishes; dA is exactly zero
    lay = synthetic.custom_layer(seed=77, d=1024, k=512, r=8, T=16, alpha=16.0, zero_b=True)
    _check(lay, 16.0)


@pytest.mark.parametrize("d,k,r,T", [(130, 128, 3, 40), (264, 256, 5, 16), (136, 192, 3, 200)])
def test_workspace_garbage_is_never_read(d, k, r, T):
    # every workspace byte a call reads is written by the same call first: a
    # workspace full of NaN patterns (0xFF bytes) must not change any output
    lay = synthetic.custom_layer(seed=d + k + r + T, d=d, k=k, r=r, T=T, alpha=2.0 * r)
    qw = q4.qlora_nf4_quantize(f32_dev(lay.W0))
    A, B, X, dY = bf16_dev(lay.A), bf16_dev(lay.B), bf16_dev(lay.X), bf16_dev(lay.dY)
    outs = []
    for fill in (0, 255):
        ws = q4.workspace(max(q4.qlora_fwd_workspace_bytes(d, k, r, T), q4.qlora_bwd_workspace_bytes(d, k, r, T)))
        ws.fill_(fill)
        Y, U = q4.qlora_fwd(qw, A, B, 2.0 * r, X, ws=ws)
        res = [Y, U]
        if d % 8 == 0:
            ws.fill_(fill)
            res += list(q4.qlora_bwd(qw, A, B, 2.0 * r, X, U, dY, ws=ws))
        torch.cuda.synchronize()
        outs.append(res)
    assert q4.qlora_get_device_status() == 0
    for a, b in zip(*outs):
        assert torch.isfinite(a.float()).all()
        assert torch.equal(a, b)
