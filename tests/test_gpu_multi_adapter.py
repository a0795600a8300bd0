"""GPU parity of a batch that uses several unmerged adapters over one frozen
NF4 base ([P2] "The LoRA hypothesis": many tasks served from one base with a
stack of small adapters chosen per request), against the float64 oracle's
forward_multi / backward_multi on the same seeded inputs and token indices."""
import numpy as np
import pytest
import torch

import synthetic
from oracle import lora, nf4
from tests.gpu_helpers import bf16_dev, bf16_host_f64, f32_dev, f32_host_f64, rows_within

pytestmark = pytest.mark.gpu

q4 = pytest.importorskip("parameter_efficient_fine_nf4_b200")


def _stack(seed, n, d, k, r, T, empty=None):
    """n adapters (A ~ N(0, 1/r), B ~ N(0, 0.01)), per-adapter alphas and a
    seeded token -> adapter index (adapter `empty` gets no token)."""
    As = np.stack([synthetic.normal_bf16(seed + 10 * i + 1, (r, k), 1.0 / r) for i in range(n)])
    Bs = np.stack([synthetic.normal_bf16(seed + 10 * i + 2, (d, r), 0.01) for i in range(n)])
    alphas = [float(2 * r * (i + 1)) for i in range(n)]
    gen = np.random.Generator(np.random.Philox(key=seed + 999))
    choices = [i for i in range(n) if i != empty] or [0]
    idx = np.array([choices[j] for j in gen.integers(0, len(choices), T)], np.int32)
    return As, Bs, alphas, idx


def _run(d, k, r, T, n, seed, empty=None):
    lay = synthetic.custom_layer(seed=seed, d=d, k=k, r=r, T=T, alpha=2.0 * r)
    As, Bs, alphas, idx = _stack(seed, n, d, k, r, T, empty)
    qw = q4.qlora_nf4_quantize(f32_dev(lay.W0))
    As_d = bf16_dev(As.reshape(n * r, k)).view(n, r, k)
    Bs_d = bf16_dev(Bs.reshape(n * d, r)).view(n, d, r)
    idx_d = torch.from_numpy(idx).cuda()
    X, dY = bf16_dev(lay.X), bf16_dev(lay.dY)
    Y, U = q4.qlora_fwd_multi(qw, As_d, Bs_d, alphas, idx_d, X)
    dX, dAs, dBs = q4.qlora_bwd_multi(qw, As_d, Bs_d, alphas, idx_d, X, U, dY)
    torch.cuda.synchronize()
    assert q4.qlora_get_device_status() == 0
    Wp = nf4.bf16_to_f64(nf4.dequantize(nf4.quantize(lay.W0)))
    Xf, dYf = nf4.bf16_to_f64(lay.X), nf4.bf16_to_f64(lay.dY)
    Af, Bf = nf4.bf16_to_f64(As), nf4.bf16_to_f64(Bs)
    ss = np.array(alphas) / r
    fw = lora.forward_multi(Xf, Wp, Af, Bf, ss, idx)
    rows_within(bf16_host_f64(Y), fw["Y"], what="Y")
    rows_within(f32_host_f64(U), fw["U"], what="U")
    bw = lora.backward_multi(Xf, Wp, Af, Bf, ss, idx, dYf)
    rows_within(bf16_host_f64(dX), bw["dX"], what="dX")
    for i in range(n):
        rows_within(f32_host_f64(dAs[i]), bw["dA"][i], what=f"dA[{i}]")
        rows_within(f32_host_f64(dBs[i]), bw["dB"][i], what=f"dB[{i}]")
    return qw, As_d, Bs_d, alphas, idx_d, X, dY, (Y, U, dX, dAs, dBs)


@pytest.mark.parametrize("n", [1, 3, 8])
@pytest.mark.parametrize("T", [16, 300])
def test_multi_adapter_against_oracle(n, T):
    _run(256, 256, 8, T, n, seed=100 * n + T)


@pytest.mark.parametrize("d,k,r,T,n", [
    (328, 192, 5, 17, 3),      # ragged tiles, r not a multiple of 8, few tokens
    (264, 512, 32, 257, 4),    # n r = 128
    (384, 256, 16, 64, 16),    # n r = 256, the largest stack
])
def test_multi_adapter_ragged(d, k, r, T, n):
    _run(d, k, r, T, n, seed=d + k + r + T + n)


@pytest.mark.parametrize("T", [16, 300])
def test_multi_adapter_unused_adapter_gets_zero_gradients(T):
    res = _run(256, 256, 8, T, 4, seed=31 + T, empty=2)[-1]
    dAs, dBs = res[3], res[4]
    assert torch.count_nonzero(dAs[2]).item() == 0 and torch.count_nonzero(dBs[2]).item() == 0


@pytest.mark.parametrize("T", [16, 300])
def test_single_adapter_stack_is_the_plain_layer(T):
    # a stack of one adapter, every token on it: the same bits as qlora_fwd/bwd
    qw, As, Bs, alphas, idx, X, dY, res = _run(256, 256, 8, T, 1, seed=5 + T)
    A, B = As[0].contiguous(), Bs[0].contiguous()
    Y, U = q4.qlora_fwd(qw, A, B, alphas[0], X)
    dX, dA, dB = q4.qlora_bwd(qw, A, B, alphas[0], X, U, dY)
    torch.cuda.synchronize()
    for a, b in zip((Y, U, dX, dA, dB), (res[0], res[1], res[2], res[3][0], res[4][0])):
        assert torch.equal(a, b)


def test_token_without_adapter_gets_the_base_output():
    d, k, r, T, n = 256, 256, 8, 40, 2
    lay = synthetic.custom_layer(seed=8, d=d, k=k, r=r, T=T, alpha=16.0)
    As, Bs, alphas, idx = _stack(8, n, d, k, r, T)
    idx[::5] = -1
    qw = q4.qlora_nf4_quantize(f32_dev(lay.W0))
    Y, U = q4.qlora_fwd_multi(qw, bf16_dev(As.reshape(n * r, k)).view(n, r, k),
                              bf16_dev(Bs.reshape(n * d, r)).view(n, d, r), alphas,
                              torch.from_numpy(idx).cuda(), bf16_dev(lay.X))
    torch.cuda.synchronize()
    Wp = nf4.bf16_to_f64(nf4.dequantize(nf4.quantize(lay.W0)))
    none = np.where(idx < 0)[0]
    rows_within(bf16_host_f64(Y)[none], nf4.bf16_to_f64(lay.X)[none] @ Wp.T, what="Y base")
    assert torch.count_nonzero(U[torch.from_numpy(none).cuda()]).item() == 0
