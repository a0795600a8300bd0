"""GPU parity of the QLoRA layer: forward, backward, merge and unmerge against
the float64 oracle on the same seeded inputs."""
import numpy as np
import pytest
import torch

import synthetic
from oracle import lora, nf4
from tests.gpu_helpers import (bf16_dev, bf16_host_bits, bf16_host_f64, f32_dev, f32_host_f64,
                               rows_within, within_one_bf16_ulp)

pytestmark = pytest.mark.gpu

q4 = pytest.importorskip("parameter_efficient_fine_nf4_b200")


_WP_CACHE = {}


def oracle_Wp(W0: np.ndarray) -> np.ndarray:
    """Oracle dequantised weight (float64), cached per seeded weight."""
    key = (W0.shape, W0[0, :16].tobytes(), W0[-1, -16:].tobytes())
    if key not in _WP_CACHE:
        if len(_WP_CACHE) > 3:
            _WP_CACHE.clear()
        qt = nf4.quantize(W0)
        _WP_CACHE[key] = nf4.bf16_to_f64(nf4.dequantize(qt))
    return _WP_CACHE[key]


class Case:
    """GPU run + oracle pieces for one layer."""

    def __init__(self, lay: synthetic.LayerInputs, alpha: float):
        self.lay = lay
        self.alpha = alpha
        self.s = alpha / lay.r
        self.qw = q4.qlora_nf4_quantize(f32_dev(lay.W0))
        self.A = bf16_dev(lay.A)
        self.B = bf16_dev(lay.B)
        self.X = bf16_dev(lay.X)
        self.dY = bf16_dev(lay.dY)
        self.Y, self.U = q4.qlora_fwd(self.qw, self.A, self.B, alpha, self.X)
        self.dX, self.dA, self.dB = q4.qlora_bwd(self.qw, self.A, self.B, alpha, self.X, self.U, self.dY)
        torch.cuda.synchronize()
        assert q4.qlora_get_device_status() == 0

    def oracle_Wp(self):
        return oracle_Wp(self.lay.W0)

    def check(self, rows=None, full_adapter_grads=True):
        lay = self.lay
        Wp = self.oracle_Wp()
        X = nf4.bf16_to_f64(lay.X)
        A = nf4.bf16_to_f64(lay.A)
        B = nf4.bf16_to_f64(lay.B)
        dY = nf4.bf16_to_f64(lay.dY)
        if rows is None:
            rows = np.arange(lay.T)
        fw = lora.forward(X[rows], Wp, A, B, self.s)
        rows_within(bf16_host_f64(self.Y)[rows], fw["Y"], what="Y")
        rows_within(f32_host_f64(self.U)[rows], fw["U"], what="U")
        gi = lora.grad_input(Wp, A, B, self.s, dY[rows])
        rows_within(bf16_host_f64(self.dX)[rows], gi["dX"], what="dX")
        if full_adapter_grads:
            ga = lora.grad_adapters(X, A, B, self.s, dY)
            rows_within(f32_host_f64(self.dA), ga["dA"], what="dA")
            rows_within(f32_host_f64(self.dB), ga["dB"], what="dB")
        return Wp


def test_config1_full():
    cfg = synthetic.config(1)
    Case(synthetic.make_layer(cfg), cfg.alpha).check()


def test_config1_b_zero_init():
    # B = 0 at initialisation: the adapter adds nothing, dA is exactly zero
    cfg = synthetic.config(1)
    c = Case(synthetic.make_layer(cfg, zero_b=True), cfg.alpha)
    Wp = c.check()
    assert torch.count_nonzero(c.dA).item() == 0
    X = nf4.bf16_to_f64(c.lay.X)
    rows_within(bf16_host_f64(c.Y), X @ Wp.T, what="Y base")


@pytest.mark.parametrize("T", [16, 300])
def test_b_zero_adds_exactly_nothing(T):
    # [P1] "The update LoRA is allowed to learn": with B = 0 the adapted layer
    # is the base layer.  On the GPU the rank-r term then adds +0 to every
    # fp32 accumulator, so Y and dX are bit-identical whatever A holds (A = 0
    # as well), and dA is exactly zero.
    cfg = synthetic.config(1)
    lay = synthetic.make_layer(cfg, T=T, zero_b=True)
    qw = q4.qlora_nf4_quantize(f32_dev(lay.W0))
    A, B, X, dY = bf16_dev(lay.A), bf16_dev(lay.B), bf16_dev(lay.X), bf16_dev(lay.dY)
    A0 = torch.zeros_like(A)
    Y, U = q4.qlora_fwd(qw, A, B, cfg.alpha, X)
    dX, dA, dB = q4.qlora_bwd(qw, A, B, cfg.alpha, X, U, dY)
    Y0, U0 = q4.qlora_fwd(qw, A0, B, cfg.alpha, X)
    dX0, dA0, dB0 = q4.qlora_bwd(qw, A0, B, cfg.alpha, X, U0, dY)
    torch.cuda.synchronize()
    assert torch.equal(Y, Y0) and torch.equal(dX, dX0)
    assert torch.count_nonzero(dA).item() == 0 and torch.count_nonzero(dA0).item() == 0
    assert torch.count_nonzero(U0).item() == 0 and torch.count_nonzero(dB0).item() == 0
    # and the base product alone is what the oracle gives
    Wp = oracle_Wp(lay.W0)
    rows_within(bf16_host_f64(Y), nf4.bf16_to_f64(lay.X) @ Wp.T, what="Y base")
    rows_within(bf16_host_f64(dX), nf4.bf16_to_f64(lay.dY) @ Wp, what="dX base")


@pytest.mark.parametrize("d,k,r,T", [
    (320, 192, 5, 200),      # ragged M and N tiles, r not a multiple of 8
    (64, 64, 1, 1),          # one token, rank 1
    (136, 128, 3, 129),      # d just past a tile, T just past a tile
    (256, 512, 100, 300),    # r > 64: two extension steps on a 128-wide N tile
    (384, 256, 256, 64),     # maximum rank
    (200, 64, 16, 1000),     # K = 64: one main step
])
def test_ragged_shapes(d, k, r, T):
    lay = synthetic.custom_layer(seed=d * 131 + k * 7 + r + T, d=d, k=k, r=r, T=T, alpha=2.0 * r)
    Case(lay, 2.0 * r).check()


def test_forward_any_d_backward_needs_d_multiple_of_8():
    # forward accepts any d; backward needs 16-byte aligned rows of dY
    lay = synthetic.custom_layer(seed=9, d=130, k=128, r=3, T=40, alpha=6.0)
    qw = q4.qlora_nf4_quantize(f32_dev(lay.W0))
    A, B, X, dY = bf16_dev(lay.A), bf16_dev(lay.B), bf16_dev(lay.X), bf16_dev(lay.dY)
    Y, U = q4.qlora_fwd(qw, A, B, 6.0, X)
    torch.cuda.synchronize()
    Wp = oracle_Wp(lay.W0)
    fw = lora.forward(nf4.bf16_to_f64(lay.X), Wp, nf4.bf16_to_f64(lay.A), nf4.bf16_to_f64(lay.B), 2.0)
    rows_within(bf16_host_f64(Y), fw["Y"], what="Y")
    with pytest.raises(q4.QloraError) as e:
        q4.qlora_bwd(qw, A, B, 6.0, X, U, dY)
    assert e.value.status == 2


@pytest.mark.parametrize("ci", [2, 3])
def test_configs_sampled_rows(ci):
    cfg = synthetic.config(ci)
    lay = synthetic.make_layer(cfg)
    rows = synthetic.sample_rows(77 + ci, lay.T, 192)
    Case(lay, cfg.alpha).check(rows=rows)


@pytest.mark.parametrize("li", [0, 1])
def test_config4_sampled_rows(li):
    cfg = synthetic.config(4)
    lay = synthetic.make_layer(cfg, li)
    rows = synthetic.sample_rows(401 + li, lay.T, 64)
    Case(lay, cfg.alpha).check(rows=rows)


@pytest.mark.parametrize("li", range(7))
@pytest.mark.parametrize("T", [16, 4096])
def test_config5_linears(li, T):
    cfg = synthetic.config(5)
    lay = synthetic.make_layer(cfg, li, T=T)
    rows = None if T == 16 else synthetic.sample_rows(500 + li, T, 64)
    Case(lay, cfg.alpha).check(rows=rows, full_adapter_grads=(li in (0, 4, 6)))


def test_bwd_deterministic_and_zero_tokens():
    cfg = synthetic.config(2)
    lay = synthetic.make_layer(cfg)
    c = Case(lay, cfg.alpha)
    dX2, dA2, dB2 = q4.qlora_bwd(c.qw, c.A, c.B, cfg.alpha, c.X, c.U, c.dY)
    torch.cuda.synchronize()
    assert torch.equal(dA2, c.dA) and torch.equal(dB2, c.dB) and torch.equal(dX2, c.dX)
    # T = 0: nothing to do, adapter gradients are overwritten with zeros
    X0 = c.X[:0]
    dA = torch.full_like(c.dA, 7.0)
    dB = torch.full_like(c.dB, 7.0)
    q4.qlora_bwd(c.qw, c.A, c.B, cfg.alpha, X0, c.U[:0], c.dY[:0], dA=dA, dB=dB)
    torch.cuda.synchronize()
    assert torch.count_nonzero(dA).item() == 0 and torch.count_nonzero(dB).item() == 0


@pytest.mark.parametrize("ci", [1, 3])
def test_merge_unmerge(ci):
    cfg = synthetic.config(ci)
    lay = synthetic.make_layer(cfg, with_acts=False)
    s = cfg.s
    qw = q4.qlora_nf4_quantize(f32_dev(lay.W0))
    A, B = bf16_dev(lay.A), bf16_dev(lay.B)
    W = q4.lora_merge(qw, A, B, cfg.alpha)
    torch.cuda.synchronize()
    qt = nf4.quantize(lay.W0)
    Wp = nf4.bf16_to_f64(nf4.dequantize(qt))
    Af, Bf = nf4.bf16_to_f64(lay.A), nf4.bf16_to_f64(lay.B)
    ref_W = lora.merge(Wp, Af, Bf, s)
    # fp32 error bound of the GPU's r-term product (accumulated on the tensor
    # core) and of the fused multiply-add, before the single bf16 rounding:
    # r * 2^-22 * s * sum_q |B_iq A_qj|  +  2^-23 * |W'_ij|
    extra = cfg.r * 2.0 ** -22 * s * (np.abs(Bf) @ np.abs(Af)) + 2.0 ** -23 * np.abs(Wp)
    within_one_bf16_ulp(bf16_host_bits(W), ref_W, "merge", abs_extra=extra)
    # unmerge of the oracle's merged weight
    W_in = bf16_dev(ref_W)
    W0pp = q4.lora_unmerge(W_in, A, B, cfg.alpha)
    torch.cuda.synchronize()
    ref_W0pp = lora.unmerge(nf4.bf16_to_f64(ref_W), Af, Bf, s)
    within_one_bf16_ulp(bf16_host_bits(W0pp), ref_W0pp, "unmerge", abs_extra=extra)
    # merge then unmerge on the GPU gives back the dequantised base (1 ulp),
    # and with B = 0 both are exactly the dequantised base
    back = q4.lora_unmerge(W, A, B, cfg.alpha)
    Wdq = q4.qlora_nf4_dequantize(qw)
    Z = torch.zeros_like(B)
    Wz = q4.lora_merge(qw, A, Z, cfg.alpha)
    Wz2 = q4.lora_unmerge(Wdq, A, Z, cfg.alpha)
    torch.cuda.synchronize()
    # two roundings (merge, then unmerge), each at most half an ulp of the
    # larger of the merged W and the result
    W_mag = bf16_host_f64(W)
    within_one_bf16_ulp(bf16_host_bits(back), nf4.dequantize(qt), "merge-unmerge", ulps=1,
                        abs_extra=2 * extra, mag_extra=W_mag)
    # the round trip re-encodes to the stored codes with the stored block scales
    a2 = nf4.block_scale(qt["absmax_q"], qt["scale2"], qt["mean"]).astype(np.float64)
    q = nf4.nf4_levels().astype(np.float64)
    x = bf16_host_f64(back).reshape(-1, 64) / a2[:, None]
    codes = np.abs(x[..., None] - q).argmin(-1).ravel().astype(np.uint8)
    assert np.array_equal(codes, nf4.unpack_codes(qt["codes"]))
    assert torch.equal(Wz, Wdq) and torch.equal(Wz2, Wdq)
    assert q4.qlora_get_device_status() == 0


@pytest.mark.parametrize("d,k,r", [
    (300, 320, 5),       # ragged tiles in both directions, r not a multiple of 8
    (128, 256, 64),      # exactly one tile
    (200, 576, 100),     # two K-steps of the rank-r product
    (136, 192, 200),     # r > 128
    (1, 64, 1),          # one row
])
def test_merge_unmerge_ragged(d, k, r):
    lay = synthetic.custom_layer(seed=d * 7 + k + r, d=d, k=k, r=r, T=1, alpha=2.0 * r)
    alpha = 2.0 * r
    s = alpha / r
    qw = q4.qlora_nf4_quantize(f32_dev(lay.W0))
    A, B = bf16_dev(lay.A), bf16_dev(lay.B)
    W = q4.lora_merge(qw, A, B, alpha)
    torch.cuda.synchronize()
    Wp = oracle_Wp(lay.W0)
    Af, Bf = nf4.bf16_to_f64(lay.A), nf4.bf16_to_f64(lay.B)
    ref_W = lora.merge(Wp, Af, Bf, s)
    extra = r * 2.0 ** -22 * s * (np.abs(Bf) @ np.abs(Af)) + 2.0 ** -23 * np.abs(Wp)
    within_one_bf16_ulp(bf16_host_bits(W), ref_W, "merge", abs_extra=extra)
    W0pp = q4.lora_unmerge(bf16_dev(ref_W), A, B, alpha)
    torch.cuda.synchronize()
    ref_W0pp = lora.unmerge(nf4.bf16_to_f64(ref_W), Af, Bf, s)
    within_one_bf16_ulp(bf16_host_bits(W0pp), ref_W0pp, "unmerge", abs_extra=extra)
    assert q4.qlora_get_device_status() == 0


def test_merged_layer_matches_unmerged_forward():
    cfg = synthetic.config(1)
    lay = synthetic.make_layer(cfg)
    c = Case(lay, cfg.alpha)
    W = q4.lora_merge(c.qw, c.A, c.B, cfg.alpha)
    Y_merged = (c.X.float() @ W.float().T)
    torch.cuda.synchronize()
    rows_within(Y_merged.double().cpu().numpy(), bf16_host_f64(c.Y).astype(np.float64), what="merged")


def test_merge_unmerge_full_size_sampled_rows():
    # the merge the benchmark times: 22016 x 8192, r = 64.  The oracle's own
    # storage for the sampled rows (constants and mean from every block,
    # codes of the sampled rows), merged in float64; the GPU unmerge is fed
    # the oracle's merged rows at those positions.
    cfg = synthetic.config(4)
    lay = synthetic.make_layer(cfg, 0, with_acts=False)
    d, k, r, s = lay.d, lay.k, lay.r, cfg.s
    qw = q4.qlora_nf4_quantize(f32_dev(lay.W0))
    A, B = bf16_dev(lay.A), bf16_dev(lay.B)
    W = q4.lora_merge(qw, A, B, cfg.alpha)
    torch.cuda.synchronize()
    assert q4.qlora_get_device_status() == 0
    rows = synthetic.sample_rows(4040, d, 48)
    kb = k // 64
    blocks = (rows[:, None] * kb + np.arange(kb)[None, :]).ravel()
    a = nf4.block_absmax(lay.W0)
    mu = nf4.block_mean(a)
    c2, s1 = nf4.double_quant(a, mu)
    packed = np.zeros(d * k // 2, np.uint8)
    packed.reshape(-1, 32)[blocks] = nf4.pack_codes(
        nf4.encode_blocks(lay.W0.reshape(-1, 64)[blocks], a[blocks]).ravel()).reshape(-1, 32)
    Wp_rows = nf4.bf16_to_f64(nf4.dequantize_blocks(packed, c2, s1, mu, blocks)).reshape(rows.size, k)
    Af = nf4.bf16_to_f64(lay.A)
    Bf = nf4.bf16_to_f64(lay.B)[rows]
    ref = lora.merge(Wp_rows, Af, Bf, s)
    extra = r * 2.0 ** -22 * s * (np.abs(Bf) @ np.abs(Af)) + 2.0 ** -23 * np.abs(Wp_rows)
    within_one_bf16_ulp(bf16_host_bits(W)[rows], ref, "merge 22016x8192", abs_extra=extra)
    W_in = W.clone()
    W_in[torch.from_numpy(rows).cuda()] = bf16_dev(ref)
    W0pp = q4.lora_unmerge(W_in, A, B, cfg.alpha)
    torch.cuda.synchronize()
    ref_back = lora.unmerge(nf4.bf16_to_f64(ref), Af, Bf, s)
    within_one_bf16_ulp(bf16_host_bits(W0pp)[rows], ref_back, "unmerge 22016x8192", abs_extra=extra)
    assert q4.qlora_get_device_status() == 0
