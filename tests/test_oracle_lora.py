"""Pins for the LoRA fwd/bwd/merge oracle: brute force on tiny shapes, finite
differences for the gradients, the B = 0 initialisation, merge/unmerge, and
the pages' parameter-count arithmetic."""
import json
import os

import numpy as np
import pytest

from oracle import lora, nf4
import synthetic


def _tiny(seed, d, k, r, T, zero_b=False):
    lay = synthetic.custom_layer(seed, d, k, r, T, alpha=2.0 * r, zero_b=zero_b)
    qt = nf4.quantize(lay.W0)
    Wp = nf4.bf16_to_f64(nf4.dequantize(qt))
    X = nf4.bf16_to_f64(lay.X)
    A = nf4.bf16_to_f64(lay.A)
    B = nf4.bf16_to_f64(lay.B)
    dY = nf4.bf16_to_f64(lay.dY)
    return lay, Wp, X, A, B, dY


def test_forward_bruteforce_loops():
    for r in (1, 2, 3, 4):
        lay, Wp, X, A, B, dY = _tiny(100 + r, d=64, k=64, r=r, T=2)
        s = lay.s
        out = lora.forward(X, Wp, A, B, s)
        T, k = X.shape
        d = Wp.shape[0]
        for t in range(T):
            for i in range(0, d, 5):
                base = 0.0
                for j in range(k):
                    base += Wp[i, j] * X[t, j]
                ba = 0.0
                for q in range(r):
                    ax = 0.0
                    for j in range(k):
                        ax += A[q, j] * X[t, j]
                    ba += B[i, q] * ax
                h = base + s * ba                  # h = W0 x + (alpha/r) B A x
                assert abs(out["Y"][t, i] - h) <= 1e-12 * (1 + abs(h))


def _loss(Y, dY):
    return float(np.sum(Y * dY))


def test_gradients_by_central_differences():
    # L = <dY, Y> is linear in X, in A and in B separately, so a central
    # difference equals the gradient up to float64 rounding.  This pins dX,
    # dA and dB without using the backward formulas.
    lay, Wp, X, A, B, dY = _tiny(7, d=64, k=128, r=4, T=3)
    s = lay.s
    g = lora.backward(X, Wp, A, B, s, dY)
    rng = np.random.Generator(np.random.Philox(key=99))
    h = 0.5
    for name, arr, grad in (("X", X, g["dX"]), ("A", A, g["dA"]), ("B", B, g["dB"])):
        for _ in range(25):
            idx = tuple(rng.integers(0, n) for n in arr.shape)
            p = arr.copy(); p[idx] += h
            m = arr.copy(); m[idx] -= h
            args = {"X": X, "A": A, "B": B}
            args[name] = p
            lp = _loss(lora.forward(args["X"], Wp, args["A"], args["B"], s)["Y"], dY)
            args[name] = m
            lm = _loss(lora.forward(args["X"], Wp, args["A"], args["B"], s)["Y"], dY)
            fd = (lp - lm) / (2 * h)
            assert abs(fd - grad[idx]) <= 1e-9 * (1 + abs(fd)), (name, idx)


def test_no_weight_gradient_and_b_zero_init():
    # B = 0 at initialisation: BA = 0, the output equals the base output
    # exactly, and A receives a zero gradient.
    lay, Wp, X, A, B, dY = _tiny(21, d=128, k=64, r=8, T=5, zero_b=True)
    out = lora.forward(X, Wp, A, B, lay.s)
    assert np.array_equal(out["Y"], X @ Wp.T)
    g = lora.backward(X, Wp, A, B, lay.s, dY)
    assert np.all(g["dA"] == 0)
    assert np.array_equal(g["dX"], dY @ Wp)
    assert set(g) == {"G", "dX", "dA", "dB"}                 # no dW is ever formed


def test_merge_then_unmerge_recovers_base():
    lay, Wp, X, A, B, dY = _tiny(33, d=128, k=128, r=8, T=4)
    s = lay.s
    Wm_bits = lora.merge(Wp, A, B, s)
    Wm = nf4.bf16_to_f64(Wm_bits)
    W0pp = nf4.bf16_to_f64(lora.unmerge(Wm, A, B, s))
    ulp = np.spacing(np.maximum(np.abs(Wm), np.abs(Wp)).astype(np.float32)).astype(np.float64) * 2 ** 16
    assert np.all(np.abs(W0pp - Wp) <= ulp)
    # the merged layer computes the same function up to bf16 rounding
    Y_merged = X @ Wm.T
    Y = lora.forward(X, Wp, A, B, s)["Y"]
    assert np.max(np.abs(Y_merged - Y)) <= 2e-2 * np.max(np.abs(Y))
    # B = 0: merge and unmerge are the identity on W'
    Z = np.zeros_like(B)
    Wp_bits = nf4.to_bf16_bits(Wp)
    assert np.array_equal(lora.merge(Wp, A, Z, s), Wp_bits)
    assert np.array_equal(lora.unmerge(Wp, A, Z, s), Wp_bits)


def test_parameter_counts_match_pages(golden_dir):
    g = json.load(open(os.path.join(golden_dir, "pages_numbers.json")))
    e = g["rank8_adapter_on_4096x4096"]
    n = lora.adapter_params(4096, 4096, 8)
    assert n == e["value"]
    assert round(4096 * 4096 / 1e6, 1) == e["matrix_params_millions"]
    assert round(100 * n / (4096 * 4096), 1) == e["fraction_percent_approx"]
    gp = g["gpt3_trainable_reduction"]
    trainable = lora.model_adapter_params(gp["n_layers"] * gp["matrices_per_layer"],
                                          gp["d_model"], gp["r"])
    ratio = gp["model_params"] / trainable
    assert 8000 < ratio < 12000                      # "about 10,000 times"
    mb = trainable * 2 / 1e6                           # 16-bit adapter file
    assert abs(mb - g["gpt3_checkpoint_MB_approx"]["value"]) < 5
    h = g["hundred_tasks_GB_approx"]
    assert round(h["base_GB"] + h["tasks"] * h["adapter_MB"] / 1e3) == h["value"]


def test_flop_formula():
    # 4Tdk + 6Tr(d+k): fwd base + dX base, plus six rank-r products
    T, d, k, r = 16384, 22016, 8192, 64
    assert lora.algorithmic_flops(T, d, k, r) == 4 * T * d * k + 6 * T * r * (d + k)
    assert round(lora.algorithmic_flops(T, d, k, r) / 1e8) == 120098   # 1.20098e13


# ---------------------------------------------------------------------------
# LoRA dropout (mask passed in): pins by special case, linearity and a
# directional derivative
# ---------------------------------------------------------------------------
def _small(seed=3, T=24, d=20, k=16, r=4):
    rng = np.random.default_rng(seed)
    X = rng.standard_normal((T, k))
    Wp = rng.standard_normal((d, k)) * 0.1
    A = rng.standard_normal((r, k)) * 0.3
    B = rng.standard_normal((d, r)) * 0.2
    dY = rng.standard_normal((T, d))
    keep = (rng.random((T, k)) < 0.5).astype(np.float64)
    return X, Wp, A, B, dY, keep


def test_dropout_zero_is_plain_lora():
    X, Wp, A, B, dY, _ = _small()
    ones = np.ones_like(X)
    f0, f1 = lora.forward(X, Wp, A, B, 0.5), lora.forward_dropout(X, Wp, A, B, 0.5, ones, 0.0)
    np.testing.assert_array_equal(f0["Y"], f1["Y"])
    b0, b1 = lora.backward(X, Wp, A, B, 0.5, dY), lora.backward_dropout(X, Wp, A, B, 0.5, dY, ones, 0.0)
    for key in ("dX", "dA", "dB"):
        np.testing.assert_allclose(b0[key], b1[key], rtol=1e-14, atol=1e-14)


def test_complementary_masks_add_up_to_twice_the_undropped_adapter():
    # p = 1/2: D_M(X) + D_{1-M}(X) = 2 X, and everything adapter-side is linear in D(X)
    X, Wp, A, B, dY, keep = _small()
    s = 0.75
    a = lora.forward_dropout(X, Wp, A, B, s, keep, 0.5)
    b = lora.forward_dropout(X, Wp, A, B, s, 1.0 - keep, 0.5)
    base = X @ Wp.T
    full = lora.forward(X, Wp, A, B, s)
    np.testing.assert_allclose((a["Y"] - base) + (b["Y"] - base), 2 * (full["Y"] - base), rtol=1e-12, atol=1e-12)
    ga = lora.backward_dropout(X, Wp, A, B, s, dY, keep, 0.5)
    gb = lora.backward_dropout(X, Wp, A, B, s, dY, 1.0 - keep, 0.5)
    gf = lora.backward(X, Wp, A, B, s, dY)
    for key in ("dA", "dB"):
        np.testing.assert_allclose(ga[key] + gb[key], 2 * gf[key], rtol=1e-12, atol=1e-12)
    base_dx = dY @ Wp
    np.testing.assert_allclose((ga["dX"] - base_dx) + (gb["dX"] - base_dx), 2 * (gf["dX"] - base_dx),
                               rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("wrt", ["X", "A", "B"])
def test_dropout_gradients_match_directional_derivatives(wrt):
    # L = <dY, Y> is linear in X and bilinear in (A, B): the central difference is exact
    # up to rounding for any step, so every mask and scale has to be in the right place
    X, Wp, A, B, dY, keep = _small(seed=9)
    s, p = 0.6, 0.1
    args = {"X": X, "A": A, "B": B}
    E = np.random.default_rng(1).standard_normal(args[wrt].shape)

    def loss(v):
        a = dict(args, **{wrt: v})
        return np.sum(dY * lora.forward_dropout(a["X"], Wp, a["A"], a["B"], s, keep, p)["Y"])

    h = 1e-3
    num = (loss(args[wrt] + h * E) - loss(args[wrt] - h * E)) / (2 * h)
    g = lora.backward_dropout(X, Wp, A, B, s, dY, keep, p)["d" + wrt]
    assert abs(num - np.sum(g * E)) <= 1e-8 * (1 + abs(num))


def test_dropout_rejects_p_one():
    X, Wp, A, B, dY, keep = _small()
    with pytest.raises(ValueError):
        lora.forward_dropout(X, Wp, A, B, 1.0, keep, 1.0)


# ---------------------------------------------------------------------------
# Several unmerged adapters in one batch: pins by reduction to the single-
# adapter routines (pinned above), permutation and directional derivatives
# ---------------------------------------------------------------------------
def _multi(seed=4, T=30, d=18, k=12, r=3, n=3):
    rng = np.random.default_rng(seed)
    X = rng.standard_normal((T, k))
    Wp = rng.standard_normal((d, k)) * 0.1
    As = rng.standard_normal((n, r, k)) * 0.3
    Bs = rng.standard_normal((n, d, r)) * 0.2
    ss = np.array([0.5, 2.0, 1.25])[:n]
    idx = rng.integers(0, n, T)
    dY = rng.standard_normal((T, d))
    return X, Wp, As, Bs, ss, idx, dY


def test_multi_with_one_adapter_is_plain_lora():
    X, Wp, As, Bs, ss, _, dY = _multi()
    idx = np.zeros(X.shape[0], int)
    f = lora.forward_multi(X, Wp, As, Bs, ss, idx)
    f1 = lora.forward(X, Wp, As[0], Bs[0], ss[0])
    np.testing.assert_allclose(f["Y"], f1["Y"], rtol=1e-13, atol=1e-13)
    b = lora.backward_multi(X, Wp, As, Bs, ss, idx, dY)
    b1 = lora.backward(X, Wp, As[0], Bs[0], ss[0], dY)
    for key in ("dX", "dA", "dB"):
        got = b[key] if key == "dX" else b[key][0]
        np.testing.assert_allclose(got, b1[key], rtol=1e-12, atol=1e-12)
    assert np.all(b["dA"][1:] == 0) and np.all(b["dB"][1:] == 0)


def test_multi_equals_separate_runs_per_adapter():
    X, Wp, As, Bs, ss, idx, dY = _multi()
    f = lora.forward_multi(X, Wp, As, Bs, ss, idx)
    b = lora.backward_multi(X, Wp, As, Bs, ss, idx, dY)
    for i in range(As.shape[0]):
        rows = np.nonzero(idx == i)[0]
        fi = lora.forward(X[rows], Wp, As[i], Bs[i], ss[i])
        np.testing.assert_allclose(f["Y"][rows], fi["Y"], rtol=1e-12, atol=1e-12)
        gi = lora.backward(X[rows], Wp, As[i], Bs[i], ss[i], dY[rows])
        np.testing.assert_allclose(b["dX"][rows], gi["dX"], rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(b["dA"][i], gi["dA"], rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(b["dB"][i], gi["dB"], rtol=1e-12, atol=1e-12)


def test_multi_is_invariant_to_token_order():
    X, Wp, As, Bs, ss, idx, dY = _multi(seed=8)
    perm = np.random.default_rng(2).permutation(X.shape[0])
    a = lora.backward_multi(X, Wp, As, Bs, ss, idx, dY)
    b = lora.backward_multi(X[perm], Wp, As, Bs, ss, idx[perm], dY[perm])
    np.testing.assert_allclose(a["dX"][perm], b["dX"], rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(a["dA"], b["dA"], rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(a["dB"], b["dB"], rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("wrt", ["X", "As", "Bs"])
def test_multi_gradients_match_directional_derivatives(wrt):
    X, Wp, As, Bs, ss, idx, dY = _multi(seed=12)
    args = {"X": X, "As": As, "Bs": Bs}
    E = np.random.default_rng(5).standard_normal(args[wrt].shape)

    def loss(v):
        a = dict(args, **{wrt: v})
        return np.sum(dY * lora.forward_multi(a["X"], Wp, a["As"], a["Bs"], ss, idx)["Y"])

    h = 1e-3
    num = (loss(args[wrt] + h * E) - loss(args[wrt] - h * E)) / (2 * h)
    g = lora.backward_multi(X, Wp, As, Bs, ss, idx, dY)[{"X": "dX", "As": "dA", "Bs": "dB"}[wrt]]
    assert abs(num - np.sum(g * E)) <= 1e-8 * (1 + abs(num))
