"""Pins for the LoRA fwd/bwd/merge oracle: brute force on tiny shapes, finite
differences for the gradients, the B = 0 initialisation, merge/unmerge, and
the pages' parameter-count arithmetic."""
import json
import os

import numpy as np

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
