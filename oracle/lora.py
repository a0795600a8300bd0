"""Oracle: the LoRA / QLoRA linear layer in float64.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__``).

Equations followed:
  * [P1] "How it works / The update LoRA is allowed to learn": h = W0 x + B A x
    with W0 d x k frozen, B d x r, A r x k; the product scaled by alpha / r;
    only A and B receive gradients.
  * [P2] "The LoRA hypothesis" figure: h = W0 x + (alpha/r) B A x.
  * [P1] "What QLoRA freezes, and in how many bits", forward equation:
    Y = X doubleDequant(c1, c2, W) + X L1 L2 (row-vector form, so L1 = A^T,
    L2 = B^T with the alpha/r scale s folded in); the activation gradient is
    also formed through the bf16-dequantised W.
  * [P5] "LoRA vs QLoRA: Parameter-Efficient Fine-Tuning Explained", run
    configuration: LoRA dropout (reading in the dropout section below).
  * [P2] "The LoRA hypothesis" and [P1] "What to choose and why": many
    unmerged adapters over one base (reading in the multi-adapter section).
  * [P1] deploy paragraph and [P2] "The LoRA hypothesis": W = W0 + (alpha/r) B A;
    switching tasks subtracts B A.  [P2] "What actually goes wrong": merge into
    the 16-bit base, keep the adapter separate (so the merged output is bf16
    and the NF4 base is kept).

Tokens are rows: X is T x k, Y is T x d.  All products are plain numpy
float64 matmuls of exactly-converted bf16 inputs; no blocking or fusion.
"""
from __future__ import annotations

from typing import Dict

import numpy as np

from .nf4 import bf16_to_f64, to_bf16_bits


def forward(X: np.ndarray, Wp: np.ndarray, A: np.ndarray, B: np.ndarray, s: float) -> Dict[str, np.ndarray]:
    """U = X A^T;  Y = X W'^T + s U B^T   (all float64 inputs)."""
    U = X @ A.T
    Y = X @ Wp.T + s * (U @ B.T)
    return {"U": U, "Y": Y}


def backward(X: np.ndarray, Wp: np.ndarray, A: np.ndarray, B: np.ndarray, s: float,
             dY: np.ndarray, U: np.ndarray = None) -> Dict[str, np.ndarray]:
    """Gradients of <dY, Y> w.r.t. X, A and B; none for W (frozen).

    G = dY B;  dX = dY W' + s G A;  dA = s G^T X;  dB = s dY^T U,  U = X A^T.
    """
    out = grad_input(Wp, A, B, s, dY)
    out.update(grad_adapters(X, A, B, s, dY, U))
    return out


def grad_input(Wp: np.ndarray, A: np.ndarray, B: np.ndarray, s: float, dY: np.ndarray) -> Dict[str, np.ndarray]:
    """dX = dY W' + s (dY B) A  (rows of dX depend only on the same rows of dY)."""
    G = dY @ B
    return {"G": G, "dX": dY @ Wp + s * (G @ A)}


def grad_adapters(X: np.ndarray, A: np.ndarray, B: np.ndarray, s: float, dY: np.ndarray,
                  U: np.ndarray = None) -> Dict[str, np.ndarray]:
    """dA = s (dY B)^T X;  dB = s dY^T (X A^T)."""
    if U is None:
        U = X @ A.T
    G = dY @ B
    return {"dA": s * (G.T @ X), "dB": s * (dY.T @ U)}


# ---------------------------------------------------------------------------
# LoRA dropout on the adapter input.  [P5] "LoRA vs QLoRA: Parameter-Efficient
# Fine-Tuning Explained", run configuration list: a LoRA dropout of 0.05-0.1
# is used for regularisation.  The pages give no formula; reading taken: the
# adapter path sees X dropped out element-wise with inverted scaling,
# D(X) = X * keep / (1 - p), keep a 0/1 mask drawn with probability 1 - p of a
# one, while the frozen path sees X itself.  The mask is an input here.
# ---------------------------------------------------------------------------
def dropout_input(X: np.ndarray, keep: np.ndarray, p: float) -> np.ndarray:
    """D(X) = X * keep / (1 - p)."""
    if not 0.0 <= p < 1.0:
        raise ValueError("dropout probability must be in [0, 1)")
    return X * keep / (1.0 - p)


def forward_dropout(X: np.ndarray, Wp: np.ndarray, A: np.ndarray, B: np.ndarray, s: float,
                    keep: np.ndarray, p: float) -> Dict[str, np.ndarray]:
    """U = D(X) A^T;  Y = X W'^T + s U B^T."""
    U = dropout_input(X, keep, p) @ A.T
    return {"U": U, "Y": X @ Wp.T + s * (U @ B.T)}


def backward_dropout(X: np.ndarray, Wp: np.ndarray, A: np.ndarray, B: np.ndarray, s: float,
                     dY: np.ndarray, keep: np.ndarray, p: float) -> Dict[str, np.ndarray]:
    """Gradients of <dY, Y> for forward_dropout:
    G = dY B;  dX = dY W' + D(s G A)  (the adapter term passes back through the
    same mask and scale);  dA = s G^T D(X);  dB = s dY^T (D(X) A^T)."""
    G = dY @ B
    Xd = dropout_input(X, keep, p)
    return {"G": G, "dX": dY @ Wp + dropout_input(s * (G @ A), keep, p),
            "dA": s * (G.T @ Xd), "dB": s * (dY.T @ (Xd @ A.T))}


# ---------------------------------------------------------------------------
# Several unmerged adapters over one frozen base in one batch.  [P2] "The LoRA
# hypothesis": serving many tasks keeps the adapters unmerged, one frozen base
# in memory with a stack of small adapters chosen per request; [P1] "What to
# choose and why": one deployed base, a small B A per task.  Reading taken:
# token t uses adapter idx[t] of a stack (A_i r x k, B_i d x r, scale s_i),
# the frozen path is shared.
# ---------------------------------------------------------------------------
def forward_multi(X: np.ndarray, Wp: np.ndarray, As: np.ndarray, Bs: np.ndarray, ss: np.ndarray,
                  idx: np.ndarray) -> Dict[str, np.ndarray]:
    """Y[t] = X[t] W'^T + s_i (X[t] A_i^T) B_i^T with i = idx[t]; U[t] = X[t] A_i^T.
    As: n x r x k, Bs: n x d x r, ss: n scales, idx: T adapter indices."""
    T = X.shape[0]
    U = np.zeros((T, As.shape[1]))
    Y = X @ Wp.T
    for t in range(T):
        i = int(idx[t])
        U[t] = As[i] @ X[t]
        Y[t] = Y[t] + ss[i] * (Bs[i] @ U[t])
    return {"U": U, "Y": Y}


def backward_multi(X: np.ndarray, Wp: np.ndarray, As: np.ndarray, Bs: np.ndarray, ss: np.ndarray,
                   idx: np.ndarray, dY: np.ndarray) -> Dict[str, np.ndarray]:
    """Gradients of <dY, Y> for forward_multi, token by token:
    G[t] = dY[t] B_i;  dX[t] = dY[t] W' + s_i G[t] A_i;
    dA_i = s_i sum over tokens of adapter i of G[t]^T X[t];
    dB_i = s_i sum over those tokens of dY[t]^T (X[t] A_i^T)."""
    dX = dY @ Wp
    dAs = np.zeros_like(As, dtype=np.float64)
    dBs = np.zeros_like(Bs, dtype=np.float64)
    for t in range(X.shape[0]):
        i = int(idx[t])
        G = dY[t] @ Bs[i]
        dX[t] = dX[t] + ss[i] * (G @ As[i])
        dAs[i] += ss[i] * np.outer(G, X[t])
        dBs[i] += ss[i] * np.outer(dY[t], As[i] @ X[t])
    return {"dX": dX, "dA": dAs, "dB": dBs}


def merge(Wp: np.ndarray, A: np.ndarray, B: np.ndarray, s: float) -> np.ndarray:
    """W = bf16(W' + s B A), computed in float64 and rounded once."""
    return to_bf16_bits(Wp + s * (B @ A))


def unmerge(W: np.ndarray, A: np.ndarray, B: np.ndarray, s: float) -> np.ndarray:
    """W0'' = bf16(W - s B A)."""
    return to_bf16_bits(W - s * (B @ A))


def as_f64(bits: np.ndarray) -> np.ndarray:
    return bf16_to_f64(bits)


# --------------------------------------------------------------------------
# Parameter-count arithmetic ([P1] "The update LoRA is allowed to learn";
# [P2] "The LoRA hypothesis")
# --------------------------------------------------------------------------
def adapter_params(d: int, k: int, r: int) -> int:
    """Trainable parameters of one adapted d x k matrix: B (d x r) + A (r x k)."""
    return d * r + r * k


def model_adapter_params(n_adapted: int, d_model: int, r: int) -> int:
    """2 * L_LoRA * d_model * r, attention projections treated as d_model x d_model."""
    return 2 * n_adapted * d_model * r


def algorithmic_flops(T: int, d: int, k: int, r: int) -> int:
    """fwd + bwd flops without any weight gradient: 4Tdk + 6Tr(d+k)."""
    return 4 * T * d * k + 6 * T * r * (d + k)
