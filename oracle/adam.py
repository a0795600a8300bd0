"""Oracle: one Adam step on the adapter factors, in float64.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__``).

What the pages fix:
  * [P1] "The update LoRA is allowed to learn": Adam keeps state per trainable
    parameter; frozen weights have neither gradient nor optimiser state, so
    only A and B carry it.
  * [P2] "Why full fine-tuning costs so much": mixed-precision Adam keeps a
    16-bit weight for the forward pass, a 32-bit master copy of it and two
    32-bit moment estimates m and v per parameter.
  * [P2] "The LoRA hypothesis": Adam only tracks moments for A and B.
The pages do not print the update rule.  Reading taken (the plainest one):
the bias-corrected Adam of Kingma and Ba ("Adam: A Method for Stochastic
Optimization", 2015, Algorithm 1), with optional decoupled weight decay
(Loshchilov and Hutter, "Decoupled Weight Decay Regularization", 2019),
applied to the fp32 master copy; the 16-bit copy is the master rounded to
bf16.  Step t counts from 1.
"""
from __future__ import annotations

from typing import Dict

import numpy as np

from .nf4 import to_bf16_bits


def adam_step(theta: np.ndarray, m: np.ndarray, v: np.ndarray, g: np.ndarray, t: int,
              lr: float, beta1: float = 0.9, beta2: float = 0.999, eps: float = 1e-8,
              weight_decay: float = 0.0) -> Dict[str, np.ndarray]:
    """One step, all in float64:
        m_t     = beta1 m + (1 - beta1) g
        v_t     = beta2 v + (1 - beta2) g^2
        m_hat   = m_t / (1 - beta1^t),  v_hat = v_t / (1 - beta2^t)
        theta_t = theta - lr (m_hat / (sqrt(v_hat) + eps) + weight_decay theta)
    Returns theta, m, v (float64) and theta_bf16 (bf16 bits of theta_t)."""
    if t < 1:
        raise ValueError("Adam steps count from 1")
    theta = np.asarray(theta, np.float64)
    m = np.asarray(m, np.float64)
    v = np.asarray(v, np.float64)
    g = np.asarray(g, np.float64)
    m_t = beta1 * m + (1.0 - beta1) * g
    v_t = beta2 * v + (1.0 - beta2) * g * g
    m_hat = m_t / (1.0 - beta1 ** t)
    v_hat = v_t / (1.0 - beta2 ** t)
    theta_t = theta - lr * (m_hat / (np.sqrt(v_hat) + eps) + weight_decay * theta)
    return {"theta": theta_t, "m": m_t, "v": v_t, "theta_bf16": to_bf16_bits(theta_t)}


def optimizer_state_bytes(n_params: int) -> int:
    """Bytes of mixed-precision Adam state per [P2]: fp32 master + m + v (4 B each)
    and the 16-bit forward copy (2 B); the gradient adds 4 B while it lives."""
    return n_params * (4 + 4 + 4 + 2)
