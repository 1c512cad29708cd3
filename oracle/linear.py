"""QLoRA linear layer forward and backward in float64.

TEST INFRASTRUCTURE ONLY. Source: "QLoRA: Efficient Finetuning of Quantized LLMs"
(Heng's Blog), opening formula h = dequant(W0^NF4) x + (alpha/r) B A x: the frozen
4-bit base is dequantized to BFloat16 on use, and only the adapters A and B receive
gradients (the base stays frozen, so there is no gradient for W0).

Layouts (row-major): W_hat [N, K], x [M, K], A [r, K], B [N, r], h [M, N].
The dequantized base enters the products as bf16 values (W_hat rounded to nearest
even); everything else is exact float64 matrix algebra.
"""
from __future__ import annotations

import numpy as np

from .numerics import round_bf16


def base_bf16(w_hat: np.ndarray) -> np.ndarray:
    """The dequantized fp32 base weight rounded to bf16, as float64."""
    return round_bf16(np.asarray(w_hat, dtype=np.float32)).astype(np.float64)


def forward(x, w_bf16, A, B, scale: float) -> np.ndarray:
    """h = x W^T + scale * (x A^T) B^T, float64."""
    x = np.asarray(x, np.float64)
    W = np.asarray(w_bf16, np.float64)
    A = np.asarray(A, np.float64)
    B = np.asarray(B, np.float64)
    u = x @ A.T
    return x @ W.T + float(scale) * (u @ B.T)


def backward(x, dY, w_bf16, A, B, scale: float):
    """Gradients of the forward above for an upstream gradient dY [M, N].

    v  = dY B                      [M, r]
    dX = dY W + scale * v A        [M, K]
    dA = scale * v^T x             [r, K]
    dB = scale * dY^T (x A^T)      [N, r]
    """
    x = np.asarray(x, np.float64)
    dY = np.asarray(dY, np.float64)
    W = np.asarray(w_bf16, np.float64)
    A = np.asarray(A, np.float64)
    B = np.asarray(B, np.float64)
    s = float(scale)
    v = dY @ B
    u = x @ A.T
    dX = dY @ W + s * (v @ A)
    dA = s * (v.T @ x)
    dB = s * (dY.T @ u)
    return dX, dA, dB


def lora_u(x, A) -> np.ndarray:
    """u = x A^T in float64 (the adapter's down-projection)."""
    return np.asarray(x, np.float64) @ np.asarray(A, np.float64).T


def close(got, ref, max_rel: float = 2e-2, fro_rel: float = 5e-3):
    """The GEMM tolerance: max|err| <= max_rel * max|ref| and
    ||err||_F <= fro_rel * ||ref||_F. Returns (ok, max_err/max_ref, fro_err/fro_ref)."""
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    err = got - ref
    mref = float(np.max(np.abs(ref))) if ref.size else 0.0
    fref = float(np.linalg.norm(ref)) if ref.size else 0.0
    merr = float(np.max(np.abs(err))) if err.size else 0.0
    ferr = float(np.linalg.norm(err)) if err.size else 0.0
    a = merr / mref if mref > 0 else merr
    b = ferr / fref if fref > 0 else ferr
    return (a <= max_rel and b <= fro_rel), a, b
