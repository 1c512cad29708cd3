"""LoftQ-style low-rank initialisation over an NF4-quantized base.

TEST INFRASTRUCTURE ONLY (see the package docstring). Source: "LowRA" article
(cloud.tencent.com.cn): its workflow quantizes each layer, computes the quantization error
and applies a low-rank initialiser, LoftQ, which it chooses over PiSSA because quantizing
first and then taking the SVD lets the low-rank tensors absorb the quantization error; it
follows LoftQ's recommendation of five alternating steps. The quantizer here is the NF4
path of "QLoRA: Efficient Finetuning of Quantized LLMs" (贡献一 NF4, 贡献二 Double
Quantization), whose adapters are B [N, r] and A [r, K] with W ~ dequant(Q) + B A.

The alternating steps, as the page's description reads plainly (A = 0, B = 0 at the start):
  1. Q_t = dequant(quantize(bf16(W - B A)))    NF4 + double quantization, as a2-a6;
  2. R_t = W - Q_t, and its best rank-r approximation U_r S_r V_r^T (a truncated SVD,
     the library primitive here, np.linalg.svd);
  3. B = U_r S_r^(1/2), A = S_r^(1/2) V_r^T.
The objective after step t is e_t = ||W - Q_t - B A||_F^2 = sum_{i > r} s_i^2 (Eckart-Young).
Readings (the page gives neither): W - B A enters the quantizer rounded to bf16 (the
quantizer's input type; parity unpinned for this rounding: no pin tells it from an
unrounded target), the SVD is of the float64 residual, and the outputs are the last step's
quantized base and adapters. Parity of the GPU path is by properties (objectives
within a tolerance, codes equal on all but a tiny fraction), not bit-exact: its SVD works in
fp32 through the Gram matrix.
"""
from __future__ import annotations

import numpy as np

from . import nf4
from .numerics import round_bf16


def quant_dequant(w: np.ndarray):
    """(codes uint8 [n], code2, scale2, mean, dequantized fp32 [N, K]) of a bf16-valued
    float array: NF4 with double quantization, as the QLoRA page describes."""
    N, K = w.shape
    codes, c = nf4.quantize(np.asarray(w, np.float32).reshape(-1))
    code2, s2, mu = nf4.double_quant(c)
    deq = nf4.dequant(nf4.pack(codes), code2, s2, mu, w.size).reshape(N, K)
    return codes, code2, s2, mu, deq.astype(np.float32)


def loftq(W: np.ndarray, r: int, steps: int = 5):
    """(codes of the last step, A [r, K], B [N, r] float64, objectives e_1..e_T float64,
    the last dequantized base Q fp32 [N, K])."""
    W = np.asarray(W, np.float64)
    N, K = W.shape
    A = np.zeros((r, K))
    B = np.zeros((N, r))
    errs = []
    codes = None
    Q = None
    for _ in range(steps):
        target = round_bf16((W - B @ A).astype(np.float32)).astype(np.float64)
        codes, _, _, _, Q = quant_dequant(target.astype(np.float32))
        R = W - Q.astype(np.float64)
        U, s, Vt = np.linalg.svd(R, full_matrices=False)
        sq = np.sqrt(s[:r])
        B = U[:, :r] * sq[None, :]
        A = sq[:, None] * Vt[:r]
        errs.append(float(np.sum(s[r:] ** 2)))
    return codes, A, B, np.array(errs), Q
