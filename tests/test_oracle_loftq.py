"""Pins of the LoftQ-style initialisation oracle ("LowRA" article: quantize first, then a
rank-r SVD of the quantization error, five alternating steps) against the pinned NF4
oracle and the mathematics of the truncated SVD."""
import numpy as np
import pytest

import synth
from oracle import loftq, nf4


def _w(N, K, seed):
    return synth.llama_weight((N, K), seed, std=0.02).float().numpy()


def test_first_step_is_plain_nf4():
    W = _w(64, 128, 1)
    codes, _, _, errs, _ = loftq.loftq(W, 4, steps=1)
    ref, _ = nf4.quantize(W.reshape(-1))
    assert np.array_equal(codes, ref)


@pytest.mark.parametrize("r", [1, 4, 8])
def test_objective_is_the_direct_residual(r):
    # e_T = sum of the discarded squared singular values (Eckart-Young) must equal the
    # residual norm computed directly from the outputs
    W = _w(48, 128, 2 + r)
    _, A, B, errs, Q = loftq.loftq(W, r, steps=3)
    direct = float(np.sum((W.astype(np.float64) - Q.astype(np.float64) - B @ A) ** 2))
    assert abs(direct - errs[-1]) <= 1e-9 * direct
    assert np.linalg.matrix_rank(B @ A) == r


def test_absorbs_quantization_error():
    # the low-rank terms absorb part of the quantization error: better than NF4 alone
    W = _w(64, 192, 5)
    _, _, _, errs, _ = loftq.loftq(W, 8, steps=5)
    Q1 = loftq.quant_dequant(W)[4].astype(np.float64)
    plain = float(np.sum((W.astype(np.float64) - Q1) ** 2))
    assert errs[0] < plain and errs[-1] < plain


def test_full_rank_leaves_no_error():
    W = _w(16, 64, 6)
    _, _, _, errs, _ = loftq.loftq(W, 16, steps=2)
    assert np.all(errs <= 1e-20)
