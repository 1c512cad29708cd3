"""GPU parity of the Llama-2-13B-shaped stack ("AQLoRA" §3.1 profiling pass with the §3.2
choice of 16-bit layers, then QLoRA's fused forward and backward).

The stack is 40 layers of {5120x5120 x4, 13824x5120 x2, 5120x13824}: 280 matrices with one
weight scale per matrix drawn from U[0.01, 0.04] (synth.llama13b_stds). Checked here:
* the two MLP shapes quantized as the profiling pass runs them (qnf4_quantize_weight:
  NF4 codes, double quantization and the reconstruction SSE in two launches), codes,
  constants and scales bit-exact and the SSE within 1e-5 relative of the oracle;
* forward and backward at 8192 tokens with r = 64, alpha = 128 on both shapes: sampled
  token rows of h and dX against the float64 oracle, dA and dB over all tokens;
* the whole-stack ranking: the SSE of every one of the 280 matrices from the GPU, the
  top-8 by SSE per parameter equal to the oracle's ranking of those values, and a gap
  between the 8th and 9th errors wide enough that SSEs within the 1e-5 tolerance of the
  oracle (checked on one matrix of each shape) cannot change the protected set.
Tolerances: bit-exact codes and constants; GEMM outputs max|err| <= 2e-2 max|ref| and
relative Frobenius error <= 5e-3.
"""
import numpy as np
import pytest
import torch

import synth
from oracle import linear as olin
from oracle import nf4 as onf4
from oracle import rank as orank

from helpers import assert_close, f32, f64

pytestmark = pytest.mark.gpu

STACK = synth.llama13b_stack()
STDS = synth.llama13b_stds()
M, R, ALPHA = 8192, 64, 128.0


@pytest.fixture(scope="module")
def q():
    import bit_nf4_quantized_04_b200 as q
    return q


def _weight(i, device="cpu"):
    sh = STACK[i]
    return synth.llama_weight((sh.N, sh.K), synth.SEED_W + 300 + i, std=float(STDS[i]),
                              device=device)


def _quant_exact(q, W):
    w, sse = q.quantize_weight(W.cuda(), sse=True)
    wf = f32(W)
    codes, c = onf4.quantize(wf)
    code2, s2, mu = onf4.double_quant(c)
    packed = onf4.pack(codes)
    torch.cuda.synchronize()
    got = w.packed.cpu().numpy()
    if not np.array_equal(got, packed):
        bad = np.nonzero(got != packed)[0]
        raise AssertionError(f"{bad.size} packed bytes differ, first at {bad[:5]}")
    assert np.array_equal(w.code2.cpu().numpy(), code2)
    assert np.array_equal(w.scale2.cpu().numpy().view(np.uint32), s2.view(np.uint32))
    assert np.float32(w.mean.item()) == mu
    ref = onf4.recon_sse(wf)
    assert abs(sse.item() - ref) <= 1e-5 * ref, (sse.item(), ref)
    return w, olin.base_bf16(onf4.dequant(packed, code2, s2, mu, wf.size).reshape(W.shape))


@pytest.mark.parametrize("idx", [4, 6])  # layer 0's gate (13824x5120) and down (5120x13824)
def test_stack13b_mlp_quantize_and_fwd_bwd(q, idx):
    sh = STACK[idx]
    N, K = sh.N, sh.K
    W = _weight(idx)
    w, Wb = _quant_exact(q, W)
    x = synth.normal_bf16((M, K), 1.0, synth.SEED_X + 300 + idx)
    dY = synth.normal_bf16((M, N), 1.0, synth.SEED_DY + 300 + idx)
    A = synth.normal_bf16((R, K), 0.01, synth.SEED_A + 300 + idx)
    B = synth.normal_bf16((N, R), 0.01, synth.SEED_B + 300 + idx)
    s = ALPHA / R
    xc, dYc, Ac, Bc = x.cuda(), dY.cuda(), A.cuda(), B.cuda()
    h = q.qlora_linear_fwd(w, xc, Ac, Bc, s)
    dX, dA, dB = q.qlora_linear_bwd(w, xc, dYc, Ac, Bc, s)
    torch.cuda.synchronize()
    rows = np.array([0, 1, 127, 128, 4095, 4096, 6000, 8191])
    xs, dYs, As, Bs = f64(x), f64(dY), f64(A), f64(B)
    assert_close(f64(h.cpu())[rows], olin.forward(xs[rows], Wb, As, Bs, s), f"h {N}x{K}")
    v = dYs @ Bs
    assert_close(f64(dX.cpu())[rows], dYs[rows] @ Wb + s * (v[rows] @ As), f"dX {N}x{K}")
    assert_close(dA.cpu().double().numpy(), s * (v.T @ xs), f"dA {N}x{K}")
    assert_close(dB.cpu().double().numpy(), s * (dYs.T @ (xs @ As.T)), f"dB {N}x{K}")


def test_stack13b_attention_shape_sse(q):
    # one 5120x5120 projection of the stack (its own weight scale) through the fused pass
    _quant_exact(q, _weight(2))


def test_stack13b_top8_ranking(q):
    n = len(STACK)
    sse = torch.zeros(n, 2, dtype=torch.float64, device="cuda")
    ws = torch.empty(q.workspace_size(q._lib.OP_QUANTIZE_WEIGHT, 13824, 5120), dtype=torch.uint8,
                     device="cuda")
    for i in range(n):
        W = _weight(i, device="cuda")
        q.quantize_weight(W, sse=True, sse_out=sse[i], ws=ws)
        del W
    q.check()
    s = sse[:, 0].cpu().numpy()
    nparams = np.array([sh.N * sh.K for sh in STACK], dtype=np.int64)
    got = q.rank_topk(s.tolist(), nparams.tolist(), 8)
    assert got == orank.top_k(s, nparams, 8).tolist()
    eps = np.sort(s / nparams)[::-1]
    # 1e-5 relative on every SSE cannot reorder the 8th and 9th layers
    assert (eps[7] - eps[8]) > 2.5e-5 * eps[7], (eps[7], eps[8])
    # the error per parameter follows the matrices' weight scales: the protected layers
    # are among those with the largest scales
    big = set(np.argsort(-STDS.numpy())[:16].tolist())
    assert set(got) <= big
