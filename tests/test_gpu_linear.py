"""GPU parity of the fused tcgen05 linear layer against the float64 oracle.

h = x bf16(W_hat)^T + s (x A^T) B^T and its backward (dX, dA, dB) through the frozen
NF4 base, the dense-base variant for protected layers and the per-channel quantized
forward. The GPU receives the oracle's quantized weight, so these tests isolate the
GEMM path. Tolerance (bf16 inputs, fp32 accumulation): max|err| <= 2e-2 max|ref| and
relative Frobenius error <= 5e-3, element by element over every output (or over
sampled token rows of the largest prefill shapes, where the oracle's float64 GEMM
would take minutes).
"""
import numpy as np
import pytest
import torch

import synth
from oracle import chanq as ochq
from oracle import linear as olin

from helpers import (assert_close, chanq_oracle, dev, f32, f64, oracle_base_bf16,
                     oracle_quant, weight_from_oracle)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def q():
    import bit_nf4_quantized_04_b200 as q
    return q


def _inputs(N, K, M, r, seed, wstd=0.02):
    W = synth.llama_weight((N, K), seed, std=wstd)
    x = synth.normal_bf16((M, K), 1.0, seed + 1)
    A = synth.normal_bf16((r, K), 0.01, seed + 2)
    B = synth.normal_bf16((N, r), 0.01, seed + 3)
    dY = synth.normal_bf16((M, N), 1.0, seed + 4)
    return W, x, A, B, dY


def _run_nf4(q, N, K, M, r, seed, bwd=True, rows=None):
    W, x, A, B, dY = _inputs(N, K, M, r, seed)
    s = 2.0 / r * 8  # an alpha/r-like scale
    oq = oracle_quant(W)
    Wb = oracle_base_bf16(oq, N, K)
    w = weight_from_oracle(q, oq, N, K)
    xc, Ac, Bc, dYc = x.cuda(), A.cuda(), B.cuda(), dY.cuda()
    h = q.qlora_linear_fwd(w, xc, Ac, Bc, s)
    sel = np.arange(M) if rows is None else rows
    xs = f64(x)
    href = olin.forward(xs[sel], Wb, f64(A), f64(B), s)
    assert_close(f64(h.cpu())[sel], href, f"h N={N} K={K} M={M} r={r}")
    if not bwd:
        return
    dX, dA, dB = q.qlora_linear_bwd(w, xc, dYc, Ac, Bc, s)
    torch.cuda.synchronize()
    dYs = f64(dY)
    v = dYs @ f64(B)
    dXref = dYs[sel] @ Wb + s * (v[sel] @ f64(A))
    assert_close(f64(dX.cpu())[sel], dXref, f"dX N={N} K={K} M={M} r={r}")
    dAref = s * (v.T @ xs)
    dBref = s * (dYs.T @ (xs @ f64(A).T))
    assert_close(dA.cpu().double().numpy(), dAref, "dA")
    assert_close(dB.cpu().double().numpy(), dBref, "dB")


def test_tiny_layer_fwd_bwd(q):
    t = synth.tiny_inputs()
    W, x, A, B, dY, r, alpha = t["W"], t["x"], t["A"], t["B"], t["dY"], t["r"], t["alpha"]
    N, K = W.shape
    s = alpha / r
    oq = oracle_quant(W)
    Wb = oracle_base_bf16(oq, N, K)
    w = weight_from_oracle(q, oq, N, K)
    h = q.qlora_linear_fwd(w, x.cuda(), A.cuda(), B.cuda(), s)
    assert_close(f64(h.cpu()), olin.forward(f64(x), Wb, f64(A), f64(B), s), "h")
    dX, dA, dB = q.qlora_linear_bwd(w, x.cuda(), dY.cuda(), A.cuda(), B.cuda(), s)
    rdX, rdA, rdB = olin.backward(f64(x), f64(dY), Wb, f64(A), f64(B), s)
    assert_close(f64(dX.cpu()), rdX, "dX")
    assert_close(dA.cpu().double().numpy(), rdA, "dA")
    assert_close(dB.cpu().double().numpy(), rdB, "dB")


@pytest.mark.parametrize("N,K,M,r", [
    (200, 192, 3, 5),      # ragged N, three contraction steps, odd rank
    (384, 640, 17, 16),
    (136, 128, 130, 33),   # M spans two token tiles, r spans three K=16 sub-steps
    (256, 256, 1, 64),     # single token, largest rank
    (128, 1024, 300, 24),
    (264, 320, 64, 8),
    # several token tiles with ragged token rows, v's contraction N = 1000 (not a multiple
    # of the 64-wide step), ranks padded to 16, 32, 48 and 64 columns
    (1000, 256, 700, 5),
    (520, 640, 512, 20),
    (264, 192, 530, 40),
    (136, 384, 600, 64),
])
def test_ragged_shapes(q, N, K, M, r):
    _run_nf4(q, N, K, M, r, seed=N * 7 + K + M + r)


@pytest.mark.parametrize("M", [1, 4, 16])
def test_llama7b_decode_shapes(q, M):
    # q_proj and down_proj (K = 11008: 172 blocks per row, unaligned constant rows)
    _run_nf4(q, 4096, 4096, M, 16, seed=1000, bwd=False)
    _run_nf4(q, 4096, 11008, M, 16, seed=1006, bwd=False)


def test_llama7b_prefill_q_proj_sampled(q):
    rows = np.array([0, 1, 255, 256, 1000, 2047, 3071, 4095])
    _run_nf4(q, 4096, 4096, 4096, 16, seed=1000, bwd=True, rows=rows)


def test_llama7b_prefill_gate_and_down_sampled(q):
    # the bench's launch configuration on the two other 7B shapes: gate (11008 x 4096: the
    # last wave's tiles cut into contraction slices) and down (4096 x 11008: a contraction
    # of 172 blocks, the backward's over N = 4096), fwd + bwd at 4096 tokens, r = 16
    rows = np.array([0, 1, 255, 256, 1000, 2047, 3071, 4095])
    _run_nf4(q, 11008, 4096, 4096, 16, seed=1001, bwd=True, rows=rows)
    _run_nf4(q, 4096, 11008, 4096, 16, seed=1006, bwd=True, rows=rows)


def test_llama13b_prefill_r64_sampled(q):
    # the 13B-shaped configuration's attention projection at 8192 tokens, r = 64 (the
    # adapter chunk spans four K = 16 sub-steps)
    rows = np.array([0, 129, 4095, 4096, 8191])
    _run_nf4(q, 5120, 5120, 8192, 64, seed=1300, bwd=True, rows=rows)


def test_zero_adapter_is_base_only(q):
    N, K, M, r = 256, 512, 40, 8
    W, x, A, B, _ = _inputs(N, K, M, r, 31)
    w = q.quantize_weight(W.cuda())
    h0 = q.qlora_linear_fwd(w, x.cuda(), A.cuda(), torch.zeros_like(B).cuda(), 2.0)
    h1 = q.qlora_linear_fwd(w, x.cuda(), torch.zeros_like(A).cuda(), B.cuda(), 2.0)
    assert torch.equal(h0, h1)


def test_dense_base_fwd_bwd(q):
    N, K, M, r = 384, 512, 100, 16
    W, x, A, B, dY = _inputs(N, K, M, r, 41)
    s = 2.0
    Wd = f64(W)
    h = q.dense_linear_fwd(W.cuda(), x.cuda(), A.cuda(), B.cuda(), s)
    assert_close(f64(h.cpu()), olin.forward(f64(x), Wd, f64(A), f64(B), s), "dense h")
    dX, dA, dB = q.dense_linear_bwd(W.cuda(), x.cuda(), dY.cuda(), A.cuda(), B.cuda(), s)
    rdX, rdA, rdB = olin.backward(f64(x), f64(dY), Wd, f64(A), f64(B), s)
    assert_close(f64(dX.cpu()), rdX, "dense dX")
    assert_close(dA.cpu().double().numpy(), rdA, "dense dA")
    assert_close(dB.cpu().double().numpy(), rdB, "dense dB")


def _chanq_case(N, K, seed):
    W = synth.llama_weight((N, K), seed)
    bits = synth.chan_bits(N)
    maps, map_off, thr, thr_off = synth.chan_tables(bits, seed=seed + 5)
    roff = torch.from_numpy(ochq.row_offsets(bits.numpy(), K))
    return W, bits, maps, map_off, thr, thr_off, roff


@pytest.mark.parametrize("N,K", [(40, 128), (200, 448), (1100, 4096)])
def test_chanq_quantize_bit_exact(q, N, K):
    W, bits, maps, map_off, thr, thr_off, roff = _chanq_case(N, K, 500 + N)
    packed, roff_o, g, _ = chanq_oracle(W, bits, thr, thr_off)
    assert np.array_equal(roff.numpy(), roff_o)
    gp, gg = q.chanq_quantize(W.cuda(), bits.cuda(), thr.cuda(), thr_off.cuda(), roff.cuda())
    torch.cuda.synchronize()
    assert np.array_equal(gg.cpu().numpy().view(np.uint32), g.view(np.uint32))
    assert np.array_equal(gp.cpu().numpy()[: packed.size], packed)


def _bf16_round(a: np.ndarray) -> np.ndarray:
    """fp32 -> nearest bf16 value (ties to even), as fp32."""
    u = a.astype(np.float32).view(np.uint32).astype(np.uint64)
    r = ((u + 0x7FFF + ((u >> 16) & 1)) >> 16) << 16
    return r.astype(np.uint32).view(np.float32)


def test_chanq_quantize_near_edges(q):
    # Rows of 4-bit codes whose thresholds are bf16 values, weights in groups with
    # absmax exactly 1 placed on each threshold and one bf16 step either side of it,
    # so the normalised value hits or straddles every threshold; a row with two
    # thresholds in one bin and one whose thresholds defeat the bin table (the exact
    # path); an all-zero group. Codes must match the oracle bit for bit.
    K = 256
    rng = np.random.default_rng(7)
    rows_thr = []
    for i in range(6):
        t = np.sort(rng.uniform(-0.95, 0.95, 15)).astype(np.float32)
        rows_thr.append(_bf16_round(t))
    t = rows_thr[0].copy()
    t[7] = _bf16_round(np.array([t[6] * np.float32(1 + 2.0 ** -7)]))[0]  # two in one bin
    rows_thr.append(np.sort(t))
    # five thresholds within 0.004 (< any bin): three share a bin at every density, so
    # the row takes the exact path throughout
    close = np.float32(0.3) + np.arange(5, dtype=np.float32) * np.float32(2.0 ** -8)
    t = np.sort(np.concatenate([close, rng.uniform(-0.9, 0.2, 10).astype(np.float32)]))
    rows_thr.append(_bf16_round(t))
    N = len(rows_thr)
    W = np.zeros((N, K), np.float32)
    for i, t in enumerate(rows_thr):
        vals = []
        for x in t:
            up = np.nextafter(x, np.float32(2), dtype=np.float32)
            dn = np.nextafter(x, np.float32(-2), dtype=np.float32)
            vals += [x, _bf16_round(np.array([up + (up - x) * 2**16]))[0],
                     _bf16_round(np.array([dn - (x - dn) * 2**16]))[0]]
        vals = np.array(vals, np.float32)
        row = np.zeros(K, np.float32)
        for gsi in range(K // 64 - 1):                           # the last group stays all zero
            seg = rng.choice(vals, 63)
            row[gsi * 64: gsi * 64 + 63] = seg
            row[gsi * 64 + 63] = 1.0 if gsi % 2 == 0 else -1.0   # absmax exactly 1
        W[i] = row
    Wt = torch.from_numpy(W).to(torch.bfloat16)
    assert np.array_equal(f32(Wt), W)
    bits = torch.full((N,), 4, dtype=torch.uint8)
    thr = torch.from_numpy(np.concatenate(rows_thr).astype(np.float32))
    thr_off = torch.arange(0, 15 * N + 1, 15, dtype=torch.int64)
    roff = torch.from_numpy(ochq.row_offsets(bits.numpy(), K))
    packed, roff_o, g, _ = chanq_oracle(Wt, bits, thr, thr_off)
    gp, gg = q.chanq_quantize(Wt.cuda(), bits.cuda(), thr.cuda(), thr_off.cuda(), roff.cuda())
    torch.cuda.synchronize()
    assert np.array_equal(gg.cpu().numpy().view(np.uint32), g.view(np.uint32))
    got = gp.cpu().numpy()[: packed.size]
    bad = np.nonzero(got != packed)[0]
    assert bad.size == 0, f"{bad.size} code bytes differ, first at {bad[:5]}"


@pytest.mark.parametrize("N,K,M,r", [(40, 128, 5, 8), (200, 448, 70, 16), (1100, 4096, 260, 16)])
def test_chanq_linear_fwd(q, N, K, M, r):
    W, bits, maps, map_off, thr, thr_off, roff = _chanq_case(N, K, 600 + N)
    packed, roff_o, g, _ = chanq_oracle(W, bits, thr, thr_off)
    x = synth.normal_bf16((M, K), 1.0, 71)
    A = synth.normal_bf16((r, K), 0.01, 72)
    B = synth.normal_bf16((N, r), 0.01, 73)
    s = 2.0
    wh = ochq.dequant(packed, roff_o, bits.numpy(), maps.numpy(), map_off.numpy(), g, N, K)
    href = olin.forward(f64(x), olin.base_bf16(wh), f64(A), f64(B), s)
    pk = np.zeros(max(packed.size, 16), np.uint8)
    pk[: packed.size] = packed
    h = q.chanq_linear_fwd(dev(pk), roff.cuda(), bits.cuda(), maps.cuda(), map_off.cuda(),
                           dev(g), N, K, x.cuda(), A.cuda(), B.cuda(), s)
    assert_close(f64(h.cpu()), href, "chanq h")


def test_chanq_linear_full_size_sampled(q):
    # the per-channel configuration in the bench's launch configuration: 11008 x 4096 at
    # 1/2/4 bits, 2048 tokens, r = 16; forward and backward on sampled token rows (dA, dB
    # over all tokens)
    N, K, M, r = 11008, 4096, 2048, 16
    W, bits, maps, map_off, thr, thr_off, roff = _chanq_case(N, K, 610)
    packed, roff_o, g, _ = chanq_oracle(W, bits, thr, thr_off)
    x = synth.normal_bf16((M, K), 1.0, 611)
    A = synth.normal_bf16((r, K), 0.01, 612)
    B = synth.normal_bf16((N, r), 0.01, 613)
    dY = synth.normal_bf16((M, N), 1.0, 614)
    s = 2.0
    wb = olin.base_bf16(ochq.dequant(packed, roff_o, bits.numpy(), maps.numpy(), map_off.numpy(),
                                     g, N, K))
    sel = np.array([0, 1, 127, 128, 1000, 2047])
    xs, dYs = f64(x), f64(dY)
    pk = np.zeros(max(packed.size, 16), np.uint8)
    pk[: packed.size] = packed
    args = (dev(pk), roff.cuda(), bits.cuda(), maps.cuda(), map_off.cuda(), dev(g), N, K)
    h = q.chanq_linear_fwd(*args, x.cuda(), A.cuda(), B.cuda(), s)
    assert_close(f64(h.cpu())[sel], olin.forward(xs[sel], wb, f64(A), f64(B), s), "chanq h (full)")
    dX, dA, dB = q.chanq_linear_bwd(*args, x.cuda(), dY.cuda(), A.cuda(), B.cuda(), s)
    torch.cuda.synchronize()
    v = dYs @ f64(B)
    assert_close(f64(dX.cpu())[sel], dYs[sel] @ wb + s * (v[sel] @ f64(A)), "chanq dX (full)")
    assert_close(dA.cpu().double().numpy(), s * (v.T @ xs), "chanq dA (full)")
    assert_close(dB.cpu().double().numpy(), s * (dYs.T @ (xs @ f64(A).T)), "chanq dB (full)")


@pytest.mark.parametrize("N,K,M,r", [
    (40, 128, 5, 8),        # thin token tile, one row tile
    (200, 448, 70, 16),     # ragged N, K = 448 (7 groups, rows of 56 b bytes)
    (1104, 4096, 260, 16),  # two token tiles, contraction slices on the last wave
    (512, 8192, 600, 24),   # more tiles than CTAs: several units per CTA
])
def test_chanq_linear_bwd(q, N, K, M, r):
    # dX = dY w_hat + s v A, dA = s v^T x, dB = s dY^T (x A^T) against the float64 oracle on
    # the oracle's dequantized per-channel weight
    W, bits, maps, map_off, thr, thr_off, roff = _chanq_case(N, K, 900 + N)
    packed, roff_o, g, _ = chanq_oracle(W, bits, thr, thr_off)
    x = synth.normal_bf16((M, K), 1.0, 81)
    A = synth.normal_bf16((r, K), 0.01, 82)
    B = synth.normal_bf16((N, r), 0.01, 83)
    dY = synth.normal_bf16((M, N), 1.0, 84)
    s = 16.0 / r
    wh = ochq.dequant(packed, roff_o, bits.numpy(), maps.numpy(), map_off.numpy(), g, N, K)
    rdX, rdA, rdB = olin.backward(f64(x), f64(dY), olin.base_bf16(wh), f64(A), f64(B), s)
    pk = np.zeros(max(packed.size, 16), np.uint8)
    pk[: packed.size] = packed
    dX, dA, dB = q.chanq_linear_bwd(dev(pk), roff.cuda(), bits.cuda(), maps.cuda(), map_off.cuda(),
                                    dev(g), N, K, x.cuda(), dY.cuda(), A.cuda(), B.cuda(), s)
    assert_close(f64(dX.cpu()), rdX, "chanq dX")
    assert_close(dA.cpu().double().numpy(), rdA, "chanq dA")
    assert_close(dB.cpu().double().numpy(), rdB, "chanq dB")


def test_chanq_linear_bwd_matches_nf4_special_case(q):
    # 4-bit rows with the NF4 levels as every row's map and each group's absmax as its
    # scale give a single-level NF4 weight; the per-channel backward must then agree with
    # the dense backward on that weight dequantized by the oracle
    N, K, M, r = 256, 512, 130, 8
    W = synth.llama_weight((N, K), 95, std=0.02)
    from oracle import nf4 as onf4
    lv = onf4.codebook().astype(np.float32)
    bits = torch.full((N,), 4, dtype=torch.uint8)
    thr_row = np.nextafter(onf4.thresholds().astype(np.float32), np.float32(-2), dtype=np.float32)
    thr = torch.from_numpy(np.tile(thr_row, N).astype(np.float32))
    thr_off = torch.arange(0, 15 * N + 1, 15, dtype=torch.int64)
    maps = torch.from_numpy(np.tile(lv, N).astype(np.float32))
    map_off = torch.arange(0, 16 * N + 1, 16, dtype=torch.int64)
    roff = torch.from_numpy(ochq.row_offsets(bits.numpy(), K))
    packed, roff_o, g, _ = chanq_oracle(W, bits, thr, thr_off)
    wh = ochq.dequant(packed, roff_o, bits.numpy(), maps.numpy(), map_off.numpy(), g, N, K)
    Wd = torch.from_numpy(olin.base_bf16(wh).astype(np.float32)).to(torch.bfloat16)
    x = synth.normal_bf16((M, K), 1.0, 96)
    A = synth.normal_bf16((r, K), 0.01, 97)
    B = synth.normal_bf16((N, r), 0.01, 98)
    dY = synth.normal_bf16((M, N), 1.0, 99)
    pk = np.zeros(max(packed.size, 16), np.uint8)
    pk[: packed.size] = packed
    got = q.chanq_linear_bwd(dev(pk), roff.cuda(), bits.cuda(), maps.cuda(), map_off.cuda(), dev(g),
                             N, K, x.cuda(), dY.cuda(), A.cuda(), B.cuda(), 2.0)
    ref = q.dense_linear_bwd(Wd.cuda(), x.cuda(), dY.cuda(), A.cuda(), B.cuda(), 2.0)
    torch.cuda.synchronize()
    # same bf16 weight, same kernels downstream of the operand: identical results
    for a, b, nm in zip(got, ref, ("dX", "dA", "dB")):
        assert torch.equal(a, b), nm

