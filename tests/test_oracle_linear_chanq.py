"""Pins for the oracle's linear layer, per-channel quantizer and layer ranking.

The linear layer is checked against torch.autograd in float64 on the CPU (a library
derivation of the gradients that the oracle's hand-written backward does not use),
plus the special cases the pages fix: with B = 0 (QLoRA's adapter init) the output
is the frozen base alone; with every code on the zero level the base vanishes.
"""
import numpy as np
import torch

from oracle import chanq, linear, nf4, rank


def _rand(shape, seed, std=1.0):
    g = torch.Generator().manual_seed(seed)
    return (torch.randn(*shape, generator=g, dtype=torch.float64) * std)


def test_linear_forward_backward_match_autograd():
    M, N, K, r, s = 7, 24, 64, 4, 2.0
    x = _rand((M, K), 1)
    W = _rand((N, K), 2, 0.1)
    A = _rand((r, K), 3, 0.1)
    B = _rand((N, r), 4, 0.1)
    dY = _rand((M, N), 5)
    xs, As, Bs = (t.clone().requires_grad_(True) for t in (x, A, B))
    h = torch.nn.functional.linear(xs, W) + s * torch.nn.functional.linear(
        torch.nn.functional.linear(xs, As), Bs)
    (h * dY).sum().backward()
    h_or = linear.forward(x.numpy(), W.numpy(), A.numpy(), B.numpy(), s)
    dX, dA, dB = linear.backward(x.numpy(), dY.numpy(), W.numpy(), A.numpy(), B.numpy(), s)
    assert np.allclose(h_or, h.detach().numpy(), rtol=1e-12, atol=1e-12)
    assert np.allclose(dX, xs.grad.numpy(), rtol=1e-12, atol=1e-12)
    assert np.allclose(dA, As.grad.numpy(), rtol=1e-12, atol=1e-12)
    assert np.allclose(dB, Bs.grad.numpy(), rtol=1e-12, atol=1e-12)


def test_linear_with_zero_B_is_base_only_and_zero_codes_is_lora_only():
    M, N, K, r = 5, 16, 128, 8
    x = _rand((M, K), 6).numpy()
    A = _rand((r, K), 7, 0.01).numpy()
    B = _rand((N, r), 8, 0.01).numpy()
    w = (_rand((N, K), 9, 0.02).float().to(torch.bfloat16).float().numpy())
    codes, c = nf4.quantize(w)
    code2, s2, mu = nf4.double_quant(c)
    wb = linear.base_bf16(nf4.dequant(nf4.pack(codes), code2, s2, mu, w.size).reshape(N, K))
    h0 = linear.forward(x, wb, A, np.zeros_like(B), 2.0)
    assert np.array_equal(h0, x @ wb.T)
    zero_codes = np.full(N * K, 7, np.uint8)  # the exact-zero level everywhere
    wz = linear.base_bf16(nf4.dequant(nf4.pack(zero_codes), code2, s2, mu, w.size).reshape(N, K))
    assert np.all(wz == 0)
    hz = linear.forward(x, wz, A, B, 2.0)
    assert np.allclose(hz, 2.0 * (x @ A.T) @ B.T, rtol=1e-13, atol=0)


def test_tolerance_helper():
    ref = np.array([1.0, -2.0, 3.0])
    ok, a, b = linear.close(ref * (1 + 1e-3), ref)
    assert ok and a < 2e-2 and b < 5e-3
    ok, _, _ = linear.close(ref + np.array([0, 0, 0.1]), ref)
    assert not ok


# ------------------------------------------------------------------- chanq
def test_chanq_threshold_indexing_matches_bruteforce():
    rng = np.random.default_rng(10)
    for b in (1, 2, 4):
        L = 1 << b
        t = np.sort(rng.uniform(-1, 1, L - 1)).astype(np.float32)
        x = np.concatenate([rng.uniform(-1, 1, 5000).astype(np.float32), t,
                            np.nextafter(t, np.float32(-2)), np.nextafter(t, np.float32(2))])
        assert np.array_equal(chanq.encode_row(x, t), chanq.encode_row_bruteforce(x, t))


def test_chanq_reduces_to_nf4_codes():
    """b = 4, mappings = NF4 levels, edges just below the NF4 decision thresholds:
    for fp32 x, x > pred(T) <=> x >= T, so the codes must equal NF4's."""
    w = _rand((8, 256), 11, 0.02).float().to(torch.bfloat16).float().numpy()
    T = nf4.thresholds()
    t = np.nextafter(T, np.float32(-np.inf)).astype(np.float32)
    bits = np.full(8, 4, np.uint8)
    thr = np.tile(t, 8)
    thr_off = np.arange(9, dtype=np.int64) * 15
    packed, roff, g, codes = chanq.quantize(w, bits, thr, thr_off)
    nf_codes, c = nf4.quantize(w)
    assert np.array_equal(codes.reshape(-1), nf_codes)
    assert np.array_equal(g, c)
    # MSB-first 4-bit packing equals the NF4 nibble order
    assert np.array_equal(packed, nf4.pack(nf_codes))
    maps = np.tile(nf4.codebook(), 8)
    map_off = np.arange(9, dtype=np.int64) * 16
    wh = chanq.dequant(packed, roff, bits, maps, map_off, g, 8, 256)
    assert np.array_equal(wh.reshape(-1), nf4.dequant_single(nf_codes, c))


def test_chanq_one_bit_is_sign_quantization():
    w = _rand((4, 128), 12, 0.02).float().to(torch.bfloat16).float().numpy()
    bits = np.ones(4, np.uint8)
    thr = np.zeros(4, np.float32)
    thr_off = np.arange(5, dtype=np.int64)
    packed, roff, g, codes = chanq.quantize(w, bits, thr, thr_off)
    assert np.array_equal(codes, (w > 0).astype(np.uint8))
    assert roff[-1] == 4 * 128 // 8
    maps = np.tile(np.array([-1, 1], np.float32), 4)
    wh = chanq.dequant(packed, roff, bits, maps, np.arange(5) * 2, g, 4, 128)
    gg = np.repeat(g, 64).reshape(4, 128)
    assert np.array_equal(wh, np.where(w > 0, gg, -gg).astype(np.float32))


def test_chanq_pack_round_trip_all_widths():
    rng = np.random.default_rng(13)
    for b in (1, 2, 4):
        c = rng.integers(0, 1 << b, 512).astype(np.uint8)
        p = chanq.pack_row(c, b)
        assert p.size == 512 * b // 8
        assert np.array_equal(chanq.unpack_row(p, b, 512), c)
    # MSB-first: first 2-bit code in bits 7..6
    assert chanq.pack_row(np.array([3, 0, 0, 1], np.uint8), 2)[0] == 0b11000001


# -------------------------------------------------------------------- ranking
def test_top_k_matches_bruteforce():
    rng = np.random.default_rng(14)
    n = rng.integers(1000, 100000, 280)
    sse = rng.uniform(0, 1, 280) * n
    sse[10] = sse[11] / n[11] * n[10]  # a tie in epsilon
    top = rank.top_k(sse, n, 8)
    eps = sse / n
    chosen = set(top.tolist())
    for i in range(280):
        for j in chosen:
            if i not in chosen:
                assert eps[j] > eps[i] or (eps[j] == eps[i] and j < i)
    assert len(chosen) == 8
    assert all(eps[top[i]] >= eps[top[i + 1]] for i in range(7))
