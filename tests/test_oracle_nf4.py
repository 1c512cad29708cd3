"""Pins for the oracle's NF4 codebook, quantizer, double quantization and dequant.

Each test checks the oracle against something other than itself: facts the QLoRA
page prints (tests/golden), closed forms, brute force on small inputs, or a library
routine (math.erfc, torch's fp8 / bf16 casts) that the oracle does not use.
"""
import math
from fractions import Fraction
import os

import numpy as np
import pytest
import torch

from oracle import nf4, numerics

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden(name):
    out = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            k, v = line.split()
            out[k] = float(v)
    return out


def _phi(z):
    """Standard normal CDF from the complementary error function (not inv_cdf)."""
    return 0.5 * math.erfc(-z / math.sqrt(2.0))


# --------------------------------------------------------------------- codebook
def test_codebook_shape_and_ends():
    g = _golden("nf4_construction.txt")
    q = nf4.codebook()
    assert q.dtype == np.float32 and q.size == int(g["levels"])
    assert np.all(np.diff(q) > 0), "levels must be strictly increasing"
    assert q[0] == np.float32(g["range_lo"]) and q[-1] == np.float32(g["range_hi"])
    assert g["has_exact_zero"] == 1 and q[7] == 0.0 and np.sum(q == 0) == 1
    # 8 negative + 9 positive quantiles, one duplicated zero dropped
    assert int(np.sum(q < 0)) == int(g["negative_quantiles"]) - 1
    assert int(np.sum(q > 0)) == int(g["positive_quantiles"]) - 1
    assert int(g["negative_quantiles"] + g["positive_quantiles"] - 1) == q.size


def test_codebook_levels_are_normal_quantiles():
    """Undo the normalisation and push each level through the normal CDF: the
    probabilities must be evenly spaced on each side, from P_MAX to 1/2."""
    q = nf4.codebook_f64()
    # find z_max from P_MAX with a bisection on the CDF (independent of inv_cdf)
    lo, hi = 0.0, 10.0
    for _ in range(200):
        mid = 0.5 * (lo + hi)
        if _phi(mid) < nf4.P_MAX:
            lo = mid
        else:
            hi = mid
    zmax = 0.5 * (lo + hi)
    pos = q[q > 0] * zmax
    neg = q[q < 0] * zmax
    p_pos = np.array([_phi(z) for z in sorted(pos, reverse=True)])
    p_neg = np.array([1.0 - _phi(z) for z in sorted(neg)])
    exp_pos = np.linspace(nf4.P_MAX, 0.5, 9)[:-1]
    exp_neg = np.linspace(nf4.P_MAX, 0.5, 8)[:-1]
    assert np.allclose(p_pos, exp_pos, atol=1e-12, rtol=0)
    assert np.allclose(p_neg, exp_neg, atol=1e-12, rtol=0)


def test_codebook_denser_near_zero():
    q = nf4.codebook().astype(np.float64)
    gaps = np.diff(q)
    # gaps shrink toward the middle on both sides (normal quantiles)
    assert np.all(np.diff(gaps[:7]) < 0)
    assert np.all(np.diff(gaps[8:]) > 0)


# ------------------------------------------------------------ thresholds/encode
def test_thresholds_are_tightest_midpoint_bounds():
    q = nf4.codebook()
    T = nf4.thresholds()
    for k in range(15):
        m = (float(q[k]) + float(q[k + 1])) / 2.0
        assert float(T[k]) > m
        below = np.nextafter(T[k], np.float32(-np.inf))
        assert float(below) <= m


def test_encode_matches_bruteforce_random():
    rng = np.random.default_rng(0)
    x = rng.uniform(-1, 1, 200000).astype(np.float32)
    assert np.array_equal(nf4.encode(x), nf4.encode_bruteforce(x))


def test_encode_matches_bruteforce_at_ties_and_neighbours():
    q = nf4.codebook()
    vals = []
    for k in range(15):
        m = np.float32((float(q[k]) + float(q[k + 1])) / 2.0)
        v = m
        for _ in range(4):
            v = np.nextafter(v, np.float32(-np.inf))
        for _ in range(9):
            vals.append(v)
            v = np.nextafter(v, np.float32(np.inf))
    vals += list(q) + [np.float32(-1), np.float32(1), np.float32(0)]
    x = np.array(vals, dtype=np.float32)
    assert np.array_equal(nf4.encode(x), nf4.encode_bruteforce(x))


def test_exact_tie_goes_low():
    # build levels whose midpoint is exactly representable in fp32
    q = np.array([-1, -0.5, 0, 0.25, 0.5, 0.75, 1] + [2.0 + i for i in range(9)], np.float32)
    T = nf4.thresholds(q)
    x = np.array([-0.75, -0.25, 0.125, 0.375], np.float32)  # exact midpoints
    assert list(nf4.encode(x, T)) == [0, 1, 2, 3]
    assert list(nf4.encode_bruteforce(x, q)) == [0, 1, 2, 3]


# ----------------------------------------------------------------- quantize
def _bf16_weight(shape, seed, std=0.02):
    g = torch.Generator().manual_seed(seed)
    return (torch.randn(*shape, generator=g) * std).to(torch.bfloat16).float().numpy()


def test_quantize_codes_are_nearest_levels_bruteforce():
    w = _bf16_weight((32, 128), 1)
    codes, c = nf4.quantize(w)
    # independent pure-Python path: per element nearest level in float64 of the
    # fp32 quotient, ties to the lower index
    q = [float(v) for v in nf4.codebook()]
    flat = w.reshape(-1)
    for i in range(flat.size):
        b = i // 64
        cb = max(abs(float(v)) for v in flat[b * 64:(b + 1) * 64])
        xn = float(np.float32(flat[i]) / np.float32(cb))
        best = min(range(16), key=lambda k: (abs(xn - q[k]), k))
        assert codes[i] == best
        assert c[b] == np.float32(cb)


def test_absmax_element_round_trips_to_plus_minus_absmax():
    w = _bf16_weight((64, 256), 2)
    codes, c = nf4.quantize(w)
    wh = nf4.dequant_single(codes, c)
    flat = w.reshape(-1)
    for b in range(c.size):
        seg = flat[b * 64:(b + 1) * 64]
        j = int(np.argmax(np.abs(seg)))
        assert wh[b * 64 + j] == np.float32(np.sign(seg[j]) * c[b])


def test_zero_block_and_constant_block():
    w = np.zeros((2, 128), np.float32)
    w[1, 64:] = 0.03125
    codes, c = nf4.quantize(w)
    assert c[0] == 0 and c[1] == 0 and np.all(codes[:128] == 7)
    assert np.all(codes[192:] == 15)  # identical values -> top level
    assert nf4.recon_sse(w) == 0.0


def test_pack_unpack_round_trip():
    rng = np.random.default_rng(3)
    codes = rng.integers(0, 16, 1000).astype(np.uint8)
    p = nf4.pack(codes)
    assert p.size == 500
    assert np.array_equal(nf4.unpack(p, 1000), codes)
    assert p[0] == (codes[0] << 4) | codes[1]


# --------------------------------------------------------- storage overheads
def test_constant_overheads_match_page_figures():
    g = _golden("qlora_dq_overhead.txt")
    assert nf4.constant_bits_per_param(False, int(g["block1"])) == g["bits_per_param_single"]
    dq = nf4.constant_bits_per_param(True, int(g["block1"]), int(g["block2"]))
    assert abs(dq - g["bits_per_param_double"]) < 5e-4
    saving = g["bits_per_param_single"] - dq
    assert abs(saving - g["saving_bits_per_param"]) < 5e-4
    gb = g["params_30b"] * saving / 8 / 1e9
    assert abs(gb - g["saving_gb_30b"]) < 0.01
    # storage_bytes agrees with the per-parameter figures on a real size
    n = 4096 * 11008
    assert nf4.storage_bytes(n, False) == n / 2 + n * g["bits_per_param_single"] / 8
    assert abs(nf4.storage_bytes(n, True) - (n / 2 + n * dq / 8)) < 1e-6


# ------------------------------------------------------------------ numerics
def test_e4m3_encoder_matches_torch_cast_in_range():
    rng = np.random.default_rng(4)
    v = np.concatenate([
        rng.uniform(-448, 448, 100000),
        rng.standard_normal(100000) * 2.0 ** rng.integers(-12, 8, 100000),
    ]).astype(np.float32)
    v = v[np.abs(v) <= 448]
    ours = numerics.e4m3_encode_satfinite(v)
    ref = torch.from_numpy(v).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(ours, ref)


def test_e4m3_all_codes_round_trip_and_saturate():
    codes = np.array([c for c in range(256) if (c & 0x7F) != 0x7F], dtype=np.uint8)
    vals = numerics.e4m3_decode(codes).astype(np.float32)
    back = numerics.e4m3_encode_satfinite(vals)
    assert np.array_equal(back, codes)
    sat = numerics.e4m3_encode_satfinite(np.array([449, 1e6, -500, 464], np.float32))
    assert list(sat) == [0x7E, 0x7E, 0xFE, 0x7E]


def test_bf16_rounding_matches_torch():
    rng = np.random.default_rng(5)
    x = (rng.standard_normal(100000) * 10.0 ** rng.integers(-6, 6, 100000)).astype(np.float32)
    ours = numerics.f32_to_bf16_bits(x)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, ref)


# ---------------------------------------------------------- double quantization
def test_double_quant_properties():
    w = _bf16_weight((256, 1024), 6)
    _, c = nf4.quantize(w)
    code2, s2, mu = nf4.double_quant(c)
    # the mean subtraction centres the constants
    assert abs(float(np.mean(c.astype(np.float64))) - float(mu)) <= 1e-6 * float(mu)
    cc = (c - mu).astype(np.float32)
    assert abs(float(np.mean(cc.astype(np.float64)))) < 1e-6 * float(np.max(c))
    # each 256-block's maximum lands on +-448
    for j in range(s2.size):
        seg = np.abs(cc[j * 256:(j + 1) * 256])
        k = int(np.argmax(seg))
        assert code2[j * 256 + k] & 0x7F == 0x7E
    # reconstruction error within half an E4M3 quantum (RNE) times the scale
    chat = nf4.dq_constants(code2, s2, mu)
    v = np.repeat(s2, 256)[: c.size]
    dec = numerics.e4m3_decode(code2)
    mag = np.abs(dec)
    e = np.floor(np.log2(np.maximum(mag, 2.0 ** -6)))
    half_q = np.exp2(np.maximum(e, -6) - 3) / 2
    # allow for the fp32 rounding of v = c'/s2 and of the final constant
    bound = (half_q * (1 + 2.0 ** -20) + 2.0 ** -22 * 448) * v + 2.0 ** -22 * np.abs(c)
    assert np.all(np.abs(chat.astype(np.float64) - c.astype(np.float64)) <= bound)


def test_double_quant_zero_spread_block():
    c = np.full(512, 0.25, np.float32)
    code2, s2, mu = nf4.double_quant(c)
    assert mu == np.float32(0.25) and np.all(s2 == 0) and np.all(code2 == 0)
    assert np.all(nf4.dq_constants(code2, s2, mu) == np.float32(0.25))


def test_dequant_error_bounded_by_half_gap():
    w = _bf16_weight((128, 512), 7)
    codes, c = nf4.quantize(w)
    code2, s2, mu = nf4.double_quant(c)
    wh = nf4.dequant(nf4.pack(codes), code2, s2, mu, w.size)
    chat = np.repeat(nf4.dq_constants(code2, s2, mu), 64)
    cb = np.repeat(c, 64)
    half_gap = float(np.max(np.diff(nf4.codebook().astype(np.float64)))) / 2
    err = np.abs(wh.astype(np.float64) - w.reshape(-1))
    bound = half_gap * cb + np.abs(chat - cb) + 1e-7 * cb
    assert np.all(err <= bound)


# ------------------------------------------------------------ recon error
def test_recon_error_zero_on_grid_and_bruteforce():
    q = nf4.codebook()
    rng = np.random.default_rng(8)
    # values exactly on the grid times a power-of-two absmax
    codes = rng.integers(0, 16, 512)
    codes[::64] = 15  # make sure each block reaches the absmax
    w = (q[codes] * np.float32(0.0625)).astype(np.float32).reshape(8, 64)
    assert nf4.recon_sse(w) == 0.0
    # brute force on a tiny random input with pure Python loops
    w = _bf16_weight((4, 128), 9)
    flat = [float(v) for v in w.reshape(-1)]
    qs = [float(v) for v in q]
    sse = 0.0
    for b in range(len(flat) // 64):
        seg = flat[b * 64:(b + 1) * 64]
        cb = max(abs(v) for v in seg)
        for v in seg:
            xn = float(np.float32(v) / np.float32(cb))
            k = min(range(16), key=lambda i: (abs(xn - qs[i]), i))
            wh = float(np.float32(np.float32(qs[k]) * np.float32(cb)))
            sse += (v - wh) ** 2
    assert abs(nf4.recon_sse(w) - sse) <= 1e-12 * sse
    # upper bound: n * (max half gap)^2 * max c^2
    _, c = nf4.quantize(w)
    hg = float(np.max(np.diff(q.astype(np.float64)))) / 2
    assert nf4.recon_sse(w) <= w.size * hg ** 2 * float(np.max(c)) ** 2


# ---------------------------------------------------------------------------
# AQLoRA §3.1 sparsity s_l = Pr[|W_ij| < tau], tau = 0.01
# ---------------------------------------------------------------------------
def _below_exact(vals, tau=Fraction(1, 100)):
    # brute force against the real number 0.01, each value taken exactly
    return sum(1 for v in vals if abs(Fraction(float(v))) < tau)


def test_sparsity_brute_force_against_real_tau():
    W = torch.randn(48, 128, generator=torch.Generator().manual_seed(5)) * 0.02
    Wb = W.to(torch.bfloat16).float().numpy()
    assert nf4.below_count(Wb) == _below_exact(Wb.reshape(-1))
    assert nf4.sparsity(Wb) == _below_exact(Wb.reshape(-1)) / Wb.size


def test_sparsity_at_the_bf16_neighbours_of_tau():
    # bf16 values in [2^-7, 2^-6) are multiples of 2^-14: 163 * 2^-14 < 0.01 < 164 * 2^-14
    lo, hi = 163 * 2.0 ** -14, 164 * 2.0 ** -14
    assert lo < 0.01 < hi
    vals = np.array([lo, -lo, hi, -hi, 0.0, -0.0, 0.01, 1.0], dtype=np.float32)
    vals = torch.from_numpy(vals).to(torch.bfloat16).float().numpy()
    assert vals[0] == np.float32(lo) and vals[2] == np.float32(hi)
    # lo, -lo, +0, -0 are below; hi, -hi, bf16(0.01) = hi, 1.0 are not
    assert nf4.below_count(vals) == 4 == _below_exact(vals)


def test_sparsity_special_cases():
    assert nf4.sparsity(np.zeros((4, 64), np.float32)) == 1.0
    assert nf4.sparsity(np.full((4, 64), 0.5, np.float32)) == 0.0
    assert nf4.sparsity(np.full((4, 64), -0.01, np.float32)) == 0.0  # |w| = tau is not below


def test_double_quant_sharded_on_256_block_boundaries_is_bit_identical():
    # a matrix split by rows across processes: each shard's constants start on a 256-block
    # boundary, the float64 sums of the shards add up exactly (bf16-derived constants), so
    # encoding each shard with the global mean reproduces the whole-matrix result
    W = torch.randn(24, 4096, generator=torch.Generator().manual_seed(11)) * 0.02
    flat = W.to(torch.bfloat16).float().numpy().reshape(-1)
    _, c = nf4.quantize(flat)
    code2, s2, mu = nf4.double_quant(c)
    cuts = [0, 4 * 64, 12 * 64, c.size]  # rows 0-3, 4-11, 12-23 (K / 64 = 64 constants per row)
    parts = [c[a:b] for a, b in zip(cuts[:-1], cuts[1:])]
    total = sum(math.fsum(p.astype(np.float64).tolist()) for p in parts)
    assert total == math.fsum(c.astype(np.float64).tolist())
    mu_g = np.float32(total / c.size)
    assert mu_g == mu
    got = [nf4.double_quant_with_mean(p, mu_g) for p in parts]
    assert np.array_equal(np.concatenate([g[0] for g in got]), code2)
    assert np.array_equal(np.concatenate([g[1] for g in got]), s2)
