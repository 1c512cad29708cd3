"""NF4 codebook, blockwise quantization, double quantization and dequantization.

TEST INFRASTRUCTURE ONLY (see the package docstring). Source: "QLoRA: Efficient
Finetuning of Quantized LLMs" (Heng's Blog), sections 贡献一 4-bit NormalFloat (NF4)
and 贡献二 Double Quantization; "AQLoRA", §3.1 for the reconstruction error and the
sparsity of a layer.

Readings of points the page leaves open (each is a convention, self-consistent on
both sides of the parity tests):
  * quantile grid: 9 evenly spaced probabilities from P_MAX down to 0.5 on the
    positive side and 8 on the negative side, P_MAX = 1 - (1/32 + 1/30) / 2; the
    union without the duplicate 0, divided by the largest magnitude (so the ends
    are exactly -1 and +1), rounded once to fp32. Parity unpinned for P_MAX.
  * nearest level with exact ties going to the lower index (decision thresholds
    are the smallest fp32 strictly above each exact midpoint);
  * normalised value = IEEE fp32 division w / absmax; an all-zero block stores
    absmax 0 and code 7 (the exact-zero level) for all its elements;
  * flattening is row-major; element 2j of the flattened weight goes in the high
    nibble of byte j, element 2j+1 in the low nibble (parity unpinned);
  * double quantization: one fp32 mean per tensor (float64 sum / count), OCP E4M3
    codes with round-to-nearest-even and saturation, block scale absmax2 / 448
    (the block maximum lands on the format maximum). A 256-block whose
    mean-subtracted constants are all zero stores scale 0 and code 0. The 8-bit
    float format is a reading: parity unpinned beyond self-consistency.
"""
from __future__ import annotations

import math
from statistics import NormalDist

import numpy as np

from .numerics import e4m3_decode, e4m3_encode_satfinite

BLOCK1 = 64
BLOCK2 = 256
P_MAX = 1.0 - 0.5 * (1.0 / 32.0 + 1.0 / 30.0)
FP8_MAX = np.float32(448.0)


# ---------------------------------------------------------------------------
# codebook (贡献一: 16 values from standard-normal quantiles, 8 + 9 - 1)
# ---------------------------------------------------------------------------
def codebook_f64() -> np.ndarray:
    """The 16 NF4 levels in float64, sorted ascending (before fp32 rounding)."""
    nd = NormalDist()
    pos_p = np.linspace(P_MAX, 0.5, 9)   # 8 positive quantiles and the median
    neg_p = np.linspace(P_MAX, 0.5, 8)   # 7 negative quantiles and the median
    pos = [nd.inv_cdf(float(p)) for p in pos_p]
    neg = [-nd.inv_cdf(float(p)) for p in neg_p]
    # the median appears in both sets; keep one exact zero
    vals = [v for v in pos if v != 0.0] + [v for v in neg if v != 0.0] + [0.0]
    vals = np.array(sorted(vals), dtype=np.float64)
    assert vals.size == 16
    return vals / nd.inv_cdf(P_MAX)


def codebook() -> np.ndarray:
    """The 16 NF4 levels as fp32 (rounded once from float64)."""
    return codebook_f64().astype(np.float32)


def thresholds(levels: np.ndarray | None = None) -> np.ndarray:
    """15 fp32 decision thresholds: T[k] = smallest fp32 strictly above the exact
    midpoint of levels k and k+1, so that code = #{k : x >= T[k]} picks the nearest
    level with exact ties going to the lower index."""
    q = codebook() if levels is None else np.asarray(levels, dtype=np.float32)
    out = np.empty(15, dtype=np.float32)
    for k in range(15):
        m = (float(q[k]) + float(q[k + 1])) / 2.0  # exact: sum of two fp32 in float64
        f = np.float32(m)
        if float(f) <= m:
            f = np.nextafter(f, np.float32(np.inf))
        out[k] = f
    return out


def encode(xn: np.ndarray, T: np.ndarray | None = None) -> np.ndarray:
    """Code of each normalised fp32 value: the number of thresholds at or below it."""
    T = thresholds() if T is None else T
    xn = np.asarray(xn, dtype=np.float32)
    code = np.zeros(xn.shape, dtype=np.uint8)
    for k in range(15):
        code += (xn >= T[k]).astype(np.uint8)
    return code


def encode_bruteforce(xn: np.ndarray, levels: np.ndarray | None = None) -> np.ndarray:
    """Nearest level by exhaustive float64 search; ties go to the lower index."""
    q = (codebook() if levels is None else levels).astype(np.float64)
    d = np.abs(np.asarray(xn, dtype=np.float64)[..., None] - q)
    return np.argmin(d, axis=-1).astype(np.uint8)  # argmin returns the first minimum


# ---------------------------------------------------------------------------
# first-level blockwise quantization
# ---------------------------------------------------------------------------
def block_absmax(w: np.ndarray, block: int = BLOCK1) -> np.ndarray:
    """Absolute maximum of each block of the row-major flattened weight (fp32).

    A partial last block takes the maximum over the elements present."""
    flat = np.asarray(w, dtype=np.float32).reshape(-1)
    n = flat.size
    nb = (n + block - 1) // block
    pad = np.zeros(nb * block, dtype=np.float32)
    pad[:n] = np.abs(flat)
    return pad.reshape(nb, block).max(axis=1)


def normalise(w: np.ndarray, absmax: np.ndarray, block: int = BLOCK1) -> np.ndarray:
    """x_n = fp32(w / c_b) by IEEE fp32 division; zero for an all-zero block."""
    flat = np.asarray(w, dtype=np.float32).reshape(-1)
    c = np.repeat(np.asarray(absmax, dtype=np.float32), block)[: flat.size]
    with np.errstate(invalid="ignore", divide="ignore"):
        xn = flat / c
    return np.where(c == 0, np.float32(0.0), xn).astype(np.float32)


def quantize(w: np.ndarray, block: int = BLOCK1):
    """Blockwise NF4 quantization of a bf16-valued weight (given as float32).

    Returns (codes uint8 [n], absmax fp32 [nb1]). Codes are in flattened order."""
    c = block_absmax(w, block)
    codes = encode(normalise(w, c, block))
    return codes, c


def pack(codes: np.ndarray) -> np.ndarray:
    """Two codes per byte: element 2j in the high nibble, 2j+1 in the low nibble."""
    codes = np.asarray(codes, dtype=np.uint8).reshape(-1)
    if codes.size % 2:
        codes = np.concatenate([codes, np.zeros(1, np.uint8)])
    return ((codes[0::2] << 4) | codes[1::2]).astype(np.uint8)


def unpack(packed: np.ndarray, n: int) -> np.ndarray:
    p = np.asarray(packed, dtype=np.uint8).reshape(-1)
    out = np.empty(p.size * 2, dtype=np.uint8)
    out[0::2] = p >> 4
    out[1::2] = p & 0xF
    return out[:n]


# ---------------------------------------------------------------------------
# double quantization (贡献二)
# ---------------------------------------------------------------------------
def dq_mean(absmax: np.ndarray) -> np.float32:
    """One fp32 mean per tensor: the float64 sum of the constants over their count."""
    c = np.asarray(absmax, dtype=np.float32).astype(np.float64)
    s = math.fsum(c.tolist())
    return np.float32(s / c.size)


def double_quant(absmax: np.ndarray, block2: int = BLOCK2):
    """Quantize the first-level constants to 8-bit floats in blocks of 256.

    Subtract the tensor mean (the constants are all positive), scale each block by
    its absolute maximum so it lands on the E4M3 maximum 448, encode with
    round-to-nearest-even. Returns (code2 uint8 [nb1], scale2 fp32 [nb2], mean fp32).
    """
    c = np.asarray(absmax, dtype=np.float32)
    return double_quant_with_mean(c, dq_mean(c), block2)


def double_quant_with_mean(absmax: np.ndarray, mu, block2: int = BLOCK2):
    """The encoding step of double_quant with the tensor mean given: what one shard of a
    matrix split across processes does once the mean of all its constants is known (its
    first constant on a 256-block boundary)."""
    c = np.asarray(absmax, dtype=np.float32)
    mu = np.float32(mu)
    nb1 = c.size
    nb2 = (nb1 + block2 - 1) // block2
    cc = (c - mu).astype(np.float32)  # fp32 subtraction
    code2 = np.zeros(nb1, dtype=np.uint8)
    s2 = np.zeros(nb2, dtype=np.float32)
    for j in range(nb2):
        seg = cc[j * block2:(j + 1) * block2]
        a2 = np.float32(np.max(np.abs(seg)))
        if a2 == 0:
            s2[j] = 0.0
            continue
        sc = np.float32(a2 / FP8_MAX)  # IEEE fp32 division
        s2[j] = sc
        v = (seg / sc).astype(np.float32)  # IEEE fp32 division
        code2[j * block2:(j + 1) * block2] = e4m3_encode_satfinite(v)
    return code2, s2, mu


def dq_constants(code2: np.ndarray, scale2: np.ndarray, mean, block2: int = BLOCK2) -> np.ndarray:
    """Reconstructed first-level constants: fp32(e4m3(code2) * scale2 + mean)."""
    e = e4m3_decode(code2)
    s = np.repeat(np.asarray(scale2, dtype=np.float32).astype(np.float64), block2)[: e.size]
    return (e * s + np.float64(np.float32(mean))).astype(np.float32)


def dequant(packed: np.ndarray, code2: np.ndarray, scale2: np.ndarray, mean, n: int,
            block1: int = BLOCK1, block2: int = BLOCK2) -> np.ndarray:
    """Two-level dequantization to fp32: w_hat = fp32(q[code] * c_hat_b), flattened."""
    q = codebook()
    codes = unpack(packed, n)
    chat = dq_constants(code2, scale2, mean, block2)
    cb = np.repeat(chat, block1)[:n]
    return (q[codes] * cb).astype(np.float32)


def dequant_single(codes: np.ndarray, absmax: np.ndarray, block1: int = BLOCK1) -> np.ndarray:
    """Single-level dequantization (no double quantization): fp32(q[code] * c_b)."""
    q = codebook()
    cb = np.repeat(np.asarray(absmax, dtype=np.float32), block1)[: codes.size]
    return (q[codes] * cb).astype(np.float32)


# ---------------------------------------------------------------------------
# AQLoRA §3.1: per-layer blockwise NF4 reconstruction error
# ---------------------------------------------------------------------------
def recon_sse(w: np.ndarray, block1: int = BLOCK1) -> float:
    """Sum over blocks of the squared error between each block and its single-level
    absmax-NF4 round trip (fp32 dequant values, float64 accumulation)."""
    flat = np.asarray(w, dtype=np.float32).reshape(-1)
    codes, c = quantize(flat, block1)
    what = dequant_single(codes, c, block1)
    d = flat.astype(np.float64) - what.astype(np.float64)
    return float(np.dot(d, d))


def recon_error(w: np.ndarray, block1: int = BLOCK1) -> float:
    """epsilon_l = SSE_l / |W_l|."""
    return recon_sse(w, block1) / np.asarray(w).size


# AQLoRA §3.1: the layer's sparsity s_l = Pr[|W_ij| < tau] with tau = 0.01. The threshold
# is taken as the fp32 value of tau (the form the kernels receive); for bf16 weights that
# is the same test as against the real 0.01, since no bf16 value lies between the two.
SPARSITY_TAU = np.float32(0.01)


def below_count(w: np.ndarray, tau=SPARSITY_TAU) -> int:
    """#{elements with |w| < tau}, tau given as fp32."""
    a = np.abs(np.asarray(w, dtype=np.float64).reshape(-1))
    return int(np.count_nonzero(a < float(np.float32(tau))))


def sparsity(w: np.ndarray, tau=SPARSITY_TAU) -> float:
    """s_l = below_count / |W_l|."""
    return below_count(w, tau) / np.asarray(w).size


# ---------------------------------------------------------------------------
# storage cost (贡献二: 0.5 bit/param of constants before DQ, ~0.127 after)
# ---------------------------------------------------------------------------
def storage_bytes(n: int, double_quant_on: bool, block1: int = BLOCK1, block2: int = BLOCK2) -> float:
    """Bytes to store n parameters: 4-bit codes plus the quantization constants."""
    codes = n / 2
    nb1 = n / block1
    if not double_quant_on:
        return codes + 4 * nb1
    return codes + nb1 + 4 * nb1 / block2


def constant_bits_per_param(double_quant_on: bool, block1: int = BLOCK1, block2: int = BLOCK2) -> float:
    n = float(block1 * block2)
    return 8.0 * (storage_bytes(n, double_quant_on, block1, block2) - n / 2) / n
