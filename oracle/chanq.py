"""Per-output-channel threshold/mapping quantizer (LowRA-style), mixed 1/2/4 bits.

TEST INFRASTRUCTURE ONLY. Source: "LowRA" article (cloud.tencent.com.cn), §4.1:
each output channel (row of W0) has its own precision, its own bin edges
("thresholds") and its own representative values ("mappings", Fig. 3); within a row,
64-element groups are normalised by their absolute maximum as in QLoRA.

Readings (self-consistent, parity unpinned beyond the pins in the tests):
  * normalised value = IEEE fp32 division w / g; an all-zero group normalises to 0;
  * code = #{k : x_n > t_i[k]} over the row's 2^b - 1 sorted fp32 edges, so a value
    exactly on an edge goes to the lower bin;
  * the row's codes are a bit stream of b bits each, first code in the most
    significant bits of the row's first byte; each row starts on a byte boundary
    (K * b / 8 bytes per row, K a multiple of 64);
  * constants: one fp32 absmax per 64-group, no double quantization;
  * dequantized value = fp32(map_i[code] * g).
"""
from __future__ import annotations

import numpy as np

GROUP = 64


def row_offsets(bits: np.ndarray, K: int) -> np.ndarray:
    """Byte offset of each row's packed codes, plus the total as the last entry."""
    b = np.asarray(bits, dtype=np.int64)
    off = np.zeros(b.size + 1, dtype=np.int64)
    off[1:] = np.cumsum(K * b // 8)
    return off


def group_absmax(w: np.ndarray) -> np.ndarray:
    w = np.asarray(w, dtype=np.float32)
    return np.abs(w.reshape(-1, GROUP)).max(axis=1)


def encode_row(xn: np.ndarray, thr: np.ndarray) -> np.ndarray:
    """code = number of edges strictly below x_n."""
    xn = np.asarray(xn, dtype=np.float32)
    code = np.zeros(xn.shape, dtype=np.uint8)
    for t in np.asarray(thr, dtype=np.float32):
        code += (xn > t).astype(np.uint8)
    return code


def encode_row_bruteforce(xn: np.ndarray, thr: np.ndarray) -> np.ndarray:
    """The same count by sorting: position of x_n among the edges, ties to the left
    (numpy.searchsorted with side='left' counts edges strictly below)."""
    return np.searchsorted(np.asarray(thr, np.float64), np.asarray(xn, np.float64),
                           side="left").astype(np.uint8)


def pack_row(codes: np.ndarray, b: int) -> np.ndarray:
    """MSB-first bit stream of b-bit codes."""
    codes = np.asarray(codes, dtype=np.uint8)
    per = 8 // b
    c = codes.reshape(-1, per).astype(np.uint32)
    out = np.zeros(c.shape[0], dtype=np.uint32)
    for j in range(per):
        out |= c[:, j] << np.uint32(8 - b * (j + 1))
    return out.astype(np.uint8)


def unpack_row(packed: np.ndarray, b: int, K: int) -> np.ndarray:
    p = np.asarray(packed, dtype=np.uint8).astype(np.uint32)
    per = 8 // b
    mask = (1 << b) - 1
    out = np.empty((p.size, per), dtype=np.uint8)
    for j in range(per):
        out[:, j] = (p >> np.uint32(8 - b * (j + 1))) & mask
    return out.reshape(-1)[:K]


def quantize(w: np.ndarray, bits: np.ndarray, thr: np.ndarray, thr_off: np.ndarray):
    """Quantize W [N, K] row by row. Returns (packed uint8, row_off int64 [N+1],
    absmax fp32 [N*K/64], codes uint8 [N, K])."""
    w = np.asarray(w, dtype=np.float32)
    N, K = w.shape
    g = group_absmax(w)
    gg = np.repeat(g, GROUP).reshape(N, K)
    with np.errstate(invalid="ignore", divide="ignore"):
        xn = (w / gg).astype(np.float32)
    xn = np.where(gg == 0, np.float32(0.0), xn)
    roff = row_offsets(bits, K)
    packed = np.zeros(int(roff[-1]), dtype=np.uint8)
    codes = np.zeros((N, K), dtype=np.uint8)
    for i in range(N):
        b = int(bits[i])
        t = thr[int(thr_off[i]):int(thr_off[i + 1])]
        assert t.size == (1 << b) - 1
        c = encode_row(xn[i], t)
        codes[i] = c
        packed[roff[i]:roff[i + 1]] = pack_row(c, b)
    return packed, roff, g, codes


def dequant(packed, row_off, bits, maps, map_off, absmax, N: int, K: int) -> np.ndarray:
    """w_hat[i, j] = fp32(map_i[code_ij] * g) as an [N, K] fp32 array."""
    out = np.zeros((N, K), dtype=np.float32)
    g = np.asarray(absmax, dtype=np.float32).reshape(N, K // GROUP)
    for i in range(N):
        b = int(bits[i])
        c = unpack_row(packed[int(row_off[i]):int(row_off[i + 1])], b, K)
        m = np.asarray(maps[int(map_off[i]):int(map_off[i + 1])], dtype=np.float32)
        out[i] = (m[c] * np.repeat(g[i], GROUP)).astype(np.float32)
    return out
