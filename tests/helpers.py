"""Shared test plumbing: run the oracle on the same seeded bf16 inputs the GPU gets,
and move oracle-produced arrays to the device. Holds none of the method's arithmetic.
"""
from __future__ import annotations

import numpy as np
import torch

from oracle import chanq as ochq
from oracle import linear as olin
from oracle import nf4 as onf4


def f32(t: torch.Tensor) -> np.ndarray:
    """bf16 (or any) tensor -> float32 numpy array of the same values."""
    return t.detach().float().cpu().numpy()


def f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().double().cpu().numpy()


def oracle_quant(W: torch.Tensor) -> dict:
    """The oracle's NF4 + double quantization of a bf16 [N, K] weight."""
    w = f32(W)
    codes, c = onf4.quantize(w)
    code2, s2, mu = onf4.double_quant(c)
    return dict(codes=codes, absmax=c, packed=onf4.pack(codes), code2=code2, scale2=s2, mean=mu)


def oracle_base_bf16(oq: dict, N: int, K: int) -> np.ndarray:
    """bf16(W_hat) as float64 [N, K] from the oracle's quantized weight."""
    wh = onf4.dequant(oq["packed"], oq["code2"], oq["scale2"], oq["mean"], N * K)
    return olin.base_bf16(wh.reshape(N, K))


def dev(a: np.ndarray, device="cuda") -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a)).to(device)


def weight_from_oracle(q, oq: dict, N: int, K: int, device="cuda"):
    """An Nf4Weight whose buffers hold the oracle's packed codes and constants."""
    mean = np.zeros(4, np.float32)
    mean[0] = oq["mean"]
    return q.Nf4Weight(N, K, dev(oq["packed"], device), dev(oq["code2"], device),
                       dev(oq["scale2"], device), dev(mean, device)[:1])


def assert_close(got, ref, what: str, max_rel=2e-2, fro_rel=5e-3):
    ok, a, b = olin.close(got, ref, max_rel, fro_rel)
    assert ok, f"{what}: max|err|/max|ref| = {a:.3e} (<= {max_rel}), fro = {b:.3e} (<= {fro_rel})"
    return a, b


def chanq_oracle(W: torch.Tensor, bits, thr, thr_off):
    return ochq.quantize(f32(W), bits.numpy(), thr.numpy(), thr_off.numpy())
