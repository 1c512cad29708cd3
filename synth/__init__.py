"""Seeded synthetic inputs shared by the CPU oracle's tests and the CUDA path.

This module only draws random numbers and shapes them into the workloads' tensors.
It contains none of the quantizer's or the linear layer's arithmetic, so both the
oracle and the GPU library can consume the same bytes without sharing method code.

Every tensor is sampled in fp32 with ``torch.Generator`` and cast to bf16 (torch's
cast rounds to nearest even). Seeds: weight matrix i -> 1000 + i, activations -> 2000,
LoRA A -> 3000, LoRA B -> 3001, upstream gradient dY -> 4000, per-channel bit widths
and tables -> 5000.

Workloads (all Llama-shaped, as the pages' experiments use Llama-2 checkpoints that
are not available here):
  * tiny: one 256x512 layer, 16 tokens, r=8, alpha=16;
  * llama2-7b layer set: q/k/v/o 4096x4096, gate/up 11008x4096, down 4096x11008;
    weights N(0, 0.02) with 0.1% entries replaced by Student-t(3) * 0.02 outliers;
  * llama2-13b stack: 40 x {5120^2 x4, 13824x5120 x2, 5120x13824}, per-matrix std
    drawn from U[0.01, 0.04];
  * per-channel mixed precision: 11008x4096 with bit widths {1,2,4} in exact counts
    3302/5504/2202 assigned by a seeded permutation.
"""
from __future__ import annotations

import math
from dataclasses import dataclass

import torch

SEED_W = 1000
SEED_X = 2000
SEED_A = 3000
SEED_B = 3001
SEED_DY = 4000
SEED_CHAN = 5000


def _gen(seed: int, device="cpu") -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def normal_bf16(shape, std: float, seed: int, device="cpu") -> torch.Tensor:
    """N(0, std^2) sampled in fp32, cast to bf16 (round to nearest even)."""
    g = _gen(seed, device)
    t = torch.randn(*shape, generator=g, device=device, dtype=torch.float32)
    return (t * std).to(torch.bfloat16)


def llama_weight(shape, seed: int, std: float = 0.02, outlier_frac: float = 0.001,
                 device="cpu") -> torch.Tensor:
    """Gaussian weight with floor(outlier_frac * n) entries replaced by t_3 * std.

    The Student-t(3) draws are z / sqrt(chi2_3 / 3), all from the same generator.
    """
    g = _gen(seed, device)
    n = int(shape[0]) * int(shape[1])
    w = torch.randn(n, generator=g, device=device, dtype=torch.float32) * std
    n_out = int(math.floor(outlier_frac * n))
    if n_out > 0:
        pos = torch.randperm(n, generator=g, device=device)[:n_out]
        z = torch.randn(n_out, generator=g, device=device, dtype=torch.float32)
        chi = torch.randn(n_out, 3, generator=g, device=device, dtype=torch.float32).pow(2).sum(1)
        t3 = z / torch.sqrt(chi / 3.0)
        w[pos] = t3 * std
    return w.view(int(shape[0]), int(shape[1])).to(torch.bfloat16)


@dataclass(frozen=True)
class LayerShape:
    name: str
    N: int  # output features (rows of W0)
    K: int  # input features (columns of W0)


LLAMA7B_SET = (
    LayerShape("q_proj", 4096, 4096),
    LayerShape("k_proj", 4096, 4096),
    LayerShape("v_proj", 4096, 4096),
    LayerShape("o_proj", 4096, 4096),
    LayerShape("gate_proj", 11008, 4096),
    LayerShape("up_proj", 11008, 4096),
    LayerShape("down_proj", 4096, 11008),
)

LLAMA13B_LAYER = (
    LayerShape("q_proj", 5120, 5120),
    LayerShape("k_proj", 5120, 5120),
    LayerShape("v_proj", 5120, 5120),
    LayerShape("o_proj", 5120, 5120),
    LayerShape("gate_proj", 13824, 5120),
    LayerShape("up_proj", 13824, 5120),
    LayerShape("down_proj", 5120, 13824),
)
LLAMA13B_LAYERS = 40


def llama13b_stack():
    """The 280 (layer, matrix) shapes of the 13B stack, in layer-major order."""
    out = []
    for layer in range(LLAMA13B_LAYERS):
        for s in LLAMA13B_LAYER:
            out.append(LayerShape(f"layers.{layer}.{s.name}", s.N, s.K))
    return out


def llama13b_stds(seed: int = SEED_W) -> torch.Tensor:
    """Per-matrix standard deviations for the 13B stack, U[0.01, 0.04], float64."""
    g = _gen(seed + 7)
    u = torch.rand(LLAMA13B_LAYERS * len(LLAMA13B_LAYER), generator=g, dtype=torch.float64)
    return 0.01 + 0.03 * u


def tiny_inputs(device="cpu"):
    """The single tiny layer: W 256x512, x 16x512, r=8, alpha=16, dY 16x256."""
    N, K, M, r = 256, 512, 16, 8
    return dict(
        W=normal_bf16((N, K), 0.02, SEED_W, device),
        x=normal_bf16((M, K), 1.0, SEED_X, device),
        A=normal_bf16((r, K), 0.01, SEED_A, device),
        B=normal_bf16((N, r), 0.01, SEED_B, device),
        dY=normal_bf16((M, N), 1.0, SEED_DY, device),
        r=r, alpha=16.0,
    )


def activations(M: int, K: int, seed: int = SEED_X, device="cpu") -> torch.Tensor:
    return normal_bf16((M, K), 1.0, seed, device)


def lora_pair(N: int, K: int, r: int, device="cpu", std: float = 0.01):
    return (normal_bf16((r, K), std, SEED_A, device),
            normal_bf16((N, r), std, SEED_B, device))


def chan_bits(N: int, counts=None, seed: int = SEED_CHAN) -> torch.Tensor:
    """Per-row bit widths in {1, 2, 4}: exact counts placed by a seeded permutation.

    The default counts 3302 / 5504 / 2202 are 0.3 / 0.5 / 0.2 of 11008 rows; other N
    scale the fractions and give the remainder to the 2-bit class.
    """
    if counts is None:
        c1 = int(round(0.3 * N)); c4 = int(round(0.2 * N)); c2 = N - c1 - c4
        counts = (c1, c2, c4)
    c1, c2, c4 = counts
    assert c1 + c2 + c4 == N
    base = torch.cat([torch.full((c1,), 1), torch.full((c2,), 2), torch.full((c4,), 4)]).to(torch.uint8)
    perm = torch.randperm(N, generator=_gen(seed))
    return base[perm].contiguous()


def chan_tables(bits: torch.Tensor, seed: int = SEED_CHAN + 1):
    """Seeded per-row mapping values and bin edges for the per-channel quantizer.

    Row i with b bits gets 2^b mapping values: sorted draws from N(0, 0.45^2) clipped
    to [-1, 1] with the two outermost forced to -1 and +1 (so every normalized value
    in [-1, 1] has a bin), and 2^b - 1 edges at the fp32 midpoints of neighbouring
    mappings. These stand in for a per-channel learned table; the kernels take any
    sorted fp32 tables as inputs.

    Returns (maps fp32 [sum 2^b], map_off int64 [N+1], thr fp32 [sum 2^b - 1],
    thr_off int64 [N+1]).
    """
    g = _gen(seed)
    N = bits.numel()
    maps, thrs = [], []
    map_off = torch.zeros(N + 1, dtype=torch.int64)
    thr_off = torch.zeros(N + 1, dtype=torch.int64)
    for i in range(N):
        b = int(bits[i])
        L = 1 << b
        v = (torch.randn(L, generator=g, dtype=torch.float32) * 0.45).clamp(-1.0, 1.0)
        v, _ = torch.sort(v)
        v[0] = -1.0
        v[-1] = 1.0
        if L > 2:
            # keep the mappings strictly increasing
            for j in range(1, L):
                if not v[j] > v[j - 1]:
                    v[j] = torch.nextafter(v[j - 1], torch.tensor(2.0))
        t = ((v[1:].double() + v[:-1].double()) * 0.5).float()
        maps.append(v)
        thrs.append(t)
        map_off[i + 1] = map_off[i] + L
        thr_off[i + 1] = thr_off[i] + (L - 1)
    return torch.cat(maps), map_off, torch.cat(thrs), thr_off
