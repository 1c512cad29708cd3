"""Multi-GPU plumbing for the hot path: one process per GPU, torch.distributed (NCCL on
GPUs) for the exchanges the path really has.

* Profiling pass ("AQLoRA", §3.1 剖析遍历, with the §3.2 choice of the layers kept in 16
  bits): the per-layer NF4 reconstruction errors are independent, so each rank computes
  those of its own layers; the ranking needs all of them, so they are all-gathered (one
  float64 per layer) and every rank ranks the same list the same way.
* Token data parallelism for the adapter training of "QLoRA: Efficient Finetuning of
  Quantized LLMs" (only A and B are trained): dA and dB are sums over tokens, so a rank
  that ran the backward on its share of the tokens all-reduces them (sum) to obtain the
  full-batch gradients; the frozen NF4 base needs no exchange.
* The same pass with the layer's sparsity s = Pr[|w| < 0.01] beside the error
  (sharded_layer_stats: two float64 per layer gathered).
* One matrix quantized as row shards ("QLoRA", 贡献二): NF4 is blockwise and local; the
  double-quantization mean needs the float64 sum of all the matrix's constants, one exact
  all-reduce of a scalar, after which each shard encodes its own constants
  (sharded_quantize_weight), bit-identical to one process.
* max_over_ranks: the timing rule of the benchmark (the slowest rank's time).

Every rank must call these functions in the same order with the same arguments' shapes.
They take an optional process group; without an initialised process group (one process)
they reduce to the local computation.
"""
from __future__ import annotations

import math
from typing import Callable, Sequence

import torch
import torch.distributed as tdist


def _world(group=None) -> tuple[int, int]:
    if not (tdist.is_available() and tdist.is_initialized()):
        return 1, 0
    return tdist.get_world_size(group), tdist.get_rank(group)


def shard(n: int, world: int, rank: int) -> list[int]:
    """The items of `rank` when n items are dealt round-robin over `world` ranks."""
    return list(range(rank, n, world))


def sharded_layer_errors(layers: Sequence[torch.Tensor],
                         sse_fn: Callable[[torch.Tensor], float] | None = None,
                         group=None, device: torch.device | None = None) -> torch.Tensor:
    """Every layer's NF4 reconstruction SSE (float64 [len(layers)], identical on all
    ranks), each computed by exactly one rank. `sse_fn` maps a bf16 weight to its SSE;
    by default the library's GPU kernel (qnf4_nf4_recon_error)."""
    world, rank = _world(group)
    if sse_fn is None:
        from . import nf4_recon_error

        def sse_fn(W):
            return float(nf4_recon_error(W).item())
    n = len(layers)
    mine = shard(n, world, rank)
    per = (n + world - 1) // world
    dev = device if device is not None else (layers[0].device if n else torch.device("cpu"))
    local = torch.zeros(per, dtype=torch.float64, device=dev)
    for i, li in enumerate(mine):
        local[i] = sse_fn(layers[li])
    if world == 1:
        return local[:n].clone()
    parts = [torch.empty_like(local) for _ in range(world)]
    tdist.all_gather(parts, local, group=group)
    out = torch.empty(n, dtype=torch.float64, device=dev)
    for r in range(world):
        for i, li in enumerate(shard(n, world, r)):
            out[li] = parts[r][i]
    return out


def sharded_layer_stats(layers: Sequence[torch.Tensor],
                        stats_fn: Callable[[torch.Tensor], Sequence[float]] | None = None,
                        group=None, device: torch.device | None = None) -> torch.Tensor:
    """Both statistics of the AQLoRA profiling pass for every layer, float64 [L, 2] =
    (reconstruction SSE, #{|w| < 0.01}), identical on all ranks, each layer computed by
    exactly one rank. `stats_fn` maps a bf16 weight to the pair; by default the library's
    one-pass GPU kernel (qnf4_nf4_layer_stats)."""
    world, rank = _world(group)
    if stats_fn is None:
        from . import nf4_layer_stats

        def stats_fn(W):
            return nf4_layer_stats(W).tolist()
    n = len(layers)
    mine = shard(n, world, rank)
    per = (n + world - 1) // world
    dev = device if device is not None else (layers[0].device if n else torch.device("cpu"))
    local = torch.zeros(per, 2, dtype=torch.float64, device=dev)
    for i, li in enumerate(mine):
        local[i] = torch.tensor([float(v) for v in stats_fn(layers[li])], dtype=torch.float64)
    if world == 1:
        return local[:n].clone()
    parts = [torch.empty_like(local) for _ in range(world)]
    tdist.all_gather(parts, local, group=group)
    out = torch.empty(n, 2, dtype=torch.float64, device=dev)
    for r in range(world):
        for i, li in enumerate(shard(n, world, r)):
            out[li] = parts[r][i]
    return out


def sharded_profile_topk(layers: Sequence[torch.Tensor], k: int,
                         sse_fn: Callable[[torch.Tensor], float] | None = None,
                         rank_fn: Callable[[list, list, int], list] | None = None,
                         group=None, device: torch.device | None = None) -> tuple[list[int], torch.Tensor]:
    """(indices of the k layers with the largest SSE per parameter, all SSEs), the same
    on every rank. `rank_fn(sse, n_params, k)` defaults to the library's host ranking
    (qnf4_rank_topk: descending error per parameter, ties to the lower index)."""
    sse = sharded_layer_errors(layers, sse_fn, group, device)
    if rank_fn is None:
        from . import rank_topk as rank_fn
    n_params = [int(W.numel()) for W in layers]
    return rank_fn(sse.cpu().tolist(), n_params, k), sse


def shard_rows(N: int, K: int, world: int, rank: int) -> tuple[int, int]:
    """Rows [r0, r1) of an [N, K] weight for `rank` when it is quantized as row shards: as
    even as possible in units of 256 / gcd(256, K / 64) rows, so that every shard's block
    constants start on a 256-constant (double-quantization block) boundary."""
    unit = 256 // math.gcd(256, K // 64)
    units = (N + unit - 1) // unit
    lo = (units * rank) // world
    hi = (units * (rank + 1)) // world
    return min(N, lo * unit), min(N, hi * unit)


def sharded_double_quant(absmax: torch.Tensor, total_count: int, group=None,
                         sum_fn: Callable | None = None, encode_fn: Callable | None = None):
    """Double quantization of this rank's row shard of one matrix ("QLoRA", 贡献二): the
    shard's float64 constant sum is all-reduced, then the shard is encoded with the
    matrix's mean. The result is bit-identical to one process when every float64 partial
    sum is exact, which holds when the constants' binades span at most
    53 - 8 - ceil(log2(count)) (8 significant bits per bf16 constant, log2(count) carry
    bits): 25 binades at 13B-layer size, far more than trained or synthetic Llama
    weights span. A matrix with both tiny and normal nonzero block maxima beyond that
    span may round its mean differently depending on the all-reduce order (all-zero
    blocks add exact zeros and do not count). `sum_fn(absmax)` -> float64 tensor [1], `encode_fn(absmax,
    total_sum, total_count)` -> (code2, scale2, mean); by default the library's qnf4_dq_sum
    and qnf4_double_quant_shard."""
    world, _ = _world(group)
    if sum_fn is None:
        from . import dq_sum as sum_fn
    if encode_fn is None:
        from . import double_quant_shard as encode_fn
    total = sum_fn(absmax)
    if world > 1:
        tdist.all_reduce(total, op=tdist.ReduceOp.SUM, group=group)
    return encode_fn(absmax, total, total_count)


def sharded_quantize_weight(W_rows: torch.Tensor, N: int, group=None):
    """NF4 + double quantization of this rank's rows (shard_rows) of an [N, K] bf16 weight:
    the rank's ``Nf4Weight`` slice (packed codes of its rows, its constants' code2 / scale2
    slices and the matrix's mean). NF4 needs no exchange; the mean needs one scalar."""
    from . import Nf4Weight, nf4_quantize
    rows, K = W_rows.shape
    packed, absmax = nf4_quantize(W_rows)
    code2, scale2, mean = sharded_double_quant(absmax, N * K // 64, group)
    return Nf4Weight(rows, K, packed, code2, scale2, mean)


def allreduce_adapter_grads(dA: torch.Tensor, dB: torch.Tensor, group=None) -> None:
    """In place: dA, dB summed over the ranks (each rank's gradients of its own tokens
    become the gradients of all the ranks' tokens)."""
    world, _ = _world(group)
    if world == 1:
        return
    tdist.all_reduce(dA, op=tdist.ReduceOp.SUM, group=group)
    tdist.all_reduce(dB, op=tdist.ReduceOp.SUM, group=group)


def max_over_ranks(x: float, device: torch.device | None = None, group=None) -> float:
    """The largest value of x over the ranks (the slowest rank's time)."""
    world, _ = _world(group)
    if world == 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64,
                     device=device if device is not None else torch.device("cpu"))
    tdist.all_reduce(t, op=tdist.ReduceOp.MAX, group=group)
    return float(t.item())
