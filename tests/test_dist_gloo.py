"""The multi-rank paths on CPU: two processes over gloo (world size 2), the exchanges of
bit_nf4_quantized_04_b200.dist checked against the single-process oracle.

* sharded profiling pass ("AQLoRA", §3.1 and the §3.2 layer choice): each rank computes the
  NF4 reconstruction SSE (and the sparsity count) of its own layers (here with the oracle),
  the results are all-gathered and both ranks must rank the same top-K as the oracle on all
  layers;
* token data parallelism (QLoRA's adapter training): each rank's dA, dB over its token
  shard, all-reduced, must equal the full-batch gradients;
* one matrix quantized as row shards ("QLoRA", 贡献二): each rank quantizes its rows, the
  float64 constant sums are all-reduced, each rank encodes its constants with the matrix's
  mean, and the concatenated codes and scales must equal the whole-matrix oracle bit for bit;
* the benchmark's timing rule: the maximum over ranks.
"""
import math
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as tdist
import torch.multiprocessing as mp

import synth

WORLD = 2


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _layers():
    # six layers of different shapes and spreads (so the ranking is not trivial)
    shapes = [(64, 128), (128, 64), (96, 192), (64, 256), (192, 64), (128, 128)]
    return [synth.llama_weight(sh, 700 + i, std=0.01 * (1 + (i * 7) % 5)) for i, sh in enumerate(shapes)]


def _shard_matrix():
    # K = 11008: 172 constants per row, shards in units of 64 rows; 150 rows -> 64 + 86
    return synth.llama_weight((150, 11008), 900, std=0.02).float().numpy()


def _grads(x, dY, Wb, A, B, s):
    from oracle import linear as olin
    _, dA, dB = olin.backward(x, dY, Wb, A, B, s)
    return dA.astype(np.float32), dB.astype(np.float32)


def _case():
    M, N, K, r = 12, 48, 64, 4
    x = synth.normal_bf16((M, K), 1.0, 801).float().numpy().astype(np.float64)
    dY = synth.normal_bf16((M, N), 1.0, 802).float().numpy().astype(np.float64)
    Wb = synth.normal_bf16((N, K), 0.02, 803).float().numpy().astype(np.float64)
    A = synth.normal_bf16((r, K), 0.01, 804).float().numpy().astype(np.float64)
    B = synth.normal_bf16((N, r), 0.01, 805).float().numpy().astype(np.float64)
    return x, dY, Wb, A, B, 2.0


def _worker(rank, port, out_dir):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    tdist.init_process_group("gloo", rank=rank, world_size=WORLD)
    try:
        from bit_nf4_quantized_04_b200 import dist
        from oracle import nf4 as onf4
        from oracle import rank as orank
        layers = _layers()
        top, sse = dist.sharded_profile_topk(
            layers, 3, sse_fn=lambda W: onf4.recon_sse(W.float().numpy()),
            rank_fn=lambda s, n, k: orank.top_k(s, n, k), device=torch.device("cpu"))
        stats = dist.sharded_layer_stats(
            layers, stats_fn=lambda W: (onf4.recon_sse(W.float().numpy()), onf4.below_count(W.float().numpy())),
            device=torch.device("cpu"))
        # one matrix quantized as row shards: local NF4, one all-reduced float64 sum
        Wm = _shard_matrix()
        N, K = Wm.shape
        r0, r1 = dist.shard_rows(N, K, WORLD, rank)
        _, c_loc = onf4.quantize(Wm[r0:r1].reshape(-1))
        code2, s2, mu = dist.sharded_double_quant(
            torch.from_numpy(c_loc), N * K // 64,
            sum_fn=lambda a: torch.tensor([math.fsum(a.double().tolist())], dtype=torch.float64),
            encode_fn=lambda a, tot, cnt: onf4.double_quant_with_mean(
                a.numpy(), np.float32(float(tot.item()) / cnt)))
        x, dY, Wb, A, B, s = _case()
        sl = slice(rank, None, WORLD)          # this rank's tokens
        dA, dB = _grads(x[sl], dY[sl], Wb, A, B, s)
        tA, tB = torch.from_numpy(dA), torch.from_numpy(dB)
        dist.allreduce_adapter_grads(tA, tB)
        mx = dist.max_over_ranks(1.0 + rank)
        np.savez(os.path.join(out_dir, f"r{rank}.npz"), top=np.array(top), sse=sse.numpy(), stats=stats.numpy(),
                 code2=code2, s2=s2, mu=np.array(mu),
                 dA=tA.numpy(), dB=tB.numpy(), mx=np.array(mx))
    finally:
        tdist.barrier()
        tdist.destroy_process_group()


def test_two_ranks_over_gloo(tmp_path):
    mp.spawn(_worker, args=(_free_port(), str(tmp_path)), nprocs=WORLD, join=True)
    res = [np.load(tmp_path / f"r{r}.npz") for r in range(WORLD)]
    from oracle import nf4 as onf4
    from oracle import rank as orank
    layers = _layers()
    sse_ref = np.array([onf4.recon_sse(W.float().numpy()) for W in layers])
    top_ref = orank.top_k(list(sse_ref), [int(W.numel()) for W in layers], 3)
    x, dY, Wb, A, B, s = _case()
    dA_ref, dB_ref = _grads(x, dY, Wb, A, B, s)
    for r in range(WORLD):
        assert np.array_equal(res[r]["sse"], sse_ref)          # each SSE computed once, gathered
        assert list(res[r]["top"]) == list(top_ref)
        # the sparsity counts travel with the errors ("AQLoRA" §3.1), each computed once
        assert np.array_equal(res[r]["stats"][:, 0], sse_ref)
        assert np.array_equal(res[r]["stats"][:, 1], [onf4.below_count(W.float().numpy()) for W in layers])
        np.testing.assert_allclose(res[r]["dA"], dA_ref, rtol=1e-5, atol=1e-6)
        np.testing.assert_allclose(res[r]["dB"], dB_ref, rtol=1e-5, atol=1e-6)
        assert float(res[r]["mx"]) == float(WORLD)
    # the row-sharded double quantization equals the whole matrix's, bit for bit
    _, c_all = onf4.quantize(_shard_matrix().reshape(-1))
    code2_ref, s2_ref, mu_ref = onf4.double_quant(c_all)
    assert np.array_equal(np.concatenate([res[r]["code2"] for r in range(WORLD)]), code2_ref)
    assert np.array_equal(np.concatenate([res[r]["s2"] for r in range(WORLD)]), s2_ref)
    assert all(np.float32(res[r]["mu"]) == mu_ref for r in range(WORLD))
    # both ranks hold bit-identical gradients after the all-reduce
    assert np.array_equal(res[0]["dA"], res[1]["dA"]) and np.array_equal(res[0]["dB"], res[1]["dB"])


def test_shard_rows_align_to_double_quant_blocks():
    from bit_nf4_quantized_04_b200.dist import shard_rows
    for N, K in ((150, 11008), (4096, 4096), (11008, 4096), (7, 64), (1, 128)):
        unit = 256 // math.gcd(256, K // 64)
        for world in (1, 2, 3, 8):
            spans = [shard_rows(N, K, world, r) for r in range(world)]
            assert spans[0][0] == 0 and spans[-1][1] == N
            for (a, b), (c, _) in zip(spans[:-1], spans[1:]):
                assert b == c and a <= b
                assert (b * K // 64) % 256 == 0  # every later shard starts on a DQ block


def test_shard_covers_every_item_once():
    from bit_nf4_quantized_04_b200.dist import shard
    for n in (0, 1, 5, 6, 7):
        for world in (1, 2, 3, 4):
            got = sorted(i for r in range(world) for i in shard(n, world, r))
            assert got == list(range(n))


def test_single_process_reduces_to_local():
    from bit_nf4_quantized_04_b200 import dist
    from oracle import nf4 as onf4
    layers = _layers()[:3]
    sse = dist.sharded_layer_errors(layers, sse_fn=lambda W: onf4.recon_sse(W.float().numpy()),
                                    device=torch.device("cpu"))
    assert np.array_equal(sse.numpy(), [onf4.recon_sse(W.float().numpy()) for W in layers])
    assert dist.max_over_ranks(3.5) == 3.5
