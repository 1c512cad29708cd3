"""GPU parity of the forward at decode sizes (M <= 16 tokens) against the float64 oracle.

Every token count of one and two 8-token groups, ragged N (a partial last row tile),
K that is not a multiple of 256, long K (up to 65536), ranks 1..64, repeated calls on
one workspace with bit-for-bit repeatability, and the zero-adapter invariance.
Tolerance as in the other linear tests: max|err| <= 2e-2 max|ref|, relative Frobenius
error <= 5e-3, over every output element.
"""
import numpy as np
import pytest
import torch

import synth
from oracle import linear as olin

from helpers import assert_close, f64, oracle_base_bf16, oracle_quant, weight_from_oracle

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def q():
    import bit_nf4_quantized_04_b200 as q
    return q


def _case(N, K, M, r, seed):
    W = synth.llama_weight((N, K), seed, std=0.02)
    x = synth.normal_bf16((M, K), 1.0, seed + 1)
    A = synth.normal_bf16((r, K), 0.01, seed + 2)
    B = synth.normal_bf16((N, r), 0.01, seed + 3)
    oq = oracle_quant(W)
    Wb = oracle_base_bf16(oq, N, K)
    s = 16.0 / r
    href = olin.forward(f64(x), Wb, f64(A), f64(B), s)
    return oq, x, A, B, s, href


@pytest.mark.parametrize("N,K,M,r", [
    (16, 64, 1, 1),        # one tile, one block, one token
    (40, 448, 2, 5),       # ragged N, 7 blocks (partial group)
    (200, 192, 7, 16),
    (136, 1024, 8, 8),     # full first column tile
    (264, 960, 9, 16),     # second column tile with one token
    (520, 2048, 15, 33),
    (1000, 4096, 16, 64),
    (48, 8192, 12, 16),
    (24, 16384, 16, 4),
    (72, 16384, 5, 16),
    (40, 65536, 1, 16),
    (160000, 64, 1, 4),    # many row tiles, one column block
])
def test_decode_parity(q, N, K, M, r):
    oq, x, A, B, s, href = _case(N, K, M, r, seed=N + 3 * K + 7 * M + r)
    w = weight_from_oracle(q, oq, N, K)
    h = q.qlora_linear_fwd(w, x.cuda(), A.cuda(), B.cuda(), s)
    assert_close(f64(h.cpu()), href, f"decode h N={N} K={K} M={M} r={r}")


def test_decode_repeatable_and_workspace_reuse(q):
    # two shapes alternating on one workspace: counters and partial tiles of one call
    # must not leak into the next, and the ordered split-K reduction gives identical bits
    cases = [_case(1000, 4096, 16, 16, 71), _case(300, 1216, 3, 8, 72)]
    ws = torch.empty(max(q.workspace_size(q._lib.OP_FWD, 1000, 4096, 16, 16),
                         q.workspace_size(q._lib.OP_FWD, 300, 1216, 3, 8)),
                     dtype=torch.uint8, device="cuda")
    shapes = [(1000, 4096), (300, 1216)]
    ws_list = [weight_from_oracle(q, c[0], N, K) for c, (N, K) in zip(cases, shapes)]
    outs = {0: [], 1: []}
    for rep in range(3):
        for i, (oq, x, A, B, s, href) in enumerate(cases):
            h = q.qlora_linear_fwd(ws_list[i], x.cuda(), A.cuda(), B.cuda(), s, ws=ws)
            outs[i].append(h.clone())
    torch.cuda.synchronize()
    for i, (oq, x, A, B, s, href) in enumerate(cases):
        assert_close(f64(outs[i][0].cpu()), href, f"case {i}")
        for h in outs[i][1:]:
            assert torch.equal(h, outs[i][0])


def test_decode_zero_adapter_is_base_only(q):
    N, K, M, r = 256, 512, 5, 8
    W = synth.llama_weight((N, K), 31, std=0.02)
    x = synth.normal_bf16((M, K), 1.0, 32)
    A = synth.normal_bf16((r, K), 0.01, 33)
    B = synth.normal_bf16((N, r), 0.01, 34)
    w = q.quantize_weight(W.cuda())
    h0 = q.qlora_linear_fwd(w, x.cuda(), A.cuda(), torch.zeros_like(B).cuda(), 2.0)
    h1 = q.qlora_linear_fwd(w, x.cuda(), torch.zeros_like(A).cuda(), B.cuda(), 2.0)
    assert torch.equal(h0, h1)


def test_decode_long_k(q):
    N, K, M, r = 64, 16640, 16, 16
    oq, x, A, B, s, href = _case(N, K, M, r, seed=5)
    w = weight_from_oracle(q, oq, N, K)
    h = q.qlora_linear_fwd(w, x.cuda(), A.cuda(), B.cuda(), s)
    assert_close(f64(h.cpu()), href, "h at K = 16640")


def test_group_matches_single_calls_bit_exactly(q):
    """n independent layers in one grouped launch give exactly the single calls' outputs
    (each row's arithmetic is the same), and one layer is checked against the oracle."""
    shapes = [(520, 2048), (40, 448), (1000, 4096), (264, 960), (200, 192), (136, 1024), (16, 64)]
    for M in (1, 5, 16):
        cases = [_case(N, K, M, 16, seed=900 + 7 * i + M) for i, (N, K) in enumerate(shapes)]
        ws_ = [weight_from_oracle(q, c[0], N, K) for c, (N, K) in zip(cases, shapes)]
        xs = [c[1].cuda() for c in cases]
        As = [c[2].cuda() for c in cases]
        Bs = [c[3].cuda() for c in cases]
        s = cases[0][4]
        single = [q.qlora_linear_fwd(w, x, A, B, s) for w, x, A, B in zip(ws_, xs, As, Bs)]
        group = q.qlora_linear_fwd_group(ws_, xs, As, Bs, s)
        torch.cuda.synchronize()
        for i, (a, b) in enumerate(zip(single, group)):
            assert torch.equal(a, b), f"layer {i} M={M}: grouped output differs from the single call"
        assert_close(f64(group[2].cpu()), cases[2][5], f"group layer 2 M={M}")


def test_group_llama7b_layer_set(q):
    """The 7B layer set (q, k, v, o, gate, up, down) at 4 tokens in one launch against
    the single calls, bit for bit."""
    ws_, xs, As, Bs = [], [], [], []
    for i, s_ in enumerate(synth.LLAMA7B_SET):
        W = synth.llama_weight((s_.N, s_.K), 3100 + i, device="cuda")
        ws_.append(q.quantize_weight(W))
        xs.append(synth.normal_bf16((4, s_.K), 1.0, 3200 + i, device="cuda"))
        As.append(synth.normal_bf16((16, s_.K), 0.01, 3300 + i, device="cuda"))
        Bs.append(synth.normal_bf16((s_.N, 16), 0.01, 3400 + i, device="cuda"))
    single = [q.qlora_linear_fwd(w, x, A, B, 2.0) for w, x, A, B in zip(ws_, xs, As, Bs)]
    group = q.qlora_linear_fwd_group(ws_, xs, As, Bs, 2.0)
    torch.cuda.synchronize()
    for i, (a, b) in enumerate(zip(single, group)):
        assert torch.equal(a, b), f"layer {i}"
