"""GPU parity of the bandwidth kernels against the CPU oracle, element by element:
NF4 codes and packed bytes, block constants, double-quantization codes/scales/mean
(bit-exact), two-level dequantization (fp32 within 1e-6 relative, bf16 exact) and
the AQLoRA reconstruction error (1e-5 relative), on the tiny layer, ragged shapes and
full Llama-2-7B matrix shapes.
"""
import numpy as np
import pytest
import torch

import synth
from oracle import nf4 as onf4
from oracle import numerics as onum

from helpers import dev, f32, oracle_quant, weight_from_oracle

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def q():
    import bit_nf4_quantized_04_b200 as q
    return q


def _check_quant(q, W):
    N, K = W.shape
    oq = oracle_quant(W)
    packed, absmax = q.nf4_quantize(W.cuda())
    torch.cuda.synchronize()
    assert np.array_equal(absmax.cpu().numpy().view(np.uint32), oq["absmax"].view(np.uint32))
    got = packed.cpu().numpy()
    if not np.array_equal(got, oq["packed"]):
        bad = np.nonzero(got != oq["packed"])[0]
        raise AssertionError(f"{bad.size} packed bytes differ, first at {bad[:5]}")
    return oq


def _crafted(N, K, seed):
    g = torch.Generator().manual_seed(seed)
    w = torch.randn(N, K, generator=g) * 0.02
    flat = w.view(-1)
    if flat.numel() >= 64:
        flat[0:64] = 0.0                      # all-zero block
    if flat.numel() >= 128:
        flat[64:128] = 0.03125                # identical values
    if flat.numel() >= 192:
        flat[128:160] = -1e-30                # tiny constants (absmax < 2^-64: the
        flat[130] = 1e-30                     # kernels decide on scaled values)
        flat[160:192] = 3e-33
    if flat.numel() >= 256:
        q = torch.tensor(onf4.codebook())     # values on the grid and at midpoints
        mid = (q[1:] + q[:-1]) / 2
        blk = torch.cat([q, mid, q[:16] * 0.5, mid[:15] * 0.25, torch.tensor([1.0, -1.0])])[:64]
        flat[192:256] = blk * 0.5
    return w.to(torch.bfloat16)


def _near_threshold_blocks(nblocks, seed):
    """bf16 blocks whose normalised values w / absmax fall within 2^-19 of an NF4
    decision threshold (found by search over the bf16 grid): the values where a
    rounding slip in the kernels' division-free decision would show."""
    T = onf4.thresholds().astype(np.float64)
    rng = np.random.default_rng(seed)
    mant = np.arange(128, dtype=np.uint32)
    bf = lambda e: ((np.uint32(127 + e) << 23) | (mant << 16)).view(np.float32)  # noqa: E731
    cands = []
    for c in bf(-5)[::3]:                      # absmax values in [1/32, 1/16)
        ws = np.concatenate([bf(e) for e in range(-13, -4)])
        ws = ws[ws <= c]
        ws = np.concatenate([ws, -ws])
        x = (ws / np.float32(c)).astype(np.float32).astype(np.float64)
        d = np.min(np.abs(x[:, None] - T[None, :]), axis=1)
        for w in ws[d <= 2.0 ** -19]:
            cands.append((np.float32(c), np.float32(w)))
    assert len(cands) > 0
    out = np.zeros((nblocks, 64), np.float32)
    for i in range(nblocks):
        c, w0 = cands[rng.integers(len(cands))]
        blk = [c] + [cands[rng.integers(len(cands))][1] for _ in range(63)]
        # keep absmax = c: drop values whose magnitude exceeds it
        blk = [v if abs(v) <= c else np.float32(0) for v in blk]
        out[i] = rng.permutation(np.array(blk, np.float32))
    return torch.from_numpy(out.reshape(-1, 128 if nblocks % 2 == 0 else 64)).to(torch.bfloat16)


def test_quantize_near_thresholds(q):
    W = _near_threshold_blocks(64, 11)
    assert np.array_equal(f32(W), f32(W).astype(np.float32))
    _check_quant(q, W)


def _exhaustive_blocks(cbits_list):
    """For each bf16 block constant c (given by its bit pattern), every bf16 value w with
    |w| <= c, both signs and zero, in blocks of 63 such values plus c itself."""
    blocks = []
    for cb in cbits_list:
        mags = np.arange(1, cb + 1, dtype=np.uint32)
        ws = np.concatenate([mags, mags | 0x8000, [0]]).astype(np.uint32)
        ws = (ws << 16).view(np.float32)
        pad = (-ws.size) % 63
        ws = np.concatenate([ws, np.zeros(pad, np.float32)]).reshape(-1, 63)
        c = np.full((ws.shape[0], 1), (np.uint32(cb) << 16).view(np.float32))
        blk = np.concatenate([ws, c], axis=1)
        for i in range(blk.shape[0]):  # move c around the block
            j = i % 64
            blk[i, [j, 63]] = blk[i, [63, j]]
        blocks.append(blk)
    out = np.concatenate(blocks)
    if out.shape[0] % 2:
        out = np.concatenate([out, np.zeros((1, 64), np.float32)])
    return torch.from_numpy(out.reshape(-1, 128)).to(torch.bfloat16)


def test_quantize_every_bf16_value_under_chosen_constants(q):
    """Brute force over the bf16 grid: under each block constant c below, every value
    |w| <= c is coded, and the codes must equal the oracle's IEEE division and threshold
    count. The constants span subnormals, the scaling edges at 2^-64 and 2^64, 1, and
    the largest finite bf16, plus random patterns."""
    rng = np.random.default_rng(123)
    cbits = [0x0001, 0x0055, 0x0080, 0x0D2B, 0x1F7F, 0x1F80, 0x1F81, 0x3C80, 0x3D4C, 0x3F80,
             0x3FC0, 0x4000, 0x5F7F, 0x5F80, 0x5FFF, 0x7E80, 0x7F00, 0x7F7F]
    cbits += [int(v) for v in rng.integers(1, 0x7F80, 14)]
    W = _exhaustive_blocks(cbits)
    assert np.array_equal(f32(W), f32(W).astype(np.float32))
    _check_quant(q, W)


def test_quantize_non_finite_blocks(q):
    """Blocks holding an infinity or a NaN: the codes are those of the IEEE quotient
    (a finite w over an infinite constant gives a signed zero, code 7; inf / inf and NaN
    give code 0), the block constant is the infinity or a NaN."""
    g = torch.Generator().manual_seed(5)
    w = (torch.randn(8, 64, generator=g) * 0.5)
    w[0, 3] = float("inf")
    w[1, 0] = float("-inf")
    w[2, 10], w[2, 20] = float("inf"), float("-inf")
    w[3, 7] = float("nan")
    w[4, :] = float("nan")
    w[5, 63] = float("inf")
    w[5, 0] = float("nan")
    W = w.reshape(4, 128).to(torch.bfloat16)
    codes, b = onf4.quantize(f32(W))
    packed, absmax = q.nf4_quantize(W.cuda())
    torch.cuda.synchronize()
    assert np.array_equal(packed.cpu().numpy(), onf4.pack(codes))
    a = absmax.cpu().numpy()
    assert np.array_equal(np.isnan(a), np.isnan(b))
    ok = ~np.isnan(b)
    assert np.array_equal(a[ok].view(np.uint32), b[ok].view(np.uint32))


def test_quantize_tiny_layer(q):
    _check_quant(q, synth.tiny_inputs()["W"])


@pytest.mark.parametrize("N,K", [(1, 64), (3, 128), (5, 192), (7, 640), (33, 320), (300, 448)])
def test_quantize_ragged_and_crafted(q, N, K):
    _check_quant(q, _crafted(N, K, N * 1000 + K))


@pytest.mark.parametrize("idx", [0, 4, 6])
def test_quantize_llama7b_shapes(q, idx):
    s = synth.LLAMA7B_SET[idx]
    W = synth.llama_weight((s.N, s.K), synth.SEED_W + idx)
    _check_quant(q, W)


def _check_dq(q, absmax):
    c2, s2, mu = onf4.double_quant(absmax)
    g2, gs2, gmu = q.double_quant(dev(absmax))
    torch.cuda.synchronize()
    assert np.float32(gmu.item()) == mu
    assert np.array_equal(gs2.cpu().numpy().view(np.uint32), s2.view(np.uint32))
    diff = int(np.sum(g2.cpu().numpy() != c2))
    assert diff == 0, f"{diff} of {c2.size} double-quantization codes differ"


def test_double_quant_tiny_and_ragged(q):
    _check_dq(q, oracle_quant(synth.tiny_inputs()["W"])["absmax"])
    for N, K in [(3, 128), (7, 640), (300, 448)]:
        _check_dq(q, oracle_quant(_crafted(N, K, 7 + N))["absmax"])
    _check_dq(q, np.full(700, 0.25, np.float32))  # zero-spread blocks


def test_double_quant_llama7b_gate(q):
    W = synth.llama_weight((11008, 4096), synth.SEED_W + 4)
    _, absmax = q.nf4_quantize(W.cuda())
    _check_dq(q, absmax.cpu().numpy())


@pytest.mark.parametrize("N,K", [(256, 512), (7, 640), (4096, 4096)])
def test_dequant_two_level(q, N, K):
    W = synth.llama_weight((N, K), 77 + N) if N > 8 else _crafted(N, K, 5)
    oq = oracle_quant(W)
    w = weight_from_oracle(q, oq, N, K)
    ref = onf4.dequant(oq["packed"], oq["code2"], oq["scale2"], oq["mean"], N * K).reshape(N, K)
    got = q.dequant(w, torch.float32).cpu().numpy()
    rel = np.abs(got.astype(np.float64) - ref) / np.maximum(np.abs(ref).astype(np.float64), 1e-30)
    assert float(rel.max()) <= 1e-6
    gb = q.dequant(w, torch.bfloat16).view(torch.int16).cpu().numpy().view(np.uint16)
    assert np.array_equal(gb, onum.f32_to_bf16_bits(ref))


@pytest.mark.parametrize("N,K", [(256, 512), (33, 320), (4096, 11008)])
def test_recon_error(q, N, K):
    W = synth.llama_weight((N, K), 99 + N, std=0.013)
    ref = onf4.recon_sse(f32(W))
    got = q.nf4_recon_error(W.cuda()).item()
    assert abs(got - ref) <= 1e-5 * ref
    # the same figure from the quantize pass with its SSE output on
    _, _, s = q.nf4_quantize(W.cuda(), sse=True)
    assert abs(s.item() - ref) <= 1e-5 * ref


@pytest.mark.parametrize("N,K", [(256, 512), (33, 320), (4096, 11008)])
def test_layer_stats(q, N, K):
    # AQLoRA §3.1 in one pass: the SSE bit-identical to the reconstruction-error kernel's,
    # the count of |w| < 0.01 exact
    W = synth.llama_weight((N, K), 199 + N, std=0.013)
    st = q.nf4_layer_stats(W.cuda()).cpu().numpy()
    assert st[0] == q.nf4_recon_error(W.cuda()).item()
    assert st[1] == onf4.below_count(f32(W))
    ref = onf4.recon_sse(f32(W))
    assert abs(st[0] - ref) <= 1e-5 * ref


def test_layer_stats_crafted_and_degenerate(q):
    # the bf16 neighbours of tau, signed zeros, a whole zero row (its blocks all below),
    # and a partial last chunk of the streamed kernel (N * K / 64 not a multiple of 128)
    lo, hi = 163 * 2.0 ** -14, 164 * 2.0 ** -14
    W = synth.llama_weight((3, 192), 7, std=0.02).float()
    W[0, :8] = torch.tensor([lo, -lo, hi, -hi, 0.0, -0.0, 0.01, -0.01])
    W[1] = 0.0
    Wb = W.to(torch.bfloat16)
    st = q.nf4_layer_stats(Wb.cuda()).cpu().numpy()
    assert st[1] == onf4.below_count(f32(Wb))
    assert abs(st[0] - onf4.recon_sse(f32(Wb))) <= 1e-5 * onf4.recon_sse(f32(Wb))
    z = torch.zeros(5, 128, dtype=torch.bfloat16, device="cuda")
    stz = q.nf4_layer_stats(z).cpu().numpy()
    assert stz[0] == 0.0 and stz[1] == z.numel()
    # another threshold: every element with |w| < 1 counts
    st1 = q.nf4_layer_stats(Wb.cuda(), tau=1.0).cpu().numpy()
    assert st1[1] == onf4.below_count(f32(Wb), np.float32(1.0)) == Wb.numel()


@pytest.mark.parametrize("N,K,world", [(150, 11008, 2), (4096, 4096, 3), (33, 320, 4)])
def test_row_sharded_quantization_is_bit_identical(q, N, K, world):
    # one matrix quantized as row shards (one per process in production; here in turn on
    # one GPU): NF4 codes and constants per shard, float64 constant sums added (what the
    # all-reduce does), each shard encoded with the matrix's sum and count
    from bit_nf4_quantized_04_b200 import dist
    W = synth.llama_weight((N, K), 300 + N, std=0.02).cuda()
    whole = q.quantize_weight(W)
    spans = [dist.shard_rows(N, K, world, r) for r in range(world)]
    parts = [q.nf4_quantize(W[a:b].contiguous()) for a, b in spans if b > a]
    total = torch.zeros(2, dtype=torch.float64, device="cuda")
    for _, absmax in parts:
        total[:1] += q.dq_sum(absmax)
    enc = [q.double_quant_shard(absmax, total, N * K // 64) for _, absmax in parts]
    torch.cuda.synchronize()
    assert torch.equal(torch.cat([p for p, _ in parts]), whole.packed)
    assert torch.equal(torch.cat([e[0] for e in enc]), whole.code2)
    assert torch.equal(torch.cat([e[1] for e in enc]), whole.scale2)
    assert all(torch.equal(e[2], whole.mean) for e in enc)
    # one process: the dist entry point reduces to the whole-matrix quantization
    w1 = dist.sharded_quantize_weight(W, N)
    assert torch.equal(w1.code2, whole.code2) and torch.equal(w1.mean, whole.mean)


@pytest.mark.parametrize("N,K", [(33, 320), (4096, 11008), (300, 4096)])
def test_fused_quantize_weight_matches_the_separate_calls(q, N, K):
    # qnf4_quantize_weight (two launches: the quantizer hands its constant sums to the
    # encoder, which also folds the SSE) against qnf4_nf4_quantize + qnf4_double_quant,
    # bit for bit, and against the oracle
    W = synth.llama_weight((N, K), 500 + N, std=0.02)
    if N == 300:
        W[7] = 0  # an all-zero row (zero constants) inside the tensor
    Wc = W.cuda()
    w, sse = q.quantize_weight(Wc, sse=True)
    packed, absmax, sse2 = q.nf4_quantize(Wc, sse=True)
    code2, scale2, mean = q.double_quant(absmax)
    torch.cuda.synchronize()
    assert torch.equal(w.packed, packed)
    assert torch.equal(w.code2, code2) and torch.equal(w.scale2, scale2)
    assert torch.equal(w.mean, mean)
    assert sse.item() == sse2.item()
    oq = oracle_quant(W)
    assert np.array_equal(w.code2.cpu().numpy(), oq["code2"])
    ref = onf4.recon_sse(f32(W))
    assert abs(sse.item() - ref) <= 1e-5 * ref
    # without the SSE output
    w2 = q.quantize_weight(Wc)
    assert torch.equal(w2.packed, packed) and torch.equal(w2.code2, code2)


def test_fused_quantize_weight_all_zero(q):
    z = torch.zeros(8, 256, dtype=torch.bfloat16, device="cuda")
    w, sse = q.quantize_weight(z, sse=True)
    torch.cuda.synchronize()
    assert sse.item() == 0.0 and w.mean.item() == 0.0
    assert torch.all(w.code2 == 0) and torch.all(w.scale2 == 0)
    assert torch.all(w.packed == 0x77)


@pytest.mark.parametrize("shapes", [
    [(33, 320)],                                              # one weight (the single call's grid)
    [(33, 320), (4096, 11008), (300, 4096), (8, 64)],         # ragged chunk and 256-block ends
    [(16, 64 * k) for k in range(1, 9)],                      # eight tiny weights: CTAs span several
])
def test_quantize_weight_group_matches_single_calls(q, shapes):
    # qnf4_quantize_weight_group: codes, constants, code2, scale2 and mean equal the
    # single call's bit for bit; each SSE equals it up to float64 rounding (the per-CTA
    # partials group the same fp32 block sums differently) and matches the oracle
    Ws = []
    for i, (N, K) in enumerate(shapes):
        W = synth.llama_weight((N, K), 900 + 7 * i + N, std=0.02)
        if N == 300:
            W[5] = 0
        Ws.append(W.cuda())
    outs, sses = q.quantize_weight_group(Ws, sse=True)
    plain = q.quantize_weight_group(Ws)
    torch.cuda.synchronize()
    for i, W in enumerate(Ws):
        w, sse = q.quantize_weight(W, sse=True)
        torch.cuda.synchronize()
        for a, b in ((outs[i].packed, w.packed), (outs[i].code2, w.code2), (outs[i].scale2, w.scale2),
                     (outs[i].mean, w.mean), (plain[i].packed, w.packed), (plain[i].code2, w.code2)):
            assert torch.equal(a, b), f"weight {i} {shapes[i]}"
        assert abs(sses[i].item() - sse.item()) <= 1e-12 * max(sse.item(), 1e-300)
    # one weight of the mixed set against the oracle
    oq = oracle_quant(Ws[-1].cpu())
    assert np.array_equal(outs[-1].code2.cpu().numpy(), oq["code2"])
    ref = onf4.recon_sse(f32(Ws[-1].cpu()))
    assert abs(sses[-1].item() - ref) <= 1e-5 * ref


@pytest.mark.parametrize("with_count", [True, False])
def test_layer_stats_group_matches_single_calls(q, with_count):
    # qnf4_nf4_layer_stats_group: the counts equal the single calls' exactly, each SSE equals
    # qnf4_nf4_recon_error's up to float64 rounding and the oracle's within its bound
    shapes = [(33, 320), (4096, 11008), (256, 512), (8, 64)]
    Ws = []
    for i, (N, K) in enumerate(shapes):
        W = synth.llama_weight((N, K), 700 + 5 * i + N, std=0.013)
        if N == 256:
            W[3] = 0
        Ws.append(W.cuda())
    sse, cnt = q.nf4_layer_stats_group(Ws, tau=0.01 if with_count else None)
    torch.cuda.synchronize()
    assert (cnt is None) != with_count
    for i, W in enumerate(Ws):
        one = q.nf4_recon_error(W).item()
        assert abs(sse[i].item() - one) <= 1e-12 * max(one, 1e-300), f"weight {i}"
        if with_count:
            st = q.nf4_layer_stats(W)
            assert cnt[i].item() == st[1].item() == onf4.below_count(f32(W.cpu()))
    ref = onf4.recon_sse(f32(Ws[1].cpu()))
    assert abs(sse[1].item() - ref) <= 1e-5 * ref
