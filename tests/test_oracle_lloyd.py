"""Pins of the weighted Lloyd-Max learner oracle (per-channel mappings and thresholds,
"LowRA" article, 第五部分) against facts that do not come from the oracle itself:
the NF4 codebook, a brute-force optimum, closed forms and the per-channel quantizer."""
import numpy as np
import pytest

from oracle import chanq, lloyd, nf4

pytestmark = pytest.mark.filterwarnings("ignore")


def _row(K, seed, std=0.02):
    rng = np.random.default_rng(seed)
    return (rng.standard_normal(K) * std).astype(np.float32)


def test_nf4_levels_from_the_general_construction():
    # the b-bit NormalFloat construction at b = 4 is NF4 (pinned in test_oracle_nf4)
    assert np.array_equal(lloyd.nf_levels(4), nf4.codebook())


def test_nf2_levels_shape():
    q = lloyd.nf_levels(2)
    assert q.size == 4 and q[0] == -1 and q[-1] == 1 and 0.0 in q
    assert np.all(np.diff(q) > 0)
    t = lloyd.initial_thresholds(2)
    assert np.all((t > q[:-1]) & (t < q[1:]))
    assert np.array_equal(lloyd.initial_thresholds(1), np.zeros(1, np.float32))


def _weighted_sse_bruteforce_1bit(x, wt):
    """Minimum over all two-bin splits of the sorted values of the weighted SSE with
    each bin at its weighted mean (the global 1-bit optimum), divided by sum(wt)."""
    o = np.argsort(x, kind="stable")
    xs, ws = x[o].astype(np.float64), wt[o].astype(np.float64)
    best = np.inf
    for s in range(1, xs.size):
        e = 0.0
        for a, b in ((0, s), (s, xs.size)):
            W = ws[a:b].sum()
            mu = (ws[a:b] * xs[a:b]).sum() / W
            e += (ws[a:b] * (xs[a:b] - mu) ** 2).sum()
        best = min(best, e)
    return best / wt.sum()


@pytest.mark.parametrize("seed", [1, 2, 3])
def test_one_bit_reaches_the_bruteforce_optimum(seed):
    w = _row(192, seed)
    x, g = lloyd.normalise_row(w)
    wt = np.repeat(g, lloyd.GROUP)
    ref = _weighted_sse_bruteforce_1bit(x, wt)
    _, _, _, _, hist = lloyd.learn_row(w, 1, lloyd.initial_thresholds(1), 200)
    assert hist[-1] >= ref * (1 - 1e-9)          # never below the global optimum
    assert hist[-1] <= ref * (1 + 1e-6)          # and Lloyd gets there on unimodal data


@pytest.mark.parametrize("bits", [1, 2, 4])
def test_error_never_increases(bits):
    w = _row(1024, 10 + bits)
    _, _, _, _, hist = lloyd.learn_row(w, bits, lloyd.initial_thresholds(bits), 30)
    h = np.array(hist)
    assert np.all(h[1:-1] <= h[:-2] * (1 + 1e-12))  # the last entry may be the stopping one
    assert h[-1] <= h[0]


def test_two_bit_converges_to_the_weighted_cluster_centres():
    # four tight clusters, each inside one initial NF2 bin, with two group weights: the
    # fixed point is each cluster's weighted centre (closed form), thresholds between them
    K = 256
    rng = np.random.default_rng(7)
    centres = np.array([-0.7, -0.2, 0.3, 0.8])
    x = np.repeat(centres, K // 4) + rng.uniform(-0.01, 0.01, K)
    rng.shuffle(x)
    w = np.empty(K, np.float32)
    # group 0..3: absmax set by one element of magnitude s (+ or -), others scaled in
    for gi, s in enumerate([0.5, 0.5, 1.0, 1.0]):
        seg = x[gi * 64:(gi + 1) * 64].astype(np.float32)
        seg[np.argmax(np.abs(seg))] = np.sign(seg[np.argmax(np.abs(seg))]) * 1.0
        w[gi * 64:(gi + 1) * 64] = (seg * s).astype(np.float32)
    m, t, _, _, _ = lloyd.learn_row(w, 2, lloyd.initial_thresholds(2), 50)
    xn, g = lloyd.normalise_row(w)
    wt = np.repeat(g, 64).astype(np.float64)
    c = np.searchsorted(centres[:-1] + np.diff(centres) / 2, xn.astype(np.float64))
    for k in range(4):
        sel = c == k
        ref = np.float32((wt[sel] * xn[sel]).sum() / wt[sel].sum())
        assert m[k] == ref
    assert np.all((t > m[:-1]) & (t < m[1:]))


@pytest.mark.parametrize("bits", [1, 2, 4])
def test_reported_error_is_the_quantizer_error(bits):
    # quantize the row with the learned edges and decode with the learned mapping
    # through the per-channel quantizer oracle: the mean squared error must match
    K = 512
    w = _row(K, 40 + bits)
    m, t, err, _, _ = lloyd.learn_row(w, bits, lloyd.initial_thresholds(bits), 8)
    b = np.array([bits], np.uint8)
    packed, roff, g, codes = chanq.quantize(w[None, :], b, t, np.array([0, t.size], np.int64))
    wh = chanq.dequant(packed, roff, b, m, np.array([0, m.size], np.int64), g, 1, K)
    ref = float(np.mean((w.astype(np.float64) - wh.reshape(-1).astype(np.float64)) ** 2))
    assert err == ref


def test_all_zero_row_keeps_the_initial_tables():
    m, t, err, done, _ = lloyd.learn_row(np.zeros(128, np.float32), 2, lloyd.initial_thresholds(2), 8)
    t0 = lloyd.initial_thresholds(2)
    assert m[0] == -1 and m[-1] == 1 and np.array_equal(m[1:-1], lloyd.midpoints(t0))
    assert err == 0.0 and done == 2
