"""GPU weighted Lloyd-Max learner (per-channel mappings and thresholds, "LowRA" article,
第五部分) against the float64 oracle: mappings, thresholds and iteration counts bit-exact
(the float64 bin sums differ from the oracle's only in summation order, far below the fp32
rounding of the centres), per-channel errors within 1e-12 relative."""
import numpy as np
import pytest
import torch

import synth
from oracle import lloyd

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def q():
    import bit_nf4_quantized_04_b200 as q
    return q


def _weights(N, K, seed):
    W = synth.llama_weight((N, K), seed, std=0.02)
    Wf = W.float().numpy()
    # an all-zero row, a row with one all-zero group, and a row at a different scale
    Wf[0] = 0.0
    Wf[1, 64:128] = 0.0
    Wf[2] *= 40.0
    return torch.from_numpy(Wf).to(torch.bfloat16)


@pytest.mark.parametrize("bits", [1, 2, 4])
@pytest.mark.parametrize("N,K", [(24, 128), (40, 448), (16, 4096)])
def test_learn_matches_oracle(q, bits, N, K):
    W = _weights(N, K, 300 + N + bits)
    t0 = lloyd.initial_thresholds(bits)
    iters = 8
    m_ref, t_ref, e_ref = lloyd.learn(W.float().numpy(), bits, t0, iters)
    it_ref = np.array([lloyd.learn_row(W.float().numpy()[i], bits, t0, iters)[3] for i in range(N)])
    mp, th, err, it = q.chanq_learn(W.cuda(), bits, torch.from_numpy(t0), iters)
    torch.cuda.synchronize()
    assert np.array_equal(it.cpu().numpy(), it_ref)
    assert np.array_equal(mp.cpu().numpy().view(np.uint32), m_ref.view(np.uint32))
    assert np.array_equal(th.cpu().numpy().view(np.uint32), t_ref.view(np.uint32))
    e = err.cpu().numpy()
    assert np.all(np.abs(e - e_ref) <= 1e-12 * np.maximum(e_ref, 1e-30))


def test_learn_tables_are_ordered(q):
    # the learned tables are valid quantizer inputs: ascending thresholds and mappings,
    # non-negative errors
    N, K, bits = 32, 256, 2
    W = _weights(N, K, 77)
    mp, th, err, _ = q.chanq_learn(W.cuda(), bits, torch.from_numpy(lloyd.initial_thresholds(bits)), 8)
    th_c = th.cpu()
    assert torch.all(th_c[:, 1:] >= th_c[:, :-1])
    mp_c = mp.cpu()
    assert torch.all(mp_c[:, 1:] >= mp_c[:, :-1])
    assert torch.all(err.cpu() >= 0)


def test_learn_argument_checks(q):
    W = torch.zeros(4, 128, dtype=torch.bfloat16, device="cuda")
    t0 = torch.from_numpy(lloyd.initial_thresholds(2))
    with pytest.raises(q._lib.Qnf4Error):
        q.chanq_learn(W, 3, t0, 8)
    with pytest.raises(q._lib.Qnf4Error):
        q.chanq_learn(W[:, :100].contiguous(), 2, t0, 8)
