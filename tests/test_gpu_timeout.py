"""Failure detection on the GPU without a fault: the library's bounded waits.

Every wait inside the library's kernels (mbarrier phases of TMA copies, MMAs and the
converter and epilogue hand-offs) gives up after the wait limit set by
qnf4_set_wait_timeout_ns. A kernel whose wait gives up records a site code in a device
flag, raises a CTA-wide abort, still waits for its own copies and MMAs in flight,
frees its memory and returns, so the context stays usable; qnf4_check then reports
QNF4_ERR_TIMEOUT with the site.

Here the limit is set far below the time the work needs (100 ns: a 4096-token forward
holds an accumulator for tens of microseconds), so waits run out on purpose. Nothing is
faulted, trapped or left hanging: the kernels end by themselves. After restoring the
default limit, the next calls must give exactly the results of calls that never timed
out. The quantization kernel is not among the cases: its only waits are each warp's
waits for its own copies, which one suspended mbarrier poll outlasts, so no limit makes
them run out.
"""
import pytest
import torch

import synth

pytestmark = pytest.mark.gpu

DEFAULT_NS = 1_000_000_000


@pytest.fixture()
def q():
    import bit_nf4_quantized_04_b200 as q
    yield q
    q.set_wait_timeout_ns(DEFAULT_NS)


def _expect_timeout(q):
    with pytest.raises(q.Qnf4Error) as ei:
        q.check()
    assert ei.value.status == 5, str(ei.value)  # QNF4_ERR_TIMEOUT
    assert "site" in str(ei.value)
    q.check()  # the flag was read and cleared: the next check is clean


def test_forward_wait_timeout_reports_and_recovers(q):
    N, K, M, r = 4096, 4096, 4096, 16
    W = synth.llama_weight((N, K), 901, device="cuda")
    x = synth.normal_bf16((M, K), 1.0, 902, device="cuda")
    A = synth.normal_bf16((r, K), 0.01, 903, device="cuda")
    B = synth.normal_bf16((N, r), 0.01, 904, device="cuda")
    w = q.quantize_weight(W)
    ref = q.qlora_linear_fwd(w, x, A, B, 2.0)
    q.check()
    q.set_wait_timeout_ns(100)
    h = torch.zeros_like(ref)
    q.qlora_linear_fwd(w, x, A, B, 2.0, h=h)
    _expect_timeout(q)
    q.set_wait_timeout_ns(DEFAULT_NS)
    h2 = q.qlora_linear_fwd(w, x, A, B, 2.0)
    q.check()
    assert torch.equal(h2, ref)


def test_backward_wait_timeout_reports_and_recovers(q):
    N, K, M, r = 4096, 4096, 2048, 16
    W = synth.llama_weight((N, K), 911, device="cuda")
    x = synth.normal_bf16((M, K), 1.0, 912, device="cuda")
    dY = synth.normal_bf16((M, N), 1.0, 913, device="cuda")
    A = synth.normal_bf16((r, K), 0.01, 914, device="cuda")
    B = synth.normal_bf16((N, r), 0.01, 915, device="cuda")
    w = q.quantize_weight(W)
    ref = q.qlora_linear_bwd(w, x, dY, A, B, 2.0)
    q.check()
    q.set_wait_timeout_ns(100)
    q.qlora_linear_bwd(w, x, dY, A, B, 2.0)
    _expect_timeout(q)
    q.set_wait_timeout_ns(DEFAULT_NS)
    got = q.qlora_linear_bwd(w, x, dY, A, B, 2.0)
    q.check()
    for g, rf in zip(got, ref):
        assert torch.equal(g, rf)
