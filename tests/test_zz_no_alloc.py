"""The allocation-free forward entry point, through the C ABI.

Callers that cannot allocate device memory (an allocator callback, a pre-planned
engine's host hook, a caller without a device allocator of its own) use
qnf4_qlora_linear_fwd_noalloc, which takes its workspace from an array built into the
library. It runs the regular entry point's kernels with the same tiling, so its
output must equal the regular call's (caller-provided workspace) bit for bit, on two
calls in a row (the second reuses the array's leftover contents, so stale scratch
leaking into the output would show). The shapes include the 7B prefill case of 4096
tokens, whose split-K partial tiles are the largest the array has to hold. This file
sorts last so a run that stops at the first failure has run every other test first.
"""
import ctypes as C

import pytest
import torch

import synth

from helpers import assert_close, f64

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("N,K,M,r", [(4096, 4096, 16, 16), (384, 640, 130, 8),
                                     (4096, 4096, 4096, 16), (11008, 4096, 4096, 16),
                                     (5120, 5120, 2048, 64)])
def test_noalloc_forward_matches_workspace_forward(N, K, M, r):
    import bit_nf4_quantized_04_b200 as q
    W = synth.llama_weight((N, K), 77 + N)
    x = synth.normal_bf16((M, K), 1.0, 78).cuda()
    A = synth.normal_bf16((r, K), 0.01, 79).cuda()
    B = synth.normal_bf16((N, r), 0.01, 80).cuda()
    s = 2.0
    w = q.quantize_weight(W.cuda())
    ref = q.qlora_linear_fwd(w, x, A, B, s)
    cw = w.c()
    stream = torch.cuda.current_stream().cuda_stream
    for _ in range(2):
        h = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
        st = q.lib.qnf4_qlora_linear_fwd_noalloc(C.byref(cw), x.data_ptr(), M, A.data_ptr(),
                                                 B.data_ptr(), r, s, h.data_ptr(), stream)
        assert st == 0, q.lib.qnf4_last_error()
        torch.cuda.synchronize()
        if not torch.equal(h, ref):
            assert_close(f64(h.cpu()), f64(ref.cpu()), "no-alloc forward")
            raise AssertionError("no-alloc forward is within tolerance but not bit-identical")


def test_noalloc_forward_rejects_oversized_shapes():
    import bit_nf4_quantized_04_b200 as q
    fake = 1 << 20  # rejected on the host before anything is launched or dereferenced
    w = q.Qnf4Weight(4096, 4096, 64, 256, fake, fake, fake, fake)
    st = q.lib.qnf4_qlora_linear_fwd_noalloc(C.byref(w), fake, 1 << 20, fake, fake, 16, 1.0,
                                             fake, None)
    assert st == 6 and b"built-in scratch" in q.lib.qnf4_last_error()
    # the documented limit: every shape up to 65536 tokens fits the 32 MiB array
    for N, K in ((4096, 4096), (11008, 4096), (4096, 11008), (13824, 5120), (5120, 13824)):
        for M in (1, 16, 4096, 8192, 65536):
            assert q.workspace_size(q._lib.OP_FWD, N, K, M, 64) <= 32 << 20, (N, K, M)


@pytest.mark.parametrize("N,K,M,r", [(4096, 4096, 16, 16), (1000, 2048, 300, 16)])
def test_noalloc_forward_captured_in_a_cuda_graph(N, K, M, r):
    # the use the header advertises: one call outside any capture (it looks up the array's
    # device address), then calls recorded into a CUDA graph and replayed on one stream;
    # every replay equals the regular forward bit for bit
    import bit_nf4_quantized_04_b200 as q
    W = synth.llama_weight((N, K), 91 + N)
    x = synth.normal_bf16((M, K), 1.0, 92).cuda()
    A = synth.normal_bf16((r, K), 0.01, 93).cuda()
    B = synth.normal_bf16((N, r), 0.01, 94).cuda()
    s = 2.0
    w = q.quantize_weight(W.cuda())
    ref = q.qlora_linear_fwd(w, x, A, B, s)
    cw = w.c()
    h = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")

    def call():
        st = q.lib.qnf4_qlora_linear_fwd_noalloc(C.byref(cw), x.data_ptr(), M, A.data_ptr(), B.data_ptr(),
                                                 r, s, h.data_ptr(), torch.cuda.current_stream().cuda_stream)
        assert st == 0, q.lib.qnf4_last_error()

    call()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        call()
    for _ in range(3):
        h.fill_(float("nan"))
        g.replay()
        torch.cuda.synchronize()
        assert torch.equal(h, ref)
