"""The C ABI without a GPU: the library loads, exports every symbol include/qnf4.h
declares, computes its host-side codebook identically to the oracle (two independent
inverse-normal implementations), and rejects bad arguments before touching a device.
"""
import ctypes as C
import os
import re
import subprocess

import numpy as np
import pytest

from oracle import nf4 as onf4, rank as orank

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "qnf4.h")


@pytest.fixture(scope="module")
def q():
    import __graft_entry__
    __graft_entry__.build()
    import bit_nf4_quantized_04_b200 as q
    return q


def _declared():
    src = open(HEADER).read()
    return sorted(set(re.findall(r"QNF4_API\s+[\w\s\*]+?\b(qnf4_\w+)\s*\(", src)))


def test_header_declares_the_abi():
    names = _declared()
    for n in ("qnf4_nf4_codebook", "qnf4_nf4_quantize", "qnf4_double_quant", "qnf4_dequant",
              "qnf4_qlora_linear_fwd", "qnf4_qlora_linear_fwd_group", "qnf4_qlora_linear_bwd",
              "qnf4_quantize_weight", "qnf4_quantize_weight_group", "qnf4_nf4_layer_stats_group",
              "qnf4_nf4_recon_error",
              "qnf4_chanq_quantize", "qnf4_chanq_linear_fwd", "qnf4_workspace_size",
              "qnf4_last_error"):
        assert n in names


def test_library_exports_every_declared_symbol(q):
    out = subprocess.run(["nm", "-D", "--defined-only", q._lib.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r"\bT (qnf4_\w+)", out))
    declared = set(_declared())
    assert declared <= exported, declared - exported
    # nothing else leaks out under the qnf4_ prefix, and every binding signature exists
    assert exported == declared
    assert set(q._lib.SIGNATURES) == declared
    # the checked build (index checks compiled into the kernels) exports the same ABI
    checked = os.path.join(os.path.dirname(q._lib.LIB_PATH), "libqnf4_checked.so")
    out = subprocess.run(["nm", "-D", "--defined-only", checked], capture_output=True,
                         text=True, check=True).stdout
    assert set(re.findall(r"\bT (qnf4_\w+)", out)) == declared


def test_host_codebook_matches_oracle_bit_exactly(q):
    lv, th = q.nf4_codebook()
    assert np.array_equal(lv.numpy().view(np.uint32), onf4.codebook().view(np.uint32))
    assert np.array_equal(th.numpy().view(np.uint32), onf4.thresholds().view(np.uint32))


def test_rank_topk_matches_oracle(q):
    rng = np.random.default_rng(1)
    n = rng.integers(1000, 100000, 280)
    sse = rng.uniform(0, 1, 280) * n
    sse[20] = sse[21] / n[21] * n[20]
    assert q.rank_topk(sse, n, 8) == list(orank.top_k(sse, n, 8))


def _st(q, name, *args):
    return getattr(q.lib, name)(*args)


def test_argument_checks_fail_before_any_launch(q):
    fake = 1 << 20  # never dereferenced: every call below fails its host-side checks
    # K not a multiple of 64
    assert _st(q, "qnf4_nf4_quantize", fake, 4, 63, 64, fake, fake, None, None, 0, None) == 2
    # block size other than 64
    assert _st(q, "qnf4_nf4_quantize", fake, 4, 64, 32, fake, fake, None, None, 0, None) == 1
    # NULL and misaligned buffers
    assert _st(q, "qnf4_nf4_quantize", None, 4, 64, 64, fake, fake, None, None, 0, None) == 1
    assert _st(q, "qnf4_nf4_quantize", fake + 2, 4, 64, 64, fake, fake, None, None, 0, None) == 3
    # sse requested without workspace
    assert _st(q, "qnf4_nf4_quantize", fake, 4, 64, 64, fake, fake, fake, None, 0, None) == 6
    assert _st(q, "qnf4_double_quant", fake, 10, 128, fake, fake, fake, fake, 1 << 20, None) == 1
    assert _st(q, "qnf4_nf4_recon_error", fake, 4, 64, 64, fake, None, 0, None) == 6
    w = q.Qnf4Weight(8, 64, 64, 256, fake, fake, fake, fake)
    # r out of range
    assert _st(q, "qnf4_qlora_linear_fwd", C.byref(w), fake, 4, fake, fake, 0, 1.0, fake, fake,
               1 << 20, None) == 1
    assert _st(q, "qnf4_qlora_linear_fwd", C.byref(w), fake, 4, fake, fake, 65, 1.0, fake, fake,
               1 << 20, None) == 1
    # M = 0 is a no-op that never launches
    assert _st(q, "qnf4_qlora_linear_fwd", C.byref(w), fake, 0, fake, fake, 8, 1.0, fake, fake,
               0, None) == 0
    # backward needs N % 8 == 0
    w2 = q.Qnf4Weight(12, 64, 64, 256, fake, fake, fake, fake)
    assert _st(q, "qnf4_qlora_linear_bwd", C.byref(w2), fake, fake, 4, fake, fake, 8, 1.0, fake,
               fake, fake, fake, 1 << 20, None) == 2
    # bad block sizes in the weight descriptor
    w3 = q.Qnf4Weight(8, 64, 64, 128, fake, fake, fake, fake)
    assert _st(q, "qnf4_dequant", C.byref(w3), fake, 0, None) == 1
    assert _st(q, "qnf4_dequant", C.byref(w), fake, 7, None) == 1
    assert _st(q, "qnf4_chanq_quantize", fake, 4, 100, fake, fake, fake, fake, fake, fake,
               None) == 2
    assert _st(q, "qnf4_rank_topk", None, None, 3, 1, None) == 1
    assert _st(q, "qnf4_set_wait_timeout_ns", 0) == 1
    assert b"positive" in q.lib.qnf4_last_error()
    # grouped forward: n in 1..8, M in 1..16, per-layer checks as for the single call
    arr = (q.Qnf4Weight * 2)(w, w)
    ptrs = (C.c_void_p * 2)(fake, fake)
    assert _st(q, "qnf4_qlora_linear_fwd_group", 0, arr, ptrs, 4, ptrs, ptrs, 8, 1.0, ptrs, fake,
               1 << 20, None) == 1
    assert _st(q, "qnf4_qlora_linear_fwd_group", 9, arr, ptrs, 4, ptrs, ptrs, 8, 1.0, ptrs, fake,
               1 << 20, None) == 1
    assert _st(q, "qnf4_qlora_linear_fwd_group", 2, arr, ptrs, 17, ptrs, ptrs, 8, 1.0, ptrs, fake,
               1 << 20, None) == 2
    assert _st(q, "qnf4_qlora_linear_fwd_group", 2, arr, ptrs, 4, ptrs, ptrs, 65, 1.0, ptrs, fake,
               1 << 20, None) == 1
    assert _st(q, "qnf4_qlora_linear_fwd_group", 2, arr, ptrs, 4, ptrs, ptrs, 8, 1.0, ptrs, fake,
               16, None) == 6
    # grouped quantization: n in 1..8, per-weight shape, NULL and alignment checks, workspace
    i64 = lambda *v: (C.c_int64 * len(v))(*v)  # noqa: E731
    N2, K2 = i64(4, 8), i64(64, 128)
    gq = lambda n, N, K, p, ws_bytes: _st(q, "qnf4_quantize_weight_group", n, p, N, K, p, p, p, p, p,  # noqa: E731
                                          None, fake, ws_bytes, None)
    assert gq(0, N2, K2, ptrs, 1 << 20) == 1
    assert gq(9, N2, K2, ptrs, 1 << 20) == 1
    assert gq(2, N2, i64(64, 100), ptrs, 1 << 20) == 2
    assert gq(2, i64(4, 0), K2, ptrs, 1 << 20) == 2
    assert gq(2, N2, K2, (C.c_void_p * 2)(fake, None), 1 << 20) == 1
    assert gq(2, N2, K2, (C.c_void_p * 2)(fake, fake + 8), 1 << 20) == 3
    assert gq(2, N2, K2, ptrs, 16) == 6
    assert _st(q, "qnf4_quantize_weight_group", 2, None, N2, K2, ptrs, ptrs, ptrs, ptrs, ptrs, None,
               fake, 1 << 20, None) == 1
    assert q.workspace_size(q._lib.OP_QUANTIZE_WEIGHT_GROUP, 0, 0) >= 2 * 8 * 1024 * 8
    # grouped profiling statistics: n, shape, NULL, alignment, tau, workspace
    gs = lambda n, N, K, tau, p, b, ws_bytes: _st(q, "qnf4_nf4_layer_stats_group", n, p, N, K, tau, p, b,  # noqa: E731
                                                  fake, ws_bytes, None)
    assert gs(0, N2, K2, 0.01, ptrs, ptrs, 1 << 20) == 1
    assert gs(9, N2, K2, 0.01, ptrs, ptrs, 1 << 20) == 1
    assert gs(2, N2, i64(64, 96), 0.01, ptrs, ptrs, 1 << 20) == 2
    assert gs(2, N2, K2, -1.0, ptrs, ptrs, 1 << 20) == 1
    assert gs(2, N2, K2, 0.01, (C.c_void_p * 2)(fake, None), ptrs, 1 << 20) == 1
    assert gs(2, N2, K2, 0.01, ptrs, (C.c_void_p * 2)(fake, fake + 8), 1 << 20) == 3
    assert gs(2, N2, K2, 0.01, ptrs, None, 16) == 6


def test_argument_checks_of_the_next_rows(q):
    fake = 1 << 20  # never dereferenced: every call below fails its host-side checks
    nan = float("nan")
    # layer statistics (error + sparsity): shape, NULL, alignment, tau, workspace
    assert _st(q, "qnf4_nf4_layer_stats", fake, 4, 100, 0.01, fake, fake, fake, 1 << 20, None) == 2
    assert _st(q, "qnf4_nf4_layer_stats", fake, 4, 64, 0.01, fake, None, fake, 1 << 20, None) == 1
    assert _st(q, "qnf4_nf4_layer_stats", fake, 4, 64, 0.01, fake, fake + 8, fake, 1 << 20, None) == 3
    assert _st(q, "qnf4_nf4_layer_stats", fake, 4, 64, -1.0, fake, fake, fake, 1 << 20, None) == 1
    assert _st(q, "qnf4_nf4_layer_stats", fake, 4, 64, nan, fake, fake, fake, 1 << 20, None) == 1
    assert _st(q, "qnf4_nf4_layer_stats", fake, 4, 64, 0.01, fake, fake, fake, 16, None) == 6
    # row-sharded double quantization
    assert _st(q, "qnf4_dq_sum", fake, 0, fake, fake, 1 << 20, None) == 2
    assert _st(q, "qnf4_dq_sum", fake, 10, None, fake, 1 << 20, None) == 1
    assert _st(q, "qnf4_dq_sum", fake, 10, fake, fake, 8, None) == 6
    assert _st(q, "qnf4_double_quant_shard", fake, 10, 128, fake, 10, fake, fake, fake, None) == 1
    assert _st(q, "qnf4_double_quant_shard", fake, 10, 256, fake, 9, fake, fake, fake, None) == 2
    assert _st(q, "qnf4_double_quant_shard", fake, 10, 256, None, 10, fake, fake, fake, None) == 1
    # LoftQ initialisation: shape, rank, steps, the Gram-matrix size limit
    args = (fake, fake, fake, fake, fake, fake, fake, fake, 1 << 30, None)
    assert _st(q, "qnf4_loftq_nf4", fake, 32, 100, 4, 5, *args) == 2
    assert _st(q, "qnf4_loftq_nf4", fake, 32, 128, 0, 5, *args) == 1
    assert _st(q, "qnf4_loftq_nf4", fake, 32, 128, 33, 5, *args) == 1
    assert _st(q, "qnf4_loftq_nf4", fake, 32, 128, 4, 0, *args) == 1
    assert _st(q, "qnf4_loftq_nf4", fake, 20000, 20032, 4, 5, *args) == 2
    # per-channel table learner: bit width
    assert _st(q, "qnf4_chanq_learn", fake, 4, 128, 3, fake, 8, fake, fake, fake, fake, None) == 1


def test_workspace_sizes_are_positive_and_monotone(q):
    a = q.workspace_size(q._lib.OP_FWD, 4096, 4096, 16, 16)
    b = q.workspace_size(q._lib.OP_FWD, 4096, 4096, 4096, 16)
    c = q.workspace_size(q._lib.OP_BWD, 4096, 4096, 4096, 16)
    assert 0 < a and 0 < b < c
    # the decode path (M <= 16) fits the allocation-free forward's 8 MiB scratch on
    # every Llama-2-7B layer shape
    for N, K in [(4096, 4096), (11008, 4096), (4096, 11008)]:
        for M in (1, 8, 9, 16):
            assert 0 < q.workspace_size(q._lib.OP_FWD, N, K, M, 64) <= 8 << 20
    assert q.workspace_size(q._lib.OP_QUANTIZE, 4096, 4096) > 0
    assert q.workspace_size(q._lib.OP_LAYER_STATS, 4096, 4096) > q.workspace_size(q._lib.OP_QUANTIZE, 4096, 4096)
    # LoftQ: at least the bf16 target, the fp32 residual and the Gram matrix
    N, K, r = 11008, 4096, 16
    assert q.workspace_size(q._lib.OP_LOFTQ, N, K, 0, r) >= N * K * 6 + K * K * 4
