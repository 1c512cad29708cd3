"""Python binding of libqnf4: the QLoRA NF4 quantized linear layer on B200 (sm_100a).

Each function marshals torch tensors (device memory) and the current CUDA stream into
one call of the C ABI declared in include/qnf4.h, under the same name without the
``qnf4_`` prefix. All arithmetic runs in the library's CUDA kernels; nothing here
computes. Outputs are allocated with torch unless passed in.

Sources (page title, section): "QLoRA: Efficient Finetuning of Quantized LLMs"
(Heng's Blog) opening formula, 贡献一 NF4, 贡献二 Double Quantization; "AQLoRA" §3.1;
"LowRA" §4.1.
"""
from __future__ import annotations

import ctypes as C
from dataclasses import dataclass

import torch

from . import _lib
from ._lib import Qnf4Error, Qnf4Weight, lib  # noqa: F401

BLOCK1 = 64
BLOCK2 = 256

__all__ = [
    "Nf4Weight", "nf4_codebook", "nf4_quantize", "double_quant", "dequant", "quantize_weight",
    "qlora_linear_fwd", "qlora_linear_bwd", "nf4_recon_error", "rank_topk",
    "dense_linear_fwd", "dense_linear_bwd", "chanq_quantize", "chanq_linear_fwd", "chanq_linear_bwd", "chanq_learn",
    "workspace_size", "check", "set_wait_timeout_ns", "Qnf4Error",
]


def _stream(t: torch.Tensor | None = None) -> int:
    dev = t.device if t is not None else None
    return torch.cuda.current_stream(dev).cuda_stream


def _p(t: torch.Tensor | None) -> int | None:
    return None if t is None else t.data_ptr()


def _req(t: torch.Tensor, dtype: torch.dtype, name: str) -> torch.Tensor:
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t


def _ws(nbytes: int, like: torch.Tensor, ws: torch.Tensor | None) -> torch.Tensor:
    if ws is not None:
        if ws.numel() * ws.element_size() < nbytes:
            raise ValueError(f"workspace of {ws.numel() * ws.element_size()} bytes < {nbytes}")
        return ws
    return torch.empty(max(nbytes, 16), dtype=torch.uint8, device=like.device)


@dataclass
class Nf4Weight:
    """A double-quantized NF4 weight (the fields of ``qnf4_weight``), device tensors."""
    N: int
    K: int
    packed: torch.Tensor   # uint8 [N*K/2]
    code2: torch.Tensor    # uint8 [N*K/64]
    scale2: torch.Tensor   # fp32 [ceil(N*K/64/256)]
    mean: torch.Tensor     # fp32 [1]

    def c(self) -> Qnf4Weight:
        return Qnf4Weight(self.N, self.K, BLOCK1, BLOCK2, self.packed.data_ptr(),
                          self.code2.data_ptr(), self.scale2.data_ptr(), self.mean.data_ptr())

    def nbytes(self) -> int:
        return sum(t.numel() * t.element_size() for t in (self.packed, self.code2, self.scale2,
                                                          self.mean))


def workspace_size(op: int, N: int, K: int, M: int = 0, r: int = 0) -> int:
    return int(lib.qnf4_workspace_size(op, N, K, M, r))


def nf4_codebook():
    """(levels fp32 [16], thresholds fp32 [15]) on the host."""
    lv = (C.c_float * 16)()
    th = (C.c_float * 15)()
    _lib.call("qnf4_nf4_codebook", C.addressof(lv), C.addressof(th))
    return torch.tensor(list(lv), dtype=torch.float32), torch.tensor(list(th), dtype=torch.float32)


def nf4_quantize(W: torch.Tensor, sse: bool = False, packed=None, absmax=None, sse_out=None,
                 ws=None):
    """Blockwise NF4 codes of a bf16 [N, K] weight: (packed u8, absmax fp32[, sse f64])."""
    _req(W, torch.bfloat16, "W")
    N, K = W.shape
    n = N * K
    packed = packed if packed is not None else torch.empty(n // 2, dtype=torch.uint8, device=W.device)
    absmax = absmax if absmax is not None else torch.empty(n // 64, dtype=torch.float32, device=W.device)
    s = None
    wsb = None
    if sse:
        s = sse_out if sse_out is not None else torch.empty(2, dtype=torch.float64, device=W.device)
        wsb = _ws(workspace_size(_lib.OP_QUANTIZE, N, K), W, ws)
    _lib.call("qnf4_nf4_quantize", W.data_ptr(), N, K, BLOCK1, packed.data_ptr(), absmax.data_ptr(),
              _p(s), _p(wsb), 0 if wsb is None else wsb.numel(), _stream(W))
    return (packed, absmax, s[:1]) if sse else (packed, absmax)


def double_quant(absmax: torch.Tensor, code2=None, scale2=None, mean=None, ws=None):
    """(code2 u8 [nb1], scale2 fp32 [nb2], mean fp32 [1]) from the first-level constants."""
    _req(absmax, torch.float32, "absmax")
    nb1 = absmax.numel()
    nb2 = (nb1 + BLOCK2 - 1) // BLOCK2
    dev = absmax.device
    code2 = code2 if code2 is not None else torch.empty(nb1, dtype=torch.uint8, device=dev)
    scale2 = scale2 if scale2 is not None else torch.empty(nb2, dtype=torch.float32, device=dev)
    mean = mean if mean is not None else torch.empty(4, dtype=torch.float32, device=dev)
    wsb = _ws(workspace_size(_lib.OP_DOUBLE_QUANT, 0, 0), absmax, ws)
    _lib.call("qnf4_double_quant", absmax.data_ptr(), nb1, BLOCK2, code2.data_ptr(),
              scale2.data_ptr(), mean.data_ptr(), wsb.data_ptr(), wsb.numel(), _stream(absmax))
    return code2, scale2, mean[:1]


def dq_sum(absmax: torch.Tensor, out=None, ws=None) -> torch.Tensor:
    """Float64 sum of a (shard's) first-level constants, device tensor [1]."""
    _req(absmax, torch.float32, "absmax")
    o = out if out is not None else torch.empty(2, dtype=torch.float64, device=absmax.device)
    wsb = _ws(workspace_size(_lib.OP_DOUBLE_QUANT, 0, 0), absmax, ws)
    _lib.call("qnf4_dq_sum", absmax.data_ptr(), absmax.numel(), o.data_ptr(), wsb.data_ptr(),
              wsb.numel(), _stream(absmax))
    return o[:1]


def double_quant_shard(absmax: torch.Tensor, total_sum: torch.Tensor, total_count: int,
                       code2=None, scale2=None, mean=None):
    """Double quantization of one row shard's constants with the whole matrix's constant
    sum (float64 device tensor, 16-byte aligned) and count: (code2, scale2, mean)."""
    _req(absmax, torch.float32, "absmax")
    nb1 = absmax.numel()
    nb2 = (nb1 + BLOCK2 - 1) // BLOCK2
    dev = absmax.device
    code2 = code2 if code2 is not None else torch.empty(nb1, dtype=torch.uint8, device=dev)
    scale2 = scale2 if scale2 is not None else torch.empty(nb2, dtype=torch.float32, device=dev)
    mean = mean if mean is not None else torch.empty(4, dtype=torch.float32, device=dev)
    _lib.call("qnf4_double_quant_shard", absmax.data_ptr(), nb1, BLOCK2, total_sum.data_ptr(),
              int(total_count), code2.data_ptr(), scale2.data_ptr(), mean.data_ptr(),
              _stream(absmax))
    return code2, scale2, mean[:1]


def quantize_weight(W: torch.Tensor, sse: bool = False, out: Nf4Weight | None = None,
                    absmax=None, sse_out=None, ws=None):
    """NF4 + double quantization of a bf16 [N, K] weight into an ``Nf4Weight`` (two
    launches, qnf4_quantize_weight); with sse=True also the reconstruction SSE (float64
    [1]): returns (weight, sse) then."""
    _req(W, torch.bfloat16, "W")
    N, K = W.shape
    n = N * K
    dev = W.device
    if out is None:
        out = Nf4Weight(N, K, torch.empty(n // 2, dtype=torch.uint8, device=dev),
                        torch.empty(n // BLOCK1, dtype=torch.uint8, device=dev),
                        torch.empty((n // BLOCK1 + BLOCK2 - 1) // BLOCK2, dtype=torch.float32, device=dev),
                        torch.empty(4, dtype=torch.float32, device=dev)[:1])
    absmax = absmax if absmax is not None else torch.empty(n // BLOCK1, dtype=torch.float32, device=dev)
    s = None
    if sse:
        s = sse_out if sse_out is not None else torch.empty(2, dtype=torch.float64, device=dev)
    wsb = _ws(workspace_size(_lib.OP_QUANTIZE_WEIGHT, N, K), W, ws)
    _lib.call("qnf4_quantize_weight", W.data_ptr(), N, K, out.packed.data_ptr(), absmax.data_ptr(),
              out.code2.data_ptr(), out.scale2.data_ptr(), out.mean.data_ptr(), _p(s),
              wsb.data_ptr(), wsb.numel(), _stream(W))
    return (out, s[:1]) if sse else out


def quantize_weight_group(Ws: list, sse: bool = False, outs=None, absmax=None, sse_out=None,
                          ws=None):
    """quantize_weight for up to 8 bf16 weights in two launches (qnf4_quantize_weight_group):
    returns the list of ``Nf4Weight``, and with sse=True also the list of float64 [1] SSEs.
    outs, absmax and sse_out, when given, are lists with one entry per weight."""
    n = len(Ws)
    for W in Ws:
        _req(W, torch.bfloat16, "W")
    dev = Ws[0].device
    if outs is None:
        outs = []
        for W in Ws:
            m = W.shape[0] * W.shape[1]
            outs.append(Nf4Weight(W.shape[0], W.shape[1], torch.empty(m // 2, dtype=torch.uint8, device=dev),
                                  torch.empty(m // BLOCK1, dtype=torch.uint8, device=dev),
                                  torch.empty((m // BLOCK1 + BLOCK2 - 1) // BLOCK2, dtype=torch.float32,
                                              device=dev),
                                  torch.empty(4, dtype=torch.float32, device=dev)[:1]))
    if absmax is None:
        absmax = [torch.empty(W.shape[0] * W.shape[1] // BLOCK1, dtype=torch.float32, device=dev) for W in Ws]
    ss = None
    if sse:
        ss = sse_out if sse_out is not None else [torch.empty(2, dtype=torch.float64, device=dev) for _ in Ws]
    wsb = _ws(workspace_size(_lib.OP_QUANTIZE_WEIGHT_GROUP, 0, 0), Ws[0], ws)
    ptrs = lambda ts: (C.c_void_p * n)(*[t.data_ptr() for t in ts])  # noqa: E731
    i64 = lambda v: (C.c_int64 * n)(*v)  # noqa: E731
    _lib.call("qnf4_quantize_weight_group", n, ptrs(Ws), i64([W.shape[0] for W in Ws]),
              i64([W.shape[1] for W in Ws]), ptrs([o.packed for o in outs]), ptrs(absmax),
              ptrs([o.code2 for o in outs]), ptrs([o.scale2 for o in outs]), ptrs([o.mean for o in outs]),
              ptrs(ss) if sse else None, wsb.data_ptr(), wsb.numel(), _stream(Ws[0]))
    return (outs, [t[:1] for t in ss]) if sse else outs


def dequant(w: Nf4Weight, dtype: torch.dtype = torch.float32, out=None) -> torch.Tensor:
    """Two-level dequantization to an [N, K] fp32 or bf16 tensor (test/export path)."""
    code = {torch.float32: _lib.OUT_F32, torch.bfloat16: _lib.OUT_BF16}[dtype]
    out = out if out is not None else torch.empty(w.N, w.K, dtype=dtype, device=w.packed.device)
    cw = w.c()
    _lib.call("qnf4_dequant", C.byref(cw), out.data_ptr(), code, _stream(out))
    return out


def qlora_linear_fwd(w: Nf4Weight, x: torch.Tensor, A: torch.Tensor, B: torch.Tensor,
                     scale: float, h=None, ws=None) -> torch.Tensor:
    """h = x dequant(W)^T + scale (x A^T) B^T, bf16 [M, N]."""
    for t, nm in ((x, "x"), (A, "A"), (B, "B")):
        _req(t, torch.bfloat16, nm)
    M = x.shape[0]
    r = A.shape[0]
    h = h if h is not None else torch.empty(M, w.N, dtype=torch.bfloat16, device=x.device)
    wsb = _ws(workspace_size(_lib.OP_FWD, w.N, w.K, M, r), x, ws)
    cw = w.c()
    _lib.call("qnf4_qlora_linear_fwd", C.byref(cw), x.data_ptr(), M, A.data_ptr(), B.data_ptr(),
              r, float(scale), h.data_ptr(), wsb.data_ptr(), wsb.numel(), _stream(x))
    return h


def qlora_linear_fwd_group(ws_: list, xs: list, As: list, Bs: list, scale: float, hs=None,
                           ws=None) -> list:
    """The decode-size forward (1..16 tokens) of up to 8 independent layers in one launch:
    h[l] = x[l] dequant(W_l)^T + scale (x[l] A[l]^T) B[l]^T; every layer has the same
    token count and rank."""
    n = len(ws_)
    if not (len(xs) == len(As) == len(Bs) == n):
        raise ValueError("one x, A and B per layer")
    for i in range(n):
        for t, nm in ((xs[i], "x"), (As[i], "A"), (Bs[i], "B")):
            _req(t, torch.bfloat16, nm)
    M = xs[0].shape[0]
    r = As[0].shape[0]
    dev = xs[0].device
    hs = hs if hs is not None else [torch.empty(M, w.N, dtype=torch.bfloat16, device=dev) for w in ws_]
    need = sum(workspace_size(_lib.OP_FWD, w.N, w.K, M, r) for w in ws_)
    wsb = _ws(need, xs[0], ws)
    arr = (_lib.Qnf4Weight * n)(*[w.c() for w in ws_])
    ptrs = lambda ts: (C.c_void_p * n)(*[t.data_ptr() for t in ts])  # noqa: E731
    _lib.call("qnf4_qlora_linear_fwd_group", n, arr, ptrs(xs), M, ptrs(As), ptrs(Bs), r, float(scale),
              ptrs(hs), wsb.data_ptr(), wsb.numel(), _stream(xs[0]))
    return hs


def qlora_linear_bwd(w: Nf4Weight, x: torch.Tensor, dY: torch.Tensor, A: torch.Tensor,
                     B: torch.Tensor, scale: float, dX=None, dA=None, dB=None, ws=None):
    """(dX bf16 [M, K], dA fp32 [r, K], dB fp32 [N, r]) through the frozen NF4 base."""
    for t, nm in ((x, "x"), (dY, "dY"), (A, "A"), (B, "B")):
        _req(t, torch.bfloat16, nm)
    M = x.shape[0]
    r = A.shape[0]
    dev = x.device
    dX = dX if dX is not None else torch.empty(M, w.K, dtype=torch.bfloat16, device=dev)
    dA = dA if dA is not None else torch.empty(r, w.K, dtype=torch.float32, device=dev)
    dB = dB if dB is not None else torch.empty(w.N, r, dtype=torch.float32, device=dev)
    wsb = _ws(workspace_size(_lib.OP_BWD, w.N, w.K, M, r), x, ws)
    cw = w.c()
    _lib.call("qnf4_qlora_linear_bwd", C.byref(cw), x.data_ptr(), dY.data_ptr(), M, A.data_ptr(),
              B.data_ptr(), r, float(scale), dX.data_ptr(), dA.data_ptr(), dB.data_ptr(),
              wsb.data_ptr(), wsb.numel(), _stream(x))
    return dX, dA, dB


def nf4_recon_error(W: torch.Tensor, sse=None, ws=None) -> torch.Tensor:
    """Single-level NF4 round-trip sum of squared errors of a bf16 weight (f64 [1])."""
    _req(W, torch.bfloat16, "W")
    N, K = W.shape
    sse = sse if sse is not None else torch.empty(2, dtype=torch.float64, device=W.device)
    wsb = _ws(workspace_size(_lib.OP_QUANTIZE, N, K), W, ws)
    _lib.call("qnf4_nf4_recon_error", W.data_ptr(), N, K, BLOCK1, sse.data_ptr(), wsb.data_ptr(),
              wsb.numel(), _stream(W))
    return sse[:1]


def nf4_layer_stats(W: torch.Tensor, tau: float = 0.01, out=None, ws=None):
    """The AQLoRA profiling statistics of a bf16 [N, K] weight in one pass: float64 [2] =
    (NF4 reconstruction SSE, #{|w| < tau}); epsilon and the sparsity are these / (N K)."""
    _req(W, torch.bfloat16, "W")
    N, K = W.shape
    o = out if out is not None else torch.empty(4, dtype=torch.float64, device=W.device)
    wsb = _ws(workspace_size(_lib.OP_LAYER_STATS, N, K), W, ws)
    # the two doubles 16 bytes apart (the ABI wants 16-byte aligned outputs)
    _lib.call("qnf4_nf4_layer_stats", W.data_ptr(), N, K, float(tau), o.data_ptr(),
              o.data_ptr() + 16, wsb.data_ptr(), wsb.numel(), _stream(W))
    return o[0::2]


def nf4_layer_stats_group(Ws: list, tau: float | None = 0.01, sse=None, below=None, ws=None):
    """The profiling pass over up to 8 bf16 weights in one quantizer launch
    (qnf4_nf4_layer_stats_group): the list of NF4 reconstruction SSEs (float64 [1] each) and,
    unless tau is None, the list of #{|w| < tau} counts; returns (sse list, count list or
    None). sse and below, when given, are lists of float64 tensors (one per weight)."""
    n = len(Ws)
    for W in Ws:
        _req(W, torch.bfloat16, "W")
    dev = Ws[0].device
    sse = sse if sse is not None else [torch.empty(2, dtype=torch.float64, device=dev) for _ in Ws]
    cnt = None
    if tau is not None:
        cnt = below if below is not None else [torch.empty(2, dtype=torch.float64, device=dev) for _ in Ws]
    wsb = _ws(workspace_size(_lib.OP_LAYER_STATS_GROUP, 0, 0), Ws[0], ws)
    ptrs = lambda ts: (C.c_void_p * n)(*[t.data_ptr() for t in ts])  # noqa: E731
    i64 = lambda v: (C.c_int64 * n)(*v)  # noqa: E731
    _lib.call("qnf4_nf4_layer_stats_group", n, ptrs(Ws), i64([W.shape[0] for W in Ws]),
              i64([W.shape[1] for W in Ws]), float(tau if tau is not None else 0.0), ptrs(sse),
              ptrs(cnt) if cnt is not None else None, wsb.data_ptr(), wsb.numel(), _stream(Ws[0]))
    return [t[:1] for t in sse], ([t[:1] for t in cnt] if cnt is not None else None)


def rank_topk(sse, n_params, k: int) -> list[int]:
    """Host ranking: indices of the k layers with the largest sse/n, ties to the lower index."""
    s = [float(v) for v in sse]
    n = [int(v) for v in n_params]
    L = len(s)
    sa = (C.c_double * L)(*s)
    na = (C.c_int64 * L)(*n)
    out = (C.c_int32 * max(k, 1))()
    _lib.call("qnf4_rank_topk", C.addressof(sa), C.addressof(na), L, k, C.addressof(out))
    return [int(out[i]) for i in range(k)]


def dense_linear_fwd(W: torch.Tensor, x, A, B, scale: float, h=None, ws=None) -> torch.Tensor:
    """The linear layer over a 16-bit (protected) base W bf16 [N, K]."""
    for t, nm in ((W, "W"), (x, "x"), (A, "A"), (B, "B")):
        _req(t, torch.bfloat16, nm)
    N, K = W.shape
    M, r = x.shape[0], A.shape[0]
    h = h if h is not None else torch.empty(M, N, dtype=torch.bfloat16, device=x.device)
    wsb = _ws(workspace_size(_lib.OP_FWD, N, K, M, r), x, ws)
    _lib.call("qnf4_dense_linear_fwd", W.data_ptr(), N, K, x.data_ptr(), M, A.data_ptr(),
              B.data_ptr(), r, float(scale), h.data_ptr(), wsb.data_ptr(), wsb.numel(), _stream(x))
    return h


def dense_linear_bwd(W: torch.Tensor, x, dY, A, B, scale: float, dX=None, dA=None, dB=None,
                     ws=None):
    for t, nm in ((W, "W"), (x, "x"), (dY, "dY"), (A, "A"), (B, "B")):
        _req(t, torch.bfloat16, nm)
    N, K = W.shape
    M, r = x.shape[0], A.shape[0]
    dev = x.device
    dX = dX if dX is not None else torch.empty(M, K, dtype=torch.bfloat16, device=dev)
    dA = dA if dA is not None else torch.empty(r, K, dtype=torch.float32, device=dev)
    dB = dB if dB is not None else torch.empty(N, r, dtype=torch.float32, device=dev)
    wsb = _ws(workspace_size(_lib.OP_BWD, N, K, M, r), x, ws)
    _lib.call("qnf4_dense_linear_bwd", W.data_ptr(), N, K, x.data_ptr(), dY.data_ptr(), M,
              A.data_ptr(), B.data_ptr(), r, float(scale), dX.data_ptr(), dA.data_ptr(),
              dB.data_ptr(), wsb.data_ptr(), wsb.numel(), _stream(x))
    return dX, dA, dB


def chanq_quantize(W: torch.Tensor, bits: torch.Tensor, thr: torch.Tensor, thr_off: torch.Tensor,
                   row_off: torch.Tensor, packed=None, absmax=None):
    """Per-output-channel threshold quantization: (packed u8, absmax fp32 [N*K/64])."""
    _req(W, torch.bfloat16, "W")
    _req(bits, torch.uint8, "bits")
    _req(thr, torch.float32, "thr")
    _req(thr_off, torch.int64, "thr_off")
    _req(row_off, torch.int64, "row_off")
    N, K = W.shape
    total = int(row_off[-1].item()) if packed is None else packed.numel()
    packed = packed if packed is not None else torch.empty(max(total, 16), dtype=torch.uint8, device=W.device)
    absmax = absmax if absmax is not None else torch.empty(N * K // 64, dtype=torch.float32, device=W.device)
    _lib.call("qnf4_chanq_quantize", W.data_ptr(), N, K, bits.data_ptr(), thr.data_ptr(),
              thr_off.data_ptr(), packed.data_ptr(), row_off.data_ptr(), absmax.data_ptr(),
              _stream(W))
    return packed, absmax


def chanq_linear_fwd(packed, row_off, bits, maps, map_off, absmax, N: int, K: int, x, A, B,
                     scale: float, h=None, ws=None) -> torch.Tensor:
    for t, nm in ((x, "x"), (A, "A"), (B, "B")):
        _req(t, torch.bfloat16, nm)
    M, r = x.shape[0], A.shape[0]
    h = h if h is not None else torch.empty(M, N, dtype=torch.bfloat16, device=x.device)
    wsb = _ws(workspace_size(_lib.OP_CHANQ_FWD, N, K, M, r), x, ws)
    _lib.call("qnf4_chanq_linear_fwd", packed.data_ptr(), row_off.data_ptr(), bits.data_ptr(),
              maps.data_ptr(), map_off.data_ptr(), absmax.data_ptr(), N, K, x.data_ptr(), M,
              A.data_ptr(), B.data_ptr(), r, float(scale), h.data_ptr(), wsb.data_ptr(),
              wsb.numel(), _stream(x))
    return h


def chanq_linear_bwd(packed, row_off, bits, maps, map_off, absmax, N: int, K: int, x, dY, A, B,
                     scale: float, dX=None, dA=None, dB=None, ws=None):
    """(dX bf16 [M, K], dA fp32 [r, K], dB fp32 [N, r]) through the frozen per-channel base."""
    for t, nm in ((x, "x"), (dY, "dY"), (A, "A"), (B, "B")):
        _req(t, torch.bfloat16, nm)
    M, r = x.shape[0], A.shape[0]
    dev = x.device
    dX = dX if dX is not None else torch.empty(M, K, dtype=torch.bfloat16, device=dev)
    dA = dA if dA is not None else torch.empty(r, K, dtype=torch.float32, device=dev)
    dB = dB if dB is not None else torch.empty(N, r, dtype=torch.float32, device=dev)
    wsb = _ws(workspace_size(_lib.OP_CHANQ_BWD, N, K, M, r), x, ws)
    _lib.call("qnf4_chanq_linear_bwd", packed.data_ptr(), row_off.data_ptr(), bits.data_ptr(),
              maps.data_ptr(), map_off.data_ptr(), absmax.data_ptr(), N, K, x.data_ptr(),
              dY.data_ptr(), M, A.data_ptr(), B.data_ptr(), r, float(scale), dX.data_ptr(),
              dA.data_ptr(), dB.data_ptr(), wsb.data_ptr(), wsb.numel(), _stream(x))
    return dX, dA, dB


def chanq_learn(W: torch.Tensor, bits: int, thr0: torch.Tensor, iters: int = 8):
    """Weighted Lloyd-Max tables of every row at one bit width: (map fp32 [N, 2^b],
    thr fp32 [N, 2^b - 1], err float64 [N], iterations int32 [N])."""
    _req(W, torch.bfloat16, "W")
    N, K = W.shape
    L = 1 << bits
    dev = W.device
    thr0 = thr0.to(device=dev, dtype=torch.float32).contiguous()
    mp = torch.empty(N, L, dtype=torch.float32, device=dev)
    th = torch.empty(N, L - 1, dtype=torch.float32, device=dev)
    err = torch.empty(N, dtype=torch.float64, device=dev)
    it = torch.empty(N, dtype=torch.int32, device=dev)
    _lib.call("qnf4_chanq_learn", W.data_ptr(), N, K, bits, thr0.data_ptr(), iters, mp.data_ptr(),
              th.data_ptr(), err.data_ptr(), it.data_ptr(), _stream(W))
    return mp, th, err, it


def loftq_nf4(W: torch.Tensor, r: int, steps: int = 5, ws=None):
    """LoftQ-style initialisation over the NF4 base: (the last step's ``Nf4Weight``,
    A fp32 [r, K], B fp32 [N, r], objectives ||W - Q - B A||_F^2 float64 [steps])."""
    _req(W, torch.bfloat16, "W")
    N, K = W.shape
    dev = W.device
    n = N * K
    packed = torch.empty(n // 2, dtype=torch.uint8, device=dev)
    code2 = torch.empty(n // BLOCK1, dtype=torch.uint8, device=dev)
    scale2 = torch.empty((n // BLOCK1 + BLOCK2 - 1) // BLOCK2, dtype=torch.float32, device=dev)
    mean = torch.empty(4, dtype=torch.float32, device=dev)
    A = torch.empty(r, K, dtype=torch.float32, device=dev)
    B = torch.empty(N, r, dtype=torch.float32, device=dev)
    errs = torch.empty(steps, dtype=torch.float64, device=dev)
    wsb = _ws(workspace_size(_lib.OP_LOFTQ, N, K, 0, r), W, ws)
    _lib.call("qnf4_loftq_nf4", W.data_ptr(), N, K, r, steps, packed.data_ptr(), code2.data_ptr(),
              scale2.data_ptr(), mean.data_ptr(), A.data_ptr(), B.data_ptr(), errs.data_ptr(),
              wsb.data_ptr(), wsb.numel(), _stream(W))
    return Nf4Weight(N, K, packed, code2, scale2, mean[:1]), A, B, errs


def check(stream: int | None = None) -> None:
    """Synchronise the stream and raise if a kernel's bounded wait gave up."""
    _lib.call("qnf4_check", torch.cuda.current_stream().cuda_stream if stream is None else stream)


def set_wait_timeout_ns(ns: int) -> None:
    _lib.call("qnf4_set_wait_timeout_ns", int(ns))
