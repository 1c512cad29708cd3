"""Out-of-bounds writes on ragged shapes, caught two ways.

* Canaries: every output of every entry point, and the workspace, is a view into a larger
  buffer whose 4 KB before and after it are filled with a byte pattern; after the call
  (and qnf4_check) those guard bytes must be unchanged.
* The checked build: libqnf4_checked.so is the same library compiled with -DQNF4_CHECKED,
  whose kernels test the indices of their global accesses (outputs, split-K partial tiles,
  arrival counters, block constants, streamed chunks) and skip and report any access
  outside its buffer as QNF4_ERR_BOUNDS. The same cases run in a child process with
  QNF4_LIB=checked; qnf4_check must stay clean there and every output must equal the
  default build's bit for bit (the checks change no arithmetic).

Shapes: N not a multiple of the 128-row tile, K not a multiple of 256 (a partial
double-quantization block), token counts that leave a partial column tile, ranks that
are not multiples of 16, and split contraction slices.
"""
import os
import subprocess
import sys

import pytest
import torch

import synth

pytestmark = pytest.mark.gpu

GUARD = 4096
PATTERN = 0xA5
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

NF4_CASES = [(40, 448, 3, 5), (200, 192, 17, 16), (264, 960, 130, 33), (136, 1024, 300, 8),
             (1000, 4096, 16, 64)]
CHANQ_CASES = [(40, 448, 5, 4), (200, 1024, 130, 16)]


class Guarded:
    """A tensor of `shape`/`dtype` inside a byte buffer with GUARD pattern bytes around it."""

    def __init__(self, shape, dtype):
        n = int(torch.Size(shape).numel()) * torch.empty(0, dtype=dtype).element_size()
        self.n = n
        self.buf = torch.full((n + 2 * GUARD,), PATTERN, dtype=torch.uint8, device="cuda")
        self.t = self.buf[GUARD:GUARD + n].view(dtype).view(shape)

    def intact(self) -> bool:
        return bool((self.buf[:GUARD] == PATTERN).all()) and \
            bool((self.buf[GUARD + self.n:] == PATTERN).all())


def _check_all(q, named):
    q.check()
    torch.cuda.synchronize()
    bad = [k for k, g in named.items() if not g.intact()]
    assert not bad, f"guard bytes overwritten around: {bad}"


def _nf4_case(q, N, K, M, r, seed):
    W = synth.llama_weight((N, K), seed, device="cuda")
    x = synth.normal_bf16((M, K), 1.0, seed + 1, device="cuda")
    A = synth.normal_bf16((r, K), 0.01, seed + 2, device="cuda")
    B = synth.normal_bf16((N, r), 0.01, seed + 3, device="cuda")
    dY = synth.normal_bf16((M, N), 1.0, seed + 4, device="cuda")
    n = N * K
    nb1 = n // 64
    nb2 = (nb1 + 255) // 256
    g = {k: Guarded(s, d) for k, (s, d) in {
        "packed": ((n // 2,), torch.uint8), "absmax": ((nb1,), torch.float32),
        "code2": ((nb1,), torch.uint8), "scale2": ((nb2,), torch.float32),
        "mean": ((4,), torch.float32), "sse": ((2,), torch.float64),
        "stats": ((4,), torch.float64), "deq32": ((N, K), torch.float32),
        "deq16": ((N, K), torch.bfloat16), "h": ((M, N), torch.bfloat16),
        "dX": ((M, K), torch.bfloat16), "dA": ((r, K), torch.float32),
        "dB": ((N, r), torch.float32), "hd": ((M, N), torch.bfloat16),
        "dXd": ((M, K), torch.bfloat16), "dAd": ((r, K), torch.float32),
        "dBd": ((N, r), torch.float32),
    }.items()}
    wsz = max(q.workspace_size(op, N, K, M, r) for op in
              (q._lib.OP_QUANTIZE_WEIGHT, q._lib.OP_LAYER_STATS, q._lib.OP_FWD, q._lib.OP_BWD))
    g["ws"] = Guarded((wsz,), torch.uint8)
    w = q.Nf4Weight(N, K, g["packed"].t, g["code2"].t, g["scale2"].t, g["mean"].t[:1])
    s = 16.0 / r
    q.quantize_weight(W, sse=True, out=w, absmax=g["absmax"].t, sse_out=g["sse"].t, ws=g["ws"].t)
    q.nf4_layer_stats(W, out=g["stats"].t, ws=g["ws"].t)
    q.dequant(w, torch.float32, out=g["deq32"].t)
    q.dequant(w, torch.bfloat16, out=g["deq16"].t)
    q.qlora_linear_fwd(w, x, A, B, s, h=g["h"].t, ws=g["ws"].t)
    q.qlora_linear_bwd(w, x, dY, A, B, s, dX=g["dX"].t, dA=g["dA"].t, dB=g["dB"].t, ws=g["ws"].t)
    q.dense_linear_fwd(W, x, A, B, s, h=g["hd"].t, ws=g["ws"].t)
    q.dense_linear_bwd(W, x, dY, A, B, s, dX=g["dXd"].t, dA=g["dAd"].t, dB=g["dBd"].t,
                       ws=g["ws"].t)
    _check_all(q, g)
    return {k: v.t.clone() for k, v in g.items() if k != "ws"}


def _chanq_case(q, N, K, M, r, seed):
    W = synth.llama_weight((N, K), seed, device="cuda")
    bits = synth.chan_bits(N)
    maps, map_off, thr, thr_off = synth.chan_tables(bits, seed=seed + 5)
    roff = torch.zeros(N + 1, dtype=torch.int64)
    roff[1:] = torch.cumsum(K * bits.to(torch.int64) // 8, 0)
    bits, maps, map_off, thr, thr_off, roff = (t.cuda() for t in (bits, maps, map_off, thr, thr_off, roff))
    x = synth.normal_bf16((M, K), 1.0, seed + 1, device="cuda")
    A = synth.normal_bf16((r, K), 0.01, seed + 2, device="cuda")
    B = synth.normal_bf16((N, r), 0.01, seed + 3, device="cuda")
    dY = synth.normal_bf16((M, N), 1.0, seed + 4, device="cuda")
    total = int(roff[-1].item())
    g = {k: Guarded(s, d) for k, (s, d) in {
        "packed": ((total,), torch.uint8), "absmax": ((N * K // 64,), torch.float32),
        "h": ((M, N), torch.bfloat16), "dX": ((M, K), torch.bfloat16),
        "dA": ((r, K), torch.float32), "dB": ((N, r), torch.float32)}.items()}
    wsz = max(q.workspace_size(q._lib.OP_CHANQ_FWD, N, K, M, r),
              q.workspace_size(q._lib.OP_CHANQ_BWD, N, K, M, r))
    g["ws"] = Guarded((wsz,), torch.uint8)
    s = 16.0 / r
    q.chanq_quantize(W, bits, thr, thr_off, roff, packed=g["packed"].t, absmax=g["absmax"].t)
    q.chanq_linear_fwd(g["packed"].t, roff, bits, maps, map_off, g["absmax"].t, N, K, x, A, B, s,
                       h=g["h"].t, ws=g["ws"].t)
    q.chanq_linear_bwd(g["packed"].t, roff, bits, maps, map_off, g["absmax"].t, N, K, x, dY, A, B,
                       s, dX=g["dX"].t, dA=g["dA"].t, dB=g["dB"].t, ws=g["ws"].t)
    _check_all(q, g)
    return {k: v.t.clone() for k, v in g.items() if k != "ws"}


def _all_cases(q):
    out = {}
    for i, (N, K, M, r) in enumerate(NF4_CASES):
        for k, v in _nf4_case(q, N, K, M, r, 6000 + 17 * i).items():
            out[f"nf4{i}.{k}"] = v
    for i, (N, K, M, r) in enumerate(CHANQ_CASES):
        for k, v in _chanq_case(q, N, K, M, r, 6500 + 17 * i).items():
            out[f"chanq{i}.{k}"] = v
    return out


def test_guard_bytes_survive_every_entry_point():
    import bit_nf4_quantized_04_b200 as q
    out = _all_cases(q)
    dump = os.environ.get("QNF4_GUARD_DUMP")
    if dump:  # the child run below: hand the outputs to the parent
        torch.save({k: v.cpu() for k, v in out.items()}, dump)


@pytest.mark.skipif(os.environ.get("QNF4_LIB") == "checked", reason="runs in the child only")
def test_checked_build_reports_nothing_and_matches(tmp_path):
    import bit_nf4_quantized_04_b200 as q
    lib = os.path.join(ROOT, "bit_nf4_quantized_04_b200", "libqnf4_checked.so")
    assert os.path.exists(lib), "libqnf4_checked.so missing: build with bit_nf4_quantized_04_b200/build.py"
    dump = str(tmp_path / "checked.pt")
    env = dict(os.environ, QNF4_LIB="checked", QNF4_GUARD_DUMP=dump)
    res = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
                          os.path.abspath(__file__), "-k", "guard_bytes_survive"],
                         cwd=ROOT, env=env, capture_output=True, text=True, timeout=900)
    assert res.returncode == 0, res.stdout[-3000:] + res.stderr[-3000:]
    theirs = torch.load(dump)
    ours = _all_cases(q)
    assert set(theirs) == set(ours)
    diff = [k for k in ours if not torch.equal(ours[k].cpu(), theirs[k])]
    assert not diff, f"checked build differs from the default build in: {diff[:10]}"
