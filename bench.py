#!/usr/bin/env python
"""Throughput of the QLoRA NF4 linear-layer hot path on B200.

One step = one pass of the whole hot path over the Llama-2-7B layer set
(q, k, v, o 4096x4096; gate, up 11008x4096; down 4096x11008; synthetic N(0, 0.02)
weights with 0.1% Student-t(3) outliers):
  * NF4 blockwise quantization of every bf16 weight, with the single-level
    reconstruction error (AQLoRA layer-ranking statistic) from the same pass,
    then double quantization of the block constants;
  * the fused forward h = x W^T + s (x A^T) B^T and backward (dX, dA, dB) of every
    layer at 4096 tokens (batch 4 x 1024), r = 16, alpha = 32;
  * the per-output-channel 1/2/4-bit quantizer and its forward on an 11008x4096
    weight at 2048 tokens.
value = fwd + bwd + per-channel-forward FLOPs of the step / step time (TFLOP/s),
with every other piece of the step inside the timed region.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Multi-GPU: ``--gpus N`` without a torchrun environment relaunches itself under
torch.distributed.run with N ranks on this node (127.0.0.1); each rank runs its own copy
of the step (independent layer sets, no collective on the data path: weak scaling) and
the time is the max over ranks.
--impl reference times the CPU oracle (the plain NumPy restatement of the pages) on
a bounded sample of the same step on the host cores.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import torch  # noqa: E402

M_TOK = 4096          # 4 x 1024 tokens
RANK = 16
ALPHA = 32.0
CQ_N, CQ_K, CQ_M = 11008, 4096, 2048
WORKLOAD = ("llama2-7b layer set (q,k,v,o 4096x4096; gate,up 11008x4096; down 4096x11008), "
            "4096 tokens, LoRA r=16 alpha=32: NF4 quantize + recon error + double quant, "
            "fused fwd+bwd; plus per-channel 1/2/4-bit quantize + fwd (11008x4096, 2048 tokens)")


# ----------------------------------------------------------------------------- helpers
def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return (float(d["hbm_gbs"]), float(d["bf16_tflops"]), float(d["bf16_tflops_sustained"]),
                "measured")
    return 6650.0, 1590.0, 1400.0, "fallback"


def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


class Clocks:
    """nvidia-smi sampler of SM clock and throttle reasons while work runs."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device: int):
        self.proc = None
        self.rows = []
        try:
            uuid = "GPU-" + str(torch.cuda.get_device_properties(device).uuid)
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", uuid, f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except Exception:
            self.proc.kill()
            out = ""
        for line in out.strip().splitlines():
            parts = [x.strip() for x in line.split(",")]
            if len(parts) >= 9:
                self.rows.append(parts)

    def summary(self):
        if not self.rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}

        def num(x):
            try:
                return float(x)
            except ValueError:
                return None
        sm = [num(r[1]) for r in self.rows if num(r[1]) is not None]
        mx = [num(r[2]) for r in self.rows if num(r[2]) is not None]
        load = [s for s in sm if s > 500] or sm
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in self.rows for i in range(4)
                          if r[5 + i].lower() == "active"})
        return {"sm_mhz": statistics.median(load) if load else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons,
                "samples": len(self.rows)}


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        info = threadpool_info()
        n = [d.get("num_threads", 1) for d in info if d.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return len(os.sched_getaffinity(0))


# ------------------------------------------------------------------------ flop / byte models
def layer_shapes():
    import synth
    return [(s.N, s.K) for s in synth.LLAMA7B_SET]


def fwd_flops(N, K, M, r):
    return 2.0 * M * N * K + 2.0 * M * r * (N + K)


def bwd_flops(N, K, M, r):
    return 2.0 * M * N * K + 4.0 * M * r * (N + K)


def step_flops():
    f = sum(fwd_flops(N, K, M_TOK, RANK) + bwd_flops(N, K, M_TOK, RANK) for N, K in layer_shapes())
    return f + fwd_flops(CQ_N, CQ_K, CQ_M, RANK)


# ------------------------------------------------------------------------------ CPU oracle
def oracle_sample(rows: int = 4096, m: int = 128):
    """Time the oracle, as it stands, on a bounded sample of the step: NF4 quantize +
    double quant + recon error of the first `rows` rows of the q_proj matrix (4096
    columns), and its fwd + bwd for m of the 4096 tokens.
    Returns (TFLOP/s, seconds, description, flops)."""
    import synth
    from oracle import linear as olin
    from oracle import nf4 as onf4
    N, K, r = rows, 4096, RANK
    W = synth.llama_weight((4096, K), synth.SEED_W)[:N].float().numpy()
    x = synth.normal_bf16((m, K), 1.0, synth.SEED_X).double().numpy()
    A = synth.normal_bf16((r, K), 0.01, synth.SEED_A).double().numpy()
    B = synth.normal_bf16((N, r), 0.01, synth.SEED_B).double().numpy()
    dY = synth.normal_bf16((m, N), 1.0, synth.SEED_DY).double().numpy()
    s = ALPHA / r
    t0 = time.perf_counter()
    codes, c = onf4.quantize(W)
    code2, s2, mu = onf4.double_quant(c)
    onf4.recon_sse(W)
    wb = olin.base_bf16(onf4.dequant(onf4.pack(codes), code2, s2, mu, N * K).reshape(N, K))
    olin.forward(x, wb, A, B, s)
    olin.backward(x, dY, wb, A, B, s)
    dt = time.perf_counter() - t0
    flops = fwd_flops(N, K, m, r) + bwd_flops(N, K, m, r)
    desc = (f"q_proj rows 0..{N} of 4096 (x4096 cols): NF4 quantize + double quant + recon "
            f"error + dequant, then fwd+bwd on {m} of 4096 tokens (r={r}); "
            "TFLOP/s = sample fwd+bwd FLOPs / time")
    return flops / dt / 1e12, dt, desc, flops


ORACLE_ROWS = 512  # the bounded sample both the reference arm and cpu_baseline time


def oracle_repeated(seconds: float):
    """The oracle on the step's bounded sample (ORACLE_ROWS rows of q_proj, 128 tokens),
    repeated until `seconds` have passed: (TFLOP/s, seconds, description, repeats)."""
    tot, fl, n, desc = 0.0, 0.0, 0, ""
    while tot < seconds or n == 0:
        _, dt, desc, f = oracle_sample(rows=ORACLE_ROWS)
        tot += dt
        fl += f
        n += 1
    return fl / tot / 1e12, tot, desc, n


# ------------------------------------------------------------------------------ GPU arm
class Workload:
    """Device-resident inputs, outputs and workspace of one step."""

    def __init__(self, q, dev, seed_offset=0):
        import synth
        self.q = q
        self.dev = dev
        self.s = ALPHA / RANK
        self.layers = []
        wsz = 0
        for i, (N, K) in enumerate(layer_shapes()):
            L = {}
            L["N"], L["K"] = N, K
            L["W"] = synth.llama_weight((N, K), synth.SEED_W + i + seed_offset, device=dev)
            L["x"] = synth.normal_bf16((M_TOK, K), 1.0, synth.SEED_X + i, device=dev)
            L["dY"] = synth.normal_bf16((M_TOK, N), 1.0, synth.SEED_DY + i, device=dev)
            L["A"] = synth.normal_bf16((RANK, K), 0.01, synth.SEED_A + i, device=dev)
            L["B"] = synth.normal_bf16((N, RANK), 0.01, synth.SEED_B + i, device=dev)
            n = N * K
            L["packed"] = torch.empty(n // 2, dtype=torch.uint8, device=dev)
            L["absmax"] = torch.empty(n // 64, dtype=torch.float32, device=dev)
            L["sse"] = torch.empty(2, dtype=torch.float64, device=dev)
            nb2 = (n // 64 + 255) // 256
            L["code2"] = torch.empty(n // 64, dtype=torch.uint8, device=dev)
            L["scale2"] = torch.empty(nb2, dtype=torch.float32, device=dev)
            L["mean"] = torch.empty(4, dtype=torch.float32, device=dev)
            L["w"] = q.Nf4Weight(N, K, L["packed"], L["code2"], L["scale2"], L["mean"][:1])
            L["h"] = torch.empty(M_TOK, N, dtype=torch.bfloat16, device=dev)
            L["dX"] = torch.empty(M_TOK, K, dtype=torch.bfloat16, device=dev)
            L["dA"] = torch.empty(RANK, K, dtype=torch.float32, device=dev)
            L["dB"] = torch.empty(N, RANK, dtype=torch.float32, device=dev)
            for op, m in ((q._lib.OP_QUANTIZE, 0), (q._lib.OP_DOUBLE_QUANT, 0), (q._lib.OP_LAYER_STATS, 0),
                          (q._lib.OP_QUANTIZE_WEIGHT, 0), (q._lib.OP_QUANTIZE_WEIGHT_GROUP, 0),
                          (q._lib.OP_LAYER_STATS_GROUP, 0),
                          (q._lib.OP_FWD, M_TOK), (q._lib.OP_BWD, M_TOK)):
                wsz = max(wsz, q.workspace_size(op, N, K, m, RANK))
            self.layers.append(L)
        # per-channel mixed precision layer
        bits = synth.chan_bits(CQ_N)
        maps, map_off, thr, thr_off = synth.chan_tables(bits)
        rowbytes = CQ_K * bits.to(torch.int64) // 8
        roff = torch.zeros(CQ_N + 1, dtype=torch.int64)
        roff[1:] = torch.cumsum(rowbytes, 0)
        self.cq = dict(
            W=synth.llama_weight((CQ_N, CQ_K), synth.SEED_W + 100 + seed_offset, device=dev),
            bits=bits.to(dev), maps=maps.to(dev), map_off=map_off.to(dev), thr=thr.to(dev),
            thr_off=thr_off.to(dev), roff=roff.to(dev),
            packed=torch.empty(int(roff[-1]) + 16, dtype=torch.uint8, device=dev),
            absmax=torch.empty(CQ_N * CQ_K // 64, dtype=torch.float32, device=dev),
            x=synth.normal_bf16((CQ_M, CQ_K), 1.0, synth.SEED_X + 50, device=dev),
            A=synth.normal_bf16((RANK, CQ_K), 0.01, synth.SEED_A + 50, device=dev),
            B=synth.normal_bf16((CQ_N, RANK), 0.01, synth.SEED_B + 50, device=dev),
            h=torch.empty(CQ_M, CQ_N, dtype=torch.bfloat16, device=dev),
            # backward through the per-channel base (a breakdown row, not in the step)
            dY=synth.normal_bf16((CQ_M, CQ_N), 1.0, synth.SEED_DY + 50, device=dev),
            dX=torch.empty(CQ_M, CQ_K, dtype=torch.bfloat16, device=dev),
            dA=torch.empty(RANK, CQ_K, dtype=torch.float32, device=dev),
            dB=torch.empty(CQ_N, RANK, dtype=torch.float32, device=dev))
        wsz = max(wsz, q.workspace_size(q._lib.OP_CHANQ_FWD, CQ_N, CQ_K, CQ_M, RANK),
                  q.workspace_size(q._lib.OP_CHANQ_BWD, CQ_N, CQ_K, CQ_M, RANK))
        self.ws = torch.empty(wsz, dtype=torch.uint8, device=dev)

    # the pieces of one step
    def quantize(self):
        # NF4 codes, constants, double quantization and the reconstruction SSE of the 7
        # layers: two launches for the set (qnf4_quantize_weight_group)
        L = self.layers
        self.q.quantize_weight_group([x["W"] for x in L], sse=True, outs=[x["w"] for x in L],
                                     absmax=[x["absmax"] for x in L], sse_out=[x["sse"] for x in L],
                                     ws=self.ws)

    def fwd(self, ev=None):
        for i, L in enumerate(self.layers):
            if ev is not None:
                self.q.lib.qnf4_set_timing_events(ev[i][0].cuda_event, ev[i][1].cuda_event)
            self.q.qlora_linear_fwd(L["w"], L["x"], L["A"], L["B"], self.s, h=L["h"], ws=self.ws)
        if ev is not None:
            self.q.lib.qnf4_set_timing_events(None, None)

    def bwd(self, ev=None):
        for i, L in enumerate(self.layers):
            if ev is not None:
                self.q.lib.qnf4_set_timing_events(ev[i][0].cuda_event, ev[i][1].cuda_event)
            self.q.qlora_linear_bwd(L["w"], L["x"], L["dY"], L["A"], L["B"], self.s, dX=L["dX"],
                                    dA=L["dA"], dB=L["dB"], ws=self.ws)
        if ev is not None:
            self.q.lib.qnf4_set_timing_events(None, None)

    def chanq(self):
        c = self.cq
        self.q.chanq_quantize(c["W"], c["bits"], c["thr"], c["thr_off"], c["roff"],
                              packed=c["packed"], absmax=c["absmax"])
        self.q.chanq_linear_fwd(c["packed"], c["roff"], c["bits"], c["maps"], c["map_off"],
                                c["absmax"], CQ_N, CQ_K, c["x"], c["A"], c["B"], self.s, h=c["h"],
                                ws=self.ws)

    def step(self, evf=None, evb=None):
        self.quantize()
        self.fwd(evf)
        self.bwd(evb)
        self.chanq()

    def layer_step(self, L):
        """One layer's share of the step (quantize + double quant, fwd, bwd): the unit the
        end-to-end run pipelines behind that layer's host-to-device copies."""
        q = self.q
        q.quantize_weight(L["W"], sse=True, out=L["w"], absmax=L["absmax"], sse_out=L["sse"],
                          ws=self.ws)
        q.qlora_linear_fwd(L["w"], L["x"], L["A"], L["B"], self.s, h=L["h"], ws=self.ws)
        q.qlora_linear_bwd(L["w"], L["x"], L["dY"], L["A"], L["B"], self.s, dX=L["dX"], dA=L["dA"],
                           dB=L["dB"], ws=self.ws)

    def input_groups(self):
        """inputs(), grouped by the unit that first needs them: one group per layer, then
        the per-channel layer's."""
        c = self.cq
        return [[L["W"], L["x"], L["A"], L["B"], L["dY"]] for L in self.layers] + \
            [[c["W"], c["bits"], c["thr"], c["thr_off"], c["roff"], c["maps"], c["map_off"],
              c["x"], c["A"], c["B"]]]

    def inputs(self):
        """Every tensor the step reads from outside (for the end-to-end copies)."""
        out = []
        for L in self.layers:
            out += [L["W"], L["x"], L["dY"], L["A"], L["B"]]
        c = self.cq
        out += [c["W"], c["x"], c["A"], c["B"], c["bits"], c["maps"], c["map_off"], c["thr"],
                c["thr_off"], c["roff"]]
        return out

    def results(self):
        """The step's training result read back by the host: adapter gradients and the
        per-layer reconstruction errors."""
        out = []
        for L in self.layers:
            out += [L["dA"], L["dB"], L["sse"][:1]]
        return out


def nbytes(ts):
    return sum(t.numel() * t.element_size() for t in ts)


def time_loop(fn, iters, stream):
    s = torch.cuda.Event(enable_timing=True)
    e = torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    s.record(stream)
    for _ in range(iters):
        fn()
    e.record(stream)
    e.synchronize()
    return s.elapsed_time(e) / 1e3 / iters


def lloyd_t0(bits: int):
    """Initial thresholds of the learner: 0.0 for 1 bit, the NormalFloat midpoints for
    2 and 4 bits (the page's initialisation), from the library's host-side codebook for
    4 bits and fixed values for 2 bits."""
    if bits == 1:
        return [0.0]
    if bits == 2:
        return [-0.5, 0.21790908, 0.7179091]
    import bit_nf4_quantized_04_b200 as q
    lv = q.nf4_codebook()[0]
    return [float((float(lv[k]) + float(lv[k + 1])) * 0.5) for k in range(15)]


def breakdown(wl, q, hbm, tc):
    """Per-row throughput, each timed alone (short loops, L2-exceeding inputs). Tensor
    rows are fractions of `tc`, the burst bf16 peak (each loop runs well under a second at
    full clock). The HBM-bound rows over the layer set replay a CUDA graph of their calls
    (as the protocol arms do), so the host's launch work does not leave the GPU idle."""
    st = torch.cuda.current_stream()
    out = {}
    nparam = sum(N * K for N, K in layer_shapes())
    t = time_loop(graphed(wl.quantize), 10, st)
    gbs = nparam * (2 + 0.5 + 1 / 64 + 4 / 16384) / t / 1e9
    out["quant_dq_sse"] = {"GBps": round(gbs, 1), "frac_hbm": round(gbs / hbm, 3),
                           "bytes_per_param": 2.5159}
    # the AQLoRA profiling pass over the layer set in one quantizer launch
    # (qnf4_nf4_layer_stats_group): the error alone, then with the sparsity count beside it
    Wl = [L["W"] for L in wl.layers]
    sl = [L["sse"] for L in wl.layers]
    cl = [torch.empty(2, dtype=torch.float64, device=wl.dev) for _ in wl.layers]
    t = time_loop(graphed(lambda: q.nf4_layer_stats_group(Wl, tau=None, sse=sl, ws=wl.ws)), 10, st)
    gbs = nparam * 2 / t / 1e9
    out["recon_error"] = {"GBps": round(gbs, 1), "frac_hbm": round(gbs / hbm, 3)}
    t = time_loop(graphed(lambda: q.nf4_layer_stats_group(Wl, tau=0.01, sse=sl, below=cl, ws=wl.ws)), 10, st)
    gbs = nparam * 2 / t / 1e9
    out["layer_stats"] = {"GBps": round(gbs, 1), "frac_hbm": round(gbs / hbm, 3)}
    ff = sum(fwd_flops(N, K, M_TOK, RANK) for N, K in layer_shapes())
    bf = sum(bwd_flops(N, K, M_TOK, RANK) for N, K in layer_shapes())
    t = time_loop(wl.fwd, 5, st)
    out["fwd_prefill"] = {"TFLOPs": round(ff / t / 1e12, 1), "frac_tc": round(ff / t / 1e12 / tc, 3)}
    t = time_loop(wl.bwd, 5, st)
    out["bwd_prefill"] = {"TFLOPs": round(bf / t / 1e12, 1), "frac_tc": round(bf / t / 1e12 / tc, 3)}
    c = wl.cq
    t = time_loop(lambda: q.chanq_quantize(c["W"], c["bits"], c["thr"], c["thr_off"], c["roff"],
                                           packed=c["packed"], absmax=c["absmax"]), 10, st)
    nb = CQ_N * CQ_K * (2 + 4 / 64) + float(c["roff"][-1].item())
    out["chanq_quantize"] = {"GBps": round(nb / t / 1e9, 1), "frac_hbm": round(nb / t / 1e9 / hbm, 3)}
    cf = fwd_flops(CQ_N, CQ_K, CQ_M, RANK)
    t = time_loop(lambda: q.chanq_linear_fwd(c["packed"], c["roff"], c["bits"], c["maps"],
                                             c["map_off"], c["absmax"], CQ_N, CQ_K, c["x"], c["A"],
                                             c["B"], wl.s, h=c["h"], ws=wl.ws), 5, st)
    out["chanq_fwd"] = {"TFLOPs": round(cf / t / 1e12, 1), "frac_tc": round(cf / t / 1e12 / tc, 3)}
    cb = bwd_flops(CQ_N, CQ_K, CQ_M, RANK)
    t = time_loop(lambda: q.chanq_linear_bwd(c["packed"], c["roff"], c["bits"], c["maps"],
                                             c["map_off"], c["absmax"], CQ_N, CQ_K, c["x"], c["dY"],
                                             c["A"], c["B"], wl.s, dX=c["dX"], dA=c["dA"],
                                             dB=c["dB"], ws=wl.ws), 5, st)
    out["chanq_bwd"] = {"TFLOPs": round(cb / t / 1e12, 1), "frac_tc": round(cb / t / 1e12 / tc, 3)}
    # the weighted Lloyd-Max learner of that layer's tables at 1, 2 and 4 bits (8
    # iterations each), e.g. for the precision allocation's per-channel errors; bound by
    # float64 arithmetic, reported as weight bytes read per second and time per layer
    t0s = {b: torch.tensor(lloyd_t0(b)) for b in (1, 2, 4)}
    t = time_loop(lambda: [q.chanq_learn(c["W"], b, t0s[b], 8) for b in (1, 2, 4)], 3, st)
    out["chanq_learn"] = {"GBps": round(3 * CQ_N * CQ_K * 2 / t / 1e9, 1), "ms": round(t * 1e3, 3),
                          "bound": "fp64 alu"}
    # LoftQ-style initialisation of that layer over the NF4 base (five alternating steps at
    # the adapter rank): time per layer; the Gram matrix and its eigensolve are library calls
    lws = torch.empty(q.workspace_size(q._lib.OP_LOFTQ, CQ_N, CQ_K, 0, RANK), dtype=torch.uint8,
                      device=wl.dev)
    q.loftq_nf4(c["W"], RANK, 5, ws=lws)
    t = time_loop(lambda: q.loftq_nf4(c["W"], RANK, 5, ws=lws), 2, st)
    out["loftq_init"] = {"ms": round(t * 1e3, 2), "steps": 5, "rank": RANK}
    del lws
    # decode (memory-bound): rotate over weight copies totalling at least 4x the L2
    l2 = torch.cuda.get_device_properties(wl.dev).L2_cache_size
    wbytes = sum(L["w"].nbytes() for L in wl.layers)
    copies = max(2, -(-4 * l2 // wbytes))
    pool = [[q.Nf4Weight(L["N"], L["K"], L["packed"].clone(), L["code2"].clone(),
                         L["scale2"].clone(), L["mean"].clone()[:1]) for L in wl.layers]
            for _ in range(copies)]
    dec = {}
    for m in (1, 4, 16):
        xs = [L["x"][:m].contiguous() for L in wl.layers]
        hs = [torch.empty(m, L["N"], dtype=torch.bfloat16, device=wl.dev) for L in wl.layers]
        ctr = [0]

        As = [L["A"] for L in wl.layers]
        Bs = [L["B"] for L in wl.layers]

        def run_group():  # the 7 layers in one grouped launch pair
            ws_ = pool[ctr[0] % copies]
            ctr[0] += 1
            q.qlora_linear_fwd_group(ws_, xs, As, Bs, wl.s, hs=hs, ws=wl.ws)

        def run_single():  # one call per layer
            ws_ = pool[ctr[0] % copies]
            ctr[0] += 1
            for i, L in enumerate(wl.layers):
                q.qlora_linear_fwd(ws_[i], xs[i], L["A"], L["B"], wl.s, h=hs[i], ws=wl.ws)
        byt = sum(N * K * (0.5 + 1 / 64 + 4 / 16384) + m * K * 2 + RANK * (N + K) * 2 + m * N * 2
                  for N, K in layer_shapes())
        res = {}
        for nm, run in (("group", run_group), ("single_calls", run_single)):
            run()
            torch.cuda.synchronize()
            # one decode pass is a few microseconds of GPU work per layer, far below the
            # host's per-call cost: capture the 7-layer passes over every weight copy in
            # one CUDA graph and time its replays
            graph = torch.cuda.CUDAGraph()
            with torch.cuda.graph(graph):
                for _ in range(copies):
                    run()
            graph.replay()
            torch.cuda.synchronize()
            t = time_loop(graph.replay, 3, torch.cuda.current_stream()) / copies
            res[nm] = {"GBps": round(byt / t / 1e9, 1), "frac_hbm": round(byt / t / 1e9 / hbm, 3),
                       "us": round(t * 1e6, 1)}
            del graph
        dec[f"M{m}"] = dict(res["group"], single_calls=res["single_calls"])
    out["decode_fwd"] = dec
    out["decode_fwd"]["pool_copies"] = copies
    out["decode_fwd"]["launch"] = ("CUDA graph of all copies; per copy one qnf4_qlora_linear_fwd_group "
                                   "call over the 7 layers (single_calls: one call per layer)")
    q.check()
    return out


def graphed(fn):
    """fn captured once into a CUDA graph (after one eager call, so every lazy set-up of
    the library and of torch has happened); returns the graph's replay."""
    fn()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        fn()
    g.replay()
    torch.cuda.synchronize()
    return g.replay


def arm_seconds(fn, seconds, stream):
    """Seconds per call of fn over a region of at least `seconds` (the iteration count is
    taken from one calibration call)."""
    t1 = time_loop(fn, 1, stream)
    iters = max(1, int(-(-seconds // max(t1, 1e-7))))
    return time_loop(fn, iters, stream), iters


def protocol(wl, q, hbm, tc_burst, tc_sus, dev, seconds=2.0, sessions=3):
    """The timing protocol of the AQLoRA page's speed measurements: every arm runs for a
    fixed duration (>= `seconds`), a duplicate of the step arm measures the noise floor,
    and the whole session of arms is repeated `sessions` times; per arm the median and
    the spread (max - min) / median over sessions. Quantize, forward, backward and decode
    arms replay CUDA graphs; the decode arm rotates over weight copies totalling >= 4x L2."""
    st = torch.cuda.current_stream()
    nparam = sum(N * K for N, K in layer_shapes())
    ff = sum(fwd_flops(N, K, M_TOK, RANK) for N, K in layer_shapes())
    bf = sum(bwd_flops(N, K, M_TOK, RANK) for N, K in layer_shapes())
    quant = graphed(wl.quantize)
    fwd = graphed(wl.fwd)
    bwd = graphed(wl.bwd)
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    wbytes = sum(L["w"].nbytes() for L in wl.layers)
    copies = max(2, -(-4 * l2 // wbytes))
    pool = [[q.Nf4Weight(L["N"], L["K"], L["packed"].clone(), L["code2"].clone(),
                         L["scale2"].clone(), L["mean"].clone()[:1]) for L in wl.layers]
            for _ in range(copies)]
    xs = [L["x"][:16].contiguous() for L in wl.layers]
    hs = [torch.empty(16, L["N"], dtype=torch.bfloat16, device=dev) for L in wl.layers]

    As = [L["A"] for L in wl.layers]
    Bs = [L["B"] for L in wl.layers]

    def dec_all():
        for ws_ in pool:
            q.qlora_linear_fwd_group(ws_, xs, As, Bs, wl.s, hs=hs, ws=wl.ws)
    dec = graphed(dec_all)
    dbytes = sum(N * K * (0.5 + 1 / 64 + 4 / 16384) + 16 * K * 2 + RANK * (N + K) * 2 + 16 * N * 2
                 for N, K in layer_shapes())
    sf = step_flops()
    arms = {
        "step": (wl.step, lambda t: sf / t / 1e12, "TFLOP/s"),
        "step_dup": (wl.step, lambda t: sf / t / 1e12, "TFLOP/s"),
        "quant_dq_sse": (quant, lambda t: nparam * 2.5159 / t / 1e9, "GB/s"),
        "fwd_prefill": (fwd, lambda t: ff / t / 1e12, "TFLOP/s"),
        "bwd_prefill": (bwd, lambda t: bf / t / 1e12, "TFLOP/s"),
        "decode_M16": (dec, lambda t: dbytes * copies / t / 1e9, "GB/s"),
    }
    vals = {k: [] for k in arms}
    clocks = Clocks(dev.index if dev.index is not None else 0)
    for _ in range(sessions):
        for k, (fn, conv, _) in arms.items():
            t, _ = arm_seconds(fn, seconds, st)
            vals[k].append(conv(t))
    clocks.stop()
    q.check()
    out = {"seconds_per_arm": seconds, "sessions": sessions, "clocks": clocks.summary(),
           "decode_pool_copies": copies, "arms": {}}
    for k, (_, _, unit) in arms.items():
        v = vals[k]
        med = statistics.median(v)
        row = {"median": round(med, 2), "unit": unit,
               "spread": round((max(v) - min(v)) / med, 4), "sessions": [round(x, 2) for x in v]}
        if unit == "GB/s":
            row["frac_hbm"] = round(med / hbm, 3)
        else:
            row["frac_tc_burst"] = round(med / tc_burst, 3)
            row["frac_tc_sustained"] = round(med / tc_sus, 3)
        out["arms"][k] = row
    out["noise_floor"] = round(statistics.median(
        [abs(a - b) / a for a, b in zip(vals["step"], vals["step_dup"])]), 4)
    return out


def stack13b(q, dev, hbm, tc, seconds=2.0):
    """The Llama-2-13B-shaped stack (40 layers x {5120^2 x4, 13824x5120 x2, 5120x13824},
    280 matrices, 12.69 B parameters, per-matrix std drawn from U[0.01, 0.04]): the
    AQLoRA profiling pass over the whole stack (NF4 + double quantization + the NF4
    reconstruction SSE of every matrix, qnf4_quantize_weight), the ranking that keeps the
    top-8 matrices by SSE per parameter in 16-bit, then forward + backward of every
    matrix at 8192 tokens with r = 64, alpha = 128, the 8 protected ones through the dense
    path. Timed: the profiling pass (GB/s at 2.5159 B/param) and the fwd + bwd pass
    (TFLOP/s), each over a region of at least `seconds`."""
    import synth
    st = torch.cuda.current_stream()
    shapes = synth.llama13b_stack()
    stds = synth.llama13b_stds()
    M, r, alpha, topk = 8192, 64, 128.0, 8
    s = alpha / r
    Ws, wq = [], []
    for i, sh in enumerate(shapes):
        Ws.append(synth.llama_weight((sh.N, sh.K), synth.SEED_W + 300 + i, std=float(stds[i]),
                                     device=dev))
        n = sh.N * sh.K
        wq.append(q.Nf4Weight(sh.N, sh.K, torch.empty(n // 2, dtype=torch.uint8, device=dev),
                              torch.empty(n // 64, dtype=torch.uint8, device=dev),
                              torch.empty((n // 64 + 255) // 256, dtype=torch.float32, device=dev),
                              torch.empty(4, dtype=torch.float32, device=dev)[:1]))
    nmax = max(sh.N * sh.K for sh in shapes)
    absmax = [torch.empty(nmax // 64, dtype=torch.float32, device=dev) for _ in range(8)]
    sse = torch.zeros(len(shapes), 2, dtype=torch.float64, device=dev)
    kinds = sorted({(sh.N, sh.K) for sh in shapes})
    io = {}
    wsz = q.workspace_size(q._lib.OP_QUANTIZE_WEIGHT_GROUP, 0, 0)
    for j, (N, K) in enumerate(kinds):
        io[(N, K)] = dict(
            x=synth.normal_bf16((M, K), 1.0, synth.SEED_X + 300 + j, device=dev),
            dY=synth.normal_bf16((M, N), 1.0, synth.SEED_DY + 300 + j, device=dev),
            A=synth.normal_bf16((r, K), 0.01, synth.SEED_A + 300 + j, device=dev),
            B=synth.normal_bf16((N, r), 0.01, synth.SEED_B + 300 + j, device=dev),
            h=torch.empty(M, N, dtype=torch.bfloat16, device=dev),
            dX=torch.empty(M, K, dtype=torch.bfloat16, device=dev),
            dA=torch.empty(r, K, dtype=torch.float32, device=dev),
            dB=torch.empty(N, r, dtype=torch.float32, device=dev))
        wsz = max(wsz, q.workspace_size(q._lib.OP_FWD, N, K, M, r),
                  q.workspace_size(q._lib.OP_BWD, N, K, M, r))
    ws = torch.empty(wsz, dtype=torch.uint8, device=dev)

    def profile_pass():
        # groups of 8 matrices, two launches per group (qnf4_quantize_weight_group); the
        # group's first-level constants go to per-matrix slices of one buffer
        for g0 in range(0, len(Ws), 8):
            ids = range(g0, min(g0 + 8, len(Ws)))
            q.quantize_weight_group([Ws[i] for i in ids], sse=True, outs=[wq[i] for i in ids],
                                    absmax=[absmax[k] for k in range(len(ids))],
                                    sse_out=[sse[i] for i in ids], ws=ws)
    profile = graphed(profile_pass)
    nparams = [sh.N * sh.K for sh in shapes]
    protected = q.rank_topk(sse[:, 0].cpu().tolist(), nparams, topk)
    prot = set(protected)

    def train_pass():
        for i, sh in enumerate(shapes):
            d = io[(sh.N, sh.K)]
            if i in prot:
                q.dense_linear_fwd(Ws[i], d["x"], d["A"], d["B"], s, h=d["h"], ws=ws)
                q.dense_linear_bwd(Ws[i], d["x"], d["dY"], d["A"], d["B"], s, dX=d["dX"],
                                   dA=d["dA"], dB=d["dB"], ws=ws)
            else:
                q.qlora_linear_fwd(wq[i], d["x"], d["A"], d["B"], s, h=d["h"], ws=ws)
                q.qlora_linear_bwd(wq[i], d["x"], d["dY"], d["A"], d["B"], s, dX=d["dX"],
                                   dA=d["dA"], dB=d["dB"], ws=ws)
    train_pass()
    torch.cuda.synchronize()
    tp, ip = arm_seconds(profile, seconds, st)
    tt, it = arm_seconds(train_pass, seconds, st)
    q.check()
    ptot = sum(nparams)
    fl = sum(fwd_flops(sh.N, sh.K, M, r) + bwd_flops(sh.N, sh.K, M, r) for sh in shapes)
    gbs = ptot * 2.5159 / tp / 1e9
    tfs = fl / tt / 1e12
    out = {"matrices": len(shapes), "params": ptot, "tokens": M, "r": r, "alpha": alpha,
           "profile_pass": {"GBps": round(gbs, 1), "frac_hbm": round(gbs / hbm, 3),
                            "ms": round(tp * 1e3, 2), "passes": ip,
                            "launch": "CUDA graph of 35 x qnf4_quantize_weight_group (8 matrices each)"},
           "protected_top8": protected,
           "fwd_bwd": {"TFLOPs": round(tfs, 1), "frac_tc": round(tfs / tc, 3),
                       "tflop_per_pass": round(fl / 1e12, 2), "ms": round(tt * 1e3, 1),
                       "passes": it}}
    del Ws, wq, io, ws, absmax
    torch.cuda.empty_cache()
    return out


def traffic_for(kernel: str):
    """DRAM bytes per unit of work from the committed ncu summary, if it was taken on
    the current source of the GEMM kernel; else None."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    try:
        d = json.load(open(p))
        src = open(os.path.join(ROOT, "bit_nf4_quantized_04_b200", "csrc", "gemm.cuh"), "rb").read()
        if d.get("gemm_sha1") != hashlib.sha1(src).hexdigest():
            return None
        return d["kernels"].get(kernel)
    except Exception:
        return None


def run_ours(args):
    ws_, rank, local = dist_env()
    if ws_ > 1:
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    import bit_nf4_quantized_04_b200 as q
    hbm, tc_burst, tc_sus, peak_kind = peaks()
    wl = Workload(q, dev, seed_offset=0)
    stream = torch.cuda.current_stream()
    K, W = args.steps, args.warmup
    evf = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(K * 7)]
    evb = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(K * 7)]
    # torch creates the CUDA event behind an Event on its first record: do that now, so
    # the library's hook receives live handles
    for a, b in evf + evb:
        a.record(stream)
        b.record(stream)
    torch.cuda.synchronize()
    # clock samples (every 200 ms) from the warm-up through the timed region and the
    # per-row breakdown that follows it
    clocks = Clocks(local)
    time.sleep(0.5)
    for _ in range(W):
        wl.step()
    q.check()
    if ws_ > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    t_start = torch.cuda.Event(enable_timing=True)
    t_stop = torch.cuda.Event(enable_timing=True)
    n0 = q.lib.qnf4_launch_count()
    t_start.record(stream)
    for k in range(K):
        wl.step(evf[7 * k:7 * k + 7], evb[7 * k:7 * k + 7])
    t_stop.record(stream)
    torch.cuda.synchronize()
    n1 = q.lib.qnf4_launch_count()
    if ws_ > 1:
        torch.distributed.barrier()
    elapsed = t_start.elapsed_time(t_stop) / 1e3
    q.check()
    from bit_nf4_quantized_04_b200.dist import max_over_ranks
    elapsed = max_over_ranks(elapsed, dev)
    # dominant kernel: the fwd h GEMM or the bwd dX GEMM, whichever took longer
    tf = sum(a.elapsed_time(b) for a, b in evf) / 1e3
    tb = sum(a.elapsed_time(b) for a, b in evb) / 1e3
    shapes = layer_shapes()
    per_f = sum(2.0 * M_TOK * N * Kk + 2.0 * M_TOK * RANK * N for N, Kk in shapes)
    per_b = sum(2.0 * M_TOK * N * Kk + 2.0 * M_TOK * RANK * Kk for N, Kk in shapes)
    if tf >= tb:
        kname, evs, per = "k_gemm<A_NF4_K> (fwd h = x W^T + LoRA)", evf, per_f
    else:
        kname, evs, per = "k_gemm<A_NF4_MN> (bwd dX = dY W + LoRA)", evb, per_b
    kt = sum(a.elapsed_time(b) for a, b in evs) / 1e3
    achieved = per * K / kt / 1e12
    # per-step achieved rate of that kernel (7 launches a step): its spread over the steps
    per_step = [per / (sum(a.elapsed_time(b) for a, b in evs[7 * k:7 * k + 7]) / 1e3) / 1e12
                for k in range(K)]
    tr = traffic_for("k_gemm<A_NF4_K>" if tf >= tb else "k_gemm<A_NF4_MN>")
    flops = step_flops()
    value = flops * K * ws_ / elapsed / 1e12
    extra = {}
    if ws_ == 1 and not args.no_breakdown:
        extra = breakdown(wl, q, hbm, tc_burst)
    else:
        time.sleep(0.5)
    clocks.stop()
    clk = clocks.summary()
    # The burst bf16 peak applies to a kernel timed in a short region at full clock; a
    # region of seconds under the power cap (SM clock held well below max) takes the
    # sustained one.
    smhz, smax = clk.get("sm_mhz"), clk.get("sm_max_mhz")
    long_region = elapsed >= 2.0 or (smhz is not None and smax and smhz < 0.9 * smax)
    tc_peak = tc_sus if long_region else tc_burst
    peak_kind = f"{peak_kind} bf16 {'sustained' if long_region else 'burst'}"
    proto = None
    stack = None
    if ws_ == 1 and not args.no_breakdown:
        if not args.no_stack:
            stack = stack13b(q, dev, hbm, tc_burst)
        if not args.no_protocol:
            proto = protocol(wl, q, hbm, tc_burst, tc_sus, dev)
    # end to end through the public API: pinned host inputs in, gradients out, per step.
    # The host-to-device copies run on a side stream in the order the layers need them;
    # each layer's kernels wait only for that layer's copies, so later copies overlap
    # earlier layers' compute. A step's copies start once the previous step's kernels are
    # done (the device buffers are reused).
    groups = wl.input_groups()
    ins = [t for g in groups for t in g]
    assert nbytes(ins) == nbytes(wl.inputs())
    host_groups = [[t.cpu().pin_memory() for t in g] for g in groups]
    res = wl.results()
    host_out = [torch.empty(t.shape, dtype=t.dtype, pin_memory=True) for t in res]
    h2d, d2h = nbytes(ins), nbytes(res)
    ke = max(1, min(K, 5))
    copy_stream = torch.cuda.Stream(device=dev)
    landed = [torch.cuda.Event() for _ in groups]

    def e2e_step():
        copy_stream.wait_stream(stream)
        with torch.cuda.stream(copy_stream):
            for g, hg, ev in zip(groups, host_groups, landed):
                for d, h in zip(g, hg):
                    d.copy_(h, non_blocking=True)
                ev.record(copy_stream)
        for L, ev in zip(wl.layers, landed):
            stream.wait_event(ev)
            wl.layer_step(L)
        stream.wait_event(landed[-1])
        wl.chanq()
        for h, d in zip(host_out, res):
            h.copy_(d, non_blocking=True)
    e2e_step()
    torch.cuda.synchronize()
    if ws_ > 1:
        torch.distributed.barrier()
    te = max_over_ranks(time_loop(e2e_step, ke, stream), dev)
    e2e_value = flops * ws_ / te / 1e12
    cpu = None
    if rank == 0 and ws_ == 1 and not args.no_cpu:
        v, dt, desc, n = oracle_repeated(10.0)
        cpu = {"value": round(v, 6), "unit": "TFLOP/s", "cores": blas_threads(), "kind": "oracle",
               "sample": desc + f"; repeated {n} times", "seconds": round(dt, 2)}
    if rank == 0:
        l2 = torch.cuda.get_device_properties(dev).L2_cache_size
        touched = sum(nbytes([L["W"], L["x"], L["dY"], L["h"], L["dX"], L["packed"]]) for L in wl.layers)
        line = {
            "metric": "QLoRA NF4 linear fwd+bwd TFLOP/s & GB/s (% roofline); NF4 quant+DQ GB/s",
            "value": round(value, 2), "unit": "TFLOP/s", "n_gpus": ws_, "steps": K, "warmup": W,
            "ms_per_step": round(elapsed / K * 1e3, 3), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": WORKLOAD, "tokens": M_TOK, "r": RANK, "alpha": ALPHA,
                       "layers": 7, "params": sum(N * K for N, K in shapes),
                       "flops_per_step": flops, "parallelism": f"independent replicas x{ws_}",
                       "l2": f"inputs larger than L2: {touched / 1e9:.2f} GB touched per step "
                             f"vs {l2 / 1e6:.0f} MB L2"},
            "roofline": {"bound": "tensor", "kernel": kname, "achieved": round(achieved, 1),
                         "peak": tc_peak, "unit": "TFLOP/s", "frac": round(achieved / tc_peak, 3),
                         "peak_kind": peak_kind,
                         "timed_region_s": round(elapsed, 4),
                         "spread": round((max(per_step) - min(per_step)) / statistics.median(per_step), 4),
                         "achieved_per_step_median": round(statistics.median(per_step), 1),
                         # dram bytes per algorithmic FLOP (ncu, gate-shaped launch) x the
                         # average FLOPs of one of this kernel's launches in the step
                         "traffic": round(tr * per / len(shapes)) if tr else None},
            "e2e": {"value": round(e2e_value, 2), "unit": "TFLOP/s", "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h},
            "gpu_launches": int(n1 - n0),
            "clocks": clk,
            "cpu_baseline": cpu,
            "breakdown": extra,
        }
        if stack is not None:
            line["stack13b"] = stack
        if proto is not None:
            line["protocol"] = proto
        print(json.dumps(line), flush=True)
    if ws_ > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()


def run_case(args):
    """One operation on one gate-shaped layer (11008x4096 NF4 weight), or a grouped call
    over the 7-layer set (quant_group, decode_group), warmup + steps calls and nothing
    else: the small, L2-exceeding case for ncu captures."""
    import synth
    import bit_nf4_quantized_04_b200 as q
    dev = torch.device("cuda", 0)
    if args.case in ("quant_group", "decode_group"):
        shapes = layer_shapes()
        Ws = [synth.llama_weight((N, K), synth.SEED_W + i, device=dev) for i, (N, K) in enumerate(shapes)]
        gws = torch.empty(1 << 26, dtype=torch.uint8, device=dev)
        if args.case == "quant_group":
            outs, sses = q.quantize_weight_group(Ws, sse=True, ws=gws)
            fn = lambda: q.quantize_weight_group(Ws, sse=True, outs=outs, sse_out=sses, ws=gws)  # noqa: E731
            m = 0
        else:
            m = 16
            wq = q.quantize_weight_group(Ws, ws=gws)
            xs = [synth.normal_bf16((m, K), 1.0, synth.SEED_X + i, device=dev) for i, (N, K) in enumerate(shapes)]
            As = [synth.normal_bf16((RANK, K), 0.01, synth.SEED_A + i, device=dev) for i, (N, K) in enumerate(shapes)]
            Bs = [synth.normal_bf16((N, RANK), 0.01, synth.SEED_B + i, device=dev) for i, (N, K) in enumerate(shapes)]
            hs = [torch.empty(m, N, dtype=torch.bfloat16, device=dev) for N, K in shapes]
            fn = lambda: q.qlora_linear_fwd_group(wq, xs, As, Bs, ALPHA / RANK, hs=hs, ws=gws)  # noqa: E731
        for _ in range(args.warmup):
            fn()
        t = time_loop(fn, args.steps, torch.cuda.current_stream())
        q.check()
        print(json.dumps({"case": args.case, "layers": len(shapes), "M": m,
                          "calls": args.warmup + args.steps, "us_per_call": round(t * 1e6, 2)}))
        return
    N, K = 11008, 4096
    m = {"fwd": M_TOK, "bwd": M_TOK, "decode": 16}.get(args.case, M_TOK)
    W = synth.llama_weight((N, K), synth.SEED_W + 4, device=dev)
    x = synth.normal_bf16((m, K), 1.0, synth.SEED_X, device=dev)
    dY = synth.normal_bf16((m, N), 1.0, synth.SEED_DY, device=dev)
    A = synth.normal_bf16((RANK, K), 0.01, synth.SEED_A, device=dev)
    B = synth.normal_bf16((N, RANK), 0.01, synth.SEED_B, device=dev)
    w = q.quantize_weight(W)
    s = ALPHA / RANK
    wsz = max(q.workspace_size(q._lib.OP_FWD, N, K, m, RANK),
              q.workspace_size(q._lib.OP_BWD, N, K, m, RANK),
              q.workspace_size(q._lib.OP_QUANTIZE_WEIGHT, N, K))
    ws = torch.empty(wsz, dtype=torch.uint8, device=dev)
    h = torch.empty(m, N, dtype=torch.bfloat16, device=dev)
    if args.case in ("chanq_quant", "chanq_fwd", "chanq_bwd"):
        # the per-channel 1/2/4-bit layer of the step (11008 x 4096, 2048 tokens)
        bits = synth.chan_bits(CQ_N)
        maps, map_off, thr, thr_off = synth.chan_tables(bits)
        roff = torch.zeros(CQ_N + 1, dtype=torch.int64)
        roff[1:] = torch.cumsum(CQ_K * bits.to(torch.int64) // 8, 0)
        bits, maps, map_off, thr, thr_off, roff = (t.to(dev) for t in (bits, maps, map_off, thr, thr_off, roff))
        cW = synth.llama_weight((CQ_N, CQ_K), synth.SEED_W + 100, device=dev)
        cp = torch.empty(int(roff[-1]) + 16, dtype=torch.uint8, device=dev)
        cg = torch.empty(CQ_N * CQ_K // 64, dtype=torch.float32, device=dev)
        cx = synth.normal_bf16((CQ_M, CQ_K), 1.0, synth.SEED_X + 50, device=dev)
        cA = A[:, :CQ_K].contiguous()
        cB = synth.normal_bf16((CQ_N, RANK), 0.01, synth.SEED_B + 50, device=dev)
        ch = torch.empty(CQ_M, CQ_N, dtype=torch.bfloat16, device=dev)
        cws = torch.empty(max(q.workspace_size(q._lib.OP_CHANQ_FWD, CQ_N, CQ_K, CQ_M, RANK),
                              q.workspace_size(q._lib.OP_CHANQ_BWD, CQ_N, CQ_K, CQ_M, RANK)),
                          dtype=torch.uint8, device=dev)
        q.chanq_quantize(cW, bits, thr, thr_off, roff, packed=cp, absmax=cg)
        if args.case == "chanq_quant":
            fn = lambda: q.chanq_quantize(cW, bits, thr, thr_off, roff, packed=cp, absmax=cg)  # noqa: E731
        elif args.case == "chanq_bwd":
            cdY = synth.normal_bf16((CQ_M, CQ_N), 1.0, synth.SEED_DY + 50, device=dev)
            fn = lambda: q.chanq_linear_bwd(cp, roff, bits, maps, map_off, cg, CQ_N, CQ_K, cx, cdY,  # noqa: E731
                                            cA, cB, s, ws=cws)
        else:
            fn = lambda: q.chanq_linear_fwd(cp, roff, bits, maps, map_off, cg, CQ_N, CQ_K, cx, cA, cB, s,  # noqa: E731
                                            h=ch, ws=cws)
        N, K, m = CQ_N, CQ_K, (0 if args.case == "chanq_quant" else CQ_M)
    elif args.case in ("fwd", "decode"):
        fn = lambda: q.qlora_linear_fwd(w, x, A, B, s, h=h, ws=ws)  # noqa: E731
    elif args.case == "bwd":
        fn = lambda: q.qlora_linear_bwd(w, x, dY, A, B, s, ws=ws)  # noqa: E731
    else:  # quant
        fn = lambda: q.quantize_weight(W, sse=True, ws=ws)  # noqa: E731  (one weight alone)
    for _ in range(args.warmup):
        fn()
    t = time_loop(fn, args.steps, torch.cuda.current_stream())
    q.check()
    print(json.dumps({"case": args.case, "N": N, "K": K, "M": m, "calls": args.warmup + args.steps,
                      "us_per_call": round(t * 1e6, 2)}))


def run_reference(args):
    ws_, rank, _ = dist_env()
    if rank != 0:
        return
    K, W = args.steps, args.warmup
    # each step: a ~1 s sample of the step (512 weight rows, 128 tokens)
    for _ in range(W):
        oracle_sample(rows=ORACLE_ROWS)
    times = []
    desc = ""
    flops = 0.0
    for _ in range(K):
        _, dt, desc, flops = oracle_sample(rows=ORACLE_ROWS)
        times.append(dt)
    tot = sum(times)
    value = flops * K / tot / 1e12
    line = {
        "impl": "reference",
        "metric": "QLoRA NF4 linear fwd+bwd TFLOP/s & GB/s (% roofline); NF4 quant+DQ GB/s",
        "value": round(value, 6), "unit": "TFLOP/s", "n_gpus": ws_, "steps": K, "warmup": W,
        "ms_per_step": round(tot / K * 1e3, 1), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": WORKLOAD, "tokens": M_TOK, "r": RANK, "alpha": ALPHA,
                   "sample": desc},
        "cpu_baseline": {"value": round(value, 6), "unit": "TFLOP/s", "cores": blas_threads(),
                         "kind": "oracle", "sample": desc},
        "e2e": {"value": round(value, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def relaunch(n: int) -> int:
    """Run this command again as n ranks of torch.distributed.run on this node."""
    import socket
    with socket.socket() as so:
        so.bind(("127.0.0.1", 0))
        port = so.getsockname()[1]
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", f"--nproc-per-node={n}",
           "--master-addr", "127.0.0.1", f"--master-port={port}", os.path.abspath(__file__),
           *sys.argv[1:]]
    return subprocess.run(cmd).returncode


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-breakdown", action="store_true")
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--no-stack", action="store_true", help="skip the 13B-stack row")
    ap.add_argument("--no-protocol", action="store_true", help="skip the 2 s x 3 session arms")
    ap.add_argument("--case", choices=["fwd", "bwd", "decode", "quant", "chanq_quant", "chanq_fwd", "chanq_bwd",
                                       "quant_group", "decode_group"], default=None,
                    help="run one operation on one gate-shaped layer (for ncu captures)")
    args = ap.parse_args()
    if args.gpus > 1 and "WORLD_SIZE" not in os.environ:
        sys.exit(relaunch(args.gpus))
    if args.case:
        run_case(args)
        return
    if args.warmup < 3 and args.impl == "ours":
        args.warmup = 3
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
