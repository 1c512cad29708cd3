// Bandwidth-bound kernels: NF4 blockwise quantization (with the optional
// reconstruction error), double quantization of the block constants, and the
// stand-alone two-level dequantization.
//
// Sources: "QLoRA: Efficient Finetuning of Quantized LLMs" (Heng's Blog),
// 贡献一 4-bit NormalFloat and 贡献二 Double Quantization; "AQLoRA", §3.1.
#pragma once
#include "common.cuh"
#include "tables.h"

namespace qnf4 {

// NF4 tables passed by value to the kernels and staged in shared memory.
struct QuantTab {
  float thr[16];
  float levels[16];
  int bin_h;
  float bin_th[2 * (2 * kMaxHalfBins + 1)];
};

QNF4_DEV float rcp_approx(float x) {
  float r;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
  return r;
}


constexpr int kQuantMaxGrid = 1024;  // most quantize CTAs; the workspace holds that many partials
constexpr int kQChunkBlocks = 32;   // 64-element blocks per streamed chunk: one per lane
constexpr int kQStages = 2;         // chunks in flight per warp
constexpr int kQWorkers = 8;        // warps per CTA, each streaming its own chunks
constexpr int kQCtasPerSm = 3;      // resident CTAs per SM (registers and shared memory allow it)
constexpr int kQThreads = 32 * kQWorkers;
constexpr uint32_t kQChunkBytes = kQChunkBlocks * 128u;  // 4 KB of bf16
constexpr int kQMaxH = 16;          // largest bin count H the kernels' table holds
constexpr int kQTabCopies = 16;     // table copies, one per lane of a half warp
constexpr size_t kQSmem = static_cast<size_t>(kQWorkers) * kQStages * kQChunkBytes + 1024;
constexpr int kQMaxJobs = 8;        // weights one launch quantizes

// The weights of one quantize launch: their chunks form one list (job l's chunks are
// [chunk0[l], chunk0[l + 1])), so a group of weights streams as one. A job's partial
// sums go to part[l * kQuantMaxGrid + CTA].
struct QuantJobs {
  CUtensorMap map[kQMaxJobs];   // weight l as [nblocks, 64] bf16, boxes of kQChunkBlocks rows
  int64_t nblocks[kQMaxJobs];
  int64_t chunk0[kQMaxJobs + 1];
  uint32_t* packed[kQMaxJobs];
  float* absmax[kQMaxJobs];
  int n;
};

// Shared loads of read-only tables (filled before a CTA barrier), by 32-bit shared address;
// not volatile, so the compiler may schedule them freely.
QNF4_DEV float lds_f32q(uint32_t addr) {
  float v;
  asm("ld.shared.f32 %0, [%1];" : "=f"(v) : "r"(addr));
  return v;
}
QNF4_DEV float2 lds_f32x2q(uint32_t addr) {
  float2 v;
  asm("ld.shared.v2.f32 {%0, %1}, [%2];" : "=f"(v.x), "=f"(v.y) : "r"(addr));
  return v;
}
// A 16-byte stage load; volatile and ordered after the mbarrier wait that published it.
QNF4_DEV uint4 lds_u4(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "r"(addr));
  return v;
}
// t - [s < 0]: the sign of s (as a signed integer) taken from t's bits, one multiply-add
QNF4_DEV uint32_t sign_sub(uint32_t s, uint32_t t) {
  uint32_t r;
  asm("mad.hi.s32 %0, %1, 2, %2;" : "=r"(r) : "r"(s), "r"(t));
  return r;
}

// max(|a|, |b|) per bf16 lane, NaN if either lane is NaN; the sign bits of the result
// are not the absolute value's (xorsign), so callers mask them.
QNF4_DEV uint32_t bmax_abs2(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("max.NaN.xorsign.abs.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

// Codes of one 64-element block with finite absmax c > 0 (see k_nf4_quant): pw[u] gets
// the packed bytes of elements 8u .. 8u + 7, acc the squared residuals (SSE). SCALED
// decides on w f and c f instead (f a power of two), and acc then holds the residuals
// of the scaled values.
template <bool SCALED, bool SSE>
QNF4_DEV void nf4_block_codes(const uint4 (&v)[8], float c, float f, float hf, float2 mg2,
                              uint32_t toff, uint32_t lvb, uint32_t (&pw)[8], float2& acc) {
  const float cd = SCALED ? c * f : c;
  const float hr = hf * rcp_approx(cd);
  const float2 hr2 = make_float2(hr, hr), nc2 = make_float2(-cd, -cd);
#pragma unroll
  for (int u = 0; u < 8; ++u) {
    const uint32_t wd[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
    uint32_t ue[4], uo[4];  // codes (bits 0-3) of elements 8u + 2i and 8u + 2i + 1
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      float2 wp = make_float2(bf16lo(wd[i]), bf16hi(wd[i]));
      if (SCALED) wp = __fmul2_rn(wp, make_float2(f, f));
      const float2 kb = __ffma2_rn(wp, hr2, mg2);
      const float2 ta = lds_f32x2q(__float_as_uint(kb.x) * (8u * kQTabCopies) + toff);
      const float2 tb = lds_f32x2q(__float_as_uint(kb.y) * (8u * kQTabCopies) + toff);
      const float sx = fmaf(cd, ta.y, fmaf(-cd, ta.x, wp.x));
      const float sy = fmaf(cd, tb.y, fmaf(-cd, tb.x, wp.y));
      ue[i] = sign_sub(__float_as_uint(sx), __float_as_uint(ta.y));
      uo[i] = sign_sub(__float_as_uint(sy), __float_as_uint(tb.y));
      if (SSE) {
        const float2 r2 = __ffma2_rn(make_float2(lds_f32q(lvb + 4u * (ue[i] & 15u)),
                                                 lds_f32q(lvb + 4u * (uo[i] & 15u))),
                                     nc2, wp);
        acc = __ffma2_rn(r2, r2, acc);
      }
    }
    // byte i of each word from the i-th code; even elements into the high nibbles
    const uint32_t ev = __byte_perm(__byte_perm(ue[0], ue[1], 0x0040), __byte_perm(ue[2], ue[3], 0x0040), 0x5410);
    const uint32_t od = __byte_perm(__byte_perm(uo[0], uo[1], 0x0040), __byte_perm(uo[2], uo[3], 0x0040), 0x5410);
    pw[u] = ((ev << 4) & 0xF0F0F0F0u) | (od & 0x0F0F0F0Fu);
  }
}

// Blockwise NF4 quantization, one 64-element block per lane, of one or more weights
// (jobs) whose 32-block chunks form one list. Warp g of the grid takes the chunks
// g, g + G, ... (G = warps in the grid) through its own ring of
// kQStages shared-memory stages: its lane 0 issues one TMA tile load per chunk (the
// weight seen as a [blocks, 64] bf16 matrix, 128-byte swizzle, rows past the end
// zero-filled) as soon as the warp has finished the chunk that stage held; no copy warp
// and no barrier between warps. The swizzle puts 16-byte piece u of row r at piece
// u ^ (r mod 8), so the lanes' reads of piece u fall in eight different bank groups per
// quarter warp. Optional outputs: WRITE -> packed codes (32 bytes per block) and fp32
// absmax; SSE -> per-CTA float64 partial sums of the single-level squared round-trip
// error (fp32 within a block); CNT -> per-CTA float64 counts of the elements with
// |w| < tau (the sparsity of "AQLoRA" §3.1), exact integers; asum_part (optional, with
// WRITE) -> per-CTA float64 sums of the block constants, the partials of the double
// quantization's tensor mean. Partials are per job: a warp's chunks run through the
// jobs in order, and it adds its sums into the CTA's slot of a job when it leaves it.
//
// absmax: max of |w| on the bf16 bit patterns, two elements per instruction.
// Code search (see Nf4Tables), for a block with finite absmax c > 0: the bin
// k = round(w H/c + H) comes from one fused multiply-add with a magic constant
// (1.5 * 2^23, whose low mantissa bits then hold k), so the table entry's shared
// address is one multiply-add of those bits. The entry (t_k, h'_k) gives the decision
// without a division: d = fma(-c, t_k, w), s = fma(c, h'_k, d); s < 0 exactly when the
// IEEE quotient RN(w / c) lies below t_k, and subtracting [s < 0] from h'_k's bits
// leaves the code in the low 4 bits. Blocks with c < 2^-64 or c >= 2^64 decide on w and
// c scaled by 2^64 or 2^-64 (the same quotient, every intermediate a normal float). An
// all-zero block takes code 7 (the exact zero level); a block holding an infinity or a
// NaN takes the code of the IEEE quotient: 7 for a finite w over an infinite c, 0
// (every comparison false) for the NaN quotients. The residual of the error is
// w - c q[code], one fma with the level read by the code.
template <bool WRITE, bool SSE, bool CNT = false>
__global__ void __launch_bounds__(kQThreads, kQCtasPerSm)
    k_nf4_quant(const __grid_constant__ QuantJobs jobs,
                double* __restrict__ sse_part, QuantTab tab, unsigned long long wait_ns,
                float tau = 0.f, double* __restrict__ cnt_part = nullptr,
                double* __restrict__ asum_part = nullptr) {
  extern __shared__ uint8_t qsm_raw[];
  __shared__ __align__(8) uint64_t full[kQWorkers][kQStages];
  __shared__ float s_lv[16];
  // entry k of copy j at (k kQTabCopies + j): a half warp's lanes read different copies
  __shared__ __align__(16) float2 s_th[(2 * kQMaxH + 1) * kQTabCopies];
  __shared__ double s_red[kQWorkers][kQMaxJobs];
  __shared__ unsigned long long s_cnt[kQWorkers][kQMaxJobs];
  __shared__ double s_asum[kQWorkers][kQMaxJobs];
  __shared__ volatile int s_abort;
  uint8_t* qsm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(qsm_raw) + 1023) &
                                            ~static_cast<uintptr_t>(1023));
  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const int H = tab.bin_h;
  for (int i = tid; i < 16; i += kQThreads) s_lv[i] = tab.levels[i];
  for (int i = tid; i < (2 * H + 1) * kQTabCopies; i += kQThreads) {
    const int k = i / kQTabCopies;
    s_th[i] = make_float2(tab.bin_th[2 * k], tab.bin_th[2 * k + 1]);
  }
  if (lane == 0) {
    for (int i = 0; i < kQStages; ++i) mbar_init(&full[warp][i], 1);
  }
  if (lane < kQMaxJobs) {
    s_red[warp][lane] = 0.0;
    s_cnt[warp][lane] = 0ull;
    s_asum[warp][lane] = 0.0;
  }
  if (tid < jobs.n) tma_prefetch_desc(&jobs.map[tid]);
  if (tid == 0) s_abort = 0;
  fence_mbar_init();
  __syncthreads();
  // launched as a programmatic dependent: the prologue above overlapped the previous
  // kernel; wait for it before touching global memory, and let the next kernel start
  griddep_wait();
  griddep_launch_dependents();

  const int64_t nchunks = jobs.chunk0[jobs.n];
  // the job of chunk c
  auto job_of = [&](int64_t c) {
    int l = 0;
    while (l + 1 < jobs.n && c >= jobs.chunk0[l + 1]) ++l;
    return l;
  };
  const int64_t gw = static_cast<int64_t>(blockIdx.x) * kQWorkers + warp;  // this warp
  const int64_t GW = static_cast<int64_t>(gridDim.x) * kQWorkers;
  const int64_t my = gw < nchunks ? (nchunks - 1 - gw) / GW + 1 : 0;      // its chunks
  uint8_t* ring = qsm + warp * (kQStages * kQChunkBytes);
  uint64_t* fb = full[warp];
  // lane 0 streams chunk j of this warp into stage j % kQStages (the whole box counts
  // towards the transaction bytes, zero-filled rows included)
  auto issue = [&](int64_t j) {
    const int64_t c = gw + j * GW;
    if (!in_bounds(c < nchunks, 1)) return;
    const int l = job_of(c);
    uint64_t* bar = &fb[j % kQStages];
    mbar_expect_tx(bar, kQChunkBytes);
    tma_load_2d(ring + (j % kQStages) * kQChunkBytes, &jobs.map[l], bar, 0,
                static_cast<int32_t>((c - jobs.chunk0[l]) * kQChunkBlocks));
  };
  if (lane == 0) {
    for (int64_t j = 0; j < min(my, static_cast<int64_t>(kQStages)); ++j) issue(j);
  }

  double acc = 0.0;
  double asum = 0.0;       // this lane's block constants (asum_part)
  unsigned int below = 0;  // this lane's elements with |w| < tau (CNT)
  const uint32_t taub = __float_as_uint(tau);
  const float hf = static_cast<float>(H);
  const float2 mg2 = make_float2(hf + 12582912.0f, hf + 12582912.0f);
  // bin k's entry of this lane's copy sits at shared address kb * 8 kQTabCopies + toff,
  // kb = 0x4B400000 + k being the bits of the magic fma's result (32-bit wrap-around)
  const uint32_t toff = smem_u32(s_th) + (lane & (kQTabCopies - 1)) * 8u -
                        0x4B400000u * (8u * kQTabCopies);
  const uint32_t lvb = smem_u32(s_lv);
  // add this warp's sums for job l into the CTA's slots and restart them (all lanes)
  auto flush = [&](int l) {
    if (SSE) {
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
      if (lane == 0) s_red[warp][l] += acc;
    }
    if (CNT) {
      unsigned long long b = below;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) b += __shfl_xor_sync(0xffffffffu, b, o);
      if (lane == 0) s_cnt[warp][l] += b;
    }
    if (WRITE && asum_part) {
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) asum += __shfl_xor_sync(0xffffffffu, asum, o);
      if (lane == 0) s_asum[warp][l] += asum;
    }
    acc = 0.0;
    asum = 0.0;
    below = 0;
  };
  int cur = -1;      // job of the warp's running sums
  int64_t done = 0;  // chunks consumed (their copies have landed)
  for (int64_t j = 0; j < my; ++j) {
    if (!warp_wait(&fb[j % kQStages], static_cast<uint32_t>((j / kQStages) & 1), wait_ns, &s_abort, 51))
      break;
    done = j + 1;
    const int64_t cj = gw + j * GW;
    const int l = job_of(cj);
    if (l != cur) {
      if (cur >= 0) flush(cur);
      cur = l;
    }
    const int64_t nblocks = jobs.nblocks[l];
    const int64_t blk = (cj - jobs.chunk0[l]) * kQChunkBlocks + lane;
    const bool valid = blk < nblocks;
    // this lane's row; piece u at row ^ (u << 4) (the swizzle)
    const uint32_t row = smem_u32(ring + (j % kQStages) * kQChunkBytes) + lane * 128u +
                         ((lane & 7u) << 4);
    uint4 v[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) v[u] = lds_u4(row ^ (static_cast<uint32_t>(u) << 4));
    uint32_t m2[4];
#pragma unroll
    for (int u = 0; u < 4; ++u)
      m2[u] = bmax_abs2(bmax_abs2(bmax_abs2(v[u].x, v[u].y), bmax_abs2(v[u].z, v[u].w)),
                        bmax_abs2(bmax_abs2(v[u + 4].x, v[u + 4].y), bmax_abs2(v[u + 4].z, v[u + 4].w)));
    const uint32_t mm = bmax_abs2(bmax_abs2(m2[0], m2[1]), bmax_abs2(m2[2], m2[3]));
    const uint32_t cb = max(mm & 0x7FFFu, (mm >> 16) & 0x7FFFu);
    const float c = __uint_as_float(cb << 16);
    if (CNT && valid) {
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const uint32_t wd[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          // |w| < tau on the magnitude bits (a NaN never counts)
          below += ((wd[i] << 16) & 0x7FFF0000u) < taub ? 1u : 0u;
          below += (wd[i] & 0x7FFF0000u) < taub ? 1u : 0u;
        }
      }
    }
    uint32_t pw[8];
    float2 acc2 = make_float2(0.f, 0.f);
    float ssq = 1.f;  // a scaled block's residuals times ssq are the true ones
    if (cb - 1u < 0x7F7Fu) {  // 0 < c < inf
      if (cb >= 0x1F80u && cb < 0x5F80u) {
        nf4_block_codes<false, SSE>(v, c, 1.f, hf, mg2, toff, lvb, pw, acc2);
      } else {
        // c < 2^-64 or c >= 2^64: decide on (w f) / (c f), f = 2^64 or 2^-64, which has
        // the same quotient and keeps c f, 1 / (c f) and the residuals normal floats (a
        // w f that lands below them is so far from every threshold that its rounding
        // cannot change a decision)
        const bool tiny = cb < 0x1F80u;
        nf4_block_codes<true, SSE>(v, c, tiny ? 0x1p64f : 0x1p-64f, hf, mg2, toff, lvb, pw, acc2);
        ssq = tiny ? 0x1p-64f : 0x1p64f;
      }
    } else {
      // c = 0 (all zeros: code 7) or a non-finite block: code 7 where the quotient is
      // a signed zero (finite w, infinite c), else 0 (a NaN quotient)
      const float2 nc2 = make_float2(-c, -c);
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const uint32_t wd[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
        uint32_t by[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const uint32_t kx = (cb > 0x7F80u || (wd[i] & 0x7FFFu) >= 0x7F80u) ? 0u : 7u;
          const uint32_t ky = (cb > 0x7F80u || (wd[i] & 0x7FFF0000u) >= 0x7F800000u) ? 0u : 7u;
          by[i] = (kx << 4) | ky;
          if (SSE) {
            const float2 r2 = __ffma2_rn(make_float2(s_lv[kx], s_lv[ky]), nc2,
                                         make_float2(bf16lo(wd[i]), bf16hi(wd[i])));
            acc2 = __ffma2_rn(r2, r2, acc2);
          }
        }
        pw[u] = __byte_perm(__byte_perm(by[0], by[1], 0x0040), __byte_perm(by[2], by[3], 0x0040), 0x5410);
      }
    }
    if (WRITE && valid && in_bounds(blk < nblocks, 2)) {
      uint4* dst = reinterpret_cast<uint4*>(jobs.packed[l]) + blk * 2;
      dst[0] = make_uint4(pw[0], pw[1], pw[2], pw[3]);
      dst[1] = make_uint4(pw[4], pw[5], pw[6], pw[7]);
      jobs.absmax[l][blk] = c;
      asum += static_cast<double>(c);
    }
    if (SSE && valid) acc += static_cast<double>((acc2.x + acc2.y) * ssq * ssq);
    // the warp is done with this stage: refill it with the chunk kQStages ahead (the
    // proxy fence orders the lanes' shared reads before the copy engine's writes)
    __syncwarp();
    if (lane == 0 && j + kQStages < my) {
      fence_proxy_async();
      issue(j + kQStages);
    }
  }
  // Drain: after a give-up, the copies this warp issued but did not consume must land
  // before the CTA exits (one deadline).
  if (lane == 0 && done < my) {
    const int64_t issued = min(my, done + static_cast<int64_t>(kQStages));
    const long long t0 = wait_clock();
    for (int64_t jj = done; jj < issued; ++jj) {
      while (!mbar_try_wait_long(&fb[jj % kQStages], static_cast<uint32_t>((jj / kQStages) & 1))) {
        if (wait_clock() - t0 > ns_cycles(drain_ns(wait_ns))) {
          set_err(52);
          break;
        }
      }
    }
  }
  if (cur >= 0) flush(cur);
  __syncthreads();
  // thread l writes job l's partials of this CTA (the warps' sums in a fixed order)
  if (tid < jobs.n && in_bounds(blockIdx.x < kQuantMaxGrid, 3)) {
    const int64_t o = static_cast<int64_t>(tid) * kQuantMaxGrid + blockIdx.x;
    if (WRITE && asum_part) {
      double t = 0.0;
      for (int i = 0; i < kQWorkers; ++i) t += s_asum[i][tid];
      asum_part[o] = t;  // exact: bf16-derived constants sum exactly in float64
    }
    if (SSE) {
      double t = 0.0;
      for (int i = 0; i < kQWorkers; ++i) t += s_red[i][tid];
      sse_part[o] = t;
    }
    if (CNT) {
      unsigned long long t = 0;
      for (int i = 0; i < kQWorkers; ++i) t += s_cnt[i][tid];
      cnt_part[o] = static_cast<double>(t);  // exact below 2^53
    }
  }
}

// Sum n float64 partials in a fixed order with the 256 threads of a CTA (all must call
// it); the result is valid in thread 0.
QNF4_DEV double block_sum_partials(const double* __restrict__ part, int n) {
  __shared__ double s[256];
  double t = 0.0;
  for (int i = threadIdx.x; i < n; i += 256) t += part[i];
  s[threadIdx.x] = t;
  __syncthreads();
  for (int o = 128; o > 0; o >>= 1) {
    if (threadIdx.x < o) s[threadIdx.x] += s[threadIdx.x + o];
    __syncthreads();
  }
  return s[0];
}

// Sum n float64 partials in a fixed order (one CTA of 256 threads) into *out.
__global__ void __launch_bounds__(256) k_sum_partials(const double* __restrict__ part, int n,
                                                      double* __restrict__ out) {
  griddep_wait();  // (programmatic dependent of the kernel that wrote the partials)
  griddep_launch_dependents();
  const double t = block_sum_partials(part, n);
  if (threadIdx.x == 0) *out = t;
}

// The per-job sums of a grouped statistics pass: CTA l sums job l's npart float64
// partials (at part + l kQuantMaxGrid) into *out[l], in k_sum_partials' order.
struct SumJobs {
  double* out[kQMaxJobs];
};
__global__ void __launch_bounds__(256) k_sum_partials_jobs(const double* __restrict__ part, int npart,
                                                           const __grid_constant__ SumJobs d) {
  griddep_wait();
  griddep_launch_dependents();
  const double t = block_sum_partials(part + static_cast<int64_t>(blockIdx.x) * kQuantMaxGrid, npart);
  if (threadIdx.x == 0) *d.out[blockIdx.x] = t;
}

// ---------------------------------------------------------------------------
// Double quantization (贡献二)
// ---------------------------------------------------------------------------
constexpr int kDqPartials = 256;

// Float64 partial sums of the first-level constants over contiguous chunks.
__global__ void __launch_bounds__(256) k_dq_partial(const float* __restrict__ c, int64_t nb1,
                                                    double* __restrict__ part) {
  __shared__ double s[256];
  const int64_t chunk = (nb1 + gridDim.x - 1) / gridDim.x;
  const int64_t lo = static_cast<int64_t>(blockIdx.x) * chunk;
  const int64_t hi = min(nb1, lo + chunk);
  double t = 0.0;
  for (int64_t i = lo + threadIdx.x; i < hi; i += 256) t += static_cast<double>(c[i]);
  s[threadIdx.x] = t;
  __syncthreads();
  for (int o = 128; o > 0; o >>= 1) {
    if (threadIdx.x < o) s[threadIdx.x] += s[threadIdx.x + o];
    __syncthreads();
  }
  if (threadIdx.x == 0 && in_bounds(blockIdx.x < kDqPartials, 4)) part[blockIdx.x] = s[0];
}

// The tensors of one double-quantization launch: their 256-blocks form one list (job
// l's are [b2_0[l], b2_0[l + 1])), which the CTAs take in contiguous runs of per_cta.
struct DqJobs {
  const float* c[kQMaxJobs];         // first-level constants [nb1]
  int64_t nb1[kQMaxJobs];
  int64_t count[kQMaxJobs];          // constants behind the mean's partials
  const double* part[kQMaxJobs];     // the mean's float64 partials, npart per job
  uint8_t* code2[kQMaxJobs];
  float* scale2[kQMaxJobs];
  float* mean[kQMaxJobs];
  const double* sse_part[kQMaxJobs];  // (fused quantize path) SSE partials, nsse per job
  double* sse_out[kQMaxJobs];         // or NULL
  int64_t b2_0[kQMaxJobs + 1];
  int64_t per_cta;
  int npart, nsse, n;
};

// Each CTA reduces the partials of the jobs it touches to their tensor means
// (bf16-derived constants sum exactly in float64, so a mean is independent of the
// summation order), then one warp per 256-block: subtract the mean, block absmax,
// scale = absmax / 448 (IEEE division), code = E4M3 round-to-nearest-even with
// saturation of (c - mean)/scale. A job's count is the number of constants behind its
// partials: nb1 for a whole matrix, the matrix's total for one row shard of it (whose
// partial is then the all-reduced sum). CTA l (l < n) writes job l's mean and, on the
// fused quantize path, folds its SSE partials in k_sum_partials' order.
__global__ void __launch_bounds__(256) k_dq_encode(const __grid_constant__ DqJobs d) {
  __shared__ float s_mu[kQMaxJobs];
  griddep_wait();  // (programmatic dependent of the kernel that wrote the constants)
  griddep_launch_dependents();
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  const int64_t lo = static_cast<int64_t>(blockIdx.x) * d.per_cta;
  const int64_t hi = min(d.b2_0[d.n], lo + d.per_cta);
  auto job_of = [&](int64_t j) {
    int l = 0;
    while (l + 1 < d.n && j >= d.b2_0[l + 1]) ++l;
    return l;
  };
  const int llo = lo < hi ? job_of(lo) : d.n, lhi = lo < hi ? job_of(hi - 1) : -1;
  const int own = static_cast<int>(blockIdx.x) < d.n ? static_cast<int>(blockIdx.x) : -1;
  if (own >= 0 && d.sse_out[own]) {
    const double t = block_sum_partials(d.sse_part[own], d.nsse);
    if (threadIdx.x == 0) *d.sse_out[own] = t;
  }
  // warp w computes job w's mean if this CTA needs it
  static_assert(kQMaxJobs <= 256 / 32, "one warp per job");
  if (wid < d.n && ((wid >= llo && wid <= lhi) || wid == own)) {
    double t = 0.0;
    for (int i = lane; i < d.npart; i += 32) t += d.part[wid][i];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) t += __shfl_xor_sync(0xffffffffu, t, o);
    if (lane == 0) {
      const float mu = static_cast<float>(t / static_cast<double>(d.count[wid]));
      s_mu[wid] = mu;
      if (wid == own) *d.mean[wid] = mu;
    }
  }
  __syncthreads();
  for (int64_t jg = lo + wid; jg < hi; jg += 8) {
    const int l = job_of(jg);
    const int64_t j = jg - d.b2_0[l];
    const float mu = s_mu[l];
    const float* __restrict__ c = d.c[l];
    const int64_t nb1 = d.nb1[l], nb2 = (nb1 + 255) / 256;
    uint8_t* __restrict__ code2 = d.code2[l];
    float* __restrict__ scale2 = d.scale2[l];
    const int64_t e0 = j * 256 + lane * 8;
    float v[8];
    if (e0 + 8 <= nb1) {
      const float4 a = *reinterpret_cast<const float4*>(c + e0);
      const float4 b = *reinterpret_cast<const float4*>(c + e0 + 4);
      v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
      v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
    } else {
#pragma unroll
      for (int k = 0; k < 8; ++k) v[k] = (e0 + k < nb1) ? c[e0 + k] : mu;  // mu -> 0 after subtract
    }
    float m = 0.f;
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      v[k] = v[k] - mu;
      m = fmaxf(m, fabsf(v[k]));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    const float s = (m == 0.f) ? 0.f : __fdiv_rn(m, 448.f);
    if (lane == 0 && in_bounds(j < nb2, 5)) scale2[j] = s;
    uint8_t q[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      q[k] = (m == 0.f) ? 0
                        : static_cast<uint8_t>(__nv_cvt_float_to_fp8(__fdiv_rn(v[k], s),
                                                                      __NV_SATFINITE, __NV_E4M3));
    }
    if (e0 + 8 <= nb1) {
      uint2 pk;
      pk.x = q[0] | (q[1] << 8) | (q[2] << 16) | (static_cast<uint32_t>(q[3]) << 24);
      pk.y = q[4] | (q[5] << 8) | (q[6] << 16) | (static_cast<uint32_t>(q[7]) << 24);
      *reinterpret_cast<uint2*>(code2 + e0) = pk;
    } else {
      for (int k = 0; k < 8; ++k)
        if (e0 + k < nb1) code2[e0 + k] = q[k];
    }
  }
}

// ---------------------------------------------------------------------------
// Stand-alone two-level dequantization (tests / export). One thread per 8 weights.
// c_hat = fma(e4m3(code2), scale2, mean); w_hat = levels[code] * c_hat (fp32).
// ---------------------------------------------------------------------------
template <bool BF16>
__global__ void __launch_bounds__(256) k_dequant(const uint32_t* __restrict__ packed,
                                                 const uint8_t* __restrict__ code2,
                                                 const float* __restrict__ scale2,
                                                 const float* __restrict__ mean, int64_t n8,
                                                 void* __restrict__ out, QuantTab tab) {
  __shared__ float s_lv[16];
  if (threadIdx.x < 16) s_lv[threadIdx.x] = tab.levels[threadIdx.x];
  __syncthreads();
  const float mu = *mean;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n8;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t b = i >> 3;  // 8 groups of 8 weights per 64-block
    if (!in_bounds(b < (n8 >> 3), 6)) continue;
    const float ch = fmaf(e4m3_to_f32(code2[b]), scale2[b >> 8], mu);
    const uint32_t word = packed[i];
    float o[8];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const uint32_t byte = (word >> (8 * j)) & 0xFFu;
      o[2 * j] = s_lv[byte >> 4] * ch;
      o[2 * j + 1] = s_lv[byte & 0xF] * ch;
    }
    if (BF16) {
      uint4 pk;
      pk.x = pack_bf16x2(o[0], o[1]);
      pk.y = pack_bf16x2(o[2], o[3]);
      pk.z = pack_bf16x2(o[4], o[5]);
      pk.w = pack_bf16x2(o[6], o[7]);
      reinterpret_cast<uint4*>(out)[i] = pk;
    } else {
      float4* f = reinterpret_cast<float4*>(out) + 2 * i;
      f[0] = make_float4(o[0], o[1], o[2], o[3]);
      f[1] = make_float4(o[4], o[5], o[6], o[7]);
    }
  }
}

}  // namespace qnf4
