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
  float bin_tc[2 * kMaxHalfBins + 1];
};

QNF4_DEV uint4 ld_stream_u4(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

// Exact code of w in a block with absolute maximum c > 0: x = RN(w / c) by IEEE
// division, code = #{k : x >= thr[k]}. Kept out of line: it runs only for values
// within 2^-19 of a decision threshold (or for blocks with a tiny absmax).
__device__ __noinline__ int nf4_code_exact(float w, float c, const float* s_thr) {
  const float x = __fdiv_rn(w, c);
  int code = 0;
#pragma unroll
  for (int k = 0; k < 15; ++k) code += (x >= s_thr[k]) ? 1 : 0;
  return code;
}

QNF4_DEV float rcp_approx(float x) {
  float r;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
  return r;
}


constexpr int kQuantMaxGrid = 1024;  // most quantize CTAs; the workspace holds that many partials
constexpr int kQChunkBlocks = 128;  // 64-element blocks per streamed chunk (16 KB of bf16)
constexpr int kQStages = 4;         // chunks in flight per CTA
constexpr int kQWorkers = 8;        // worker warps; one more warp issues the copies
constexpr int kQCtasPerSm = 3;      // resident CTAs per SM (registers and shared memory allow it)
constexpr int kQThreads = 32 * (kQWorkers + 1);
constexpr uint32_t kQChunkBytes = kQChunkBlocks * 128u;
constexpr size_t kQSmem = kQStages * kQChunkBytes + 128;

// Spin on a phase with a bound, in every lane of a warp, then agree: the result is
// the same in all lanes (all observed the phase, or the warp gives up together).
QNF4_DEV bool warp_wait(uint64_t* bar, uint32_t parity, unsigned long long wait_ns,
                        volatile int* abort_flag, unsigned int site) {
  bool ok = mbar_try_wait(bar, parity);
  if (!ok) {
    const uint64_t t0 = globaltimer();
    while (!(ok = mbar_try_wait(bar, parity))) {
      if (*abort_flag) break;
      if (globaltimer() - t0 > wait_ns) {
        set_err(site);
        *abort_flag = 1;
        break;
      }
    }
  }
  return __all_sync(0xffffffffu, ok);
}

// Shared loads of read-only tables (filled before a CTA barrier), by 32-bit shared address;
// not volatile, so the compiler may schedule them freely.
QNF4_DEV uint32_t lds_u32q(uint32_t addr) {
  uint32_t v;
  asm("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(addr));
  return v;
}
QNF4_DEV float lds_f32q(uint32_t addr) {
  float v;
  asm("ld.shared.f32 %0, [%1];" : "=f"(v) : "r"(addr));
  return v;
}
// (d >> 31) + t: the sign bit of d added to t's bits (one multiply-add)
QNF4_DEV uint32_t sign_add(uint32_t d, uint32_t t) {
  uint32_t r;
  asm("mad.hi.u32 %0, %1, 2, %2;" : "=r"(r) : "r"(d), "r"(t));
  return r;
}

// max(|a|, |b|) per bf16 lane, NaN if either lane is NaN; the sign bits of the result
// are not the absolute value's (xorsign), so callers mask them.
QNF4_DEV uint32_t bmax_abs2(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("max.NaN.xorsign.abs.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

// Blockwise NF4 quantization, streamed: each CTA walks its chunks (chunk c holds
// blocks [128 c, 128 c + 128)) through a ring of shared-memory stages. One warp
// fills the ring with cp.async.bulk; eight worker warps consume it, each releasing a
// stage with one arrival when done, so no warp waits for the others. Inside a chunk,
// four threads take one 64-element block, each 16 consecutive elements as two 16-byte
// shared loads (the first piece alternates between neighbouring blocks, so a quarter
// warp's loads hit eight different bank groups), and write 8 packed bytes. Optional
// outputs: WRITE -> packed codes and fp32 absmax; SSE -> per-CTA float64 partial sums
// of the single-level squared round-trip error (fp32 over a thread's 16 elements);
// CNT -> per-CTA float64 counts of the elements with |w| < tau (the sparsity of
// "AQLoRA" §3.1), exact integers; asum_part (optional, with WRITE) -> per-CTA float64
// sums of the block constants, the partials of the double quantization's tensor mean.
//
// absmax: max of |w| on the bf16 bit patterns, two elements per instruction; a block
// holding a NaN or an infinity has magnitude bits >= 0x7F80 and takes the exact path.
// Code search (see Nf4Tables), for a block with absmax c > 0: the bin
// k = round(w H/c + H) comes from one fused multiply-add with a magic constant
// (1.5 * 2^23, whose low mantissa bits then hold k), so the table entry's shared
// address is one multiply-add of those bits; the entry t_k carries (14 - c_k) mod 16 in
// its low mantissa bits; d = fma(-c, t_k, w) = w - c t_k rounded once, so its sign is
// exactly that of w/c - t_k, and adding d's sign bit to t_k's bits leaves 15 - code in
// the low 4 bits (the packed word is complemented once at the end). If any of a
// thread's 16 values lies within 2^-18 c of its t_k, those 16 take the exact IEEE
// quotient and the full count. The residual of the error is w - c q[code], one fma
// with the level read by the (complemented) code.
template <bool WRITE, bool SSE, bool CNT = false>
__global__ void __launch_bounds__(kQThreads, kQCtasPerSm)
    k_nf4_quant(const uint16_t* __restrict__ W, int64_t nblocks, uint32_t* __restrict__ packed,
                float* __restrict__ absmax, double* __restrict__ sse_part, QuantTab tab,
                unsigned long long wait_ns, float tau = 0.f, double* __restrict__ cnt_part = nullptr,
                double* __restrict__ asum_part = nullptr) {
  extern __shared__ uint8_t qsm_raw[];
  __shared__ __align__(8) uint64_t full[kQStages], empty[kQStages];
  __shared__ float s_thr[16];
  __shared__ float s_lv[16];
  __shared__ float s_lvc[16];  // levels by complemented code: s_lvc[i] = q[15 - i]
  __shared__ __align__(16) float s_tc[2 * kMaxHalfBins + 1];
  __shared__ double s_red[kQWorkers];
  __shared__ unsigned long long s_cnt[kQWorkers];
  __shared__ double s_asum[kQWorkers];
  __shared__ volatile int s_abort;
  uint8_t* qsm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(qsm_raw) + 127) &
                                            ~static_cast<uintptr_t>(127));
  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  for (int i = tid; i < 16; i += kQThreads) {
    s_thr[i] = tab.thr[i];
    s_lv[i] = tab.levels[i];
    s_lvc[i] = tab.levels[15 - i];
  }
  for (int i = tid; i <= 2 * kMaxHalfBins; i += kQThreads) s_tc[i] = tab.bin_tc[i];
  const int64_t nchunks = (nblocks + kQChunkBlocks - 1) / kQChunkBlocks;
  const int64_t my = blockIdx.x < nchunks ? (nchunks - 1 - blockIdx.x) / gridDim.x + 1 : 0;
  if (tid == 0) {
    for (int i = 0; i < kQStages; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], kQWorkers);
    }
    s_abort = 0;
    fence_mbar_init();
  }
  __syncthreads();

  double acc = 0.0;
  double asum = 0.0;       // this thread's block constants (asum_part; block leaders only)
  unsigned int below = 0;  // this thread's elements with |w| < tau (CNT)
  if (warp == kQWorkers) {
    // ---------------------------------------------------------------- producer
    if ((tid & 31) == 0) {
      int st = 0;
      uint32_t ph = 0;
      int64_t issued = 0;
      for (int64_t j = 0; j < my; ++j) {
        if (!mbar_try_wait(&empty[st], ph ^ 1u)) {
          const uint64_t t0 = globaltimer();
          bool ok = false;
          while (!(ok = mbar_try_wait_long(&empty[st], ph ^ 1u))) {
            if (s_abort) break;
            if (globaltimer() - t0 > wait_ns) {
              set_err(53);
              s_abort = 1;
              break;
            }
          }
          if (!ok) break;
        }
        const int64_t c = blockIdx.x + j * gridDim.x;
        const int64_t nb = min(static_cast<int64_t>(kQChunkBlocks), nblocks - c * kQChunkBlocks);
        const uint32_t bytes = static_cast<uint32_t>(nb) * 128u;
        if (!in_bounds(nb > 0 && c * kQChunkBlocks + nb <= nblocks, 1)) break;
        mbar_expect_tx(&full[st], bytes);
        bulk_load(qsm + st * kQChunkBytes, W + c * kQChunkBlocks * 64, bytes, &full[st]);
        issued = j + 1;
        if (++st == kQStages) {
          st = 0;
          ph ^= 1u;
        }
      }
      // Drain: every copy issued must land before the CTA exits (one deadline).
      const uint64_t t0 = globaltimer();
      for (int64_t jj = max(static_cast<int64_t>(0), issued - kQStages); jj < issued; ++jj) {
        while (!mbar_try_wait_long(&full[jj % kQStages], static_cast<uint32_t>((jj / kQStages) & 1))) {
          if (globaltimer() - t0 > drain_ns(wait_ns)) {
            set_err(52);
            break;
          }
        }
      }
    }
  } else {
    // ---------------------------------------------------------------- workers
    const int H = tab.bin_h;
    const float hf = static_cast<float>(H);
    const float2 mg2 = make_float2(hf + 12582912.0f, hf + 12582912.0f);
    // bin k's entry sits at shared address kb * 4 + toff, kb = 0x4B400000 + k being the
    // bits of the magic fma's result (32-bit wrap-around): one multiply-add
    const uint32_t toff = smem_u32(s_tc) - 0x4B400000u * 4u;
    const uint32_t lvoff = smem_u32(s_lvc);
    const int l4 = tid & 3;     // elements 16 l4 .. 16 l4 + 15 of the block
    const int grp = tid >> 2;   // 64 groups of four threads
    const int sw = grp & 1;     // which 16-byte piece this thread loads first
    const int p0 = 2 * l4 + sw, p1 = 2 * l4 + 1 - sw;
    int st = 0;
    uint32_t ph = 0;
    for (int64_t j = 0; j < my; ++j) {
      if (!warp_wait(&full[st], ph, wait_ns, &s_abort, 51)) break;
      const int64_t c0 = (blockIdx.x + j * gridDim.x) * kQChunkBlocks;
      const int nb = static_cast<int>(min(static_cast<int64_t>(kQChunkBlocks), nblocks - c0));
      const uint8_t* chunk = qsm + st * kQChunkBytes;
#pragma unroll 1
      for (int u = 0; u < kQChunkBlocks / 64; ++u) {
        const int bl = grp + 64 * u;  // block within the chunk
        const bool valid = bl < nb;   // groups past a partial chunk's end work on zeros
        uint4 va = make_uint4(0u, 0u, 0u, 0u), vb = va;
        if (valid) {
          va = *reinterpret_cast<const uint4*>(chunk + bl * 128 + p0 * 16);
          vb = *reinterpret_cast<const uint4*>(chunk + bl * 128 + p1 * 16);
        }
        const uint32_t wd[8] = {va.x, va.y, va.z, va.w, vb.x, vb.y, vb.z, vb.w};
        if (CNT && valid) {
#pragma unroll
          for (int e = 0; e < 8; ++e)
            below += (fabsf(bf16lo(wd[e])) < tau ? 1u : 0u) + (fabsf(bf16hi(wd[e])) < tau ? 1u : 0u);
        }
        uint32_t m2 = bmax_abs2(bmax_abs2(bmax_abs2(wd[0], wd[1]), bmax_abs2(wd[2], wd[3])),
                                bmax_abs2(bmax_abs2(wd[4], wd[5]), bmax_abs2(wd[6], wd[7])));
        uint32_t cb = max(m2 & 0x7FFFu, (m2 >> 16) & 0x7FFFu);
        cb = max(cb, __shfl_xor_sync(0xffffffffu, cb, 1));
        cb = max(cb, __shfl_xor_sync(0xffffffffu, cb, 2));
        const float c = __uint_as_float(cb << 16);
        uint32_t mc[16];  // 15 - code of the thread's elements: pieces p0 (0..7), p1 (8..15)
        float sse = 0.f;
        bool exact = cb >= 0x7F80u || H == 0 || !(c >= 0x1p-100f);
        if (cb == 0u) {
#pragma unroll
          for (int e = 0; e < 16; ++e) mc[e] = 8u;  // the exact-zero level (error 0)
          exact = false;
        } else if (!exact) {
          const float hr = hf * rcp_approx(c);
          const float2 hr2 = make_float2(hr, hr), nc2 = make_float2(-c, -c);
          float2 wp[8];
          float dmin = 3.0e38f;
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            wp[e] = make_float2(bf16lo(wd[e]), bf16hi(wd[e]));
            const float2 kb = __ffma2_rn(wp[e], hr2, mg2);
            const uint32_t ta = lds_u32q(__float_as_uint(kb.x) * 4u + toff);
            const uint32_t tb = lds_u32q(__float_as_uint(kb.y) * 4u + toff);
            const float dx = fmaf(-c, __uint_as_float(ta), wp[e].x);
            const float dy = fmaf(-c, __uint_as_float(tb), wp[e].y);
            dmin = fminf(dmin, fminf(fabsf(dx), fabsf(dy)));
            mc[2 * e] = sign_add(__float_as_uint(dx), ta) & 15u;
            mc[2 * e + 1] = sign_add(__float_as_uint(dy), tb) & 15u;
          }
          exact = !(dmin > c * 0x1p-18f);
          if (SSE && !exact) {
            // r = w - c q[code], two running sums of r^2 (even and odd elements)
            float2 acc2 = make_float2(0.f, 0.f);
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              const float2 r2 = __ffma2_rn(make_float2(lds_f32q(lvoff + 4u * mc[2 * e]),
                                                       lds_f32q(lvoff + 4u * mc[2 * e + 1])),
                                           nc2, wp[e]);
              acc2 = __ffma2_rn(r2, r2, acc2);
            }
            sse = acc2.x + acc2.y;
          }
        }
        if (exact) {
          // out of line: the IEEE quotient and the full threshold count (values near a
          // threshold, tiny or non-finite absmax, or no bin table)
          float a = 0.f, b = 0.f;
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const float w0 = bf16lo(wd[e]), w1 = bf16hi(wd[e]);
            const int k0 = nf4_code_exact(w0, c, s_thr), k1 = nf4_code_exact(w1, c, s_thr);
            mc[2 * e] = static_cast<uint32_t>(15 - k0);
            mc[2 * e + 1] = static_cast<uint32_t>(15 - k1);
            if (SSE) {
              const float r0 = fmaf(s_lv[k0], -c, w0), r1 = fmaf(s_lv[k1], -c, w1);
              a = fmaf(r0, r0, a);
              b = fmaf(r1, r1, b);
            }
          }
          sse = a + b;
        }
        const int64_t blk = c0 + bl;
        if (WRITE && valid) {
          // element 2i in the high nibble of byte i; the complemented nibbles are
          // packed, then the word is complemented once
          uint32_t pw[2];
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const uint32_t b0 = mc[8 * h + 0] * 16u + mc[8 * h + 1];
            const uint32_t b1 = mc[8 * h + 2] * 16u + mc[8 * h + 3];
            const uint32_t b2 = mc[8 * h + 4] * 16u + mc[8 * h + 5];
            const uint32_t b3 = mc[8 * h + 6] * 16u + mc[8 * h + 7];
            pw[h] = ~__byte_perm(__byte_perm(b0, b1, 0x0040), __byte_perm(b2, b3, 0x0040), 0x5410);
          }
          uint2 out;
          out.x = sw ? pw[1] : pw[0];  // piece 2 l4
          out.y = sw ? pw[0] : pw[1];  // piece 2 l4 + 1
          if (in_bounds(blk < nblocks, 2)) reinterpret_cast<uint2*>(packed)[blk * 4 + l4] = out;
          if (l4 == 0 && in_bounds(blk < nblocks, 2)) {
            absmax[blk] = c;
            asum += static_cast<double>(c);
          }
        }
        if (SSE && valid) acc += static_cast<double>(sse);
      }
      __syncwarp();
      if ((tid & 31) == 0) mbar_arrive(&empty[st]);  // this warp is done with the stage
      if (++st == kQStages) {
        st = 0;
        ph ^= 1u;
      }
    }
  }
  if (SSE) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if ((tid & 31) == 0 && warp < kQWorkers) s_red[warp] = acc;
  }
  if (CNT) {
    unsigned long long b = below;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) b += __shfl_xor_sync(0xffffffffu, b, o);
    if ((tid & 31) == 0 && warp < kQWorkers) s_cnt[warp] = b;
  }
  if (WRITE && asum_part) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) asum += __shfl_xor_sync(0xffffffffu, asum, o);
    if ((tid & 31) == 0 && warp < kQWorkers) s_asum[warp] = asum;
  }
  __syncthreads();
  if (WRITE && asum_part && tid == 0 && in_bounds(blockIdx.x < kQuantMaxGrid, 3)) {
    double t = 0.0;
    for (int i = 0; i < kQWorkers; ++i) t += s_asum[i];
    asum_part[blockIdx.x] = t;  // exact: bf16-derived constants sum exactly in float64
  }
  if (SSE && tid == 0 && in_bounds(blockIdx.x < kQuantMaxGrid, 3)) {
    double t = 0.0;
    for (int i = 0; i < kQWorkers; ++i) t += s_red[i];
    sse_part[blockIdx.x] = t;
  }
  if (CNT && tid == 0 && in_bounds(blockIdx.x < kQuantMaxGrid, 3)) {
    unsigned long long t = 0;
    for (int i = 0; i < kQWorkers; ++i) t += s_cnt[i];
    cnt_part[blockIdx.x] = static_cast<double>(t);  // exact below 2^53
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
  const double t = block_sum_partials(part, n);
  if (threadIdx.x == 0) *out = t;
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

// Each CTA reduces the partials to the tensor mean (bf16-derived constants sum
// exactly in float64, so the mean is independent of the summation order), then one
// warp per 256-block: subtract the mean, block absmax, scale = absmax / 448 (IEEE
// division), code = E4M3 round-to-nearest-even with saturation of (c - mean)/scale.
// count is the number of constants behind the partials: nb1 for a whole matrix, the
// matrix's total for one row shard of it (whose partial is then the all-reduced sum).
__global__ void __launch_bounds__(256) k_dq_encode(const float* __restrict__ c, int64_t nb1,
                                                   const double* __restrict__ part, int npart,
                                                   int64_t count, uint8_t* __restrict__ code2,
                                                   float* __restrict__ scale2,
                                                   float* __restrict__ mean_out,
                                                   const double* __restrict__ sse_part = nullptr,
                                                   int nsse = 0, double* __restrict__ sse_out = nullptr) {
  __shared__ float s_mu;
  const int lane = threadIdx.x & 31;
  // (fused quantize path) CTA 0 also folds the quantizer's SSE partials, in the same
  // order as k_sum_partials
  if (sse_out && blockIdx.x == 0) {
    const double t = block_sum_partials(sse_part, nsse);
    if (threadIdx.x == 0) *sse_out = t;
  }
  if (threadIdx.x < 32) {
    double t = 0.0;
    for (int i = lane; i < npart; i += 32) t += part[i];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) t += __shfl_xor_sync(0xffffffffu, t, o);
    if (lane == 0) {
      const float mu = static_cast<float>(t / static_cast<double>(count));
      s_mu = mu;
      if (blockIdx.x == 0) *mean_out = mu;
    }
  }
  __syncthreads();
  const float mu = s_mu;
  const int64_t nb2 = (nb1 + 255) / 256;
  const int64_t warp = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
  for (int64_t j = warp; j < nb2; j += nwarps) {
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
