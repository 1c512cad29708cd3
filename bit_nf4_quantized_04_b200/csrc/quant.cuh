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

// One group of 8 threads per 64-element block; each thread owns 8 consecutive
// elements (one 16-byte load) and writes 4 packed bytes. Optional outputs:
// WRITE -> packed codes and fp32 absmax; SSE -> per-CTA float64 partial sums of the
// single-level squared round-trip error (fp32 within a block).
//
// Code search (see Nf4Tables): q0 = RN(w * RN(1/c)) is within 3 ulp of the exact
// quotient x. Its bin k = round(H q0 + H), read off a magic-number float add, gives
// one table entry t_k | c_k; the code is c_k + (q0 >= t_k) unless |q0 - t_k| <= 2^-19,
// in which case the exact quotient and all thresholds decide.
template <bool WRITE, bool SSE>
__global__ void __launch_bounds__(256) k_nf4_quant(const uint16_t* __restrict__ W,
                                                   int64_t nblocks, uint32_t* __restrict__ packed,
                                                   float* __restrict__ absmax,
                                                   double* __restrict__ sse_part, QuantTab tab) {
  __shared__ float s_thr[16];
  __shared__ float s_lv[16];
  __shared__ float s_tc[2 * kMaxHalfBins + 1];
  __shared__ double s_red[8];
  for (int i = threadIdx.x; i < 16; i += blockDim.x) {
    s_thr[i] = tab.thr[i];
    s_lv[i] = tab.levels[i];
  }
  for (int i = threadIdx.x; i <= 2 * kMaxHalfBins; i += blockDim.x) s_tc[i] = tab.bin_tc[i];
  __syncthreads();

  const int H = tab.bin_h;
  const float hf = static_cast<float>(H);
  const float magic = hf + 12582912.0f;  // 1.5 * 2^23: the low bits of the sum hold round(H q0 + H)
  const int lane8 = threadIdx.x & 7;
  const int grp = (threadIdx.x >> 3) & 3;  // group within the warp
  // Loop bounds are per warp (4 consecutive blocks per warp-step) so that every
  // lane reaches the shuffles; groups past the end work on zeros and store nothing.
  const int64_t w0 = ((static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5) * 4;
  const int64_t gstride = ((static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5) * 4;
  double acc = 0.0;

  constexpr int U = 4;
  for (int64_t base = w0; base < nblocks; base += U * gstride) {
    uint4 v[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int64_t b = base + u * gstride + grp;
      v[u] = make_uint4(0u, 0u, 0u, 0u);
      if (b < nblocks) v[u] = ld_stream_u4(W + b * 64 + lane8 * 8);
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      if (base + u * gstride >= nblocks) break;  // uniform across the warp
      const int64_t b = base + u * gstride + grp;
      const bool valid = b < nblocks;
      float w[8];
      const uint32_t words[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        w[2 * j] = bf16lo(words[j]);
        w[2 * j + 1] = bf16hi(words[j]);
      }
      float m = 0.f;
#pragma unroll
      for (int j = 0; j < 8; ++j) m = fmaxf(m, fabsf(w[j]));
      m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 1));
      m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 2));
      m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 4));
      const float c = m;
      int code[8];
      if (c == 0.f) {
#pragma unroll
        for (int j = 0; j < 8; ++j) code[j] = 7;  // the exact-zero level
      } else {
        const float r = __frcp_rn(c);
        uint32_t amb = (H == 0 || !(c >= 0x1p-100f)) ? 0xFFu : 0u;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const float q0 = w[j] * r;
          const int k = __float_as_int(fmaf(q0, hf, magic)) - 0x4B400000;
          const float tk = s_tc[min(max(k, 0), 2 * kMaxHalfBins)];
          const float d = q0 - tk;
          code[j] = (__float_as_int(tk) & 15) + (d >= 0.f ? 1 : 0);
          amb |= (fabsf(d) <= 0x1p-19f ? 1u : 0u) << j;
        }
        if (amb) {
#pragma unroll
          for (int j = 0; j < 8; ++j)
            if ((amb >> j) & 1u) code[j] = nf4_code_exact(w[j], c, s_thr);
        }
      }
      if (WRITE && valid) {
        uint32_t word = 0;
#pragma unroll
        for (int j = 0; j < 4; ++j)
          word |= static_cast<uint32_t>((code[2 * j] << 4) | code[2 * j + 1]) << (8 * j);
        packed[b * 8 + lane8] = word;
        if (lane8 == 0) absmax[b] = c;
      }
      if (SSE) {
        float sse = 0.f;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const float e = w[j] - s_lv[code[j]] * c;
          sse = fmaf(e, e, sse);
        }
        sse += __shfl_xor_sync(0xffffffffu, sse, 1);
        sse += __shfl_xor_sync(0xffffffffu, sse, 2);
        sse += __shfl_xor_sync(0xffffffffu, sse, 4);
        if (lane8 == 0) acc += static_cast<double>(sse);
      }
    }
  }
  if (SSE) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if ((threadIdx.x & 31) == 0) s_red[threadIdx.x >> 5] = acc;
    __syncthreads();
    if (threadIdx.x == 0) {
      double t = 0.0;
      for (int i = 0; i < static_cast<int>(blockDim.x >> 5); ++i) t += s_red[i];
      sse_part[blockIdx.x] = t;
    }
  }
}

// Sum n float64 partials in a fixed order (one CTA of 256 threads) into *out.
__global__ void __launch_bounds__(256) k_sum_partials(const double* __restrict__ part, int n,
                                                      double* __restrict__ out) {
  __shared__ double s[256];
  double t = 0.0;
  for (int i = threadIdx.x; i < n; i += 256) t += part[i];
  s[threadIdx.x] = t;
  __syncthreads();
  for (int o = 128; o > 0; o >>= 1) {
    if (threadIdx.x < o) s[threadIdx.x] += s[threadIdx.x + o];
    __syncthreads();
  }
  if (threadIdx.x == 0) *out = s[0];
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
  if (threadIdx.x == 0) part[blockIdx.x] = s[0];
}

// Each CTA reduces the partials to the tensor mean (bf16-derived constants sum
// exactly in float64, so the mean is independent of the summation order), then one
// warp per 256-block: subtract the mean, block absmax, scale = absmax / 448 (IEEE
// division), code = E4M3 round-to-nearest-even with saturation of (c - mean)/scale.
__global__ void __launch_bounds__(256) k_dq_encode(const float* __restrict__ c, int64_t nb1,
                                                   const double* __restrict__ part, int npart,
                                                   uint8_t* __restrict__ code2,
                                                   float* __restrict__ scale2,
                                                   float* __restrict__ mean_out) {
  __shared__ float s_mu;
  const int lane = threadIdx.x & 31;
  if (threadIdx.x < 32) {
    double t = 0.0;
    for (int i = lane; i < npart; i += 32) t += part[i];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) t += __shfl_xor_sync(0xffffffffu, t, o);
    if (lane == 0) {
      const float mu = static_cast<float>(t / static_cast<double>(nb1));
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
    if (lane == 0) scale2[j] = s;
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
