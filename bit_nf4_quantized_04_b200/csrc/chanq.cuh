// Per-output-channel threshold quantizer with mixed 1/2/4-bit rows.
//
// Source: "LowRA" article (cloud.tencent.com.cn), §4.1: each output channel has its
// own precision, bin edges ("thresholds") and representative values ("mappings",
// Fig. 3); 64-element groups inside a row are normalised by their absmax as in QLoRA.
#pragma once
#include "common.cuh"
#include "quant.cuh"

namespace qnf4 {

constexpr int kCqTable = 256;  // table entries per warp (bins 0..2 H + 1 used, H <= 61)

// The four bin densities a row may use: odd, so that H t + H is never a half-integer
// (a bin edge) for a threshold t with a power-of-two denominator (any fp32 or bf16 t).
QNF4_DEV float chanq_h(int o) { return o == 0 ? 61.f : o == 1 ? 59.f : o == 2 ? 53.f : 47.f; }

// Code of x = fp32(w / g) against the row's nt sorted thresholds, exactly: IEEE
// quotient, then #{k : x > t_k}. Kept out of line (only values near a threshold, rows
// whose thresholds defeat the bin table, and tiny or zero groups take it).
__device__ __noinline__ int chanq_code_exact(float w, float g, const float* s_t, int nt) {
  const float x = g == 0.f ? 0.f : __fdiv_rn(w, g);
  int code = 0;
  for (int k = 0; k < nt; ++k) code += (x > s_t[k]) ? 1 : 0;
  return code;
}

// One warp per row (grid-stride over rows). Each lane owns 8 consecutive elements
// per step (one 16-byte load); 8 lanes form a 64-element group. A lane's 8 codes
// are b bytes of the row's MSB-first bit stream, stored with one 1/2/4-byte write.
//
// Code search per row: bins of width 1/H over the normalised range, bin
// j = round(x H + H) for the first H of chanq_h that keeps every threshold at least
// 2^-12 of a bin from a bin edge and puts at most two thresholds in one bin (the warp
// checks the four densities at once; a row where none qualifies takes the exact
// path). Table entry j holds the first two thresholds t, t' at or above the bin's lower
// edge (2.0 where there are none), with (number of thresholds below the edge) + 1 in
// the low 5 mantissa bits of t. For x in bin j, code = that count + [x > t] + [x > t']:
// no third threshold lies in the bin, and a value one bin off (only within 2^-16 of an
// edge) gets the same code, as no threshold is that close to an edge. d = fma(-g, t, w)
// has the sign of w/g - t exactly; values within 2^-17 g of t or t' (the low-bit
// perturbation of t and the rounding of the quotient both lie inside) take the exact
// path.
__global__ void __launch_bounds__(256) k_chanq_quant(const uint16_t* __restrict__ W, int64_t N,
                                                     int64_t K, const uint8_t* __restrict__ bits,
                                                     const float* __restrict__ thr,
                                                     const int64_t* __restrict__ thr_off,
                                                     uint8_t* __restrict__ packed,
                                                     const int64_t* __restrict__ row_off,
                                                     float* __restrict__ absmax) {
  __shared__ float s_t[8][16];
  __shared__ __align__(2048) float2 s_bin[8][kCqTable];
  const int lane = threadIdx.x & 31;
  const int wib = threadIdx.x >> 5;
  const int64_t warp = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
  const char* tbase = reinterpret_cast<const char*>(s_bin[wib]);
  for (int64_t i = warp; i < N; i += nwarps) {
    const int b = bits[i];
    const int nt = (1 << b) - 1;
    const int64_t t0 = thr_off[i];
    __syncwarp();
    if (lane < nt) s_t[wib][lane] = thr[t0 + lane];
    __syncwarp();
    // ---- the row's bin density: lane o < 4 checks chanq_h(o)
    bool good = false;
    if (lane < 4) {
      good = true;
      int prev = -1, prev2 = -2;
      const float hl = chanq_h(lane);
      for (int k = 0; k < nt; ++k) {
        const float v = fmaf(s_t[wib][k], hl, hl);  // rounding error far below the margin
        const float f = v - floorf(v);
        if (fabsf(f - 0.5f) < 0x1p-12f) good = false;  // near a bin edge
        const int j = static_cast<int>(floorf(v + 0.5f));
        if (j == prev2) good = false;                 // three thresholds in one bin
        prev2 = prev;
        prev = j;
      }
    }
    const unsigned ok = __ballot_sync(0xffffffffu, good) & 0xFu;
    const bool row_exact = ok == 0u;
    const float kH = chanq_h(row_exact ? 0 : __ffs(ok) - 1);
    // ---- the row's bin table: bins 0 .. 2 H + 1 (finite weights index no others; a
    // non-finite weight indexes entry 0 and its NaN or infinite residual sends the
    // group to the exact path)
    const int nbin = 2 * static_cast<int>(kH) + 2;
    for (int e = lane; e < nbin; e += 32) {
      const float lo = (static_cast<float>(e) - 0.5f) / kH - 1.f;  // bin e's lower edge
      int cnt = 0;
      float tn = 2.0f, tn2 = 2.0f;
      for (int k = nt - 1; k >= 0; --k) {
        const float t = s_t[wib][k];
        if (t < lo) {
          ++cnt;
        } else {
          tn2 = tn;
          tn = t;
        }
      }
      s_bin[wib][e] = make_float2(__uint_as_float((__float_as_uint(tn) & ~31u) | static_cast<uint32_t>(cnt + 1)), tn2);
    }
    __syncwarp();
    const float mg = kH + 12582912.0f;
    uint8_t* prow = packed + row_off[i];
    const uint16_t* wrow = W + i * K;
    for (int64_t base = 0; base < K; base += 256) {
      // The loop is uniform across the warp; with K a multiple of 64 a step past the
      // row's end idles whole 8-lane groups, which still join the shuffles.
      const int64_t e0 = base + lane * 8;
      const bool active = e0 < K;
      uint4 v = make_uint4(0u, 0u, 0u, 0u);
      if (active) v = *reinterpret_cast<const uint4*>(wrow + e0);
      const uint32_t words[4] = {v.x, v.y, v.z, v.w};
      float w[8];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        w[2 * j] = bf16lo(words[j]);
        w[2 * j + 1] = bf16hi(words[j]);
      }
      float m = fmaxf(fabsf(w[0]), fabsf(w[1]));
#pragma unroll
      for (int j = 2; j < 8; ++j) m = fmaxf(m, fabsf(w[j]));
      m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 1));
      m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 2));
      m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 4));
      int code[8];
      const float hr = kH * rcp_approx(m);
      float dmin = 3.0e38f;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const uint32_t kb = __float_as_uint(fmaf(w[j], hr, mg));
        const float2 tk = *reinterpret_cast<const float2*>(tbase + ((kb << 3) & 0x7F8u));
        const float d = fmaf(-m, tk.x, w[j]), d2 = fmaf(-m, tk.y, w[j]);
        // count + [d > 0] + [d2 > 0] (d, d2 = 0 fall in the exact path's window)
        code[j] = (__float_as_int(tk.x) & 31) + (__float_as_int(d) >> 31) + 1 + (__float_as_int(d2) >> 31);
        dmin = fminf(dmin, fminf(fabsf(d), fabsf(d2)));
      }
      if (row_exact || !(dmin > m * 0x1p-17f) || !(m >= 0x1p-100f)) {
#pragma unroll
        for (int j = 0; j < 8; ++j) code[j] = chanq_code_exact(w[j], m, s_t[wib], nt);
      }
      uint32_t stream = 0;  // the lane's 8 codes, first code in the top bits
#pragma unroll
      for (int j = 0; j < 8; ++j) stream = (stream << b) | static_cast<uint32_t>(code[j]);
      if (active) {
        // stream holds 8*b bits; byte 0 of the row stream is its most significant byte
        const int64_t off = e0 * b / 8;
        if (b == 4) {
          const uint32_t be = __byte_perm(stream, 0, 0x0123);
          *reinterpret_cast<uint32_t*>(prow + off) = be;
        } else if (b == 2) {
          const uint32_t be = __byte_perm(stream, 0, 0x3201) & 0xFFFFu;
          *reinterpret_cast<uint16_t*>(prow + off) = static_cast<uint16_t>(be);
        } else {
          prow[off] = static_cast<uint8_t>(stream);
        }
        if ((lane & 7) == 0) absmax[(i * K + e0) >> 6] = m;
      }
    }
  }
}


// Widen a per-channel weight into the NF4 storage layout for the transposed
// (backward dX) GEMM, which reads it like an NF4 weight: row n's codes (bits[n] in
// {1, 2, 4}, MSB-first at packed + row_off[n]) become 4-bit codes, element 2j in the
// high nibble of byte j (wide [N, K/2]); its 2^b mapping values become a 16-entry fp32
// table with the unused entries 0 (tab [N, 16]). One warp per row. Row offsets are
// multiples of K b / 8, a multiple of 8 bytes, so a 4-bit row's words are aligned.
__global__ void __launch_bounds__(256) k_chanq_widen(const uint8_t* __restrict__ packed,
                                                     const int64_t* __restrict__ row_off,
                                                     const uint8_t* __restrict__ bits,
                                                     const float* __restrict__ map,
                                                     const int64_t* __restrict__ map_off, int64_t N,
                                                     int64_t K, uint8_t* __restrict__ wide,
                                                     float* __restrict__ tab) {
  const int lane = threadIdx.x & 31;
  const int64_t warps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
  for (int64_t n = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5; n < N;
       n += warps) {
    const int b = bits[n];
    const uint8_t* src = packed + row_off[n];
    uint32_t* dst = reinterpret_cast<uint32_t*>(wide + n * (K / 2));
    for (int64_t wi = lane; wi < K / 8; wi += 32) {  // one output word = 8 codes
      uint32_t word = 0;
      if (b == 4) {
        word = *reinterpret_cast<const uint32_t*>(src + 4 * wi);
      } else {
        // code k of the 8 at bit (w - b (k + 1)) of the big-endian field of width w
        const uint32_t x = b == 2 ? ((static_cast<uint32_t>(src[2 * wi]) << 8) | src[2 * wi + 1])
                                  : static_cast<uint32_t>(src[wi]);
        const int w = 8 * b;
        const uint32_t m = (1u << b) - 1u;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const uint32_t hi = (x >> (w - b * (2 * j + 1))) & m;
          const uint32_t lo = (x >> (w - b * (2 * j + 2))) & m;
          word |= ((hi << 4) | lo) << (8 * j);
        }
      }
      dst[wi] = word;
    }
    if (lane < 16) tab[n * 16 + lane] = lane < (1 << b) ? map[map_off[n] + lane] : 0.f;
  }
}

}  // namespace qnf4
