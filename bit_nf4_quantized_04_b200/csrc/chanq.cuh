// Per-output-channel threshold quantizer with mixed 1/2/4-bit rows.
//
// Source: "LowRA" article (cloud.tencent.com.cn), §4.1: each output channel has its
// own precision, bin edges ("thresholds") and representative values ("mappings",
// Fig. 3); 64-element groups inside a row are normalised by their absmax as in QLoRA.
#pragma once
#include "common.cuh"

namespace qnf4 {

// One warp per row (grid-stride over rows). Each lane owns 8 consecutive elements
// per step (one 16-byte load); 8 lanes form a 64-element group. A lane's 8 codes
// are b bytes of the row's MSB-first bit stream, stored with one 1/2/4-byte write.
__global__ void __launch_bounds__(256) k_chanq_quant(const uint16_t* __restrict__ W, int64_t N,
                                                     int64_t K, const uint8_t* __restrict__ bits,
                                                     const float* __restrict__ thr,
                                                     const int64_t* __restrict__ thr_off,
                                                     uint8_t* __restrict__ packed,
                                                     const int64_t* __restrict__ row_off,
                                                     float* __restrict__ absmax) {
  __shared__ float s_t[8][16];
  const int lane = threadIdx.x & 31;
  const int wib = threadIdx.x >> 5;
  const int64_t warp = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
  for (int64_t i = warp; i < N; i += nwarps) {
    const int b = bits[i];
    const int nt = (1 << b) - 1;
    const int64_t t0 = thr_off[i];
    __syncwarp();
    if (lane < nt) s_t[wib][lane] = thr[t0 + lane];
    __syncwarp();
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
      float m = 0.f;
#pragma unroll
      for (int j = 0; j < 8; ++j) m = fmaxf(m, fabsf(w[j]));
      m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 1));
      m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 2));
      m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 4));
      uint32_t stream = 0;  // the lane's 8 codes, first code in the top bits
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const float x = (m == 0.f) ? 0.f : __fdiv_rn(w[j], m);
        int code = 0;
        for (int k = 0; k < nt; ++k) code += (x > s_t[wib][k]) ? 1 : 0;
        stream = (stream << b) | static_cast<uint32_t>(code);
      }
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

}  // namespace qnf4
