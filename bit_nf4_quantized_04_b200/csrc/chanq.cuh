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
      if (row_exact || !(dmin > m * 0x1p-17f) || !(m >= 0x1p-100f && m < 0x1p64f)) {
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


// ---------------------------------------------------------------------------
// Weighted Lloyd-Max learner of a row's mapping and thresholds ("LowRA", 第五部分
// 映射与阈值学习器, with the §4.1 group normalisation). One CTA per row, L = 2^b levels.
// Values x = fp32(w / g) (0 in an all-zero group), weight g = the 64-group absmax.
// Each iteration: bin = #{k : x > t_k}; per bin S0 = sum g, S1 = sum g x in float64
// (the products of two fp32 values are exact there, so only the summation order, which
// is fixed here, differs from a sequential sum); centre m_k = fp32(S1 / S0) or the
// previous value for an empty bin; thresholds fp32((m_k + m_{k+1}) / 2); error
// E = (sum (g x) x - sum_k (2 m_k S1_k - m_k^2 S0_k)) / sum g, evaluated with explicit
// roundings (no contraction); from the second iteration on, E not below the previous
// one stops after that iteration. Initial centres: -1, midpoints of the initial
// thresholds, +1. Output: the last tables, the iterations run, and the mean over the
// row of (w - fp32(m[c] g))^2 (float64) with c from the output thresholds.
// ---------------------------------------------------------------------------
constexpr int kLearnThreads = 256;

// Fixed-order block sum of NV doubles per thread: warp butterflies, then the warps'
// results in warp order; the sums land in s_out[0..NV). Every thread of the block calls it.
template <int NV, int NW>
QNF4_DEV void learn_block_sum(double (&v)[NV], double* s_red, double* s_out) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
#pragma unroll
  for (int i = 0; i < NV; ++i) {
#pragma unroll
    for (int o = 16; o; o >>= 1) v[i] = __dadd_rn(v[i], __shfl_xor_sync(0xffffffffu, v[i], o));
  }
  if (lane == 0) {
#pragma unroll
    for (int i = 0; i < NV; ++i) s_red[warp * NV + i] = v[i];
  }
  __syncthreads();
  if (tid < NV) {
    double a = 0.0;
    for (int w = 0; w < NW; ++w) a = __dadd_rn(a, s_red[w * NV + tid]);
    s_out[tid] = a;
  }
  __syncthreads();
}

template <int L>
__global__ void __launch_bounds__(kLearnThreads) k_chanq_learn(
    const uint16_t* __restrict__ W, int64_t N, int64_t K, const float* __restrict__ thr0, int iters,
    float* __restrict__ map_out, float* __restrict__ thr_out, double* __restrict__ err_out,
    int* __restrict__ done_out) {
  constexpr int NW = kLearnThreads / 32;
  extern __shared__ float lsm[];
  float* sx = lsm;          // normalised values [K]
  float* sg = lsm + K;      // group absmax [K / 64]
  __shared__ double s_red[NW * 2 * L];
  __shared__ double s_S[2 * L];
  __shared__ double s_tot[2];
  __shared__ double s_term[L];
  __shared__ float s_t[L], s_m[L];
  __shared__ int s_stop;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

  for (int64_t n = blockIdx.x; n < N; n += gridDim.x) {
    const uint16_t* wr = W + n * K;
    // values and weights: a warp per 64-group, two elements per lane
    for (int64_t grp = warp; grp < K / 64; grp += NW) {
      const uint32_t pr = *reinterpret_cast<const uint32_t*>(wr + grp * 64 + 2 * lane);
      const float a = bf16lo(pr), b = bf16hi(pr);
      float mx = fmaxf(fabsf(a), fabsf(b));
#pragma unroll
      for (int o = 16; o; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
      sx[grp * 64 + 2 * lane] = mx > 0.f ? __fdiv_rn(a, mx) : 0.f;
      sx[grp * 64 + 2 * lane + 1] = mx > 0.f ? __fdiv_rn(b, mx) : 0.f;
      if (lane == 0) sg[grp] = mx;
    }
    __syncthreads();
    {
      double v[2] = {0.0, 0.0};  // sum g, sum (g x) x
      for (int64_t j = tid; j < K; j += kLearnThreads) {
        const double gg = sg[j >> 6], xx = sx[j];
        v[0] = __dadd_rn(v[0], gg);
        v[1] = __dadd_rn(v[1], __dmul_rn(__dmul_rn(gg, xx), xx));
      }
      learn_block_sum<2, NW>(v, s_red, s_S);
      if (tid == 0) {
        s_tot[0] = s_S[0];
        s_tot[1] = s_S[1];
      }
    }
    if (tid < L - 1) s_t[tid] = thr0[tid];
    __syncthreads();
    if (tid < L)
      s_m[tid] = tid == 0 ? -1.f
               : tid == L - 1 ? 1.f
                              : __double2float_rn(__dmul_rn(__dadd_rn(static_cast<double>(s_t[tid - 1]),
                                                                      static_cast<double>(s_t[tid])), 0.5));
    if (tid == 0) s_stop = 0;
    __syncthreads();
    double eprev = 0.0;  // thread 0
    int done = 0;
    for (int it = 0; it < iters; ++it) {
      float tr[L - 1];
#pragma unroll
      for (int k = 0; k < L - 1; ++k) tr[k] = s_t[k];
      // every bin's sums in registers, predicated (only bin c gains; the others add
      // exact zeros)
      double v[2 * L];
#pragma unroll
      for (int k = 0; k < 2 * L; ++k) v[k] = 0.0;
      for (int64_t j = tid; j < K; j += kLearnThreads) {
        const float xx = sx[j];
        int c = 0;
#pragma unroll
        for (int k = 0; k < L - 1; ++k) c += xx > tr[k] ? 1 : 0;
        const double gg = sg[j >> 6];
        const double gx = __dmul_rn(gg, static_cast<double>(xx));
#pragma unroll
        for (int k = 0; k < L; ++k) {
          v[k] = __dadd_rn(v[k], c == k ? gg : 0.0);
          v[L + k] = __dadd_rn(v[L + k], c == k ? gx : 0.0);
        }
      }
      learn_block_sum<2 * L, NW>(v, s_red, s_S);
      // centre k and its error term on thread k; thresholds on threads 0..L-2; the
      // terms summed in bin order on thread 0
      if (tid < L) {
        const double S0 = s_S[tid], S1 = s_S[L + tid];
        if (S0 > 0.0) s_m[tid] = __double2float_rn(__ddiv_rn(S1, S0));
        const double mk = s_m[tid];
        s_term[tid] = __dsub_rn(__dmul_rn(__dmul_rn(2.0, mk), S1), __dmul_rn(__dmul_rn(mk, mk), S0));
      }
      __syncthreads();
      if (tid < L - 1)
        s_t[tid] = __double2float_rn(__dmul_rn(__dadd_rn(static_cast<double>(s_m[tid]),
                                                         static_cast<double>(s_m[tid + 1])), 0.5));
      if (tid == 0) {
        double acc = 0.0;
        for (int k = 0; k < L; ++k) acc = __dadd_rn(acc, s_term[k]);
        const double E = s_tot[0] > 0.0 ? __ddiv_rn(__dsub_rn(s_tot[1], acc), s_tot[0]) : 0.0;
        if (it > 0 && E >= eprev) s_stop = 1;
        eprev = E;
      }
      done = it + 1;
      __syncthreads();
      if (s_stop) break;
    }
    // the error of the quantization the output tables give
    {
      float tr[L - 1];
#pragma unroll
      for (int k = 0; k < L - 1; ++k) tr[k] = s_t[k];
      double v[1] = {0.0};
      for (int64_t j = tid; j < K; j += kLearnThreads) {
        const float xx = sx[j];
        int c = 0;
#pragma unroll
        for (int k = 0; k < L - 1; ++k) c += xx > tr[k] ? 1 : 0;
        const float deq = __fmul_rn(s_m[c], sg[j >> 6]);
        const float wv = __uint_as_float(static_cast<uint32_t>(wr[j]) << 16);
        const double d = __dsub_rn(static_cast<double>(wv), static_cast<double>(deq));
        v[0] = __dadd_rn(v[0], __dmul_rn(d, d));
      }
      learn_block_sum<1, NW>(v, s_red, s_S);
      if (tid == 0) {
        err_out[n] = __ddiv_rn(s_S[0], static_cast<double>(K));
        if (done_out) done_out[n] = done;
      }
    }
    if (tid < L) map_out[n * L + tid] = s_m[tid];
    if (tid < L - 1) thr_out[n * (L - 1) + tid] = s_t[tid];
    __syncthreads();  // the next row reuses the shared arrays
  }
}

}  // namespace qnf4
