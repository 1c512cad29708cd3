// LoftQ-style low-rank initialisation over the NF4 base ("LowRA" article: quantize the
// weight, take the quantization error, let a rank-r SVD of it initialise the adapters;
// five alternating steps, LoftQ's recommendation). One step:
//   target = bf16(W - B A)                   k_loftq_target
//   Q = dequant(NF4 + double quant(target))  the quantizer, double quantization, k_dequant
//   R = W - Q                                k_loftq_residual
//   rank-r SVD of R through its Gram matrix  cuBLAS sgemm + cuSOLVER syevd (library)
//   B = U S^(1/2), A = S^(1/2) V^T           k_loftq_factor (+ one sgemm)
//   e = sum of the discarded eigenvalues     k_loftq_err  (= ||W - Q - B A||_F^2)
#pragma once
#include "common.cuh"
#include "gemm.cuh"  // f2bf

namespace qnf4 {

// Device error code of a failed eigensolve (qnf4_check reports it as a CUDA error).
constexpr unsigned int kErrEigensolve = 90;

// target[n, k] = bf16(fp32(W[n, k] - sum_j B[n, j] A[j, k])), the sum in float64.
__global__ void __launch_bounds__(256) k_loftq_target(const uint16_t* __restrict__ W,
                                                      const float* __restrict__ B,
                                                      const float* __restrict__ A, int64_t N,
                                                      int64_t K, int r, uint16_t* __restrict__ out) {
  const int64_t total = N * K;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t n = i / K, k = i - n * K;
    double acc = 0.0;
    for (int j = 0; j < r; ++j)
      acc = fma(static_cast<double>(B[n * r + j]), static_cast<double>(A[j * K + k]), acc);
    const double w = __uint_as_float(static_cast<uint32_t>(W[i]) << 16);
    out[i] = f2bf(__double2float_rn(w - acc));
  }
}

// Q[i] = fp32(W[i]) - Q[i]: the quantization error of the step, in place.
__global__ void __launch_bounds__(256) k_loftq_residual(const uint16_t* __restrict__ W,
                                                        float* __restrict__ Q, int64_t total) {
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x)
    Q[i] = __uint_as_float(static_cast<uint32_t>(W[i]) << 16) - Q[i];
}

// From the Gram eigenvectors E (m x m, column-major, eigenvalues ascending) take the top r:
// column c_i = m - 1 - i, lambda_i = max(w[c_i], 0), rho_i = lambda_i^(1/4). P (m x r,
// column-major) = E[:, c_i] / rho_i (0 when rho_i = 0) feeds the sgemm that builds the other
// factor; F gets rho_i E[:, c_i]: B [N, r] row-major (F[n * r + i]) when the Gram side is N,
// A [r, K] row-major (F[i * m + k]) when it is K.
__global__ void __launch_bounds__(256) k_loftq_factor(const float* __restrict__ E,
                                                      const float* __restrict__ w, int64_t m,
                                                      int r, float* __restrict__ P,
                                                      float* __restrict__ F, int f_rowmajor_nr) {
  const int64_t total = m * r;
  for (int64_t t = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; t < total;
       t += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int i = static_cast<int>(t / m);
    const int64_t row = t - static_cast<int64_t>(i) * m;
    const int64_t c = m - 1 - i;
    const float lam = fmaxf(w[c], 0.f);
    const float rho = sqrtf(sqrtf(lam));
    const float e = E[c * m + row];
    P[static_cast<int64_t>(i) * m + row] = rho > 0.f ? e / rho : 0.f;
    const float f = rho * e;
    if (f_rowmajor_nr) F[row * r + i] = f;
    else F[static_cast<int64_t>(i) * m + row] = f;
  }
}

// err = sum of the m - r smallest eigenvalues (clamped at 0), float64; a failed
// eigensolve (info != 0) raises the device error flag instead.
__global__ void k_loftq_err(const float* __restrict__ w, int64_t m, int r,
                            const int* __restrict__ info, double* __restrict__ err) {
  __shared__ double part[256];
  double a = 0.0;
  for (int64_t i = threadIdx.x; i < m - r; i += blockDim.x) a += fmax(static_cast<double>(w[i]), 0.0);
  part[threadIdx.x] = a;
  __syncthreads();
  for (int s = blockDim.x / 2; s > 0; s >>= 1) {
    if (static_cast<int>(threadIdx.x) < s) part[threadIdx.x] += part[threadIdx.x + s];
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    *err = part[0];
    if (*info != 0) set_err(kErrEigensolve);
  }
}

}  // namespace qnf4
