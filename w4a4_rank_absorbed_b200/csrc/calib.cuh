// Calibration statistics on the GPU: the offline quantities of an SVDQuant layer ("From SmoothQuant
// to SVDQuant", quantization scheme: the smoothing factors, the weight-side split and the activation
// global scale are fixed before inference from calibration data).
//
//   amax_x[j] = max_m |X[m, j]|               (activation channel maxima, bf16 X, batches merged by max)
//   amax_w[j] = max_n |W[j, n]|               (weight input-channel maxima, float64 W)
//   s_j       = amax_x[j]^alpha / amax_w[j]^(1 - alpha), 1 when either is 0   ("Smooth Quant (W8A8)")
//   W_hat     = diag(s) W                     (float64, one rounding per element)
//   amax_xh   = max |f32(X * inv_s)|          (gives the static activation global scale)
//
// Maxima of magnitudes are merged with an integer atomic max on the float bit pattern (non-negative
// IEEE values order like their bit patterns), so every result is exact and independent of the order
// in which blocks finish.
#pragma once
#include "common.cuh"

namespace svdq {

SVDQ_DEV void atomic_max_nonneg(float* addr, float v) {
  atomicMax(reinterpret_cast<unsigned int*>(addr), __float_as_uint(v));
}

// Column maxima of |X| (bf16, M x K).  Block: 256 threads = 32 column groups of 8 (one 16-byte load
// each) x 8 row lanes; grid (ceil(K / 256), row slices).  K % 8 == 0.
__global__ void __launch_bounds__(256) k_absmax_cols(const uint16_t* __restrict__ X, int64_t M, int K,
                                                     int rows_per_slice, float* __restrict__ amax) {
  const int cg = threadIdx.x & 31, rl = threadIdx.x >> 5;
  const int col = (blockIdx.x * 32 + cg) * 8;
  const int64_t r0 = (int64_t)blockIdx.y * rows_per_slice;
  const int64_t r1 = M < r0 + rows_per_slice ? M : r0 + rows_per_slice;
  float m[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  if (col < K) {
    for (int64_t r = r0 + rl; r < r1; r += 8) {
      const uint4 v = __ldg(reinterpret_cast<const uint4*>(X + r * K + col));
      const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        m[2 * i] = fmaxf(m[2 * i], fabsf(bf16_lo(w[i])));
        m[2 * i + 1] = fmaxf(m[2 * i + 1], fabsf(bf16_hi(w[i])));
      }
    }
  }
  __shared__ float red[8][256 + 8];
#pragma unroll
  for (int i = 0; i < 8; ++i) red[rl][cg * 8 + i] = m[i];
  __syncthreads();
  const int c = threadIdx.x;                              // one column of the block's 256
  float v = red[0][c];
#pragma unroll
  for (int i = 1; i < 8; ++i) v = fmaxf(v, red[i][c]);
  const int gc = blockIdx.x * 256 + c;
  if (gc < K) atomic_max_nonneg(amax + gc, v);
}

// Row maxima of |W| (float64, K x N): one block of 256 threads per row.
__global__ void __launch_bounds__(256) k_absmax_rows(const double* __restrict__ W, int64_t N,
                                                     double* __restrict__ amax) {
  const double* row = W + (int64_t)blockIdx.x * N;
  double m = 0.0;
  for (int64_t n = threadIdx.x; n < N; n += 256) m = fmax(m, fabs(__ldg(row + n)));
#pragma unroll
  for (int o = 16; o; o >>= 1) m = fmax(m, __shfl_xor_sync(0xffffffffu, m, o));
  __shared__ double red[8];
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = m;
  __syncthreads();
  if (threadIdx.x == 0) {
    double v = red[0];
    for (int i = 1; i < 8; ++i) v = fmax(v, red[i]);
    amax[blockIdx.x] = v;
  }
}

// s and inv_s = f32(1/s) from the two maxima (float32 activation maxima, float64 weight maxima).
__global__ void k_smooth(const float* __restrict__ amax_x, const double* __restrict__ amax_w, int K, double alpha,
                         double* __restrict__ s, float* __restrict__ inv_s) {
  const int j = blockIdx.x * blockDim.x + threadIdx.x;
  if (j >= K) return;
  const double ax = (double)amax_x[j], aw = amax_w[j];
  const double v = (ax == 0.0 || aw == 0.0) ? 1.0 : pow(ax, alpha) / pow(aw, 1.0 - alpha);
  s[j] = v;
  inv_s[j] = (float)(1.0 / v);
}

// W_hat = diag(s) W (float64, K x N), one block row-slice per block.
__global__ void __launch_bounds__(256) k_scale_rows(const double* __restrict__ W, const double* __restrict__ s,
                                                    int64_t K, int64_t N, double* __restrict__ W_hat) {
  const int64_t total = K * N;
  for (int64_t i = (int64_t)blockIdx.x * 256 + threadIdx.x; i < total; i += (int64_t)gridDim.x * 256)
    W_hat[i] = __dmul_rn(__ldg(s + i / N), __ldg(W + i));
}

// max |f32(X * inv_s)| over a bf16 M x K matrix (K % 8 == 0).
__global__ void __launch_bounds__(256) k_act_amax(const uint16_t* __restrict__ X, int64_t M, int K,
                                                  const float* __restrict__ inv_s, float* __restrict__ amax) {
  const int64_t nv = M * (K / 8);
  float m = 0.0f;
  for (int64_t i = (int64_t)blockIdx.x * 256 + threadIdx.x; i < nv; i += (int64_t)gridDim.x * 256) {
    const int c = (int)(i % (K / 8)) * 8;
    const uint4 v = __ldg(reinterpret_cast<const uint4*>(X) + i);
    const float4 s0 = __ldg(reinterpret_cast<const float4*>(inv_s + c));
    const float4 s1 = __ldg(reinterpret_cast<const float4*>(inv_s + c + 4));
    m = fmaxf(m, fabsf(__fmul_rn(bf16_lo(v.x), s0.x)));
    m = fmaxf(m, fabsf(__fmul_rn(bf16_hi(v.x), s0.y)));
    m = fmaxf(m, fabsf(__fmul_rn(bf16_lo(v.y), s0.z)));
    m = fmaxf(m, fabsf(__fmul_rn(bf16_hi(v.y), s0.w)));
    m = fmaxf(m, fabsf(__fmul_rn(bf16_lo(v.z), s1.x)));
    m = fmaxf(m, fabsf(__fmul_rn(bf16_hi(v.z), s1.y)));
    m = fmaxf(m, fabsf(__fmul_rn(bf16_lo(v.w), s1.z)));
    m = fmaxf(m, fabsf(__fmul_rn(bf16_hi(v.w), s1.w)));
  }
#pragma unroll
  for (int o = 16; o; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  if ((threadIdx.x & 31) == 0) atomic_max_nonneg(amax, m);
}

}  // namespace svdq
