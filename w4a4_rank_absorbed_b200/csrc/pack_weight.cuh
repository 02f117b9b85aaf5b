// Kernel 1: static NVFP4 packing of the residual weight R (K x N float32).
//
// SVDQuant review, §4.2: only the residual R = W_hat - L1 L2 is quantized to
// 4 bits; "From SmoothQuant to SVDQuant", quantization scheme item 1: weight
// scales are computed once, offline.  NVFP4 grouping ("From SmoothQuant to
// SVDQuant", section Personal view): groups of 16 along K, UE4M3 block scale,
// float32 global scale gs_w = amax / 2688.
//
// Four launches, all HBM-bound:
//   1. zero the amax accumulator (the gs_w output float);
//   2. amax |R| over the whole tensor (vectorised grid-stride loads, atomicMax on the bits);
//   3. gs_w = amax / 2688 (or 1);
//   4. encode: one thread per (column n, 64 consecutive k): 4 groups of 16,
//      32 bytes of codes and one 32-bit word of scales; also the up-projection
//      laid out K-major for the GEMM, L2p = L2^T (N x r).
#pragma once
#include "common.cuh"

namespace svdq {

__global__ void k_zero_u32(unsigned int* p) { *p = 0u; }

// amax of |R| as the bit pattern of a non-negative float (ordered like unsigned ints).
__global__ void __launch_bounds__(256) k_absmax_f32(const float* __restrict__ R, int64_t n,
                                                    unsigned int* __restrict__ out_bits) {
  float m = 0.0f;
  const int64_t n4 = n >> 2;
  const float4* R4 = reinterpret_cast<const float4*>(R);
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n4; i += (int64_t)gridDim.x * blockDim.x) {
    const float4 v = __ldg(R4 + i);
    m = fmaxf(m, fmaxf(fmaxf(fabsf(v.x), fabsf(v.y)), fmaxf(fabsf(v.z), fabsf(v.w))));
  }
  for (int64_t i = (n4 << 2) + blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n;
       i += (int64_t)gridDim.x * blockDim.x)
    m = fmaxf(m, fabsf(R[i]));
#pragma unroll
  for (int o = 16; o; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  __shared__ float wmax[8];
  if ((threadIdx.x & 31) == 0) wmax[threadIdx.x >> 5] = m;
  __syncthreads();
  if (threadIdx.x == 0) {
    for (int w = 1; w < (int)(blockDim.x >> 5); ++w) m = fmaxf(m, wmax[w]);
    atomicMax(out_bits, __float_as_uint(m));
  }
}

// gs = amax / 2688 (one IEEE division), 1 when amax == 0.
__global__ void k_global_scale(float* gs_inout) {
  const float amax = __uint_as_float(*reinterpret_cast<unsigned int*>(gs_inout));
  *gs_inout = amax > 0.0f ? __fdiv_rn(amax, 2688.0f) : 1.0f;
}

// Quantize 16 float32 values in registers (one NVFP4 group) with per-tensor scale
// constants gs and c = f32(1 / f32(6 gs)); returns the UE4M3 scale, writes the
// 64-bit code word (element i in nibble i).
SVDQ_DEV uint32_t encode_group16(const float (&x)[16], float gs, float c, uint2& codes) {
  float a = 0.0f;
#pragma unroll
  for (int i = 0; i < 16; ++i) a = fmaxf(a, fabsf(x[i]));
  const uint32_t sb = cvt_ue4m3(__fmul_rn(a, c));
  if (sb == 0u) {
    codes = make_uint2(0u, 0u);
    return 0u;
  }
  const float rinv = __frcp_rn(__fmul_rn(dec_ue4m3(sb), gs));
  float q0[8], q1[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    q0[i] = __fmul_rn(x[i], rinv);
    q1[i] = __fmul_rn(x[8 + i], rinv);
  }
  codes = make_uint2(cvt_e2m1x8(q0), cvt_e2m1x8(q1));
  return sb;
}

// grid: (ceil(Npad/128), K/64); block 128.  Thread = (column n, 64-row slab kb of R).
__global__ void __launch_bounds__(128) k_pack_weight(const float* __restrict__ R, int K, int N, int Npad,
                                                     const float* __restrict__ gs_ptr,
                                                     uint8_t* __restrict__ Wq, uint8_t* __restrict__ SFw) {
  const int n = blockIdx.x * 128 + threadIdx.x;
  const int kb = blockIdx.y;
  if (n >= Npad) return;
  const uint32_t KS4 = (uint32_t)(K >> 6);
  uint8_t* sfw = SFw + sf_word_offset((uint32_t)n, (uint32_t)kb, KS4);
  if (n >= N) {  // padding row of the scale buffer
    *reinterpret_cast<uint32_t*>(sfw) = 0u;
    return;
  }
  const float gs = *gs_ptr;
  const float c = __frcp_rn(__fmul_rn(6.0f, gs));
  uint32_t sfword = 0u;
  uint4 out[2];
  uint32_t* ow = reinterpret_cast<uint32_t*>(out);
#pragma unroll
  for (int g = 0; g < 4; ++g) {
    float x[16];
    const float* src = R + (int64_t)(kb * 64 + g * 16) * N + n;
#pragma unroll
    for (int i = 0; i < 16; ++i) x[i] = __ldg(src + (int64_t)i * N);
    uint2 cw;
    const uint32_t sb = encode_group16(x, gs, c, cw);
    sfword |= sb << (8 * g);
    ow[2 * g] = cw.x;
    ow[2 * g + 1] = cw.y;
  }
  uint4* dst = reinterpret_cast<uint4*>(Wq + (int64_t)n * (K >> 1) + kb * 32);
  dst[0] = out[0];
  dst[1] = out[1];
  *reinterpret_cast<uint32_t*>(sfw) = sfword;
}

// MXFP4 packing of R (no global scale): one thread per (column n, 128 consecutive k), four blocks of
// 32 along K, each with its E8M0 scale (mx_scale) and codes E2M1_rne_sat(x * 2^-X) (the product is
// exact); 64 bytes of codes and one 32-bit word of four scales.  grid: (ceil(Npad/128), K/128).
__global__ void __launch_bounds__(128) k_pack_weight_mx(const float* __restrict__ R, int K, int N, int Npad,
                                                        uint8_t* __restrict__ Wq, uint8_t* __restrict__ SFw) {
  const int n = blockIdx.x * 128 + threadIdx.x;
  const int kb = blockIdx.y;
  if (n >= Npad) return;
  uint8_t* sfw = SFw + sf_word_offset((uint32_t)n, (uint32_t)kb, (uint32_t)(K >> 7));
  if (n >= N) {
    *reinterpret_cast<uint32_t*>(sfw) = 0u;
    return;
  }
  uint32_t sfword = 0u;
  uint4* dst = reinterpret_cast<uint4*>(Wq + (int64_t)n * (K >> 1) + kb * 64);
#pragma unroll
  for (int g = 0; g < 4; ++g) {
    float x[32];
    const float* src = R + (int64_t)(kb * 128 + g * 32) * N + n;
    float a = 0.0f;
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      x[i] = __ldg(src + (int64_t)i * N);
      a = fmaxf(a, fabsf(x[i]));
    }
    float mul;
    sfword |= mx_scale(a, mul) << (8 * g);
    uint32_t w[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      float v[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) v[i] = __fmul_rn(x[8 * q + i], mul);
      w[q] = a > 0.0f ? cvt_e2m1x8(v) : 0u;     // an all-zero block: codes 0
    }
    dst[g] = make_uint4(w[0], w[1], w[2], w[3]);
  }
  *reinterpret_cast<uint32_t*>(sfw) = sfword;
}

// Q(R) from a packed weight: R_q[k, n] = f32(e2m1(code) * f32(dec(sb) * gs)), K x N row-major.
// grid: (ceil(N/128), K/64); block 128; thread = (column n, 64-row slab kb), so a warp writes 32
// consecutive columns of one row at a time.
__global__ void __launch_bounds__(128) k_dequant_weight(const uint8_t* __restrict__ Wq,
                                                        const uint8_t* __restrict__ SFw,
                                                        const float* __restrict__ gs_ptr, int K, int N,
                                                        float* __restrict__ Rq) {
  const int n = blockIdx.x * 128 + threadIdx.x;
  const int kb = blockIdx.y;
  if (n >= N) return;
  const float gs = *gs_ptr;
  const uint32_t sfword = *reinterpret_cast<const uint32_t*>(SFw + sf_word_offset((uint32_t)n, (uint32_t)kb,
                                                                                  (uint32_t)(K >> 6)));
  const uint4* src = reinterpret_cast<const uint4*>(Wq + (int64_t)n * (K >> 1) + kb * 32);
  const uint4 c0 = src[0], c1 = src[1];
  const uint32_t cw[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
  // E2M1 magnitudes of codes 0..7 (bit 3 is the sign)
  const float mag[8] = {0.0f, 0.5f, 1.0f, 1.5f, 2.0f, 3.0f, 4.0f, 6.0f};
#pragma unroll
  for (int g = 0; g < 4; ++g) {
    const float d = __fmul_rn(dec_ue4m3((sfword >> (8 * g)) & 0xFFu), gs);
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const uint32_t code = (cw[2 * g + (i >> 3)] >> (4 * (i & 7))) & 0xFu;
      const float v = __fmul_rn(mag[code & 7u], d);
      Rq[(int64_t)(kb * 64 + g * 16 + i) * N + n] = (code & 8u) ? -v : v;
    }
  }
}

// L2p[n, t] = L2b[t, n] for t < r (r even).  grid: ceil(N/128); block 128.
__global__ void __launch_bounds__(128) k_layout_l2(const uint16_t* __restrict__ L2b, int N, int r,
                                                   uint16_t* __restrict__ L2p) {
  const int n = blockIdx.x * 128 + threadIdx.x;
  if (n >= N) return;
  uint16_t* row = L2p + (int64_t)n * r;
  for (int t = 0; t < r; t += 2) {
    const uint32_t v = (uint32_t)L2b[(int64_t)t * N + n] | ((uint32_t)L2b[(int64_t)(t + 1) * N + n] << 16);
    *reinterpret_cast<uint32_t*>(row + t) = v;
  }
}

}  // namespace svdq
