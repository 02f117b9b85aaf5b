// GELU (tanh form) between the two layers of an MLP, and the reduction that completes the next
// layer's low-rank down-projection when it is computed in pieces by the fused GEMM epilogue.
//
// The activation: GELU(y) = 0.5 y (1 + tanh(sqrt(2/pi) (y + 0.044715 y^3))), evaluated as
// y * sigma(t) with t = 2 sqrt(2/pi) (y + 0.044715 y^3) (the same function; no cancellation for
// negative y).  Every step is one correctly rounded binary32 operation (the _rn intrinsics are
// never contracted into fused multiply-adds), so the result is a fixed function of y:
//
//   y2 = y*y; y3 = y2*y; w = C1*y3; inner = y + w; t = C2*inner
//   e = exp(-|t|); d = 1 + e; q = 1/d; sigma = t >= 0 ? q : e*q; GELU = y*sigma
//
// exp of a non-positive argument x (0 below -80): Cody-Waite reduction x = n ln2 + f with
// n = rint(x log2 e) and ln2 split into a 16-bit high part (n * high is exact) and a low part
// (W. J. Cody and W. Waite, "Software Manual for the Elementary Functions", 1980), then the
// degree-7 Taylor polynomial of e^f in Horner form (|f| <= ln2/2: truncation below 6e-9), times
// 2^n built from its exponent bits.  The constants are log2(e), ln2 and 1/k! rounded to binary32.
#pragma once
#include "common.cuh"

namespace svdq {

struct GeluConst {
  static constexpr uint32_t kLog2e = 0x3fb8aa3bu;   // log2(e)
  static constexpr uint32_t kLn2Hi = 0x3f317200u;   // 0.693145751953125
  static constexpr uint32_t kLn2Lo = 0x35bfbe8eu;   // ln2 - kLn2Hi
  static constexpr uint32_t kC1 = 0x3d372713u;      // 0.044715
  static constexpr uint32_t kC2 = 0x3fcc422au;      // 2 sqrt(2/pi)
};

// 1/k!, k = 0..7, rounded to binary32.
SVDQ_DEV float taylor_coef(int k) {
  return __uint_as_float(k == 0 ? 0x3f800000u : k == 1 ? 0x3f800000u : k == 2 ? 0x3f000000u
                         : k == 3 ? 0x3e2aaaabu : k == 4 ? 0x3d2aaaabu : k == 5 ? 0x3c088889u
                         : k == 6 ? 0x3ab60b61u : 0x39500d01u);
}

SVDQ_DEV float exp_nonpos(float x) {
  const float nf = rintf(__fmul_rn(x, __uint_as_float(GeluConst::kLog2e)));
  float f = __fsub_rn(x, __fmul_rn(nf, __uint_as_float(GeluConst::kLn2Hi)));
  f = __fsub_rn(f, __fmul_rn(nf, __uint_as_float(GeluConst::kLn2Lo)));
  float p = taylor_coef(7);
#pragma unroll
  for (int k = 6; k >= 0; --k) p = __fadd_rn(__fmul_rn(p, f), taylor_coef(k));
  const int n = (int)nf;                                          // in [-116, 0] when x >= -80
  const float r = __fmul_rn(p, __uint_as_float((uint32_t)(n + 127) << 23));
  return x < -80.0f ? 0.0f : r;
}

SVDQ_DEV float gelu_f32(float y) {
  const float y2 = __fmul_rn(y, y);
  const float y3 = __fmul_rn(y2, y);
  const float w = __fmul_rn(__uint_as_float(GeluConst::kC1), y3);
  const float inner = __fadd_rn(y, w);
  const float t = __fmul_rn(__uint_as_float(GeluConst::kC2), inner);
  const float e = exp_nonpos(-fabsf(t));
  const float q = __frcp_rn(__fadd_rn(1.0f, e));
  const float sigma = t >= 0.0f ? q : __fmul_rn(e, q);
  return __fmul_rn(y, sigma);
}

// The same sequence on a pair of values, with packed float32 instructions.  rint(z) for |z| < 2^22
// is z + 1.5 2^23 - 1.5 2^23 (the addition rounds to an integer, ties to even, like rint), and the
// integer n is read from the low bits of z + 1.5 2^23; each remaining step is the operation of
// gelu_f32, so both give the same bits.
SVDQ_DEV float2 gelu_f32x2(float2 y) {
  const float2 c1 = make_float2(__uint_as_float(GeluConst::kC1), __uint_as_float(GeluConst::kC1));
  const float2 c2 = make_float2(__uint_as_float(GeluConst::kC2), __uint_as_float(GeluConst::kC2));
  const float2 y3 = mul_f32x2(mul_f32x2(y, y), y);
  const float2 t = mul_f32x2(c2, add_f32x2(y, mul_f32x2(c1, y3)));
  const float2 x = make_float2(-fabsf(t.x), -fabsf(t.y));
  const float2 magic = make_float2(12582912.0f, 12582912.0f);           // 1.5 * 2^23
  const float2 a = add_f32x2(mul_f32x2(x, make_float2(__uint_as_float(GeluConst::kLog2e),
                                                      __uint_as_float(GeluConst::kLog2e))), magic);
  const float2 nf = sub_f32x2(a, magic);
  float2 f = sub_f32x2(x, mul_f32x2(nf, make_float2(__uint_as_float(GeluConst::kLn2Hi),
                                                     __uint_as_float(GeluConst::kLn2Hi))));
  f = sub_f32x2(f, mul_f32x2(nf, make_float2(__uint_as_float(GeluConst::kLn2Lo), __uint_as_float(GeluConst::kLn2Lo))));
  float2 p = make_float2(taylor_coef(7), taylor_coef(7));
#pragma unroll
  for (int k = 6; k >= 0; --k) p = add_f32x2(mul_f32x2(p, f), make_float2(taylor_coef(k), taylor_coef(k)));
  // 2^n: n = bits(a) - bits(1.5 2^23) (a holds 1.5 2^23 + n, n in [-116, 0] when x >= -80)
  const float2 two_n = make_float2(__uint_as_float((__float_as_uint(a.x) - 0x4B400000u + 127u) << 23),
                                   __uint_as_float((__float_as_uint(a.y) - 0x4B400000u + 127u) << 23));
  float2 e = mul_f32x2(p, two_n);
  e.x = x.x < -80.0f ? 0.0f : e.x;
  e.y = x.y < -80.0f ? 0.0f : e.y;
  const float2 d = add_f32x2(make_float2(1.0f, 1.0f), e);
  const float2 q = make_float2(__frcp_rn(d.x), __frcp_rn(d.y));
  const float2 eq = mul_f32x2(e, q);
  const float2 sigma = make_float2(t.x >= 0.0f ? q.x : eq.x, t.y >= 0.0f ? q.y : eq.y);
  return mul_f32x2(y, sigma);
}

// bf16 pair (packed, low half first) -> GELU of each -> bf16 pair.
SVDQ_DEV uint32_t gelu_bf16x2(uint32_t w) {
  const float2 g = gelu_f32x2(make_float2(bf16_lo(w), bf16_hi(w)));
  return pack_bf16x2(g.x, g.y);
}

// bf16 -> GELU -> bf16 (round to nearest even), on the float value of a bf16.
SVDQ_DEV float gelu_bf16(float yb) { return __bfloat162float(__float2bfloat16_rn(gelu_f32(yb))); }

// Y = GELU(X) element-wise on bf16 tensors; 8 elements (16 bytes) per thread and step, the tail
// element by element.  X and Y 16-byte aligned.
__global__ void __launch_bounds__(256) k_gelu_bf16(const uint16_t* __restrict__ X, int64_t n,
                                                   uint16_t* __restrict__ Y) {
  griddep_wait();
  const int64_t nv = n >> 3;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < nv; i += stride) {
    const uint4 x = __ldg(reinterpret_cast<const uint4*>(X) + i);
    const uint32_t xw[4] = {x.x, x.y, x.z, x.w};
    uint32_t o[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) o[j] = gelu_bf16x2(xw[j]);
    reinterpret_cast<uint4*>(Y)[i] = make_uint4(o[0], o[1], o[2], o[3]);
  }
  for (int64_t i = (nv << 3) + (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += stride) {
    const float g = gelu_f32(__uint_as_float((uint32_t)X[i] << 16));
    Y[i] = (uint16_t)(pack_bf16x2(g, 0.0f) & 0xFFFFu);
  }
}

// LAs of the next layer from the fused epilogue's pieces: part holds S slices of Mpad x r float32
// partial products (slice s = the output column tile s of the producing GEMM); the sum runs over
// the slices in order (a fixed order: the result does not depend on scheduling), then
// v = f32(sum * lr_scale) is split into bf16 hi = bf16(v) and lo = bf16(v - hi), stored
// interleaved by 16 columns as the activation kernel stores them.  Thread = (row, 4 columns).
__global__ void __launch_bounds__(256) k_lowrank_finalize(const float* __restrict__ part, int S, int M, int Mpad,
                                                          int r, float lr_scale, uint16_t* __restrict__ LAs) {
  griddep_wait();
  const int per_row = r >> 2;
  const int idx = blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= M * per_row) return;
  const int row = idx / per_row, c4 = 4 * (idx - row * per_row);
  const float4* src = reinterpret_cast<const float4*>(part + (int64_t)row * r + c4);
  const int64_t slice = (int64_t)Mpad * r / 4;
  float4 acc = __ldg(src);
#pragma unroll 8
  for (int s = 1; s < S; ++s) {
    const float4 v = __ldg(src + s * slice);
    acc.x = __fadd_rn(acc.x, v.x);
    acc.y = __fadd_rn(acc.y, v.y);
    acc.z = __fadd_rn(acc.z, v.z);
    acc.w = __fadd_rn(acc.w, v.w);
  }
  const float v4[4] = {__fmul_rn(acc.x, lr_scale), __fmul_rn(acc.y, lr_scale), __fmul_rn(acc.z, lr_scale),
                       __fmul_rn(acc.w, lr_scale)};
  float hh[4];
#pragma unroll
  for (int e = 0; e < 4; ++e) hh[e] = __bfloat162float(__float2bfloat16_rn(v4[e]));
  uint16_t* d = LAs + (int64_t)row * (2 * r) + 32 * (c4 >> 4) + (c4 & 15);
  *reinterpret_cast<uint2*>(d) = make_uint2(pack_bf16x2(hh[0], hh[1]), pack_bf16x2(hh[2], hh[3]));
  *reinterpret_cast<uint2*>(d + 16) = make_uint2(pack_bf16x2(__fsub_rn(v4[0], hh[0]), __fsub_rn(v4[1], hh[1])),
                                                 pack_bf16x2(__fsub_rn(v4[2], hh[2]), __fsub_rn(v4[3], hh[3])));
}

}  // namespace svdq
