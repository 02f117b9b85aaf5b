// GELU (tanh form) between the two layers of an MLP, and the reduction that completes the next
// layer's low-rank down-projection when it is computed in pieces by the fused GEMM epilogue.
//
// The activation: GELU(y) = 0.5 y (1 + tanh(sqrt(2/pi) (y + 0.044715 y^3))), evaluated as
// y * sigma(t) with t = 2 sqrt(2/pi) (y + 0.044715 y^3) (the same function; no cancellation for
// negative y).  Every step is one correctly rounded binary32 operation (a fused multiply-add counts
// as one; the _rn intrinsics and the explicitly rounded PTX below are never contracted or split),
// so the result is a fixed function of y:
//
//   y2 = y*y; h = fma(C3, y2, C2); t = y*h;  x = -|t|
//   a = fma(x, log2 e, 1.5 2^23); n = a - 1.5 2^23            (n = rint(x log2 e))
//   f = fma(-n, ln2_hi, x); f = fma(-n, ln2_lo, f)            (Cody-Waite reduction)
//   p = 1/6!; p = fma(p, f, 1/k!) for k = 5 .. 0               (Taylor polynomial of e^f)
//   e = x < -80 ? 0 : p * 2^n;  d = 1 + e
//   q = fma(-8/17, d, 24/17); 3 x { r = fma(-d, q, 1); q = fma(q, r, q) }   (Newton: q -> 1/d)
//   sigma = t >= 0 ? q : e*q;  GELU = y*sigma
//
// Cody-Waite: W. J. Cody and W. Waite, "Software Manual for the Elementary Functions", 1980 (ln2 in a
// 16-bit high part, so n * ln2_hi is exact, and a low part).  The constants are log2(e), ln2, 1/k!,
// 24/17, 8/17, C2 = 2 sqrt(2/pi) and C3 = 0.044715 C2, each rounded to binary32.
#pragma once
#include "common.cuh"

namespace svdq {

struct GeluConst {
  static constexpr uint32_t kLog2e = 0x3fb8aa3bu;   // log2(e)
  static constexpr uint32_t kLn2Hi = 0x3f317200u;   // 0.693145751953125
  static constexpr uint32_t kLn2Lo = 0x35bfbe8eu;   // ln2 - kLn2Hi
  static constexpr uint32_t kC2 = 0x3fcc422au;      // 2 sqrt(2/pi)
  static constexpr uint32_t kC3 = 0x3d922279u;      // 0.044715 * 2 sqrt(2/pi)
  static constexpr uint32_t kR0A = 0x3fb4b4b5u;     // 24/17: seed of 1/d on [1, 2] is 24/17 - 8/17 d
  static constexpr uint32_t kR0B = 0x3ef0f0f1u;     // 8/17
  static constexpr uint32_t kMagic = 0x4b400000u;   // 1.5 * 2^23
};

// 1/k!, k = 0..6, rounded to binary32.
SVDQ_DEV float taylor_coef(int k) {
  return __uint_as_float(k == 0 ? 0x3f800000u : k == 1 ? 0x3f800000u : k == 2 ? 0x3f000000u
                         : k == 3 ? 0x3e2aaaabu : k == 4 ? 0x3d2aaaabu : k == 5 ? 0x3c088889u
                         : 0x3ab60b61u);
}

SVDQ_DEV float2 f2(float v) { return make_float2(v, v); }
SVDQ_DEV float2 f2c(uint32_t bits) { return f2(__uint_as_float(bits)); }

SVDQ_DEV float gelu_f32(float y) {
  const float t = __fmul_rn(y, __fmaf_rn(__uint_as_float(GeluConst::kC3), __fmul_rn(y, y),
                                         __uint_as_float(GeluConst::kC2)));
  const float x = -fabsf(t);
  const float magic = __uint_as_float(GeluConst::kMagic);
  const float a = __fmaf_rn(x, __uint_as_float(GeluConst::kLog2e), magic);
  const float nf = __fsub_rn(a, magic);
  float f = __fmaf_rn(-nf, __uint_as_float(GeluConst::kLn2Hi), x);
  f = __fmaf_rn(-nf, __uint_as_float(GeluConst::kLn2Lo), f);
  float p = taylor_coef(6);
#pragma unroll
  for (int k = 5; k >= 0; --k) p = __fmaf_rn(p, f, taylor_coef(k));
  // 2^n from the integer in a's low bits (garbage below x = -80, where e is cut to 0 anyway)
  const float two_n = __uint_as_float((__float_as_uint(a) - GeluConst::kMagic + 127u) << 23);
  const float e = x < -80.0f ? 0.0f : __fmul_rn(p, two_n);
  const float d = __fadd_rn(1.0f, e);
  float q = __fmaf_rn(-__uint_as_float(GeluConst::kR0B), d, __uint_as_float(GeluConst::kR0A));
#pragma unroll
  for (int i = 0; i < 3; ++i) q = __fmaf_rn(q, __fmaf_rn(-d, q, 1.0f), q);
  const float sigma = t >= 0.0f ? q : __fmul_rn(e, q);
  return __fmul_rn(y, sigma);
}

// The same sequence on a pair of values, with packed float32 instructions (each element of each
// instruction is the operation of gelu_f32, so both give the same bits).
SVDQ_DEV float2 gelu_f32x2(float2 y) {
  const float2 t = mul_f32x2(y, fma_f32x2(f2c(GeluConst::kC3), mul_f32x2(y, y), f2c(GeluConst::kC2)));
  const float2 x = make_float2(-fabsf(t.x), -fabsf(t.y));
  const float2 magic = f2c(GeluConst::kMagic);
  const float2 a = fma_f32x2(x, f2c(GeluConst::kLog2e), magic);
  const float2 nneg = sub_f32x2(magic, a);                          // -n (exact)
  float2 f = fma_f32x2(nneg, f2c(GeluConst::kLn2Hi), x);
  f = fma_f32x2(nneg, f2c(GeluConst::kLn2Lo), f);
  float2 p = f2(taylor_coef(6));
#pragma unroll
  for (int k = 5; k >= 0; --k) p = fma_f32x2(p, f, f2(taylor_coef(k)));
  const float2 two_n = make_float2(__uint_as_float((__float_as_uint(a.x) - GeluConst::kMagic + 127u) << 23),
                                   __uint_as_float((__float_as_uint(a.y) - GeluConst::kMagic + 127u) << 23));
  float2 e = mul_f32x2(p, two_n);
  e.x = x.x < -80.0f ? 0.0f : e.x;
  e.y = x.y < -80.0f ? 0.0f : e.y;
  const float2 d = add_f32x2(f2(1.0f), e);
  const float2 dneg = make_float2(-d.x, -d.y);
  float2 q = fma_f32x2(f2(-__uint_as_float(GeluConst::kR0B)), d, f2c(GeluConst::kR0A));
#pragma unroll
  for (int i = 0; i < 3; ++i) q = fma_f32x2(q, fma_f32x2(dneg, q, f2(1.0f)), q);
  const float2 eq = mul_f32x2(e, q);
  const float2 sigma = make_float2(t.x >= 0.0f ? q.x : eq.x, t.y >= 0.0f ? q.y : eq.y);
  return mul_f32x2(y, sigma);
}

// bf16 pair (packed, low half first) -> GELU of each -> bf16 pair.
SVDQ_DEV uint32_t gelu_bf16x2(uint32_t w) {
  const float2 g = gelu_f32x2(make_float2(bf16_lo(w), bf16_hi(w)));
  return pack_bf16x2(g.x, g.y);
}

// Y = GELU(X) element-wise on bf16 tensors.  A thread moves four 16-byte vectors per step (all four
// loads issued before any arithmetic, so that 64 bytes per thread are in flight), a warp's four loads
// covering four consecutive 512-byte runs; the tail element by element.  X and Y 16-byte aligned.
constexpr int GELU_VEC = 4;
__global__ void __launch_bounds__(256) k_gelu_bf16(const uint16_t* __restrict__ X, int64_t n,
                                                   uint16_t* __restrict__ Y) {
  griddep_wait();
  const int64_t nv = n >> 3;                                   // 16-byte vectors
  const int64_t nchunk = nv / (GELU_VEC * 256);                // whole block-steps
  const uint4* xv = reinterpret_cast<const uint4*>(X);
  uint4* yv = reinterpret_cast<uint4*>(Y);
  for (int64_t c = blockIdx.x; c < nchunk; c += gridDim.x) {
    const int64_t base = c * (GELU_VEC * 256) + threadIdx.x;
    uint4 x[GELU_VEC];
#pragma unroll
    for (int j = 0; j < GELU_VEC; ++j) x[j] = __ldg(xv + base + 256 * j);
#pragma unroll
    for (int j = 0; j < GELU_VEC; ++j)
      yv[base + 256 * j] = make_uint4(gelu_bf16x2(x[j].x), gelu_bf16x2(x[j].y), gelu_bf16x2(x[j].z),
                                      gelu_bf16x2(x[j].w));
  }
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t i = nchunk * (GELU_VEC * 256) + (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < nv; i += stride) {
    const uint4 x = __ldg(xv + i);
    yv[i] = make_uint4(gelu_bf16x2(x.x), gelu_bf16x2(x.y), gelu_bf16x2(x.z), gelu_bf16x2(x.w));
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
