// Kernel 2: activation quantization fused with the low-rank down-projection.
//
// SVDQuant review, §4.3 (Nunchaku): the down-projection is merged into the
// quantization kernel, so the 16-bit activations are read from HBM once and
// shared by both branches.  Per element x_hat = f32(x * inv_s) (the smoothing
// divide, "From SmoothQuant to SVDQuant", section Smooth Quant (W8A8));
// per group of 16 along K the NVFP4 codec of SVDQuant review §3 (q_max = 6)
// with a UE4M3 block scale; the down-projection LA = X L1f (L1f =
// diag(s)^-1 L1, so X L1f = X_hat L1) on the tensor cores (bf16 in, fp32
// accumulate), pre-scaled by lr_scale and split into bf16 hi/lo halves.
//
// CTA = 32 rows x all of K; 14 warps in 7 pairs.  The K axis is cut into
// 64-column chunks; chunk c goes through ring stage c % S and is consumed by
// warp pair c % 7, so seven chunks are processed at once.  S is a multiple of
// 7 (up to 49): as many stages as fit in 200 KB, 21 for r = 32, 7 for r = 128,
// so each pair keeps S/7 chunks in flight.  A pair loads its own chunks: once
// both of its warps are done with a stage, warp 0 of the pair issues the copies
// of the chunk S further on into that stage (three lanes in one converged
// instruction, rotating with the round so no thread has two copies in flight:
// a thread's copies are serviced one after another).  No producer warp, and no
// lanes waiting on different barriers in divergent branches.  A stage holds
// the X box (32 x 64 bf16, 128-byte swizzle), the L1f^T box (r x 64 bf16, same
// swizzle) and the chunk's 64 smoothing factors.  Warp h of a pair owns rows
// 16h..16h+15 of the chunk: two lanes per row quantize two groups of 16 each,
// and the warp runs the 16 x r down-projection of its rows for the chunk's 64
// columns (mma.sync m16n8k16), keeping a partial sum in registers.  After the
// last chunk the seven partial sums of every row are added in shared memory and
// written as LAs.
#pragma once
#include "common.cuh"

namespace svdq {

constexpr int QA_ROWS = 32;
constexpr int QA_CHUNK = 64;          // bf16 columns per chunk (128 bytes)
constexpr int QA_PAIRS = 7;
constexpr int QA_CONSUMER_WARPS = 2 * QA_PAIRS;
constexpr int QA_THREADS = QA_CONSUMER_WARPS * 32;
constexpr int QA_RING_BYTES = 200 * 1024;

template <int R>
struct QaCfg {
  static constexpr int kXBytes = QA_ROWS * 128;
  static constexpr int kLBytes = R * 128;
  static constexpr int kStageBytes = kXBytes + kLBytes;
  // The ring size is a multiple of the pair count, so a ring slot is always loaded and consumed
  // by the same warp pair, one round after another.
  static constexpr int kPerPair = QA_RING_BYTES / (QA_PAIRS * (kStageBytes + 256));
  static constexpr int kStages = QA_PAIRS * (kPerPair < 1 ? 1 : kPerPair > 7 ? 7 : kPerPair);
  static constexpr int kNT = R / 8;                                  // n8 tiles of the r columns
  static constexpr int kAcc = R > 0 ? kNT : 1;                      // (m16, n8) tiles per warp
  static constexpr int kRedBytes = QA_PAIRS * QA_ROWS * R * 4;
  static constexpr int kRingBytes = kStages * kStageBytes;
  static_assert(kRedBytes <= kRingBytes, "reduction buffer must fit in the ring");
  static constexpr int kInvOff = kRingBytes;                        // S x 64 smoothing factors
  static constexpr int kRcpOff = kInvOff + kStages * 256;           // 128-entry 1/d table
  static constexpr int kBarOff = kRcpOff + 128 * 4;
  static constexpr int kSmem = kBarOff + 2 * kStages * 8 + 16 + 1024;
};

SVDQ_DEV void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
SVDQ_DEV void ldsm_x2(uint32_t addr, uint32_t& r0, uint32_t& r1) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x2.shared.b16 {%0, %1}, [%2];" : "=r"(r0), "=r"(r1) : "r"(addr));
}
SVDQ_DEV void mma_bf16_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t b0,
                             uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
SVDQ_DEV void named_bar_sync(int id, int threads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}

// Byte offset of 16-byte chunk `c16` of row `row` in a 128-byte-swizzled tile.
SVDQ_DEV uint32_t sw128(uint32_t row, uint32_t c16) { return row * 128u + ((c16 ^ (row & 7u)) << 4); }

// One group of 16 values of X (two 16-byte smem chunks) times 16 smoothing factors:
// returns the UE4M3 scale and the two 32-bit code words.
// d = a * b element-wise on two float32 pairs (two correctly rounded products).
SVDQ_DEV float2 mul_f32x2(float2 a, float2 b) {
  uint64_t d;
  const uint64_t x = (uint64_t)__float_as_uint(a.x) | ((uint64_t)__float_as_uint(a.y) << 32);
  const uint64_t y = (uint64_t)__float_as_uint(b.x) | ((uint64_t)__float_as_uint(b.y) << 32);
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(x), "l"(y));
  return make_float2(__uint_as_float((uint32_t)d), __uint_as_float((uint32_t)(d >> 32)));
}

// One group of 16 values of X (two 16-byte smem chunks) times 16 smoothing factors:
// returns the UE4M3 scale and the two 32-bit code words.
SVDQ_DEV uint32_t quant_group(const uint4& r0, const uint4& r1, const float4 (&inv)[4], float c_x,
                              uint32_t rcp_table, uint32_t& w0, uint32_t& w1) {
  const uint32_t xw[8] = {r0.x, r0.y, r0.z, r0.w, r1.x, r1.y, r1.z, r1.w};
  float2 xh[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const float4 s4 = inv[i >> 1];
    const float2 sp = (i & 1) ? make_float2(s4.z, s4.w) : make_float2(s4.x, s4.y);
    xh[i] = mul_f32x2(make_float2(bf16_lo(xw[i]), bf16_hi(xw[i])), sp);
  }
  float a = 0.0f;
#pragma unroll
  for (int i = 0; i < 8; ++i) a = fmaxf(a, fmaxf(fabsf(xh[i].x), fabsf(xh[i].y)));
  const uint32_t sb = cvt_ue4m3(__fmul_rn(a, c_x));
  const float rinv = lds_f32(rcp_table + 4 * sb);   // f32(1 / f32(dec(sb) * gs)); entry 0 is 0
  const float2 rr = make_float2(rinv, rinv);
  float q0[8], q1[8];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 p0 = mul_f32x2(xh[i], rr);
    const float2 p1 = mul_f32x2(xh[4 + i], rr);
    q0[2 * i] = p0.x; q0[2 * i + 1] = p0.y;
    q1[2 * i] = p1.x; q1[2 * i + 1] = p1.y;
  }
  // rinv = 0 for an all-zero scale: every product is +-0; the codes are forced to 0.
  w0 = sb ? cvt_e2m1x8(q0) : 0u;
  w1 = sb ? cvt_e2m1x8(q1) : 0u;
  return sb;
}

template <int R>
__global__ void __launch_bounds__(QA_THREADS, 1) k_quantize_act(
    const __grid_constant__ CUtensorMap tm_x,   // bf16 {K, M}, box {64, 32}, 128B swizzle
    const __grid_constant__ CUtensorMap tm_l1,  // bf16 {K, R}, box {64, R}, 128B swizzle
    const float* __restrict__ inv_s, float gs_x, float lr_scale, int M, int K, int Mpad,
    uint8_t* __restrict__ Xq, uint8_t* __restrict__ SFx, uint16_t* __restrict__ LAs, uint64_t timeout_ns) {
  using Cfg = QaCfg<R>;
  constexpr int S = Cfg::kStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  float* s_inv = reinterpret_cast<float*>(smem + Cfg::kInvOff);
  float* s_rcp = reinterpret_cast<float*>(smem + Cfg::kRcpOff);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + Cfg::kBarOff);
  uint64_t* consumed = full + S;           // both warps of the owning pair are done with the stage
  volatile int* abort_flag = reinterpret_cast<volatile int*>(consumed + S);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int m0 = blockIdx.x * QA_ROWS;
  const int nchunks = K / QA_CHUNK;
  const int pairi = warp >> 1;             // warp pair: consumes chunks pairi, pairi + 7, ...
  const int half = warp & 1;               // rows 16*half .. 16*half + 15 of the chunk

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&consumed[s], 2);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  // 1/d for every possible block scale: d = f32(dec(sb) * gs_x), same operations as the per-group path.
  if (threadIdx.x < 128) {
    const uint32_t sb = threadIdx.x;
    s_rcp[sb] = sb == 0 ? 0.0f : __frcp_rn(__fmul_rn(dec_ue4m3(sb), gs_x));
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tm_x);
    if (R > 0) tma_prefetch_desc(&tm_l1);
  }
  __syncthreads();

  // Copies of chunk c into its stage, by lanes 3j .. 3j + 2 of warp 0 of the owning pair (j
  // rotates with the round): X box and L1f^T box in one converged instruction, then the chunk's
  // 64 smoothing factors.
  auto issue = [&](int c) {
    const int g = c % S;
    const int j = (c / S) % 10;
    if (lane >= 3 * j && lane < 3 * j + 3) {
      const int k = lane - 3 * j;
      uint8_t* st = smem + g * Cfg::kStageBytes;
      if (k == 0) mbar_arrive_expect_tx(&full[g], Cfg::kStageBytes + 256);
      __syncwarp(7u << (3 * j));
      if (k == 0 || (k == 1 && R > 0))
        tma_load_2d(k == 0 ? st : st + Cfg::kXBytes, k == 0 ? &tm_x : &tm_l1, &full[g], c * QA_CHUNK,
                    k == 0 ? m0 : 0);
      else if (k == 2)
        bulk_load(s_inv + g * 64, inv_s + (int64_t)c * QA_CHUNK, 256, &full[g]);
    }
    __syncwarp();
  };
  int hi = pairi;                          // the pair's chunks below hi have been issued
  for (; hi < nchunks && hi < S; hi += QA_PAIRS)
    if (half == 0) issue(hi);

  const int qrow = 16 * half + (lane >> 1);
  const int qg = 2 * (lane & 1);           // first of the two groups this lane quantizes
  const int m = m0 + qrow;
  const float c_x = __frcp_rn(__fmul_rn(6.0f, gs_x));
  const uint32_t KS4 = (uint32_t)(K >> 6);
  const uint32_t rcp_u32 = smem_u32(s_rcp);

  float acc[Cfg::kAcc][4];
#pragma unroll
  for (int i = 0; i < Cfg::kAcc; ++i) acc[i][0] = acc[i][1] = acc[i][2] = acc[i][3] = 0.0f;

  bool ok = true;
  int c = pairi;
  for (; c < nchunks; c += QA_PAIRS) {
    const int s = c % S;
    if (!mbar_wait(&full[s], (uint32_t)((c / S) & 1), timeout_ns, abort_flag, 0x202)) {
      ok = false;
      break;
    }
    const uint8_t* st = smem + s * Cfg::kStageBytes;
    const uint32_t st_u32 = smem_u32(st);
    const uint32_t inv_u32 = smem_u32(s_inv + s * 64 + 16 * qg);

    // ---- quantize two groups of row qrow ------------------------------------
    uint32_t w[4];
    uint32_t sb2 = 0u;
#pragma unroll
    for (int g = 0; g < 2; ++g) {
      const int gg = qg + g;
      const uint4 r0 = lds_v4(st_u32 + sw128(qrow, 2 * gg));
      const uint4 r1 = lds_v4(st_u32 + sw128(qrow, 2 * gg + 1));
      float4 inv[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) inv[j] = lds_v4f(inv_u32 + 64 * g + 16 * j);
      const uint32_t sb = quant_group(r0, r1, inv, c_x, rcp_u32, w[2 * g], w[2 * g + 1]);
      sb2 |= sb << (8 * g);
    }
    const uint32_t other = __shfl_xor_sync(0xffffffffu, sb2, 1);
    if (m < M)
      *reinterpret_cast<uint4*>(Xq + (int64_t)m * (K >> 1) + c * 32 + 8 * qg) = make_uint4(w[0], w[1], w[2], w[3]);
    if ((lane & 1) == 0 && m < Mpad)
      *reinterpret_cast<uint32_t*>(SFx + sf_word_offset((uint32_t)m, (uint32_t)c, KS4)) = sb2 | (other << 16);

    // ---- down-projection of this warp's 16 rows on the tensor cores ---------
    if constexpr (R > 0) {
      const uint32_t sl_u32 = st_u32 + Cfg::kXBytes;
#pragma unroll
      for (int ks = 0; ks < 4; ++ks) {
        uint32_t a0, a1, a2, a3;
        const uint32_t arow = 16 * half + (lane & 7) + ((lane >> 3) & 1) * 8;
        ldsm_x4(st_u32 + sw128(arow, ks * 2 + (lane >> 4)), a0, a1, a2, a3);
#pragma unroll
        for (int nt = 0; nt < Cfg::kNT; nt += 2) {
          uint32_t b[4];
          const uint32_t brow = (nt + (lane >> 4)) * 8 + (lane & 7);
          ldsm_x4(sl_u32 + sw128(brow, ks * 2 + ((lane >> 3) & 1)), b[0], b[1], b[2], b[3]);
          mma_bf16_16816(acc[nt], a0, a1, a2, a3, b[0], b[1]);
          mma_bf16_16816(acc[nt + 1], a0, a1, a2, a3, b[2], b[3]);
        }
      }
    }
    // Once both warps of the pair are done with stage s, warp 0 refills it with the chunk S
    // further on.
    if (c + S < nchunks) {
      __syncwarp();
      if (lane == 0) mbar_arrive(&consumed[s]);
      if (half == 0) {
        int done = 1;
        if (lane == 0) done = mbar_wait(&consumed[s], (uint32_t)((c / S) & 1), timeout_ns, abort_flag, 0x201) ? 1 : 0;
        if (!__shfl_sync(0xffffffffu, done, 0)) {
          ok = false;
          c += QA_PAIRS;                   // chunk c was consumed; the loads still owed start after it
          break;
        }
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        issue(c + S);
      }
      hi = c + S + QA_PAIRS;
    }
  }
  if (!ok && half == 0) {
    // Let the loads this pair issued but did not consume land before the CTA exits.
    int never = 0;
    for (int c2 = c; c2 < hi; c2 += QA_PAIRS)
      mbar_wait(&full[c2 % S], (uint32_t)((c2 / S) & 1), timeout_ns, &never, 0x203);
  }

  // ---- LAs = [hi | lo] of lr_scale * sum over pairs of the partial X L1f ----
  if constexpr (R > 0) {
    // Every chunk has been consumed, so no load is in flight into the ring: reuse it.
    named_bar_sync(1, QA_CONSUMER_WARPS * 32);
    float* red = reinterpret_cast<float*>(smem);            // [pair][row][R]
    if (ok) {
#pragma unroll
      for (int nt = 0; nt < Cfg::kNT; ++nt) {
        const int row = 16 * half + (lane >> 2);
        const int col = nt * 8 + 2 * (lane & 3);
        float* p = red + ((pairi * QA_ROWS + row) * R + col);
        *reinterpret_cast<float2*>(p) = make_float2(acc[nt][0], acc[nt][1]);
        *reinterpret_cast<float2*>(p + 8 * R) = make_float2(acc[nt][2], acc[nt][3]);
      }
    }
    named_bar_sync(1, QA_CONSUMER_WARPS * 32);
    if (ok && !*abort_flag) {
      for (int p = threadIdx.x; p < QA_ROWS * R / 2; p += QA_CONSUMER_WARPS * 32) {
        const int row = p / (R / 2);
        const int col = 2 * (p % (R / 2));
        float v0 = 0.0f, v1 = 0.0f;
#pragma unroll
        for (int w2 = 0; w2 < QA_PAIRS; ++w2) {
          const float2 t = *reinterpret_cast<const float2*>(red + ((w2 * QA_ROWS + row) * R + col));
          v0 += t.x;
          v1 += t.y;
        }
        const int mm = m0 + row;
        if (mm < M) {
          v0 = __fmul_rn(v0, lr_scale);
          v1 = __fmul_rn(v1, lr_scale);
          const float h0 = __bfloat162float(__float2bfloat16_rn(v0));
          const float h1 = __bfloat162float(__float2bfloat16_rn(v1));
          uint16_t* dst = LAs + (int64_t)mm * (2 * R);
          *reinterpret_cast<uint32_t*>(dst + col) = pack_bf16x2(h0, h1);
          *reinterpret_cast<uint32_t*>(dst + R + col) = pack_bf16x2(v0 - h0, v1 - h1);
        }
      }
    }
  }
}

}  // namespace svdq
