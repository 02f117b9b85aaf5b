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
// CTA = 32 rows x all of K; 8 consumer warps + 1 TMA producer warp.
// Stage = one 64-column chunk: X box 32 x 64 bf16 (4 KB) and L1f^T box
// r x 64 bf16, both 128-byte swizzled.  Consumer thread t handles row t/8,
// columns 8(t%8)..+7 of the chunk (half a group; the pair of threads of a
// group combine their maxima with one shuffle).  Warp w owns the (16-row,
// 8-column) tiles p = w, w+8, ... of the 32 x r down-projection output and
// keeps them in registers across the whole K loop (mma.sync m16n8k16).
#pragma once
#include "common.cuh"

namespace svdq {

constexpr int QA_ROWS = 32;
constexpr int QA_CHUNK = 64;          // bf16 columns per stage (128 bytes)
constexpr int QA_CONSUMER_WARPS = 8;
constexpr int QA_THREADS = (QA_CONSUMER_WARPS + 1) * 32;

template <int R>
struct QaCfg {
  static constexpr int kStages = R <= 32 ? 8 : (R <= 64 ? 6 : 4);
  static constexpr int kXBytes = QA_ROWS * 128;
  static constexpr int kLBytes = R * 128;
  static constexpr int kStageBytes = kXBytes + kLBytes;
  static constexpr int kTiles = 2 * (R / 8);                        // (m16, n8) tiles of the 32 x R output
  static constexpr int kTilesPerWarp = (kTiles + QA_CONSUMER_WARPS - 1) / QA_CONSUMER_WARPS;
  static constexpr int kSmem = kStages * kStageBytes + 2 * kStages * 8 + 16 + 1024;
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

// Byte offset of 16-byte chunk `c16` of row `row` in a 128-byte-swizzled tile.
SVDQ_DEV uint32_t sw128(uint32_t row, uint32_t c16) { return row * 128u + ((c16 ^ (row & 7u)) << 4); }

template <int R>
__global__ void __launch_bounds__(QA_THREADS) k_quantize_act(
    const __grid_constant__ CUtensorMap tm_x,   // bf16 {K, M}, box {64, 32}, 128B swizzle
    const __grid_constant__ CUtensorMap tm_l1,  // bf16 {K, R}, box {64, R}, 128B swizzle
    const float* __restrict__ inv_s, float gs_x, float lr_scale, int M, int K, int Mpad,
    uint8_t* __restrict__ Xq, uint8_t* __restrict__ SFx, uint16_t* __restrict__ LAs, uint64_t timeout_ns) {
  using Cfg = QaCfg<R>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + Cfg::kStages * Cfg::kStageBytes);
  uint64_t* empty = full + Cfg::kStages;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(empty + Cfg::kStages);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int m0 = blockIdx.x * QA_ROWS;
  const int nchunks = K / QA_CHUNK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < Cfg::kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], QA_CONSUMER_WARPS);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();

  if (warp == QA_CONSUMER_WARPS) {
    // ---------------------------------------------------------- producer --
    if (lane == 0) {
      tma_prefetch_desc(&tm_x);
      if (R > 0) tma_prefetch_desc(&tm_l1);
      int stage = 0;
      uint32_t phase = 0;
      for (int c = 0; c < nchunks; ++c) {
        if (!mbar_wait(&empty[stage], phase ^ 1u, timeout_ns, abort_flag, 0x201)) break;
        uint8_t* sx = smem + stage * Cfg::kStageBytes;
        mbar_arrive_expect_tx(&full[stage], Cfg::kStageBytes);
        tma_load_2d(sx, &tm_x, &full[stage], c * QA_CHUNK, m0);
        if (R > 0) tma_load_2d(sx + Cfg::kXBytes, &tm_l1, &full[stage], c * QA_CHUNK, 0);
        if (++stage == Cfg::kStages) { stage = 0; phase ^= 1u; }
      }
    }
    return;
  }

  // -------------------------------------------------------------- consumers --
  const int t = threadIdx.x;
  const int row = t >> 3;            // 0..31
  const int j = t & 7;               // 8-column slice of the 64-column chunk
  const int m = m0 + row;
  const float c_x = __frcp_rn(__fmul_rn(6.0f, gs_x));
  const uint32_t KS4 = (uint32_t)(K >> 6);
  const int64_t xq_row = (int64_t)m * (K >> 1);

  float acc[Cfg::kTilesPerWarp > 0 ? Cfg::kTilesPerWarp : 1][4];
#pragma unroll
  for (int i = 0; i < (Cfg::kTilesPerWarp > 0 ? Cfg::kTilesPerWarp : 1); ++i)
    acc[i][0] = acc[i][1] = acc[i][2] = acc[i][3] = 0.0f;

  int stage = 0;
  uint32_t phase = 0;
  bool ok = true;
  for (int c = 0; c < nchunks; ++c) {
    if (!mbar_wait(&full[stage], phase, timeout_ns, abort_flag, 0x202)) { ok = false; break; }
    const uint8_t* sx = smem + stage * Cfg::kStageBytes;
    const uint32_t sx_u32 = smem_u32(sx);

    // ---- quantize 8 elements (half a group) -------------------------------
    const int k0 = c * QA_CHUNK + 8 * j;
    const uint4 raw = *reinterpret_cast<const uint4*>(sx + sw128(row, j));
    const float4 s0 = __ldg(reinterpret_cast<const float4*>(inv_s + k0));
    const float4 s1 = __ldg(reinterpret_cast<const float4*>(inv_s + k0 + 4));
    float xh[8];
    xh[0] = __fmul_rn(bf16_lo(raw.x), s0.x);
    xh[1] = __fmul_rn(bf16_hi(raw.x), s0.y);
    xh[2] = __fmul_rn(bf16_lo(raw.y), s0.z);
    xh[3] = __fmul_rn(bf16_hi(raw.y), s0.w);
    xh[4] = __fmul_rn(bf16_lo(raw.z), s1.x);
    xh[5] = __fmul_rn(bf16_hi(raw.z), s1.y);
    xh[6] = __fmul_rn(bf16_lo(raw.w), s1.z);
    xh[7] = __fmul_rn(bf16_hi(raw.w), s1.w);
    float a = 0.0f;
#pragma unroll
    for (int i = 0; i < 8; ++i) a = fmaxf(a, fabsf(xh[i]));
    a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, 1));
    const uint32_t sb = cvt_ue4m3(__fmul_rn(a, c_x));
    uint32_t code = 0u;
    if (sb != 0u) {
      const float rinv = __frcp_rn(__fmul_rn(dec_ue4m3(sb), gs_x));
      float q[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) q[i] = __fmul_rn(xh[i], rinv);
      code = cvt_e2m1x8(q);
    }
    if (m < M) *reinterpret_cast<uint32_t*>(Xq + xq_row + (k0 >> 1)) = code;
    const uint32_t s2 = __shfl_down_sync(0xffffffffu, sb, 2);
    const uint32_t s4 = __shfl_down_sync(0xffffffffu, sb, 4);
    const uint32_t s6 = __shfl_down_sync(0xffffffffu, sb, 6);
    if (j == 0 && m < Mpad)
      *reinterpret_cast<uint32_t*>(SFx + sf_word_offset((uint32_t)m, (uint32_t)c, KS4)) =
          sb | (s2 << 8) | (s4 << 16) | (s6 << 24);

    // ---- down-projection on the tensor cores ------------------------------
    if constexpr (R > 0) {
      const uint32_t sl_u32 = sx_u32 + Cfg::kXBytes;
#pragma unroll
      for (int i = 0; i < Cfg::kTilesPerWarp; ++i) {
        const int p = warp + QA_CONSUMER_WARPS * i;
        if (p < Cfg::kTiles) {
          const int mt = p / (R / 8);
          const int nt = p % (R / 8);
#pragma unroll
          for (int ks = 0; ks < 4; ++ks) {
            uint32_t a0, a1, a2, a3, b0, b1;
            const uint32_t arow = mt * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
            ldsm_x4(sx_u32 + sw128(arow, ks * 2 + (lane >> 4)), a0, a1, a2, a3);
            const uint32_t brow = nt * 8 + (lane & 7);
            ldsm_x2(sl_u32 + sw128(brow, ks * 2 + ((lane >> 3) & 1)), b0, b1);
            mma_bf16_16816(acc[i], a0, a1, a2, a3, b0, b1);
          }
        }
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[stage]);
    if (++stage == Cfg::kStages) { stage = 0; phase ^= 1u; }
  }

  // ---- LAs = [hi | lo] of lr_scale * (X L1f) -------------------------------
  if constexpr (R > 0) {
    if (ok) {
#pragma unroll
      for (int i = 0; i < Cfg::kTilesPerWarp; ++i) {
        const int p = warp + QA_CONSUMER_WARPS * i;
        if (p < Cfg::kTiles) {
          const int mt = p / (R / 8);
          const int nt = p % (R / 8);
          const int col = nt * 8 + 2 * (lane & 3);
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const int mm = m0 + mt * 16 + (lane >> 2) + 8 * h;
            if (mm < M) {
              const float v0 = __fmul_rn(acc[i][2 * h], lr_scale);
              const float v1 = __fmul_rn(acc[i][2 * h + 1], lr_scale);
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
  }
}

}  // namespace svdq
