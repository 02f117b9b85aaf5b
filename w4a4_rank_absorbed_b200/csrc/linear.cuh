// Kernel 3: block-scaled NVFP4 GEMM on the tcgen05 tensor cores with the
// low-rank up-projection fused into the same accumulator.
//
// SVDQuant review, §4.3 (Nunchaku): the up-projection is merged into the 4-bit
// GEMM kernel.  §4.2 output: X_hat L1 L2 (16-bit branch) + Q(X_hat) Q(R).
// §3: XW ~ s_X s_W Q_X Q_W, here in block-scaled form with a UE4M3 scale per
// 16 values along K on both operands and the global scales gs_x, gs_w.
//
//   acc  = sum over K tiles of  tcgen05.mma.kind::mxf4nvf4 (A = Xq, B = Wq, scales SFx, SFw)
//        + sum over rank tiles of tcgen05.mma.kind::f16 (A = LAs, B = L2p)        (same TMEM accumulator)
//   Y    = f32(gs_x gs_w) * acc + bias
// LAs was pre-scaled by 1/(gs_x gs_w) in kernel 2, so a single scale serves both branches.
//
// Persistent, warp-specialised kernel on CTA pairs (clusters of 2, tcgen05 cta_group::2):
// a pair owns a 256 x 256 output tile; CTA r holds rows 128r..128r+127 of the A tile
// and rows 128r..+127 of the B tile (its half of N), and receives in its TMEM the
// 128 x 256 accumulator of its A rows.  Per CTA:
//   warp 0      TMA producer: A box 128 rows x 128 B, B box 128 x 128 B (128-byte swizzle),
//               scale blocks (SFA for its rows, SFB for all 256 columns) as 3-D boxes of
//               4 K-atoms.  Loads of both CTAs count on the first CTA's "full" barrier.
//   warp 1      TMEM owner; in the first CTA also the MMA issuer (one thread): scale
//               blocks smem -> TMEM (tcgen05.cp, both CTAs), then 4 MMAs (K = 64 each) per
//               256-wide K tile, then the rank tiles; commits release the stage in both CTAs.
//   warps 2-9   epilogue: TMEM -> registers (two warps per 32-lane quarter, 128 columns
//               each), release the accumulator to the first CTA, scale + bias, store.
// 5-stage smem ring (38 KB a stage).  TMEM: accumulator in columns 0-255, per-stage
// scale slots of 48 columns from column 256.  No load uses cluster multicast.
#pragma once
#include "common.cuh"

namespace svdq {

constexpr int LN_BM = 256;                       // rows of a pair tile (128 per CTA)
constexpr int LN_BN = 256;
constexpr int LN_STAGES = 5;
constexpr int LN_A_BYTES = 128 * 128;            // 128 rows x 256 FP4 (or 64 bf16)
constexpr int LN_B_BYTES = 128 * 128;            // this CTA's half of N
constexpr int LN_SFA_BYTES = 4 * 512;            // 4 K-atoms of this CTA's 128 rows
constexpr int LN_SFB_BYTES = 2 * 4 * 512;        // 2 row blocks (all 256 columns) x 4 K-atoms
constexpr int LN_STAGE_BYTES = LN_A_BYTES + LN_B_BYTES + LN_SFA_BYTES + LN_SFB_BYTES;
constexpr int LN_THREADS = 320;
constexpr int LN_EPI_WARPS = 8;
constexpr int LN_TMEM_COLS = 512;
constexpr int LN_SF_COL0 = 256;
constexpr int LN_SF_COLS_PER_STAGE = 48;
constexpr int LN_OFF_B = LN_STAGES * LN_A_BYTES;
constexpr int LN_OFF_SFA = LN_OFF_B + LN_STAGES * LN_B_BYTES;
constexpr int LN_OFF_SFB = LN_OFF_SFA + LN_STAGES * LN_SFA_BYTES;
constexpr int LN_OFF_BAR = LN_OFF_SFB + LN_STAGES * LN_SFB_BYTES;
constexpr int LN_SMEM = LN_OFF_BAR + 256 + 1024;
constexpr uint64_t LN_DEFAULT_TIMEOUT_NS = 2000000000ull;
static_assert(LN_SF_COL0 + LN_STAGES * LN_SF_COLS_PER_STAGE <= LN_TMEM_COLS, "TMEM budget");

enum : int { LN_DBG_NO_LOADS = 1 };

struct LinearArgs {
  const uint16_t* bias;
  void* Y;
  int y_fp32;
  int M, N, K, r;
  float gs;
  int debug;
  uint64_t timeout_ns;
};

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(LN_THREADS, 1) k_linear(
    const __grid_constant__ CUtensorMap tm_xq,   // uint8 {K/2, M},  box {128, 128}, SW128
    const __grid_constant__ CUtensorMap tm_wq,   // uint8 {K/2, N},  box {128, 128}, SW128
    const __grid_constant__ CUtensorMap tm_las,  // bf16  {2r, M},   box {64, 128},  SW128
    const __grid_constant__ CUtensorMap tm_l2p,  // bf16  {2r, N},   box {64, 128},  SW128
    const __grid_constant__ CUtensorMap tm_sfx,  // uint8 {256, 2, atoms}, box {256, 2, 4}
    const __grid_constant__ CUtensorMap tm_sfw,  // uint8 {256, 2, atoms}, box {256, 2, 4}
    const LinearArgs args) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + LN_OFF_B;
  uint8_t* sSFA = smem + LN_OFF_SFA;
  uint8_t* sSFB = smem + LN_OFF_SFB;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + LN_OFF_BAR);
  uint64_t* empty = full + LN_STAGES;
  uint64_t* acc_full = empty + LN_STAGES;
  uint64_t* acc_empty = acc_full + 1;
  uint64_t* drain = acc_empty + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();      // 0: issues the MMAs of the pair
  const int M = args.M, N = args.N, K = args.K, r = args.r;
  const int KA = K >> 6;                          // K atoms of 64
  const int nkt = (KA + 3) >> 2;                  // K tiles of 256
  const int nlr = r > 0 ? (2 * r + 63) / 64 : 0;  // rank tiles of 64 bf16
  const int num_m = (M + LN_BM - 1) / LN_BM;
  const int num_n = (N + LN_BN - 1) / LN_BN;
  const int total = num_m * num_n;
  const int pair = blockIdx.x >> 1;
  const int npairs = gridDim.x >> 1;
  const uint64_t tmo = args.timeout_ns;

  if (threadIdx.x == 0) {
    for (int s = 0; s < LN_STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(acc_full, 1);
    mbar_init(acc_empty, 2 * LN_EPI_WARPS);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_slot, LN_TMEM_COLS);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync_all();
  tc_fence_after();
  const uint32_t tbase = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ producer --
    if (lane == 0 && !(args.debug & LN_DBG_NO_LOADS)) {
      tma_prefetch_desc(&tm_xq);
      tma_prefetch_desc(&tm_wq);
      tma_prefetch_desc(&tm_sfx);
      tma_prefetch_desc(&tm_sfw);
      if (r > 0) {
        tma_prefetch_desc(&tm_las);
        tma_prefetch_desc(&tm_l2p);
      }
      int stage = 0;
      uint32_t phase = 0;
      uint32_t issued = 0, issued_parity = 0;
      bool ok = true;
      for (int t = pair; t < total && ok; t += npairs) {
        const int mb = t / num_n, nb = t % num_n;
        const int arow = mb * LN_BM + 128 * (int)rank;    // this CTA's A rows
        const int brow = nb * LN_BN + 128 * (int)rank;    // this CTA's half of the B rows
        for (int kt = 0; kt < nkt + nlr; ++kt) {
          if (!mbar_wait(&empty[stage], phase ^ 1u, tmo, abort_flag, 0x301)) { ok = false; break; }
          const uint32_t fb = mapa_shared(smem_u32(&full[stage]), 0);
          uint8_t* a = sA + stage * LN_A_BYTES;
          uint8_t* b = sB + stage * LN_B_BYTES;
          if (kt < nkt) {
            if (rank == 0) mbar_arrive_expect_tx(&full[stage], 2 * LN_STAGE_BYTES);
            tma_load_2d_pair(a, &tm_xq, fb, kt * 128, arow);
            tma_load_2d_pair(b, &tm_wq, fb, kt * 128, brow);
            tma_load_3d_pair(sSFA + stage * LN_SFA_BYTES, &tm_sfx, fb, 0, 0, (arow >> 7) * KA + 4 * kt);
            tma_load_3d_pair(sSFB + stage * LN_SFB_BYTES, &tm_sfw, fb, 0, 0, (2 * nb) * KA + 4 * kt);
            tma_load_3d_pair(sSFB + stage * LN_SFB_BYTES + 2048, &tm_sfw, fb, 0, 0, (2 * nb + 1) * KA + 4 * kt);
          } else {
            const int i = kt - nkt;
            if (rank == 0) mbar_arrive_expect_tx(&full[stage], 2 * (LN_A_BYTES + LN_B_BYTES));
            tma_load_2d_pair(a, &tm_las, fb, i * 64, arow);
            tma_load_2d_pair(b, &tm_l2p, fb, i * 64, brow);
          }
          issued |= 1u << stage;
          issued_parity = (issued_parity & ~(1u << stage)) | (phase << stage);
          if (++stage == LN_STAGES) { stage = 0; phase ^= 1u; }
        }
      }
      if (*abort_flag && rank == 0) {
        // Give every load already issued the chance to land before the CTAs exit.
        int never = 0;
        for (int s = 0; s < LN_STAGES; ++s)
          if (issued & (1u << s)) mbar_wait(&full[s], (issued_parity >> s) & 1u, tmo, &never, 0x302);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------- MMA issuer (first CTA) --
    if (rank == 0 && lane == 0) {
      constexpr uint32_t IDESC_F4 = idesc_nvf4(LN_BM, LN_BN);
      constexpr uint32_t IDESC_BF16 = idesc_bf16(LN_BM, LN_BN);
      int stage = 0;
      uint32_t phase = 0;
      int it = 0;
      bool ok = true;
      for (int t = pair; t < total && ok; t += npairs, ++it) {
        if (it > 0 && !mbar_wait(acc_empty, (uint32_t)((it - 1) & 1), tmo, abort_flag, 0x311)) break;
        tc_fence_after();
        for (int kt = 0; kt < nkt + nlr; ++kt) {
          if (!mbar_wait(&full[stage], phase, tmo, abort_flag, 0x312)) { ok = false; break; }
          tc_fence_after();
          const uint64_t adesc = sdesc_kmajor_sw128(smem_u32(sA + stage * LN_A_BYTES));
          const uint64_t bdesc = sdesc_kmajor_sw128(smem_u32(sB + stage * LN_B_BYTES));
          if (kt < nkt) {
            const int ka = min(4, KA - 4 * kt);
            const uint32_t sfa_col = tbase + LN_SF_COL0 + LN_SF_COLS_PER_STAGE * stage;
            const uint32_t sfb_col = sfa_col + 16;
            const uint32_t sfa_s = smem_u32(sSFA + stage * LN_SFA_BYTES);
            const uint32_t sfb_s = smem_u32(sSFB + stage * LN_SFB_BYTES);
            for (int j = 0; j < ka; ++j) {
              tc_cp_32x128b_x4_pair(sfa_col + 4 * j, sdesc_sf_block(sfa_s + 512 * j));
              tc_cp_32x128b_x4_pair(sfb_col + 8 * j, sdesc_sf_block(sfb_s + 512 * j));
              tc_cp_32x128b_x4_pair(sfb_col + 8 * j + 4, sdesc_sf_block(sfb_s + 2048 + 512 * j));
            }
            for (int j = 0; j < ka; ++j)
              tc_mma_nvf4_pair(tbase, adesc + 2 * j, bdesc + 2 * j, IDESC_F4, sfa_col + 4 * j, sfb_col + 8 * j,
                               (kt | j) != 0 ? 1u : 0u);
          } else {
#pragma unroll
            for (int j = 0; j < 4; ++j) tc_mma_bf16_pair(tbase, adesc + 2 * j, bdesc + 2 * j, IDESC_BF16, 1u);
          }
          tc_commit_pair_mc(&empty[stage], 0x3);
          if (++stage == LN_STAGES) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        tc_commit_pair_mc(acc_full, 0x3);
      }
      if (*abort_flag) {
        int never = 0;
        tc_commit_pair(drain);
        mbar_wait(drain, 0, tmo, &never, 0x313);
      }
    }
  } else {
    // ------------------------------------------------------------- epilogue --
    const int ew = warp - 2;
    const int q = warp & 3;              // TMEM lane quarter this warp may access
    const int h = ew >> 2;               // column half of the 256-wide tile
    const float gs = args.gs;
    const uint32_t acc_empty_leader = mapa_shared(smem_u32(acc_empty), 0);
    int it = 0;
    for (int t = pair; t < total; t += npairs, ++it) {
      const int mb = t / num_n, nb = t % num_n;
      if (!mbar_wait(acc_full, (uint32_t)(it & 1), tmo, abort_flag, 0x321)) break;
      tc_fence_after();
      uint32_t v[4][32];
      const uint32_t taddr = tbase + ((uint32_t)(32 * q) << 16) + (uint32_t)(h * 128);
#pragma unroll
      for (int i = 0; i < 4; ++i) tmem_ld_32x32b_x32(taddr + 32 * i, v[i]);
      tmem_ld_wait();
#pragma unroll
      for (int i = 0; i < 4; ++i) reg_fence(v[i]);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(acc_empty_leader);

      const int row = mb * LN_BM + 128 * (int)rank + 32 * q + lane;
      if (row < M) {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
#pragma unroll
          for (int g = 0; g < 4; ++g) {
            const int n = nb * LN_BN + h * 128 + 32 * i + 8 * g;
            if (n < N) {
              float bv[8];
              if (args.bias) {
                const uint4 bw = __ldg(reinterpret_cast<const uint4*>(args.bias + n));
                bv[0] = bf16_lo(bw.x); bv[1] = bf16_hi(bw.x); bv[2] = bf16_lo(bw.y); bv[3] = bf16_hi(bw.y);
                bv[4] = bf16_lo(bw.z); bv[5] = bf16_hi(bw.z); bv[6] = bf16_lo(bw.w); bv[7] = bf16_hi(bw.w);
              } else {
#pragma unroll
                for (int e = 0; e < 8; ++e) bv[e] = 0.0f;
              }
              float y[8];
#pragma unroll
              for (int e = 0; e < 8; ++e) y[e] = __fmaf_rn(gs, __uint_as_float(v[i][8 * g + e]), bv[e]);
              if (args.y_fp32) {
                float4* dst = reinterpret_cast<float4*>(static_cast<float*>(args.Y) + (int64_t)row * N + n);
                dst[0] = make_float4(y[0], y[1], y[2], y[3]);
                dst[1] = make_float4(y[4], y[5], y[6], y[7]);
              } else {
                uint4 o;
                o.x = pack_bf16x2(y[0], y[1]);
                o.y = pack_bf16x2(y[2], y[3]);
                o.z = pack_bf16x2(y[4], y[5]);
                o.w = pack_bf16x2(y[6], y[7]);
                *reinterpret_cast<uint4*>(static_cast<uint16_t*>(args.Y) + (int64_t)row * N + n) = o;
              }
            }
          }
        }
      }
    }
  }

  // Both CTAs leave together: the pair shares TMEM allocation, barriers and shared memory reads.
  tc_fence_before();
  __syncwarp();
  cluster_sync_all();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tbase, LN_TMEM_COLS);
  }
}

}  // namespace svdq
