// Kernel 3, CTA-pair form: the same GEMM as k_linear (block-scaled NVFP4 on tcgen05 with
// the low-rank up-projection in the same accumulator), on pairs of CTAs (clusters of 2,
// tcgen05 cta_group::2) that own 256 x 256 output tiles.
//
// SVDQuant review, §4.3 (Nunchaku): the up-projection is merged into the 4-bit GEMM;
// §4.2 output X_hat L1 L2 + Q(X_hat) Q(R); §3 the scaled 4-bit product.
//
// Why pairs: CTA r of a pair holds rows 128r..128r+127 of the tile's A rows and of its 256
// B rows; one MMA of the first CTA multiplies the pair's 256 A rows by all 256 B rows, each
// CTA's TMEM receiving the 128 x 256 accumulator of its own A rows.  Each CTA so loads half
// of B: 38 KB a stage instead of 54 KB for the same MMA work per SM, and the L2 -> SM
// traffic that bounds the single-CTA kernel drops by 30 %.
//
// Per CTA (16 warps, same roles as k_linear):
//   warp 0      tensor producer: A box (own 128 rows) and B box (own 128 rows of N), 128-byte
//               swizzle, counted on the CTA's own "full" barrier.  (Pair-form copies counted on
//               the first CTA's barrier landed 3.7 us after issue against 1.1-1.4 us for local
//               ones.)
//   warp 3      in the second CTA: forwards each stage's "full" to the first CTA's "peer_full".
//   warp 1      TMEM owner (cta_group::2 allocation); in the first CTA the MMA issuer: 4 MMAs
//               of 256 x 256 x 64 per K tile, then the rank tiles; each commit is multicast to
//               the "empty" barrier of both CTAs.
//   warp 2      scale producer: SFA of its 128 rows, SFB of all 256 columns (its TMEM must hold
//               the scales of every column it accumulates), into its own "sf_full" barrier.
//   warps 4-11  epilogue of its own 128 rows; the accumulator is released to the first CTA.
//   warps 12-15 scale writers (tcgen05.st into the CTA's own TMEM), then an arrival on the
//               first CTA's "sf_ready" barrier (8 arrivals: 4 local, 4 from the other CTA).
// No load uses cluster multicast.  5-stage smem ring (38 KB a stage).  TMEM: accumulator in
// columns 0-255, per-stage scale slots of 48 columns from column 256.
#pragma once
#include "common.cuh"
#include "linear.cuh"

namespace svdq {

constexpr int LP_BM = 256;                       // rows of a pair tile (128 per CTA)
constexpr int LP_BN = 256;
constexpr int LP_STAGES = 5;
constexpr int LP_A_BYTES = 128 * 128;            // 128 rows x 256 FP4 (or 64 bf16)
constexpr int LP_B_BYTES = 128 * 128;            // this CTA's half of the B rows
constexpr int LP_SFA_BYTES = 4 * 512;            // 4 K-atoms of this CTA's 128 rows
constexpr int LP_SFB_BYTES = 2 * 4 * 512;        // both 128-row blocks of B x 4 K-atoms
constexpr int LP_THREADS = 512;
constexpr int LP_TMEM_COLS = 512;
constexpr int LP_SF_COL0 = 256;
constexpr int LP_SF_COLS_PER_STAGE = 48;
constexpr int LP_OFF_B = LP_STAGES * LP_A_BYTES;
constexpr int LP_OFF_SFA = LP_OFF_B + LP_STAGES * LP_B_BYTES;
constexpr int LP_OFF_SFB = LP_OFF_SFA + LP_STAGES * LP_SFA_BYTES;
constexpr int LP_OFF_BAR = LP_OFF_SFB + LP_STAGES * LP_SFB_BYTES;
constexpr int LP_SMEM = LP_OFF_BAR + 256 + 1024;
static_assert(LP_SF_COL0 + LP_STAGES * LP_SF_COLS_PER_STAGE <= LP_TMEM_COLS, "TMEM budget");
static_assert(LP_STAGES * 2 <= 32 && LP_STAGES * 3 <= 32, "one lane per slot and stream");

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(LP_THREADS, 1) k_linear_pair(
    const __grid_constant__ CUtensorMap tm_xq,   // uint8 {K/2, M},  box {128, 128}, SW128
    const __grid_constant__ CUtensorMap tm_wq,   // uint8 {K/2, N},  box {128, 128}, SW128
    const __grid_constant__ CUtensorMap tm_las,  // bf16  {2r, M},   box {64, 128},  SW128
    const __grid_constant__ CUtensorMap tm_l2p,  // bf16  {2r, N},   box {64, 128},  SW128
    const LinearArgs args) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + LP_OFF_B;
  uint8_t* sSFA = smem + LP_OFF_SFA;
  uint8_t* sSFB = smem + LP_OFF_SFB;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + LP_OFF_BAR);   // this CTA's A/B landed
  uint64_t* sf_full = full + LP_STAGES;                               // this CTA's scale blocks landed
  uint64_t* sf_ready = sf_full + LP_STAGES;                           // both CTAs' scales in TMEM (first CTA)
  uint64_t* empty = sf_ready + LP_STAGES;                             // stage consumed by the MMAs
  uint64_t* acc_full = empty + LP_STAGES;
  uint64_t* acc_empty = acc_full + 1;                                 // first CTA: both epilogues done
  uint64_t* drain = acc_empty + 1;
  uint64_t* peer_full = drain + 1;                                    // first CTA: the other CTA's A/B landed
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(peer_full + LP_STAGES);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();       // 0: issues the pair's MMAs
  const int M = args.M, N = args.N, K = args.K, r = args.r;
  const int KA = K >> 6;                          // K atoms of 64
  const int nkt = (KA + 3) >> 2;                  // K tiles of 256
  const int nlr = r > 0 ? (2 * r + 63) / 64 : 0;  // rank tiles of 64 bf16
  const int nst = nkt + nlr;                      // ring stages per output tile
  const int sfx_blocks = (M + 127) >> 7;          // 128-row blocks in the scale buffers
  const int sfw_blocks = (N + 127) >> 7;
  const int num_m = (M + LP_BM - 1) / LP_BM;
  const int num_n = (N + LP_BN - 1) / LP_BN;
  const int total = num_m * num_n;
  const int pair = blockIdx.x >> 1;
  const int npairs = gridDim.x >> 1;
  const uint64_t tmo = args.timeout_ns;

  if (threadIdx.x == 0) {
    for (int s = 0; s < LP_STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&sf_full[s], 1);
      mbar_init(&sf_ready[s], 8);                  // 4 scale writers in each CTA
      mbar_init(&empty[s], 1);
      mbar_init(&peer_full[s], 1);
    }
    mbar_init(acc_full, 1);
    mbar_init(acc_empty, 2 * LN_EPI_WARPS);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_slot, LP_TMEM_COLS);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync_all();                              // barriers of both CTAs initialised
  tc_fence_after();
  const uint32_t tbase = *tmem_slot;

  if (warp == 0 || warp == 2) {
    regs_dec<LN_REGS_LOW>();
    if (!(args.debug & LN_DBG_NO_LOADS)) {
      // --------------------------------------------------------- producers --
      // In-order, warp-uniform waits on this CTA's "empty" (multicast by the first CTA's
      // commits); lane S g + k issues stream k of slot g, the stage's lanes in one converged
      // instruction.  Warp 0: k = 0 A, 1 B (this CTA's "full").  Warp 2: k = 0 SFA, 1 SFB
      // block 0, 2 SFB block 1 (this CTA's "sf_full").
      const bool tensor_warp = warp == 0;
      const int per = tensor_warp ? 2 : 3;
      const int g = lane / per, k = lane % per;
      const bool loader = lane < LP_STAGES * per;
      if (lane == 0 && tensor_warp) {
        tma_prefetch_desc(&tm_xq);
        tma_prefetch_desc(&tm_wq);
        if (r > 0) {
          tma_prefetch_desc(&tm_las);
          tma_prefetch_desc(&tm_l2p);
        }
      }
      int gidx = 0;
      bool ok = true, issued = false;
      uint32_t last_parity = 0;
      for (int t = pair; t < total && ok; t += npairs) {
        int mb, nb;
        tile_coords(t, num_m, num_n, mb, nb);
        const int arow = mb * LP_BM + 128 * (int)rank;     // this CTA's A rows
        const int brow = nb * LP_BN + 128 * (int)rank;     // this CTA's half of the B rows
        for (int kt = 0; kt < nst; ++kt, ++gidx) {
          const int stage = gidx % LP_STAGES;
          const uint32_t phase = (uint32_t)((gidx / LP_STAGES) & 1);
          int free_slot = 1;
          if (lane == 0) free_slot = mbar_wait(&empty[stage], phase ^ 1u, tmo, abort_flag, 0x401) ? 1 : 0;
          if (!__shfl_sync(0xffffffffu, free_slot, 0)) { ok = false; break; }
          const bool mine = loader && g == stage;
          const bool lr = kt >= nkt;
          const unsigned smask = (tensor_warp ? 3u : 7u) << (per * stage);
          if (tensor_warp) {
            if (mine) {
              if (k == 0) mbar_arrive_expect_tx(&full[stage], (uint32_t)(LP_A_BYTES + LP_B_BYTES));
              const CUtensorMap* map = k == 0 ? (lr ? &tm_las : &tm_xq) : (lr ? &tm_l2p : &tm_wq);
              uint8_t* dst = k == 0 ? sA + stage * LP_A_BYTES : sB + stage * LP_B_BYTES;
              const int x = lr ? (kt - nkt) * 64 : kt * 128;
              __syncwarp(smask);
              tma_load_2d(dst, map, &full[stage], x, k == 0 ? arow : brow);
              issued = true;
              last_parity = phase;
            }
          } else if (mine) {
            const int ka = lr ? 0 : min(4, KA - 4 * kt);
            const int ablk = arow >> 7;
            const int has_a = ablk < sfx_blocks, has_b0 = 2 * nb < sfw_blocks, has_b1 = 2 * nb + 1 < sfw_blocks;
            if (k == 0) {
              if (lr) mbar_arrive(&sf_full[stage]);
              else mbar_arrive_expect_tx(&sf_full[stage], (uint32_t)((has_a + has_b0 + has_b1) * ka * 512));
            }
            const bool has = !lr && (k == 0 ? has_a : k == 1 ? has_b0 : has_b1);
            __syncwarp(smask);
            if (has) {
              uint8_t* dst = k == 0 ? sSFA + stage * LP_SFA_BYTES : sSFB + stage * LP_SFB_BYTES + 2048 * (k - 1);
              const uint8_t* src = k == 0 ? args.SFx + ((int64_t)ablk * KA + 4 * kt) * 512
                                          : args.SFw + ((int64_t)(2 * nb + k - 1) * KA + 4 * kt) * 512;
              bulk_load(dst, src, (uint32_t)(ka * 512), &sf_full[stage]);
              issued = true;
              last_parity = phase;
            }
          }
          __syncwarp();
        }
      }
      if (*abort_flag && issued) {
        // Let this lane's last copy land before the CTA exits.
        int never = 0;
        mbar_wait(tensor_warp ? &full[g] : &sf_full[g], last_parity, tmo, &never, 0x402);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------- MMA issuer (first CTA) --
    regs_dec<LN_REGS_LOW>();
    if (rank == 0 && lane == 0) {
      constexpr uint32_t IDESC_F4 = idesc_nvf4(LP_BM, LP_BN);
      constexpr uint32_t IDESC_BF16 = idesc_bf16(LP_BM, LP_BN);
      int stage = 0;
      uint32_t phase = 0;
      int it = 0;
      bool ok = true;
      for (int t = pair; t < total && ok; t += npairs, ++it) {
        if (it > 0 && !mbar_wait_cluster(acc_empty, (uint32_t)((it - 1) & 1), tmo, abort_flag, 0x411)) break;
        tc_fence_after();
        for (int kt = 0; kt < nst; ++kt) {
          if (!mbar_wait(&full[stage], phase, tmo, abort_flag, 0x412) ||
              !mbar_wait_cluster(&peer_full[stage], phase, tmo, abort_flag, 0x415) ||
              !mbar_wait_cluster(&sf_ready[stage], phase, tmo, abort_flag, 0x414)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t adesc = sdesc_kmajor_sw128(smem_u32(sA + stage * LP_A_BYTES));
          const uint64_t bdesc = sdesc_kmajor_sw128(smem_u32(sB + stage * LP_B_BYTES));
          if (kt < nkt) {
            const int ka = min(4, KA - 4 * kt);
            const uint32_t sfa_col = tbase + LP_SF_COL0 + LP_SF_COLS_PER_STAGE * stage;
            const uint32_t sfb_col = sfa_col + 16;
            for (int j = 0; j < ka; ++j)
              tc_mma_nvf4_pair(tbase, adesc + 2 * j, bdesc + 2 * j, IDESC_F4, sfa_col + 4 * j, sfb_col + 8 * j,
                               (kt | j) != 0 ? 1u : 0u);
          } else {
#pragma unroll
            for (int j = 0; j < 4; ++j) tc_mma_bf16_pair(tbase, adesc + 2 * j, bdesc + 2 * j, IDESC_BF16, 1u);
          }
          tc_commit_pair_mc(&empty[stage], 0x3);
          if (++stage == LP_STAGES) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        tc_commit_pair_mc(acc_full, 0x3);
      }
      if (*abort_flag) {
        int never = 0;
        tc_commit_pair(drain);
        mbar_wait(drain, 0, tmo, &never, 0x413);
      }
    }
  } else if (warp >= LN_SFW_WARP0) {
    // -------------------------------------------------------- scale writers --
    // Same layout as k_linear's writers: lane l of every quarter takes the 16 bytes at 16 l of
    // each 512-byte atom; SFA atom j -> columns 4j, SFB block b atom j -> 16 + 8j + 4b.
    regs_dec<LN_REGS_LOW>();
    const int q = warp & 3;
    const uint32_t lane_base = tbase + ((uint32_t)(32 * q) << 16);
    const uint32_t ready0 = mapa_shared(smem_u32(sf_ready), 0);   // sf_ready[0] of the first CTA
    int stage = 0;
    uint32_t phase = 0;
    bool ok = true;
    for (int t = pair; t < total && ok; t += npairs) {
      for (int kt = 0; kt < nst; ++kt) {
        int landed = 1;
        if (lane == 0) landed = mbar_wait(&sf_full[stage], phase, tmo, abort_flag, 0x431) ? 1 : 0;
        if (!__shfl_sync(0xffffffffu, landed, 0)) { ok = false; break; }
        if (kt < nkt) {
          const uint32_t sa = smem_u32(sSFA + stage * LP_SFA_BYTES) + 16 * lane;
          const uint32_t sb = smem_u32(sSFB + stage * LP_SFB_BYTES) + 16 * lane;
          uint32_t a[16], b0[16], b1[16];
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const uint4 x = lds_v4(sa + 512 * j);
            const uint4 y0 = lds_v4(sb + 512 * j);
            const uint4 y1 = lds_v4(sb + 2048 + 512 * j);
            a[4 * j] = x.x; a[4 * j + 1] = x.y; a[4 * j + 2] = x.z; a[4 * j + 3] = x.w;
            uint32_t* b = j < 2 ? b0 : b1;
            const int o = 8 * (j & 1);
            b[o] = y0.x; b[o + 1] = y0.y; b[o + 2] = y0.z; b[o + 3] = y0.w;
            b[o + 4] = y1.x; b[o + 5] = y1.y; b[o + 6] = y1.z; b[o + 7] = y1.w;
          }
          const uint32_t col = lane_base + LP_SF_COL0 + LP_SF_COLS_PER_STAGE * stage;
          tmem_st_32x32b_x16(col, a);
          tmem_st_32x32b_x16(col + 16, b0);
          tmem_st_32x32b_x16(col + 32, b1);
          tmem_st_wait();
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(ready0 + 8u * (uint32_t)stage);
        if (++stage == LP_STAGES) { stage = 0; phase ^= 1u; }
      }
    }
  } else if (warp >= LN_EPI_WARP0) {
    // ------------------------------------------------------------- epilogue --
    regs_inc<LN_REGS_HIGH>();
    const int ew = warp - LN_EPI_WARP0;
    const int q = warp & 3;
    const int h = ew >> 2;
    const float gs = args.gs;
    const uint32_t acc_empty0 = mapa_shared(smem_u32(acc_empty), 0);
    int it = 0;
    for (int t = pair; t < total; t += npairs, ++it) {
      int mb, nb;
      tile_coords(t, num_m, num_n, mb, nb);
      if (!mbar_wait(acc_full, (uint32_t)(it & 1), tmo, abort_flag, 0x421)) break;
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
      if (lane == 0) mbar_arrive_cluster(acc_empty0);

      const int row = mb * LP_BM + 128 * (int)rank + 32 * q + lane;
      if (row < M) store_y_row(args, v, row, nb * LP_BN + h * 128, gs);
    }
  } else {
    regs_dec<LN_REGS_LOW>();
    // warp 3 of the second CTA: forwards "this CTA's A/B of the stage landed" to the first CTA
    if (rank == 1 && lane == 0) {
      const uint32_t peer0 = mapa_shared(smem_u32(peer_full), 0);
      int gi = 0;
      bool ok = true;
      for (int t = pair; t < total && ok; t += npairs)
        for (int kt = 0; kt < nst; ++kt, ++gi) {
          const int st2 = gi % LP_STAGES;
          if (!mbar_wait(&full[st2], (uint32_t)((gi / LP_STAGES) & 1), tmo, abort_flag, 0x441)) { ok = false; break; }
          mbar_arrive_cluster(peer0 + 8u * (uint32_t)st2);
        }
    }
  }

  // Both CTAs leave together: TMEM is allocated for the pair and arrivals cross between them.
  tc_fence_before();
  __syncwarp();
  cluster_sync_all();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tbase, LP_TMEM_COLS);
  }
}

}  // namespace svdq
