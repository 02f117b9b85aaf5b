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
// Persistent, warp-specialised kernel, one CTA per SM, 128 x 256 output tiles:
//   warp 0   TMA producer, one lane per (ring slot, load stream): A box 128 rows x 128 B,
//            B box 256 rows x 128 B (128-byte swizzle), and the stage's scale blocks
//            (SFA: 4 K-atoms of the 128 rows, SFB: 4 K-atoms of each of the two 128-row
//            blocks; stored in MMA order, so plain bulk copies).  A thread's TMA copies are
//            serviced one after another, so no lane has more than one in flight.
//   warp 1   TMEM owner and MMA issuer (one thread): 4 MMAs (K = 64 each) per K tile,
//            then the rank tiles, all into one accumulator.
//   warp 2   scale copier (one thread): as soon as a stage's scale blocks land (their own
//            barrier, ahead of the larger A/B boxes), shared -> TMEM copies (tcgen05.cp,
//            replicated into the four lane quarters), then a commit that tells the MMA thread.  Copies issued by the MMA thread itself
//            stall its MMA issue; from a thread of their own they overlap the MMAs.
//   warps 4-11  epilogue: TMEM -> registers (two warps per 32-lane quarter, 128 columns
//            each), release the accumulator, scale + bias, store.
// 4-stage smem ring (54 KB a stage).  TMEM: accumulator in columns 0-255, per-stage
// scale slots of 48 columns from column 256.
#pragma once
#include "common.cuh"

namespace svdq {

constexpr int LN_BM = 128;
constexpr int LN_BN = 256;
constexpr int LN_STAGES = 4;
constexpr int LN_A_BYTES = LN_BM * 128;          // 128 rows x 256 FP4 (or 64 bf16)
constexpr int LN_B_BYTES = LN_BN * 128;
constexpr int LN_SFA_BYTES = 4 * 512;            // 4 K-atoms of 128 rows
constexpr int LN_SFB_BYTES = 2 * 4 * 512;        // 2 row blocks x 4 K-atoms
constexpr int LN_THREADS = 384;
constexpr int LN_EPI_WARP0 = 4;
constexpr int LN_EPI_WARPS = 8;
constexpr int LN_TMEM_COLS = 512;
constexpr int LN_SF_COL0 = 256;
constexpr int LN_SF_COLS_PER_STAGE = 48;
constexpr int LN_STREAMS = 5;                    // A, B, SFA, SFB block 0, SFB block 1
constexpr int LN_OFF_B = LN_STAGES * LN_A_BYTES;
constexpr int LN_OFF_SFA = LN_OFF_B + LN_STAGES * LN_B_BYTES;
constexpr int LN_OFF_SFB = LN_OFF_SFA + LN_STAGES * LN_SFA_BYTES;
constexpr int LN_OFF_BAR = LN_OFF_SFB + LN_STAGES * LN_SFB_BYTES;
constexpr int LN_SMEM = LN_OFF_BAR + 512 + 1024;
constexpr uint64_t LN_DEFAULT_TIMEOUT_NS = 2000000000ull;
static_assert(LN_SF_COL0 + LN_STAGES * LN_SF_COLS_PER_STAGE <= LN_TMEM_COLS, "TMEM budget");
static_assert(LN_STAGES * LN_STREAMS <= 32, "one producer lane per slot and stream");

enum : int { LN_DBG_NO_LOADS = 1 };

struct LinearArgs {
  const uint8_t* SFx;
  const uint8_t* SFw;
  const uint16_t* bias;
  void* Y;
  int y_fp32;
  int M, N, K, r;
  float gs;
  int debug;
  uint64_t timeout_ns;
};

__global__ void __launch_bounds__(LN_THREADS, 1) k_linear(
    const __grid_constant__ CUtensorMap tm_xq,   // uint8 {K/2, M},  box {128, 128}, SW128
    const __grid_constant__ CUtensorMap tm_wq,   // uint8 {K/2, N},  box {128, 256}, SW128
    const __grid_constant__ CUtensorMap tm_las,  // bf16  {2r, M},   box {64, 128},  SW128
    const __grid_constant__ CUtensorMap tm_l2p,  // bf16  {2r, N},   box {64, 256},  SW128
    const LinearArgs args) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + LN_OFF_B;
  uint8_t* sSFA = smem + LN_OFF_SFA;
  uint8_t* sSFB = smem + LN_OFF_SFB;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + LN_OFF_BAR);   // stage's A/B landed
  uint64_t* sf_ready = full + LN_STAGES;                              // stage scales in TMEM
  uint64_t* empty = sf_ready + LN_STAGES;                             // stage consumed by the MMAs
  uint64_t* acc_full = empty + LN_STAGES;
  uint64_t* acc_empty = acc_full + 1;
  uint64_t* drain = acc_empty + 1;                                    // MMA thread, on a time-out
  uint64_t* drain_cp = drain + 1;                                     // copier thread, on a time-out
  uint64_t* sf_full = drain_cp + 1;                                   // stage's scale blocks landed
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sf_full + LN_STAGES);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int M = args.M, N = args.N, K = args.K, r = args.r;
  const int KA = K >> 6;                          // K atoms of 64
  const int nkt = (KA + 3) >> 2;                  // K tiles of 256
  const int nlr = r > 0 ? (2 * r + 63) / 64 : 0;  // rank tiles of 64 bf16
  const int nst = nkt + nlr;                      // ring stages per output tile
  const int sfx_blocks = (M + 127) >> 7;          // 128-row blocks in the scale buffers
  const int sfw_blocks = (N + 127) >> 7;
  const int num_m = (M + LN_BM - 1) / LN_BM;
  const int num_n = (N + LN_BN - 1) / LN_BN;
  const int total = num_m * num_n;
  const uint64_t tmo = args.timeout_ns;

  if (threadIdx.x == 0) {
    for (int s = 0; s < LN_STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&sf_full[s], 1);
      mbar_init(&sf_ready[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(acc_full, 1);
    mbar_init(acc_empty, LN_EPI_WARPS);
    mbar_init(drain, 1);
    mbar_init(drain_cp, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, LN_TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tmem_slot;

  if (warp == 0) {
    if (lane < LN_STAGES * LN_STREAMS && !(args.debug & LN_DBG_NO_LOADS)) {
      // ---------------------------------------------------------- producer --
      const int g = lane / LN_STREAMS, k = lane % LN_STREAMS;   // ring slot, load stream
      if (lane == 0) {
        tma_prefetch_desc(&tm_xq);
        tma_prefetch_desc(&tm_wq);
        if (r > 0) {
          tma_prefetch_desc(&tm_las);
          tma_prefetch_desc(&tm_l2p);
        }
      }
      int gidx = 0;                 // position in this CTA's sequence of ring stages
      bool ok = true, issued = false;
      uint32_t last_parity = 0;
      for (int t = blockIdx.x; t < total && ok; t += gridDim.x) {
        const int mb = t / num_n, nb = t % num_n;
        for (int kt = 0; kt < nst; ++kt, ++gidx) {
          const int stage = gidx % LN_STAGES;
          if (stage != g) continue;
          const uint32_t phase = (uint32_t)((gidx / LN_STAGES) & 1);
          if (!mbar_wait(&empty[stage], phase ^ 1u, tmo, abort_flag, 0x301)) { ok = false; break; }
          if (kt < nkt) {
            // Scale blocks are contiguous runs of ka 512-byte atoms, copied as they are.  Blocks
            // past the end of a scale buffer (rows beyond the padded M or N) are not loaded; they
            // only feed accumulator rows or columns that are never stored.
            const int ka = min(4, KA - 4 * kt);
            const bool has_a = mb < sfx_blocks;
            const bool has_b0 = 2 * nb < sfw_blocks, has_b1 = 2 * nb + 1 < sfw_blocks;
            if (k == 0) {
              mbar_arrive_expect_tx(&full[stage], (uint32_t)(LN_A_BYTES + LN_B_BYTES));
              tma_load_2d(sA + stage * LN_A_BYTES, &tm_xq, &full[stage], kt * 128, mb * LN_BM);
            } else if (k == 1) {
              tma_load_2d(sB + stage * LN_B_BYTES, &tm_wq, &full[stage], kt * 128, nb * LN_BN);
            } else if (k == 2) {
              mbar_arrive_expect_tx(&sf_full[stage], (uint32_t)((has_a + has_b0 + has_b1) * ka * 512));
              if (has_a)
                bulk_load(sSFA + stage * LN_SFA_BYTES, args.SFx + ((int64_t)mb * KA + 4 * kt) * 512,
                          (uint32_t)(ka * 512), &sf_full[stage]);
            } else if (k == 3 ? has_b0 : has_b1) {
              const int rb = 2 * nb + (k - 3);
              bulk_load(sSFB + stage * LN_SFB_BYTES + 2048 * (k - 3), args.SFw + ((int64_t)rb * KA + 4 * kt) * 512,
                        (uint32_t)(ka * 512), &sf_full[stage]);
            }
          } else {
            const int i = kt - nkt;
            if (k == 0) {
              mbar_arrive_expect_tx(&full[stage], LN_A_BYTES + LN_B_BYTES);
              tma_load_2d(sA + stage * LN_A_BYTES, &tm_las, &full[stage], i * 64, mb * LN_BM);
            } else if (k == 1) {
              tma_load_2d(sB + stage * LN_B_BYTES, &tm_l2p, &full[stage], i * 64, nb * LN_BN);
            } else if (k == 2) {
              mbar_arrive(&sf_full[stage]);            // no scales in a rank stage
            }
          }
          issued = true;
          last_parity = phase;
        }
      }
      if (*abort_flag && issued) {
        // Give the last load of this lane's slot the chance to land before the CTA exits.
        int never = 0;
        if (k < 2) mbar_wait(&full[g], last_parity, tmo, &never, 0x302);
        else mbar_wait(&sf_full[g], last_parity, tmo, &never, 0x302);
      }
    }
  } else if (warp == 1) {
    // ----------------------------------------------------------- MMA issuer --
    if (lane == 0) {
      constexpr uint32_t IDESC_F4 = idesc_nvf4(LN_BM, LN_BN);
      constexpr uint32_t IDESC_BF16 = idesc_bf16(LN_BM, LN_BN);
      int stage = 0;
      uint32_t phase = 0;
      int it = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < total && ok; t += gridDim.x, ++it) {
        if (it > 0 && !mbar_wait(acc_empty, (uint32_t)((it - 1) & 1), tmo, abort_flag, 0x311)) break;
        tc_fence_after();
        for (int kt = 0; kt < nst; ++kt) {
          if (!mbar_wait(&full[stage], phase, tmo, abort_flag, 0x312) ||
              !mbar_wait(&sf_ready[stage], phase, tmo, abort_flag, 0x314)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t adesc = sdesc_kmajor_sw128(smem_u32(sA + stage * LN_A_BYTES));
          const uint64_t bdesc = sdesc_kmajor_sw128(smem_u32(sB + stage * LN_B_BYTES));
          if (kt < nkt) {
            const int ka = min(4, KA - 4 * kt);
            const uint32_t sfa_col = tbase + LN_SF_COL0 + LN_SF_COLS_PER_STAGE * stage;
            const uint32_t sfb_col = sfa_col + 16;
            for (int j = 0; j < ka; ++j)
              tc_mma_nvf4(tbase, adesc + 2 * j, bdesc + 2 * j, IDESC_F4, sfa_col + 4 * j, sfb_col + 8 * j,
                          (kt | j) != 0 ? 1u : 0u);
          } else {
#pragma unroll
            for (int j = 0; j < 4; ++j) tc_mma_bf16(tbase, adesc + 2 * j, bdesc + 2 * j, IDESC_BF16, 1u);
          }
          tc_commit(&empty[stage]);
          if (++stage == LN_STAGES) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        tc_commit(acc_full);
      }
      if (*abort_flag) {
        int never = 0;
        tc_commit(drain);
        mbar_wait(drain, 0, tmo, &never, 0x313);
      }
    }
  } else if (warp == 2) {
    // --------------------------------------------------------- scale copier --
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < total && ok; t += gridDim.x) {
        for (int kt = 0; kt < nst; ++kt) {
          // the stage's scales landed; the MMAs of the slot's previous round finished before its
          // loads began, so its TMEM scale slot is free
          if (!mbar_wait(&sf_full[stage], phase, tmo, abort_flag, 0x331)) { ok = false; break; }
          tc_fence_after();
          if (kt < nkt) {
            const int ka = min(4, KA - 4 * kt);
            const uint32_t sfa_col = tbase + LN_SF_COL0 + LN_SF_COLS_PER_STAGE * stage;
            const uint32_t sfb_col = sfa_col + 16;
            const uint32_t sfa_s = smem_u32(sSFA + stage * LN_SFA_BYTES);
            const uint32_t sfb_s = smem_u32(sSFB + stage * LN_SFB_BYTES);
            for (int j = 0; j < ka; ++j) {
              tc_cp_32x128b_x4(sfa_col + 4 * j, sdesc_sf_block(sfa_s + 512 * j));
              tc_cp_32x128b_x4(sfb_col + 8 * j, sdesc_sf_block(sfb_s + 512 * j));
              tc_cp_32x128b_x4(sfb_col + 8 * j + 4, sdesc_sf_block(sfb_s + 2048 + 512 * j));
            }
          }
          tc_commit(&sf_ready[stage]);
          if (++stage == LN_STAGES) { stage = 0; phase ^= 1u; }
        }
      }
      if (*abort_flag) {
        int never = 0;
        tc_commit(drain_cp);     // lets the copies issued so far finish before TMEM is released
        mbar_wait(drain_cp, 0, tmo, &never, 0x332);
      }
    }
  } else if (warp >= LN_EPI_WARP0) {
    // ------------------------------------------------------------- epilogue --
    const int ew = warp - LN_EPI_WARP0;
    const int q = warp & 3;              // TMEM lane quarter this warp may access
    const int h = ew >> 2;               // column half of the 256-wide tile
    const float gs = args.gs;
    int it = 0;
    for (int t = blockIdx.x; t < total; t += gridDim.x, ++it) {
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
      if (lane == 0) mbar_arrive(acc_empty);

      const int row = mb * LN_BM + 32 * q + lane;
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

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tbase, LN_TMEM_COLS);
  }
}

}  // namespace svdq
