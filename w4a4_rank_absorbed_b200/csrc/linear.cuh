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
// LAs was pre-scaled by 1/(gs_x gs_w) in kernel 2, so a single scale serves both branches.  It holds
// a bf16 hi/lo pair of every low-rank value, interleaved by 16 columns (hi of columns 16j..16j+15,
// then their lo), so a 64-column LAs box meets one 32-column box of L2p (N x r, a single copy of
// L2, 64-byte swizzle) twice: MMA k-steps 0 and 1 (hi, lo of columns 0-15 of the box) both read
// L2p columns 0-15, k-steps 2 and 3 columns 16-31.
//
// Persistent, warp-specialised kernel, one CTA of 16 warps per SM, 128 x 256 output tiles:
//   warp 0   TMA producer for A (box 128 rows x 128 B, 128-byte swizzle) and B (two boxes
//            of 128 rows x 128 B), issued by three lanes in one converged instruction.
//   warp 1   TMEM owner and MMA issuer (one thread): 4 MMAs (K = 64 each) per K tile,
//            then the rank tiles, all into one accumulator.
//   warp 2   producer for the stage's scale blocks (SFA: 4 K-atoms of the 128 rows, SFB:
//            4 K-atoms of each of the two 128-row blocks; stored in MMA order, so plain
//            bulk copies), again three lanes in one instruction.
//   warps 4-11   epilogue: TMEM -> registers (two warps per 32-lane quarter, 128 columns
//            each), release the accumulator, scale + bias, 32-byte stores.
//   warps 12-15  scale writers, one per TMEM lane quarter: shared -> registers ->
//            tcgen05.st of the stage's 12 scale atoms into the quarter's lanes (the MMA
//            reads each atom replicated in all four quarters).  Four warps storing in
//            parallel take about a quarter of the time of the 12 tcgen05.cp copies a
//            single thread would issue, which kept the MMAs waiting.
// Registers: launched at 128 per thread; the epilogue warpgroups raise theirs to 168 and
// the other two lower theirs to 88 (88 x 128 + 168 x 256 + 88 x 128 = 512 x 128).
// 4-stage smem ring (54 KB a stage).  TMEM: accumulator in columns 0-255, per-stage
// scale slots of 48 columns from column 256.
#pragma once
#include "common.cuh"
#include "gelu.cuh"

namespace svdq {

constexpr int LN_BM = 128;
constexpr int LN_BN = 256;
constexpr int LN_STAGES = 4;
constexpr int LN_A_BYTES = LN_BM * 128;          // 128 rows x 256 FP4 (or 64 bf16)
constexpr int LN_B_BYTES = LN_BN * 128;
constexpr int LN_B_HALF = LN_B_BYTES / 2;
constexpr int LN_LR_B_HALF = 128 * 64;           // rank stage: 128 rows of L2p x 32 bf16 (64-byte rows)
constexpr int LN_LR_BYTES = LN_A_BYTES + 2 * LN_LR_B_HALF;
constexpr int LN_SFA_BYTES = 4 * 512;            // 4 K-atoms of 128 rows
constexpr int LN_SFB_BYTES = 2 * 4 * 512;        // 2 row blocks x 4 K-atoms
constexpr int LN_THREADS = 512;
constexpr int LN_EPI_WARP0 = 4;
constexpr int LN_EPI_WARPS = 8;
constexpr int LN_SFW_WARP0 = 12;                 // scale writers: warps 12-15 (lane quarters 0-3)
constexpr int LN_TMEM_COLS = 512;
constexpr int LN_SF_COL0 = 256;
constexpr int LN_SF_COLS_PER_STAGE = 48;
constexpr int LN_REGS_LOW = 88;                  // warpgroups 0 and 3
constexpr int LN_REGS_HIGH = 168;                // warpgroups 1 and 2 (epilogue)
constexpr int LN_STREAMS = 3;                    // lanes per slot: A, B 0, B 1 (warp 0); SFA, SFB 0, SFB 1 (warp 2)
constexpr int LN_OFF_B = LN_STAGES * LN_A_BYTES;
constexpr int LN_OFF_SFA = LN_OFF_B + LN_STAGES * LN_B_BYTES;
constexpr int LN_OFF_SFB = LN_OFF_SFA + LN_STAGES * LN_SFA_BYTES;
constexpr int LN_OFF_BAR = LN_OFF_SFB + LN_STAGES * LN_SFB_BYTES;
constexpr int LN_SMEM = LN_OFF_BAR + 256 + 1024;
// Fused GELU + next-layer quantization epilogue: 1 KB of staging per epilogue warp (the x2 slab
// read back by ldmatrix; a warp pair's 2 KB also carries the pair's partial-sum hand-off).
constexpr int LN_OFF_STG = LN_OFF_BAR + 256;
constexpr int LN_STG_BYTES = 1024;
constexpr int LN_OFF_RCP = LN_OFF_STG + LN_EPI_WARPS * LN_STG_BYTES;   // 256 floats: f32(1/f32(dec(sb) gs2))
constexpr int LN_SMEM_GQ = LN_OFF_RCP + 1024 + 1024;
constexpr int LN_GQ_MAX_R = 32;
static_assert(LN_SMEM_GQ <= 232448, "shared memory budget of the fused epilogue");
constexpr uint64_t LN_DEFAULT_TIMEOUT_NS = 2000000000ull;
static_assert(LN_SF_COL0 + LN_STAGES * LN_SF_COLS_PER_STAGE <= LN_TMEM_COLS, "TMEM budget");
static_assert(LN_STAGES * LN_STREAMS <= 32 && LN_STREAMS == 3, "one lane per slot and stream");
static_assert(LN_REGS_LOW * 256 + LN_REGS_HIGH * 256 == LN_THREADS * 128, "register split = launch budget");

// Test hook (svdq_linear_debug): the load warp issues nothing, so the first wait must run out.
// Test hooks (svdq_linear_debug): the load warp issues nothing, so the first wait must run out; or
// (accepted by the check build only) the first A box of every tile is asked for at a misaligned
// innermost coordinate, which the build's copy checks must catch.
enum : int { LN_DBG_NO_LOADS = 1, LN_DBG_MISALIGN = 2 };

#ifndef LN_RASTER_GM
#define LN_RASTER_GM 12
#endif
// Output tile t -> (row block mb, column block nb).  Tiles run in groups of LN_RASTER_GM
// row blocks; within a group the row block varies fastest.
SVDQ_DEV void tile_coords(int t, int num_m, int num_n, int& mb, int& nb) {
  const int per_group = LN_RASTER_GM * num_n;
  const int first_m = (t / per_group) * LN_RASTER_GM;
  const int gm = min(LN_RASTER_GM, num_m - first_m);
  const int w = t - (t / per_group) * per_group;
  mb = first_m + w % gm;
  nb = w / gm;
}

struct LinearArgs {
  const uint8_t* SFx;
  const uint8_t* SFw;
  const uint16_t* bias;
  void* Y;
  int y_fp32;
  int y_vec32;          // Y is 32-byte aligned: 32-byte stores
  int y_accum;          // Y += result (read-modify-write, the unfused up-projection); no bias

  int M, N, K, r;
  float gs;
  int debug;
  uint64_t timeout_ns;

  // Fused GELU + quantization for the next layer (k_linear<..., true>): the next layer's
  // smoothing factors (N of them), global scale and down factor (r2 x N, K-major), its codes
  // (M x N/2), scales (MMA scale order, N/16 a row) and the partial down-projection, one
  // Mpad x r2 float32 slice per 256-column tile of this layer's output.
  const float* inv_s2;
  float gs_x2;
  const uint16_t* L1fT2;
  int r2;
  int Mpad;
  uint8_t* Xq2;
  uint8_t* SFx2;
  float* part;
};

// Both warps of a pair (64 threads, named barrier `id`) agree that `v` holds for both.
SVDQ_DEV bool pair_all(int id, bool v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\tsetp.ne.u32 p, %1, 0;\n\tbar.red.and.pred q, %2, 64, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)v), "r"(id)
      : "memory");
  return r != 0;
}
SVDQ_DEV void pair_sync(int id) { asm volatile("bar.sync %0, 64;" ::"r"(id) : "memory"); }

SVDQ_DEV void ldmatrix_x4(uint32_t (&a)[4], uint32_t saddr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(a[0]), "=r"(a[1]), "=r"(a[2]), "=r"(a[3])
               : "r"(saddr));
}

// D += A (16 x 16 bf16, row) * B (16 x 8 bf16, col), float32 accumulate.
SVDQ_DEV void mma_bf16_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

SVDQ_DEV void sts_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c), "r"(d) : "memory");
}
SVDQ_DEV void sts_v2f(uint32_t addr, float a, float b) {
  asm volatile("st.shared.v2.f32 [%0], {%1, %2};" ::"r"(addr), "f"(a), "f"(b) : "memory");
}
SVDQ_DEV float2 lds_v2f(uint32_t addr) {
  float2 v;
  asm volatile("ld.shared.v2.f32 {%0, %1}, [%2];" : "=f"(v.x), "=f"(v.y) : "r"(addr) : "memory");
  return v;
}

// Epilogue store of one accumulator row: 128 columns from n0, y = f32(gs_x gs_w) acc + bias,
// rounded to bf16 (or kept fp32 in test mode).  16 columns at a time: one 32-byte store of
// bf16 (two of fp32); N % 16 == 0, so a group is either wholly inside the matrix or wholly
// past its end.
SVDQ_DEV void store_y_row(const LinearArgs& a, const uint32_t (&v)[4][32], int row, int n0, float gs) {
#pragma unroll
  for (int i = 0; i < 4; ++i) {
#pragma unroll
    for (int gp = 0; gp < 2; ++gp) {
      const int n = n0 + 32 * i + 16 * gp;
      if (n < a.N) {
        float y[16];
        if (a.y_accum) {
          if (a.y_fp32) {
            const float4* src = reinterpret_cast<const float4*>(static_cast<const float*>(a.Y) + (int64_t)row * a.N + n);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const float4 o = src[e];
              y[4 * e] = __fmaf_rn(gs, __uint_as_float(v[i][16 * gp + 4 * e]), o.x);
              y[4 * e + 1] = __fmaf_rn(gs, __uint_as_float(v[i][16 * gp + 4 * e + 1]), o.y);
              y[4 * e + 2] = __fmaf_rn(gs, __uint_as_float(v[i][16 * gp + 4 * e + 2]), o.z);
              y[4 * e + 3] = __fmaf_rn(gs, __uint_as_float(v[i][16 * gp + 4 * e + 3]), o.w);
            }
          } else {
            const uint4* src = reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(a.Y) + (int64_t)row * a.N + n);
            const uint4 o0 = src[0], o1 = src[1];
            const uint32_t ow[8] = {o0.x, o0.y, o0.z, o0.w, o1.x, o1.y, o1.z, o1.w};
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              y[2 * e] = __fmaf_rn(gs, __uint_as_float(v[i][16 * gp + 2 * e]), bf16_lo(ow[e]));
              y[2 * e + 1] = __fmaf_rn(gs, __uint_as_float(v[i][16 * gp + 2 * e + 1]), bf16_hi(ow[e]));
            }
          }
        } else if (a.bias) {
          const uint4 b0 = __ldg(reinterpret_cast<const uint4*>(a.bias + n));
          const uint4 b1 = __ldg(reinterpret_cast<const uint4*>(a.bias + n + 8));
          const uint32_t bw[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            y[2 * e] = __fmaf_rn(gs, __uint_as_float(v[i][16 * gp + 2 * e]), bf16_lo(bw[e]));
            y[2 * e + 1] = __fmaf_rn(gs, __uint_as_float(v[i][16 * gp + 2 * e + 1]), bf16_hi(bw[e]));
          }
        } else {
#pragma unroll
          for (int e = 0; e < 16; ++e) y[e] = __fmaf_rn(gs, __uint_as_float(v[i][16 * gp + e]), 0.0f);
        }
        if (a.y_fp32) {
          float* dst = static_cast<float*>(a.Y) + (int64_t)row * a.N + n;
          if (a.y_vec32) {
            st_global_v8(dst, __float_as_uint(y[0]), __float_as_uint(y[1]), __float_as_uint(y[2]),
                         __float_as_uint(y[3]), __float_as_uint(y[4]), __float_as_uint(y[5]),
                         __float_as_uint(y[6]), __float_as_uint(y[7]));
            st_global_v8(dst + 8, __float_as_uint(y[8]), __float_as_uint(y[9]), __float_as_uint(y[10]),
                         __float_as_uint(y[11]), __float_as_uint(y[12]), __float_as_uint(y[13]),
                         __float_as_uint(y[14]), __float_as_uint(y[15]));
          } else {
            float4* d4 = reinterpret_cast<float4*>(dst);
#pragma unroll
            for (int e = 0; e < 4; ++e) d4[e] = make_float4(y[4 * e], y[4 * e + 1], y[4 * e + 2], y[4 * e + 3]);
          }
        } else {
          uint32_t o[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) o[e] = pack_bf16x2(y[2 * e], y[2 * e + 1]);
          uint16_t* dst = static_cast<uint16_t*>(a.Y) + (int64_t)row * a.N + n;
          if (a.y_vec32) {
            st_global_v8(dst, o[0], o[1], o[2], o[3], o[4], o[5], o[6], o[7]);
          } else {
            uint4* d4 = reinterpret_cast<uint4*>(dst);
            d4[0] = make_uint4(o[0], o[1], o[2], o[3]);
            d4[1] = make_uint4(o[4], o[5], o[6], o[7]);
          }
        }
      }
    }
  }
}

// MX = true: the MXFP4 form (E8M0 scales per 32 along K, no global scales; K % 128 == 0).  A stage
// of K = 256 then has two scale atoms (four scales of 32 a row each) per 128-row block, and MMA j of
// the stage reads atom j / 2 from byte 2 (j % 2) of its TMEM columns (the scale-factor ID).
// GQ = true: the epilogue does not store Y; it rounds each output to bf16, applies GELU (rounded
// to bf16 again), and quantizes the result as the next layer's activations (NVFP4 codes and
// scales with the next layer's smoothing factors and global scale), and multiplies it by the next
// layer's down factor (mma.sync, bf16 in, float32 out) into one partial slice per output column
// tile.  k_lowrank_finalize sums the slices into the next layer's LAs.
template <bool MX, bool GQ = false>
__global__ void __launch_bounds__(LN_THREADS, 1) k_linear(
    const __grid_constant__ CUtensorMap tm_xq,   // uint8 {K/2, M},  box {128, 128}, SW128
    const __grid_constant__ CUtensorMap tm_wq,   // uint8 {K/2, N},  box {128, 128}, SW128
    const __grid_constant__ CUtensorMap tm_las,  // bf16  {2r, M},   box {64, 128},  SW128
    const __grid_constant__ CUtensorMap tm_l2p,  // bf16  {r, N},    box {32, 128},  SW64
    const LinearArgs args) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + LN_OFF_B;
  uint8_t* sSFA = smem + LN_OFF_SFA;
  uint8_t* sSFB = smem + LN_OFF_SFB;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + LN_OFF_BAR);   // stage's A/B landed
  uint64_t* sf_full = full + LN_STAGES;                               // stage's scale blocks landed
  uint64_t* sf_ready = sf_full + LN_STAGES;                           // stage scales in TMEM
  uint64_t* empty = sf_ready + LN_STAGES;                             // stage consumed by the MMAs
  uint64_t* acc_full = empty + LN_STAGES;
  uint64_t* acc_empty = acc_full + 1;
  uint64_t* drain = acc_empty + 1;                                    // MMA thread, on a time-out
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
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
      mbar_init(&sf_ready[s], 4);                  // one arrival per scale-writer warp
      mbar_init(&empty[s], 1);
    }
    mbar_init(acc_full, 1);
    mbar_init(acc_empty, LN_EPI_WARPS);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (GQ && threadIdx.x < 256) {
    // The next layer's quantizer: rinv = f32(1 / f32(dec(sb) gs2)) for every UE4M3 byte (0 for sb = 0).
    float* rcp = reinterpret_cast<float*>(smem + LN_OFF_RCP);
    const uint32_t sb = threadIdx.x;
    rcp[sb] = sb ? __frcp_rn(__fmul_rn(dec_ue4m3(sb), args.gs_x2)) : 0.0f;
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, LN_TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tmem_slot;
  // Everything above overlaps the previous kernel on the stream when launched as a programmatic
  // dependent; every read of the inputs and every write of Y comes after this wait.
  griddep_wait();
  griddep_launch_dependents();

  // Register split by warpgroup: every warp of a warpgroup executes the same setmaxnreg, at
  // the top of its role so that the role's code is compiled under that budget.
  if (warp == 0 || warp == 2) {
    regs_dec<LN_REGS_LOW>();
    if (!(args.debug & LN_DBG_NO_LOADS)) {
      // --------------------------------------------------------- producers --
      // Warp 0 issues the stage's three tensor boxes (A; B rows 0-127; B rows 128-255),
      // warp 2 its three scale blocks (SFA; SFB 0; SFB 1).  Lane 3g + k serves stream k of
      // ring slot g, so no lane has two copies of the same stream in flight (a thread's
      // copies are serviced one after another).  The three lanes of a stage issue one
      // converged copy instruction with per-lane operands: an issuing warp is held for
      // about the same time by a copy instruction whether one lane or three take part,
      // so three lanes in divergent branches would take three times as long.  Both warps
      // walk the stages in order with warp-uniform waits (lane 0 polls, the verdict is
      // broadcast); lanes waiting on different barriers in divergent branches would block
      // one another inside try_wait.
      const bool tensor_warp = warp == 0;
      const int g = lane / LN_STREAMS, k = lane % LN_STREAMS;   // ring slot, stream
      const bool loader = lane < LN_STAGES * LN_STREAMS;
      if (lane == 0) {
        if (tensor_warp) {
          tma_prefetch_desc(&tm_xq);
          tma_prefetch_desc(&tm_wq);
          if (r > 0) {
            tma_prefetch_desc(&tm_las);
            tma_prefetch_desc(&tm_l2p);
          }
        }
      }
      int gidx = 0;                 // position in this CTA's sequence of ring stages
      bool ok = true, issued = false;
      uint32_t last_parity = 0;
      for (int t = blockIdx.x; t < total && ok; t += gridDim.x) {
        int mb, nb;
        tile_coords(t, num_m, num_n, mb, nb);
        for (int kt = 0; kt < nst; ++kt, ++gidx) {
          const int stage = gidx % LN_STAGES;
          const uint32_t phase = (uint32_t)((gidx / LN_STAGES) & 1);
          int free_slot = 1;
          if (lane == 0) free_slot = mbar_wait_spin(&empty[stage], phase ^ 1u, tmo, abort_flag, 0x301) ? 1 : 0;
          if (!__shfl_sync(0xffffffffu, free_slot, 0)) { ok = false; break; }
          const bool mine = loader && g == stage;
          const unsigned smask = 7u << (LN_STREAMS * stage);   // the stage's three lanes
          const bool lr = kt >= nkt;               // a rank stage: LAs x L2p in bf16
          if (tensor_warp) {
            if (mine) {
              if (k == 0)
                mbar_arrive_expect_tx(&full[stage], (uint32_t)(lr ? LN_LR_BYTES : LN_A_BYTES + LN_B_BYTES));
              const CUtensorMap* map = k == 0 ? (lr ? &tm_las : &tm_xq) : (lr ? &tm_l2p : &tm_wq);
              uint8_t* dst = k == 0 ? sA + stage * LN_A_BYTES
                                    : sB + stage * LN_B_BYTES + (k - 1) * (lr ? LN_LR_B_HALF : LN_B_HALF);
              const int x = (lr ? (kt - nkt) * (k == 0 ? 64 : 32) : kt * 128) +
                            ((args.debug & LN_DBG_MISALIGN) && k == 0 && kt == 0 ? 8 : 0);
              const int y = k == 0 ? mb * LN_BM : nb * LN_BN + (k - 1) * 128;
              __syncwarp(smask);
              const uint32_t box = k == 0 ? (lr ? LN_A_BYTES : LN_A_BYTES) : (lr ? LN_LR_B_HALF : LN_B_HALF);
              if (SVDQ_CHECK_OK((x * (lr ? 2 : 1)) % 16 == 0 && x >= 0 && y >= 0 &&
                                    (uint32_t)(dst - smem_raw) + box <= dyn_smem_bytes(), 0x3c1))
                tma_load_2d(dst, map, &full[stage], x, y);
              issued = true;
              last_parity = phase;
            }
          } else if (mine) {
            // Scale blocks are contiguous runs of ka 512-byte atoms, copied as they are.
            // Blocks past the end of a scale buffer (rows beyond the padded M or N) are not
            // loaded; they only feed accumulator rows or columns that are never stored.
            const int KAs = MX ? (K >> 7) : KA;        // scale atoms a row block holds along K
            const int per = MX ? 2 : 4;                // atoms per stage
            const int ka = lr ? 0 : min(per, KAs - per * kt);
            const int has_a = mb < sfx_blocks, has_b0 = 2 * nb < sfw_blocks, has_b1 = 2 * nb + 1 < sfw_blocks;
            if (k == 0) {
              if (lr) mbar_arrive(&sf_full[stage]);        // no scales in a rank stage
              else mbar_arrive_expect_tx(&sf_full[stage], (uint32_t)((has_a + has_b0 + has_b1) * ka * 512));
            }
            const bool has = !lr && (k == 0 ? has_a : k == 1 ? has_b0 : has_b1);
            __syncwarp(smask);
            if (has) {
              uint8_t* dst = k == 0 ? sSFA + stage * LN_SFA_BYTES : sSFB + stage * LN_SFB_BYTES + 2048 * (k - 1);
              const uint8_t* src = k == 0 ? args.SFx + ((int64_t)mb * KAs + per * kt) * 512
                                          : args.SFw + ((int64_t)(2 * nb + k - 1) * KAs + per * kt) * 512;
              const int64_t blocks = k == 0 ? sfx_blocks : sfw_blocks;
              const int64_t atom = k == 0 ? (int64_t)mb * KAs + per * kt : (int64_t)(2 * nb + k - 1) * KAs + per * kt;
              if (SVDQ_CHECK_OK(ka > 0 && atom + ka <= blocks * KAs && (reinterpret_cast<uintptr_t>(src) & 15u) == 0 &&
                                    (uint32_t)(dst - smem_raw) + ka * 512 <= dyn_smem_bytes(), 0x3c2))
                bulk_load(dst, src, (uint32_t)(ka * 512), &sf_full[stage]);
              issued = true;
              last_parity = phase;
            }
          }
          __syncwarp();
        }
      }
      if (*abort_flag && issued) {
        // Give the last load of this lane's slot the chance to land before the CTA exits.
        int never = 0;
        mbar_wait(tensor_warp ? &full[g] : &sf_full[g], last_parity, tmo, &never, 0x302);
      }
    }
  } else if (warp == 1) {
    // ----------------------------------------------------------- MMA issuer --
    regs_dec<LN_REGS_LOW>();
    if (lane == 0) {
      constexpr uint32_t IDESC_F4 = idesc_nvf4(LN_BM, LN_BN);
      constexpr uint32_t IDESC_MX0 = idesc_mxf4(LN_BM, LN_BN, 0);
      constexpr uint32_t IDESC_MX1 = idesc_mxf4(LN_BM, LN_BN, 2);
      constexpr uint32_t IDESC_BF16 = idesc_bf16(LN_BM, LN_BN);
      int stage = 0;
      uint32_t phase = 0;
      int it = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < total && ok; t += gridDim.x, ++it) {
        if (it > 0 && !mbar_wait_spin(acc_empty, (uint32_t)((it - 1) & 1), tmo, abort_flag, 0x311)) break;
        tc_fence_after();
        for (int kt = 0; kt < nst; ++kt) {
          if (!mbar_wait_spin(&full[stage], phase, tmo, abort_flag, 0x312) ||
              !mbar_wait_spin(&sf_ready[stage], phase, tmo, abort_flag, 0x314)) {
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
            for (int j = 0; j < ka; ++j) {
              if constexpr (MX)
                tc_mma_mxf4(tbase, adesc + 2 * j, bdesc + 2 * j, (j & 1) ? IDESC_MX1 : IDESC_MX0,
                            sfa_col + 4 * (j >> 1), sfb_col + 8 * (j >> 1), (kt | j) != 0 ? 1u : 0u);
              else
                tc_mma_nvf4(tbase, adesc + 2 * j, bdesc + 2 * j, IDESC_F4, sfa_col + 4 * j, sfb_col + 8 * j,
                            (kt | j) != 0 ? 1u : 0u);
            }
          } else {
            // hi and lo of the same 16 low-rank columns meet the same 16 columns of L2p.  (With no
            // K tiles, the rank-only mode, the first rank MMA starts the accumulator.)
            const uint64_t bdesc64 = sdesc_kmajor_sw64(smem_u32(sB + stage * LN_B_BYTES));
#pragma unroll
            for (int j = 0; j < 4; ++j)
              tc_mma_bf16(tbase, adesc + 2 * j, bdesc64 + 2 * (j >> 1), IDESC_BF16, (kt | j) != 0 ? 1u : 0u);
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
  } else if (warp >= LN_SFW_WARP0) {
    // -------------------------------------------------------- scale writers --
    // Warp w writes TMEM lanes 32 (w % 4) .. +31.  Atom j of a 128-row scale block holds
    // row r's 4 scales at byte 16 (r % 32) + 4 ((r / 32) % 4); lane l of every quarter
    // takes the atom's 16 bytes at 16 l into 4 consecutive columns (the replicated layout
    // the block-scaled MMA reads).  SFA atom j -> columns 4j, SFB block b atom j -> 16 + 8j + 4b.
    regs_dec<LN_REGS_LOW>();
    const int q = warp & 3;
    const uint32_t lane_base = tbase + ((uint32_t)(32 * q) << 16);
    int stage = 0;
    uint32_t phase = 0;
    bool ok = true;
    for (int t = blockIdx.x; t < total && ok; t += gridDim.x) {
      for (int kt = 0; kt < nst; ++kt) {
        // The stage's scales landed; the MMAs of the slot's previous round finished before its
        // loads began, so the slot's TMEM columns are free.
        int landed = 1;
        if (lane == 0) landed = mbar_wait(&sf_full[stage], phase, tmo, abort_flag, 0x331) ? 1 : 0;
        if (!__shfl_sync(0xffffffffu, landed, 0)) { ok = false; break; }
        if (kt < nkt) {
          const uint32_t sa = smem_u32(sSFA + stage * LN_SFA_BYTES) + 16 * lane;
          const uint32_t sb = smem_u32(sSFB + stage * LN_SFB_BYTES) + 16 * lane;
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
          const uint32_t col = lane_base + LN_SF_COL0 + LN_SF_COLS_PER_STAGE * stage;
          tmem_st_32x32b_x16(col, a);
          tmem_st_32x32b_x16(col + 16, b0);
          tmem_st_32x32b_x16(col + 32, b1);
          tmem_st_wait();
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sf_ready[stage]);
        if (++stage == LN_STAGES) { stage = 0; phase ^= 1u; }
      }
    }
  } else if (!GQ && warp >= LN_EPI_WARP0) {
    // ------------------------------------------------------------- epilogue --
    regs_inc<LN_REGS_HIGH>();
    const int ew = warp - LN_EPI_WARP0;
    const int q = warp & 3;              // TMEM lane quarter this warp may access
    const int h = ew >> 2;               // column half of the 256-wide tile
    const float gs = args.gs;
    int it = 0;
    for (int t = blockIdx.x; t < total; t += gridDim.x, ++it) {
      int mb, nb;
      tile_coords(t, num_m, num_n, mb, nb);
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
      if (row < M) store_y_row(args, v, row, nb * LN_BN + h * 128, gs);
    }
  } else if (GQ && warp >= LN_EPI_WARP0) {
    // ------------------------------------------- epilogue: GELU + next-layer quantization --
    // Warp (q, h) owns rows 32 q .. +31 of the tile (lane = row) and columns h*128 .. +127.
    regs_inc<LN_REGS_HIGH>();
    const int ew = warp - LN_EPI_WARP0;
    const int q = warp & 3;
    const int h = ew >> 2;
    const int pid = 1 + q;                           // named barrier of the warp pair (q, 0), (q, 1)
    const float gs = args.gs;
    const float gs2 = args.gs_x2;
    const float c_x2 = __frcp_rn(__fmul_rn(6.0f, gs2));
    const int r2 = args.r2;
    const int KS4 = N >> 6;                          // scale words per row of the next layer
    const uint32_t stg = smem_u32(smem + LN_OFF_STG + (2 * q + h) * LN_STG_BYTES);
    const uint32_t pairbuf = smem_u32(smem + LN_OFF_STG + 2 * q * LN_STG_BYTES);
    const uint32_t rcp_tab = smem_u32(smem + LN_OFF_RCP);
    const int gid = lane >> 2, tig = lane & 3;
    int it = 0;
    for (int t = blockIdx.x; t < total; t += gridDim.x, ++it) {
      int mb, nb;
      tile_coords(t, num_m, num_n, mb, nb);
      const bool got = mbar_wait(acc_full, (uint32_t)(it & 1), tmo, abort_flag, 0x321);
      // Both warps of the pair leave together: the named barriers below need both of them.
      if (!pair_all(pid, got)) break;
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
      const int n0 = nb * LN_BN + h * 128;
      // The down-projection's B operand for these 128 columns (r2 rows of L1f2^T, 256 bytes each) into
      // L1 now, so its fragment loads after the GELU hit L1 instead of waiting on L2.
      if (lane < r2) {
        const uint16_t* bl = args.L1fT2 + (int64_t)lane * N + n0;
        asm volatile("prefetch.global.L1 [%0];" ::"l"(bl));
        if (n0 + 64 < N) asm volatile("prefetch.global.L1 [%0];" ::"l"(bl + 64));
      }
      uint32_t p[64];                                // y, then x2 (bf16 pairs): p[8g + j] = columns 16g + 2j, +1
      uint32_t cw[4];                                // codes of two groups of 16 (two words each)
      uint32_t sw[2] = {0u, 0u};                     // scale words (4 groups each)
      // y = f32(gs acc + bias) rounded to bf16, as bf16 pairs (the accumulator registers end here,
      // which leaves room for the GELU of several pairs at a time)
#pragma unroll
      for (int g = 0; g < 8; ++g) {
        const int n = n0 + 16 * g;
        uint32_t bw[8] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};
        if (n < N && args.bias) {                    // warp-uniform; N % 64 == 0
          const uint4 b0 = __ldg(reinterpret_cast<const uint4*>(args.bias + n));
          const uint4 b1 = __ldg(reinterpret_cast<const uint4*>(args.bias + n + 8));
          bw[0] = b0.x; bw[1] = b0.y; bw[2] = b0.z; bw[3] = b0.w;
          bw[4] = b1.x; bw[5] = b1.y; bw[6] = b1.z; bw[7] = b1.w;
        }
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const float y0 = __fmaf_rn(gs, __uint_as_float(v[g >> 1][16 * (g & 1) + 2 * j]), bf16_lo(bw[j]));
          const float y1 = __fmaf_rn(gs, __uint_as_float(v[g >> 1][16 * (g & 1) + 2 * j + 1]), bf16_hi(bw[j]));
          p[8 * g + j] = pack_bf16x2(y0, y1);
        }
      }
#pragma unroll
      for (int g = 0; g < 8; ++g) {
        const int n = n0 + 16 * g;
        const bool valid = n < N;                    // warp-uniform
        // x2 = bf16(GELU(y)), in place
#pragma unroll
        for (int j = 0; j < 8; ++j) p[8 * g + j] = valid ? gelu_bf16x2(p[8 * g + j]) : 0u;
        // NVFP4 of x2 * inv_s2 with the next layer's global scale (the activation kernel's steps):
        // one pass for the group maximum, a second (products recomputed) for the codes.
        const float4* invp = reinterpret_cast<const float4*>(args.inv_s2 + (valid ? n : 0));
        float2 xh[8];
        float a = 0.0f;
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const float4 iv = __ldg(invp + k);
          const uint32_t w0 = p[8 * g + 2 * k], w1 = p[8 * g + 2 * k + 1];
          xh[2 * k] = mul_f32x2(make_float2(bf16_lo(w0), bf16_hi(w0)), make_float2(iv.x, iv.y));
          xh[2 * k + 1] = mul_f32x2(make_float2(bf16_lo(w1), bf16_hi(w1)), make_float2(iv.z, iv.w));
          a = fmaxf(a, fmaxf(fmaxf(fabsf(xh[2 * k].x), fabsf(xh[2 * k].y)),
                             fmaxf(fabsf(xh[2 * k + 1].x), fabsf(xh[2 * k + 1].y))));
        }
        const uint32_t sb = valid ? cvt_ue4m3(__fmul_rn(a, c_x2)) : 0u;
        const float rinv = lds_f32(rcp_tab + 4 * sb);
        const float2 rr = make_float2(rinv, rinv);
#pragma unroll
        for (int hb = 0; hb < 2; ++hb) {
          float qv[8];
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const float2 q2 = mul_f32x2(xh[4 * hb + i], rr);
            qv[2 * i] = q2.x;
            qv[2 * i + 1] = q2.y;
          }
          cw[2 * (g & 1) + hb] = sb ? cvt_e2m1x8(qv) : 0u;
        }
        if ((g & 1) && row < M && n0 + 16 * (g - 1) < N)    // codes of groups g-1, g: 16 bytes
          reinterpret_cast<uint4*>(args.Xq2 + (int64_t)row * (N >> 1) + (n0 >> 1))[g >> 1] =
              make_uint4(cw[0], cw[1], cw[2], cw[3]);
        sw[g >> 2] |= sb << (8 * (g & 3));
      }
#pragma unroll
      for (int kw = 0; kw < 2; ++kw)          // padding rows (M .. Mpad) hold zero scales
        if (n0 + 64 * kw < N)
          *reinterpret_cast<uint32_t*>(args.SFx2 + sf_word_offset((uint32_t)row, (uint32_t)((n0 >> 6) + kw),
                                                                  (uint32_t)KS4)) = row < M ? sw[kw] : 0u;

      if (r2 > 0) {
        // Partial down-projection of the next layer over this warp's 128 columns:
        // D[row][t] = sum_c x2[row][c] L1f2[n0 + c][t], 16 columns (one k step) per slab.
        float acc2[2][LN_GQ_MAX_R / 8][4];
#pragma unroll
        for (int mi = 0; mi < 2; ++mi)
#pragma unroll
          for (int ni = 0; ni < LN_GQ_MAX_R / 8; ++ni)
#pragma unroll
            for (int e = 0; e < 4; ++e) acc2[mi][ni][e] = 0.0f;
#pragma unroll
        for (int sl = 0; sl < 8; ++sl) {
          const int kc = n0 + 16 * sl;
          if (kc < N) {                          // warp-uniform
            // Stage the slab (32 rows x 32 bytes; 16-byte chunk c of row L at chunk c ^ ((L >> 2) & 1),
            // so that 8 consecutive rows of one chunk fall in 8 different bank groups).
            __syncwarp();
            const uint32_t sw_l = (uint32_t)((lane >> 2) & 1);
            sts_v4(stg + lane * 32 + ((0u ^ sw_l) << 4), p[8 * sl], p[8 * sl + 1], p[8 * sl + 2], p[8 * sl + 3]);
            sts_v4(stg + lane * 32 + ((1u ^ sw_l) << 4), p[8 * sl + 4], p[8 * sl + 5], p[8 * sl + 6], p[8 * sl + 7]);
            __syncwarp();
            uint32_t afr[2][4];
#pragma unroll
            for (int mi = 0; mi < 2; ++mi) {
              const int j = lane >> 3;
              const uint32_t rr = (uint32_t)(16 * mi + (j & 1) * 8 + (lane & 7));
              const uint32_t c = (uint32_t)(j >> 1);
              ldmatrix_x4(afr[mi], stg + rr * 32 + ((c ^ ((rr >> 2) & 1u)) << 4));
            }
#pragma unroll
            for (int ni = 0; ni < LN_GQ_MAX_R / 8; ++ni) {
              if (8 * ni < r2) {
                const uint16_t* bp = args.L1fT2 + (int64_t)(8 * ni + gid) * N + kc + 2 * tig;
                const uint32_t b0 = __ldg(reinterpret_cast<const unsigned int*>(bp));
                const uint32_t b1 = __ldg(reinterpret_cast<const unsigned int*>(bp + 8));
#pragma unroll
                for (int mi = 0; mi < 2; ++mi) mma_bf16_16816(acc2[mi][ni], afr[mi], b0, b1);
              }
            }
          }
        }
        // Pair hand-off, 16 columns of r2 at a time through the pair's 2 KB: warp h = 1 writes its
        // sums, warp h = 0 adds them to its own (own + other: a fixed order) and stores the slice.
#pragma unroll
        for (int rh = 0; rh < LN_GQ_MAX_R / 16; ++rh) {
          if (16 * rh < r2) {
            pair_sync(pid);
            if (h == 1) {
#pragma unroll
              for (int mi = 0; mi < 2; ++mi)
#pragma unroll
                for (int nj = 0; nj < 2; ++nj) {
                  const uint32_t rr = (uint32_t)(16 * mi + gid), cc = (uint32_t)(8 * nj + 2 * tig);
                  const float(&d)[4] = acc2[mi][2 * rh + nj];
                  sts_v2f(pairbuf + (rr * 16 + cc) * 4, d[0], d[1]);
                  sts_v2f(pairbuf + ((rr + 8) * 16 + cc) * 4, d[2], d[3]);
                }
            }
            pair_sync(pid);
            if (h == 0) {
#pragma unroll
              for (int mi = 0; mi < 2; ++mi)
#pragma unroll
                for (int nj = 0; nj < 2; ++nj) {
                  const int rr = 16 * mi + gid, cc = 8 * nj + 2 * tig;
                  const float(&d)[4] = acc2[mi][2 * rh + nj];
                  const float2 o0 = lds_v2f(pairbuf + (uint32_t)(rr * 16 + cc) * 4);
                  const float2 o1 = lds_v2f(pairbuf + (uint32_t)((rr + 8) * 16 + cc) * 4);
                  const int64_t base = ((int64_t)nb * args.Mpad + mb * LN_BM + 32 * q) * r2 + 16 * rh + cc;
                  *reinterpret_cast<float2*>(args.part + base + (int64_t)rr * r2) =
                      make_float2(__fadd_rn(d[0], o0.x), __fadd_rn(d[1], o0.y));
                  *reinterpret_cast<float2*>(args.part + base + (int64_t)(rr + 8) * r2) =
                      make_float2(__fadd_rn(d[2], o1.x), __fadd_rn(d[3], o1.y));
                }
            }
          }
        }
      }
    }
  } else {
    regs_dec<LN_REGS_LOW>();                       // warp 3: no role
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tbase, LN_TMEM_COLS);
  }
}

}  // namespace svdq
