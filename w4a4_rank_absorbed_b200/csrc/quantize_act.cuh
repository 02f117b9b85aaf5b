// Kernel 2: activation quantization fused with the low-rank down-projection.
//
// SVDQuant review, §4.3 (Nunchaku): the down-projection is merged into the
// quantization kernel, so the 16-bit activations are read from HBM once and
// shared by both branches.  Per element x_hat = f32(x * inv_s) (the smoothing
// divide, "From SmoothQuant to SVDQuant", section Smooth Quant (W8A8)); per
// group of 16 along K the NVFP4 codec of SVDQuant review §3 (q_max = 6) with a
// UE4M3 block scale; the down-projection LA = X L1f (L1f = diag(s)^-1 L1, so
// X L1f = X_hat L1) on the tcgen05 tensor cores (bf16 in, fp32 accumulate in
// TMEM), pre-scaled by lr_scale and split into bf16 hi/lo halves.
//
// Work split: a CTA owns 128 rows and a contiguous range of the K axis; `split`
// CTAs share a row block (split = 1 when there are enough row blocks to fill
// the GPU).  The K axis is read in stages of two 64-column chunks through an
// S-stage ring: one 3-D TMA box (dims: 64 columns, rows, K/64 chunks) brings
// both chunks of all 128 rows, landing as two 128-byte-swizzled 128-row tiles
// (the reads are 256 contiguous bytes a row, which streams from HBM faster than
// 128-byte pieces), and one more box the matching r x 64 L1f^T tiles.  A copy
// instruction holds its warp for a few hundred nanoseconds, so each stream has
// a producer warp of its own and a stage takes one instruction per stream; the
// smoothing factors (a few KB, L1-resident) are read by the quantizers
// directly.  Roles (19 warps):
//   warp 0      X producer, warp 18 L1f^T producer (one lane each).
//   warp 1      TMEM owner and MMA issuer (one thread): per stage eight
//               tcgen05.mma.kind::f16 of 128 x r x 16 (A = an X tile, B = the
//               chunk's L1f^T tile) into one fp32 accumulator of r TMEM columns;
//               each stage's commit is one of the arrivals that frees it.
//   warps 2-17  quantizers: thread i takes group i % 4 of chunk (i / 8) % 2 of
//               the stage for rows 2 (i / 16) + (i / 4) % 2 and that row + 64: two
//               independent groups of 16 values (two chains of work in flight)
//               that share their 16 smoothing factors.  A quarter-warp so reads
//               rows r and r ^ 1 of one chunk, whose 128-byte swizzle patterns
//               are complementary: its eight 16-byte reads hit eight different
//               bank groups.  Each group gives 8 bytes of codes and, gathered
//               over the four lanes of a row and chunk, one 32-bit word of scales.
// After the last stage, four of the quantizer warps (one per TMEM lane quarter)
// read the accumulator.  With split = 1 it goes through shared memory straight
// to LAs.  Otherwise each CTA writes its partial sums to the caller's workspace
// and takes a ticket for its row block; the CTA that takes the last ticket adds
// the `split` partials in rank order (the result does not depend on which CTA
// finishes last) and resets the ticket to 0 for the next call.  LAs holds the
// hi/lo pair of lr_scale * (X L1f), interleaved by 16 columns (hi of columns
// 16j..16j+15 at 32j, their lo at 32j + 16), the order the GEMM's rank stage
// reads.
//
// With QUANT = false the same kernel is the separate down-projection of the
// unfused pipeline (the quantizer warps only release the stages).
#pragma once
#include "common.cuh"

namespace svdq {

constexpr int QB_ROWS = 128;
constexpr int QB_CHUNK = 64;                 // bf16 columns per chunk (128 bytes)
constexpr int QB_QWARPS = 16;
constexpr int QB_WARP_Q0 = 2;                // first quantizer warp
constexpr int QB_WARP_L1 = QB_WARP_Q0 + QB_QWARPS;   // producer of the L1f^T tiles
constexpr int QB_THREADS = (QB_WARP_L1 + 1) * 32;
constexpr int QB_MAX_SPLIT = 8;                // power of two: 128 rows / split, ticket arithmetic
constexpr int QB_RING_BYTES = 200 * 1024;
constexpr int QB_MAX_STAGES = 12;

template <int R>
struct QbCfg {
  static constexpr int kChunks = 2;                              // 64-column chunks per stage
  static constexpr int kXTile = QB_ROWS * 128;                   // one chunk of 128 rows
  static constexpr int kLTile = R * 128;                         // one chunk of L1f^T
  static constexpr int kXBytes = kChunks * kXTile;
  static constexpr int kLBytes = kChunks * kLTile;
  static constexpr int kStageBytes = kXBytes + kLBytes;
  static constexpr int kStages = QB_RING_BYTES / kStageBytes < QB_MAX_STAGES ? QB_RING_BYTES / kStageBytes
                                                                             : QB_MAX_STAGES;
  static constexpr int kRingBytes = kStages * kStageBytes;
  static_assert(QB_ROWS * R * 4 + 16 <= kRingBytes, "the reduction buffer and last-CTA flag reuse the ring");
  static_assert(kStages >= 2, "ring");
  static constexpr int kRcpOff = kRingBytes;                // 128-entry 1/d table
  static constexpr int kBarOff = kRcpOff + 128 * 4;
  static constexpr int kSmem = kBarOff + (2 * kStages + 2) * 8 + 16 + 1024;
  static constexpr int kTmemCols = R <= 32 ? 32 : R <= 64 ? 64 : 128;
};

// Byte offset of 16-byte chunk `c16` of row `row` in a 128-byte-swizzled tile.
SVDQ_DEV uint32_t sw128(uint32_t row, uint32_t c16) { return row * 128u + ((c16 ^ (row & 7u)) << 4); }

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

// MXFP4: one half (16 values) of a block of 32 held by this lane and its partner (lane ^ 1): the
// smoothing multiply, the block maximum over both halves, the E8M0 scale and the two code words.
// Every lane of the warp must call it (it shuffles).
SVDQ_DEV uint32_t quant_half_mx(const uint4& r0, const uint4& r1, const float4 (&inv)[4], uint32_t& w0,
                                uint32_t& w1) {
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
  a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, 1));
  float mul;
  const uint32_t sb = mx_scale(a, mul);
  const float2 mm = make_float2(mul, mul);
  float q0[8], q1[8];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 p0 = mul_f32x2(xh[i], mm);
    const float2 p1 = mul_f32x2(xh[4 + i], mm);
    q0[2 * i] = p0.x; q0[2 * i + 1] = p0.y;
    q1[2 * i] = p1.x; q1[2 * i + 1] = p1.y;
  }
  w0 = a > 0.0f ? cvt_e2m1x8(q0) : 0u;     // an all-zero block: codes 0
  w1 = a > 0.0f ? cvt_e2m1x8(q1) : 0u;
  return sb;
}

// Warp-uniform bounded wait: lane 0 polls, the verdict is broadcast.
SVDQ_DEV bool warp_wait(uint64_t* bar, uint32_t parity, uint64_t timeout_ns, volatile int* abort, unsigned site) {
  int ok = 1;
  if ((threadIdx.x & 31) == 0) ok = mbar_wait(bar, parity, timeout_ns, abort, site) ? 1 : 0;
  return __shfl_sync(0xffffffffu, ok, 0) != 0;
}

// MX = true: the MXFP4 format (blocks of 32 with an E8M0 scale, no global scale; K % 128 == 0, so a
// stage always holds two chunks): scale bytes follow the same MMA order with K/32 scales a row.
template <int R, bool QUANT, bool MX = false>
__global__ void __launch_bounds__(QB_THREADS, 1) k_quantize_act(
    const __grid_constant__ CUtensorMap tm_x,   // bf16 {64, M, K/64} (strides 2K, 128 bytes), box {64, 128, 2}, SW128
    const __grid_constant__ CUtensorMap tm_l1,  // bf16 {64, R, K/64} (strides 2K, 128 bytes), box {64, R, 2}, SW128
    const __grid_constant__ CUtensorMap tm_x1,  // bf16 {K, M}, box {64, 128}, SW128: a lone last chunk
    const __grid_constant__ CUtensorMap tm_l11, // bf16 {K, R}, box {64, R}, SW128: a lone last chunk
    const float* __restrict__ inv_s, float gs_x, float lr_scale, int M, int K, int Mpad, int split,
    uint8_t* __restrict__ Xq, uint8_t* __restrict__ SFx, uint16_t* __restrict__ LAs,
    float* __restrict__ ws_part,            // split > 1: [split][Mpad][R] partial sums
    unsigned int* __restrict__ ws_ticket,   // split > 1: one counter per row block, 0 between calls
    uint64_t timeout_ns) {
  using Cfg = QbCfg<R>;
  constexpr int S = Cfg::kStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  float* s_rcp = reinterpret_cast<float*>(smem + Cfg::kRcpOff);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + Cfg::kBarOff);
  uint64_t* empty = full + S;              // quantizer warps done and (r > 0) the chunk's MMAs complete
  uint64_t* acc_full = empty + S;          // every MMA of this CTA complete
  uint64_t* drain = acc_full + 1;          // MMA thread, on a time-out
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int rank = (int)(blockIdx.x % (unsigned)split);   // position of this CTA in its row block
  const int rb = (int)(blockIdx.x / (unsigned)split);
  const int m0 = rb * QB_ROWS;
  const int nch = K / QB_CHUNK;
  const int nunits = (nch + 1) >> 1;                          // stages of two chunks (the last may hold one)
  const int u_begin = rank * nunits / split;
  const int my = (rank + 1) * nunits / split - u_begin;       // stages of this CTA (>= 1)
  const uint64_t tmo = timeout_ns;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], R > 0 ? 2 : 1);      // one expect-tx arrival per producer
      mbar_init(&empty[s], QB_QWARPS + (R > 0 ? 1 : 0));
    }
    mbar_init(acc_full, 1);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  // 1/d for every possible block scale: d = f32(dec(sb) * gs_x), same operations as the per-group path.
  if (threadIdx.x < 128) {
    const uint32_t sb = threadIdx.x;
    s_rcp[sb] = sb == 0 ? 0.0f : __frcp_rn(__fmul_rn(dec_ue4m3(sb), gs_x));
  }
  if constexpr (R > 0) {
    if (warp == 1) {
      tmem_alloc(tmem_slot, Cfg::kTmemCols);
      tmem_relinquish();
    }
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tm_x);
    tma_prefetch_desc(&tm_x1);
    if (R > 0) {
      tma_prefetch_desc(&tm_l1);
      tma_prefetch_desc(&tm_l11);
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = R > 0 ? *tmem_slot : 0u;
  // X may be the previous kernel's output: read nothing before it has finished.
  griddep_wait();
  griddep_launch_dependents();

  if (warp == 0 || warp == QB_WARP_L1) {
    // ------------------------------------------------------------ producers --
    // Warp 0 fetches the X tiles, warp 18 the L1f^T tiles (r > 0), each with one lane.  With an odd
    // number of chunks the last stage holds one: it is fetched with the 2-D maps, so no copy reaches
    // past the last chunk of K.
    const bool xw = warp == 0;
    if (lane == 0 && (xw || R > 0)) {
      int issued = 0;
      bool ok = true;
      for (int i = 0; i < my; ++i) {
        const int s = i % S;
        if (i >= S && !mbar_wait_spin(&empty[s], (uint32_t)(((i / S) - 1) & 1), tmo, abort_flag, 0x201)) {
          ok = false;
          break;
        }
        uint8_t* st = smem + s * Cfg::kStageBytes;
        const int c = 2 * (u_begin + i);                       // first chunk of the stage
        const bool pair = c + 1 < nch;
        const bool fits = SVDQ_CHECK_OK(c >= 0 && c < nch && m0 >= 0 && m0 < Mpad &&
                                            (uint32_t)(st - smem_raw) + Cfg::kStageBytes <= dyn_smem_bytes(), 0x2c1);
        if (xw) {
          mbar_arrive_expect_tx(&full[s], (uint32_t)((pair ? 2 : 1) * Cfg::kXTile));
          if (fits && pair) tma_load_3d(st, &tm_x, &full[s], 0, m0, c);
          else if (fits) tma_load_2d(st, &tm_x1, &full[s], c * QB_CHUNK, m0);
        } else {
          mbar_arrive_expect_tx(&full[s], (uint32_t)((pair ? 2 : 1) * Cfg::kLTile));
          if (fits && pair) tma_load_3d(st + Cfg::kXBytes, &tm_l1, &full[s], 0, 0, c);
          else if (fits) tma_load_2d(st + Cfg::kXBytes, &tm_l11, &full[s], c * QB_CHUNK, 0);
        }
        issued = i + 1;
      }
      if (!ok) {
        // Let the copies that were issued but not consumed land before the CTA exits.
        int never = 0;
        for (int i = issued > S ? issued - S : 0; i < issued; ++i)
          mbar_wait(&full[i % S], (uint32_t)((i / S) & 1), tmo, &never, 0x203);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer --
    if constexpr (R > 0) {
      if (lane == 0) {
        constexpr uint32_t IDESC = idesc_bf16(QB_ROWS, R);
        bool ok = true;
        for (int i = 0; i < my; ++i) {
          const int s = i % S;
          if (!mbar_wait_spin(&full[s], (uint32_t)((i / S) & 1), tmo, abort_flag, 0x211)) {
            ok = false;
            break;
          }
          tc_fence_after();
          uint8_t* st = smem + s * Cfg::kStageBytes;
          const int nc = 2 * (u_begin + i) + 1 < nch ? 2 : 1;     // a lone last chunk: one tile
#pragma unroll
          for (int cc = 0; cc < Cfg::kChunks; ++cc) {
            if (cc >= nc) break;
            const uint64_t adesc = sdesc_kmajor_sw128(smem_u32(st + cc * Cfg::kXTile));
            const uint64_t bdesc = sdesc_kmajor_sw128(smem_u32(st + Cfg::kXBytes + cc * Cfg::kLTile));
#pragma unroll
            for (int j = 0; j < 4; ++j)
              tc_mma_bf16(tbase, adesc + 2 * j, bdesc + 2 * j, IDESC, (i | cc | j) != 0 ? 1u : 0u);
          }
          tc_commit(&empty[s]);
        }
        if (ok) {
          tc_commit(acc_full);
          // The ring becomes the reduction buffer: the MMAs must have finished reading it.
          ok = mbar_wait(acc_full, 0, tmo, abort_flag, 0x212);
        }
        if (!ok || *abort_flag) {
          int never = 0;
          tc_commit(drain);
          mbar_wait(drain, 0, tmo, &never, 0x213);
        }
      }
    }
  } else {
    // ------------------------------------------------------------ quantizers --
    const int qi = threadIdx.x - QB_WARP_Q0 * 32;
    const int g = qi & 3;                    // group of 16 within the chunk
    const int cc = (qi >> 3) & 1;            // chunk within the stage
    const int rr = 2 * (qi >> 4) + ((qi >> 2) & 1);   // rows rr and rr + 64
    const float c_x = __frcp_rn(__fmul_rn(6.0f, gs_x));
    const uint32_t KS4 = (uint32_t)(K >> 6);
    const uint32_t rcp_u32 = smem_u32(s_rcp);
    for (int i = 0; i < my; ++i) {
      const int s = i % S;
      if (!warp_wait(&full[s], (uint32_t)((i / S) & 1), tmo, abort_flag, 0x202)) break;
      const int c = 2 * (u_begin + i) + cc;
      if constexpr (QUANT) {
        // Every lane runs the group math and the shuffles (they take the whole warp); a lane whose chunk
        // lies past K (the lone last chunk's partner, never loaded) only skips its stores.
        const bool valid = c < nch;
        {
          const uint32_t st_u32 = smem_u32(smem + s * Cfg::kStageBytes);
          const uint32_t x_u32 = st_u32 + cc * Cfg::kXTile;
          // the group's 16 smoothing factors (a lane past K reads the last chunk's, never used)
          const float4* invg =
              reinterpret_cast<const float4*>(inv_s + (int64_t)(valid ? c : nch - 1) * QB_CHUNK + 16 * g);
          float4 inv[4];
#pragma unroll
          for (int j = 0; j < 4; ++j) inv[j] = __ldg(invg + j);
          uint4 a0 = lds_v4(x_u32 + sw128(rr, 2 * g)), a1 = lds_v4(x_u32 + sw128(rr, 2 * g + 1));
          uint4 b0 = lds_v4(x_u32 + sw128(rr + 64, 2 * g)), b1 = lds_v4(x_u32 + sw128(rr + 64, 2 * g + 1));
          uint32_t wa0, wa1, wb0, wb1, sa, sb;
          if constexpr (MX) {
            // the block (g / 2) of 32 spans lanes g and g ^ 1; its byte is at 2 * cc + g / 2 of the row's
            // word for the stage (four E8M0 scales: two chunks, two blocks each)
            // (every lane runs quant_half_mx: it shuffles with the partner lane)
            const int sh = 8 * (2 * cc + (g >> 1));
            const uint32_t ta = quant_half_mx(a0, a1, inv, wa0, wa1);
            const uint32_t tb = quant_half_mx(b0, b1, inv, wb0, wb1);
            sa = (g & 1) ? 0u : ta << sh;
            sb = (g & 1) ? 0u : tb << sh;
            sa |= __shfl_xor_sync(0xffffffffu, sa, 2);
            sb |= __shfl_xor_sync(0xffffffffu, sb, 2);
            sa |= __shfl_xor_sync(0xffffffffu, sa, 8);
            sb |= __shfl_xor_sync(0xffffffffu, sb, 8);
          } else {
            sa = quant_group(a0, a1, inv, c_x, rcp_u32, wa0, wa1) << (8 * g);
            sb = quant_group(b0, b1, inv, c_x, rcp_u32, wb0, wb1) << (8 * g);
            sa |= __shfl_xor_sync(0xffffffffu, sa, 1);
            sb |= __shfl_xor_sync(0xffffffffu, sb, 1);
            sa |= __shfl_xor_sync(0xffffffffu, sa, 2);
            sb |= __shfl_xor_sync(0xffffffffu, sb, 2);
          }
          const int ma = m0 + rr, mb = m0 + rr + 64;
          if (valid && ma < M)
            *reinterpret_cast<uint2*>(Xq + (int64_t)ma * (K >> 1) + c * 32 + 8 * g) = make_uint2(wa0, wa1);
          if (valid && mb < M)
            *reinterpret_cast<uint2*>(Xq + (int64_t)mb * (K >> 1) + c * 32 + 8 * g) = make_uint2(wb0, wb1);
          if constexpr (MX) {
            if (valid && g == 0 && cc == 0) {
              const uint32_t u = (uint32_t)(c >> 1), KW = (uint32_t)(K >> 7);
              if (ma < Mpad) *reinterpret_cast<uint32_t*>(SFx + sf_word_offset((uint32_t)ma, u, KW)) = sa;
              if (mb < Mpad) *reinterpret_cast<uint32_t*>(SFx + sf_word_offset((uint32_t)mb, u, KW)) = sb;
            }
          } else if (valid && g == 0) {
            if (ma < Mpad) *reinterpret_cast<uint32_t*>(SFx + sf_word_offset((uint32_t)ma, (uint32_t)c, KS4)) = sa;
            if (mb < Mpad) *reinterpret_cast<uint32_t*>(SFx + sf_word_offset((uint32_t)mb, (uint32_t)c, KS4)) = sb;
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[s]);
    }
  }

  // ---- LAs = hi/lo of lr_scale * (sum over the row block's CTAs of the partial X L1f) ----
  if constexpr (R > 0) {
    // Every chunk has been consumed and every MMA has finished (or the CTA gave up), so the ring
    // is idle: with split = 1 it holds the accumulator rows, red[row][R].
    tc_fence_before();
    __syncthreads();
    float* red = reinterpret_cast<float*>(smem);
    volatile int* s_last = reinterpret_cast<volatile int*>(smem + QB_ROWS * R * 4);
    if (warp >= QB_WARP_Q0 && warp < QB_WARP_Q0 + 4) {
      const int q = warp & 3;                // TMEM lane quarter of this warp
      if (warp_wait(acc_full, 0, tmo, abort_flag, 0x221)) {
        tc_fence_after();
        const int row = 32 * q + lane;
        float* dst = split > 1 ? ws_part + ((size_t)rank * Mpad + m0 + row) * R : red + (size_t)row * R;
#pragma unroll
        for (int cc = 0; cc < R / 16; ++cc) {
          uint32_t v[16];
          tmem_ld_32x32b_x16(tbase + ((uint32_t)(32 * q) << 16) + 16 * cc, v);
          tmem_ld_wait();
          reg_fence16(v);
#pragma unroll
          for (int e = 0; e < 4; ++e)
            reinterpret_cast<uint4*>(dst + 16 * cc)[e] = make_uint4(v[4 * e], v[4 * e + 1], v[4 * e + 2], v[4 * e + 3]);
        }
      }
    }
    tc_fence_before();
    if (split > 1) {
      // Publish this CTA's partial, then take a ticket; the CTA that takes the last one reduces.  The
      // barrier orders every thread's partial-sum stores before thread 0's device-scope fence, which
      // then orders them before the ticket (a release by one thread, not a fence in every thread).
      __syncthreads();
      if (threadIdx.x == 0) {
        __threadfence();
        const unsigned old = atomicAdd(&ws_ticket[rb], 1u);
        const int last = (old % (unsigned)split) == (unsigned)split - 1u;
        if (last) {
          atomicExch(&ws_ticket[rb], 0u);
          __threadfence();        // acquire: the other CTAs' partials before this CTA's reads of them
        }
        *s_last = last;
      }
      __syncthreads();
    } else {
      __syncthreads();
    }
    if (!*abort_flag && (split == 1 || *s_last)) {
      // Four consecutive columns an item, two items a thread at once: with split > 1 every source's
      // partial of both items is loaded before any is added (one round of loads in flight), then the
      // sources are added in rank order.
      constexpr int kItems = QB_ROWS * (R / 4);
      for (int p0 = threadIdx.x; p0 < kItems; p0 += 2 * QB_THREADS) {
        float4 v[2];
        if (split == 1) {
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const int p = p0 + h * QB_THREADS;
            if (p < kItems) v[h] = *reinterpret_cast<const float4*>(red + (size_t)(p / (R / 4)) * R + 4 * (p % (R / 4)));
          }
        } else {
          float4 t[2][QB_MAX_SPLIT];
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const int p = p0 + h * QB_THREADS;
            if (p < kItems) {
              const float* src0 = ws_part + ((size_t)m0 + p / (R / 4)) * R + 4 * (p % (R / 4));
#pragma unroll
              for (int src = 0; src < QB_MAX_SPLIT; ++src)
                if (src < split) t[h][src] = __ldcg(reinterpret_cast<const float4*>(src0 + (size_t)src * Mpad * R));
            }
          }
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            v[h] = t[h][0];
#pragma unroll
            for (int src = 1; src < QB_MAX_SPLIT; ++src)
              if (src < split) {
                v[h].x += t[h][src].x;
                v[h].y += t[h][src].y;
                v[h].z += t[h][src].z;
                v[h].w += t[h][src].w;
              }
          }
        }
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int p = p0 + h * QB_THREADS;
          if (p >= kItems) continue;
          const int row = p / (R / 4);
          const int col = 4 * (p % (R / 4));
          const int mm = m0 + row;
          if (mm < M) {
            const float v4[4] = {__fmul_rn(v[h].x, lr_scale), __fmul_rn(v[h].y, lr_scale),
                                 __fmul_rn(v[h].z, lr_scale), __fmul_rn(v[h].w, lr_scale)};
            float hh[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) hh[e] = __bfloat162float(__float2bfloat16_rn(v4[e]));
            uint16_t* d = LAs + (int64_t)mm * (2 * R) + 32 * (col >> 4) + (col & 15);
            *reinterpret_cast<uint2*>(d) = make_uint2(pack_bf16x2(hh[0], hh[1]), pack_bf16x2(hh[2], hh[3]));
            *reinterpret_cast<uint2*>(d + 16) =
                make_uint2(pack_bf16x2(v4[0] - hh[0], v4[1] - hh[1]), pack_bf16x2(v4[2] - hh[2], v4[3] - hh[3]));
          }
        }
      }
    }
    if (warp == 1) {
      tc_fence_after();
      tmem_dealloc(tbase, Cfg::kTmemCols);
    }
  }
}

}  // namespace svdq
