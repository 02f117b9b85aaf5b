// C ABI of the SVDQuant W4A4 linear layer (declared in include/svdq.h):
// argument checks, TMA descriptor encoding and kernel launches.
// All kernels live in this one translation unit so they share one device
// error word.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>
#include <utility>

#include "../../include/svdq.h"
#include "common.cuh"
#include "calib.cuh"
#include "linear.cuh"
#include "pack_weight.cuh"
#include "quantize_act.cuh"

namespace {

using namespace svdq;

constexpr int kMaxDevices = 64;

// ----------------------------------------------------------- device info ----
struct DevInfo {
  bool init = false;
  bool ok = false;
  int sms = 0;
  bool linear_attr[3] = {};     // [NVFP4, MXFP4, NVFP4 with the GELU + next-layer quantization epilogue]
  bool qa_attr[3][9] = {};      // [NVFP4 quantize, down-projection only, MXFP4 quantize][r / 16]
};
DevInfo g_dev[kMaxDevices];
std::mutex g_mu;

svdq_status current_device(int* dev_out, DevInfo** info) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return SVDQ_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return SVDQ_ERR_DEVICE;
  std::lock_guard<std::mutex> lk(g_mu);
  DevInfo& d = g_dev[dev];
  if (!d.init) {
    int major = 0, minor = 0, sms = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return SVDQ_ERR_CUDA;
    d.ok = (major == 10 && minor == 0);
    d.sms = sms;
    d.init = true;
  }
  if (!d.ok) return SVDQ_ERR_DEVICE;
  *dev_out = dev;
  *info = &d;
  return SVDQ_OK;
}

// ------------------------------------------------------------ TMA maps ------
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// 2-D row-major tensor (rows x inner elements, row pitch in bytes), box (box_inner x box_rows),
// 128-byte swizzle unless stated.
// Tensor maps are cached on the host: a call on the same buffers with the same shapes (every forward
// pass of a layer) reuses the encoded map instead of encoding it again.  A map holds only the
// address, the shape and the box, so a cached entry stays valid for any later buffer at the same
// address with the same shape.  64 entries, least recently used replaced, one mutex.
struct MapKey {
  const void* base;
  uint32_t dt, rank, swizzle;
  uint64_t dims[3], strides[2];
  uint32_t box[3];
  bool operator==(const MapKey& o) const {
    return base == o.base && dt == o.dt && rank == o.rank && swizzle == o.swizzle &&
           std::memcmp(dims, o.dims, sizeof(dims)) == 0 && std::memcmp(strides, o.strides, sizeof(strides)) == 0 &&
           std::memcmp(box, o.box, sizeof(box)) == 0;
  }
};
struct MapEntry {
  MapKey key;
  CUtensorMap map;
  uint64_t stamp = 0;
  bool used = false;
};
constexpr int kMapCacheEntries = 64;
MapEntry g_maps[kMapCacheEntries];
uint64_t g_map_clock = 0;
uint64_t g_map_hits = 0, g_map_misses = 0;
std::mutex g_map_mu;

bool encode_map(const MapKey& k, CUtensorMap* m) {
  {
    std::lock_guard<std::mutex> lk(g_map_mu);
    for (MapEntry& e : g_maps)
      if (e.used && e.key == k) {
        e.stamp = ++g_map_clock;
        *m = e.map;
        ++g_map_hits;
        return true;
      }
  }
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {k.dims[0], k.dims[1], k.dims[2]};
  cuuint64_t strides[2] = {k.strides[0], k.strides[1]};
  cuuint32_t box[3] = {k.box[0], k.box[1], k.box[2]};
  cuuint32_t estr[3] = {1, 1, 1};
  if (fn(m, (CUtensorMapDataType)k.dt, k.rank, const_cast<void*>(k.base), dims, strides, box, estr,
         CU_TENSOR_MAP_INTERLEAVE_NONE, (CUtensorMapSwizzle)k.swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return false;
  std::lock_guard<std::mutex> lk(g_map_mu);
  MapEntry* victim = &g_maps[0];
  for (MapEntry& e : g_maps) {
    if (!e.used) {
      victim = &e;
      break;
    }
    if (e.stamp < victim->stamp) victim = &e;
  }
  victim->key = k;
  victim->map = *m;
  victim->stamp = ++g_map_clock;
  victim->used = true;
  ++g_map_misses;
  return true;
}

bool make_map_2d(CUtensorMap* m, CUtensorMapDataType dt, const void* base, uint64_t inner, uint64_t rows,
                 uint64_t pitch_bytes, uint32_t box_inner, uint32_t box_rows,
                 CUtensorMapSwizzle swizzle = CU_TENSOR_MAP_SWIZZLE_128B) {
  MapKey k{};
  k.base = base;
  k.dt = (uint32_t)dt;
  k.rank = 2;
  k.swizzle = (uint32_t)swizzle;
  k.dims[0] = inner;
  k.dims[1] = rows;
  k.strides[0] = pitch_bytes;
  k.box[0] = box_inner;
  k.box[1] = box_rows;
  return encode_map(k, m);
}

// The rows x K bf16 matrix at `base` as a 3-D tensor {64 columns, rows, K/64 chunks} (strides 2K and
// 128 bytes), box {64, box_rows, 2}, 128-byte swizzle: one copy brings two adjacent 64-column
// chunks of box_rows rows and lands them as two 128-byte-swizzled tiles, one after the other.
bool make_map_chunks(CUtensorMap* m, const void* base, uint64_t K, uint64_t rows, uint32_t box_rows) {
  MapKey k{};
  k.base = base;
  k.dt = (uint32_t)CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  k.rank = 3;
  k.swizzle = (uint32_t)CU_TENSOR_MAP_SWIZZLE_128B;
  k.dims[0] = 64;
  k.dims[1] = rows;
  k.dims[2] = K / 64;
  k.strides[0] = K * 2;
  k.strides[1] = 128;
  k.box[0] = 64;
  k.box[1] = box_rows;
  k.box[2] = 2;
  return encode_map(k, m);
}

// ------------------------------------------------------------- checks -------
bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

constexpr int64_t kMaxDim = (int64_t(1) << 31) - 1;

// M = 0 (an empty batch) passes; the per-forward entry points then return SVDQ_OK at once.
svdq_status check_shape(int64_t M, int64_t N, int64_t K, int r) {
  if (M < 0 || N < 1 || K < 1 || r < 0) return SVDQ_ERR_INVALID_ARG;
  if (M > kMaxDim || N > kMaxDim || K > kMaxDim) return SVDQ_ERR_UNSUPPORTED_SHAPE;
  if (K % 64 != 0 || N % 16 != 0 || r % 16 != 0 || r > 128) return SVDQ_ERR_UNSUPPORTED_SHAPE;
  return SVDQ_OK;
}

svdq_status launch_status() {
  return cudaGetLastError() == cudaSuccess ? SVDQ_OK : SVDQ_ERR_CUDA;
}

int64_t pad128(int64_t v) { return (v + 127) / 128 * 128; }

// Launch as a programmatic dependent of the previous kernel on the stream: the kernel's prologue
// (barrier set-up, TMEM allocation, descriptor prefetch) overlaps that kernel's tail, and the kernel
// waits for it (griddepcontrol.wait) before it touches global memory.  cluster > 1 launches
// thread-block clusters of that many CTAs along x.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s, int cluster,
                       Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  int n = 1;
  if (cluster > 1) {
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = (unsigned)cluster;
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = 1;
    n = 2;
  }
  cfg.attrs = attr;
  cfg.numAttrs = n;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// --------------------------------------------------------- quantize_act -----
// CTAs that share a 128-row block split its K chunks between them: the smallest split in
// {1, 2, 4, 8} that gives about one CTA per SM (the kernel runs one 576-thread CTA per SM, so a
// larger grid would run in two waves), with at least two chunks a CTA.
int qa_split(int64_t M, int64_t K, int sms) {
  const int64_t rb = pad128(M) / 128, nunits = (K / 64 + 1) / 2;   // stages of two 64-column chunks
  int split = 1;
  while (split < QB_MAX_SPLIT && rb * 2 * split <= (int64_t)sms && nunits >= 2 * split) split *= 2;
  return split;
}

// Workspace of kernel 2 (see include/svdq.h): the ticket words first, then the partial sums.
size_t qa_ticket_bytes(int64_t M) { return (size_t)((pad128(M) / 128 * 4 + 255) / 256 * 256); }
size_t qa_workspace_bytes(int64_t M, int r) {
  return r > 0 ? qa_ticket_bytes(M) + (size_t)QB_MAX_SPLIT * (size_t)pad128(M) * (size_t)r * 4 : 0;
}

// ------------------------------------------------ scratch of svdq_quantize_act_noalloc ---
// Device memory the library owns for callers that cannot allocate: the counters and partial sums
// of kernel 2's K split.  In host code the name stands for a host-side handle, not a device address,
// so the kernels are given the address cudaGetSymbolAddress returns for the current device.
constexpr size_t kNoAllocScratchBytes = SVDQ_NOALLOC_SCRATCH_BYTES;
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];
void* g_noalloc_ptr[kMaxDevices] = {};

// Bytes of the scratch a call uses: the counters, then the partial sums of the split the launch takes.
size_t noalloc_scratch_need(int64_t M, int64_t K, int r, int sms) {
  return qa_ticket_bytes(M) + (size_t)qa_split(M, K, sms) * (size_t)pad128(M) * (size_t)r * 4;
}

// Device address of the scratch array on device `dev` (the current device), looked up once.
svdq_status noalloc_scratch(int dev, DevInfo* d, void** out) {
  (void)d;
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_noalloc_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return SVDQ_ERR_CUDA;
    g_noalloc_ptr[dev] = p;
  }
  *out = g_noalloc_ptr[dev];
  return SVDQ_OK;
}

template <int R, bool QUANT, bool MX = false>
svdq_status launch_qa(DevInfo* d, const uint16_t* X, int64_t M, int64_t K, const float* inv_s, float gs_x,
                      const uint16_t* L1fT, float lr_scale, uint8_t* Xq, uint8_t* SFx, uint16_t* LAs,
                      void* ws, cudaStream_t s) {
  using Cfg = QbCfg<R>;
  CUtensorMap tm_x, tm_l1, tm_x1, tm_l11;
  if (!make_map_chunks(&tm_x, X, (uint64_t)K, (uint64_t)M, QB_ROWS) ||
      !make_map_2d(&tm_x1, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, X, (uint64_t)K, (uint64_t)M, (uint64_t)K * 2, 64,
                   QB_ROWS))
    return SVDQ_ERR_CUDA;
  if (R > 0) {
    if (!make_map_chunks(&tm_l1, L1fT, (uint64_t)K, (uint64_t)R, R > 0 ? R : 1) ||
        !make_map_2d(&tm_l11, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, L1fT, (uint64_t)K, (uint64_t)R, (uint64_t)K * 2, 64,
                     R > 0 ? R : 1))
      return SVDQ_ERR_CUDA;
  } else {
    tm_l1 = tm_x;
    tm_l11 = tm_x1;
  }
  bool& attr = d->qa_attr[MX ? 2 : QUANT ? 0 : 1][R / 16];
  if (!attr) {
    if (cudaFuncSetAttribute(k_quantize_act<R, QUANT, MX>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             Cfg::kSmem) != cudaSuccess)
      return SVDQ_ERR_CUDA;
    attr = true;
  }
  const int64_t Mpad = pad128(M);
  const int split = qa_split(M, K, d->sms);   // with r = 0 the CTAs of a row block only share out K
  unsigned int* ticket = reinterpret_cast<unsigned int*>(ws);
  float* part = ws ? reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(ws) + qa_ticket_bytes(M)) : nullptr;
  if (R > 0 && split > 1 && !ws) return SVDQ_ERR_INVALID_ARG;
  const dim3 grid((unsigned)(Mpad / QB_ROWS * split));
  if (launch_pdl(k_quantize_act<R, QUANT, MX>, grid, dim3(QB_THREADS), (size_t)Cfg::kSmem, s, 1, tm_x, tm_l1, tm_x1,
                 tm_l11, inv_s, gs_x, lr_scale, (int)M, (int)K, (int)Mpad, split, Xq, SFx, LAs, part, ticket,
                 LN_DEFAULT_TIMEOUT_NS) != cudaSuccess)
    return SVDQ_ERR_CUDA;
  return launch_status();
}

template <bool QUANT, bool MX = false>
svdq_status dispatch_qa(DevInfo* d, int r, const uint16_t* X, int64_t M, int64_t K, const float* inv_s, float gs_x,
                        const uint16_t* L1fT, float lr_scale, uint8_t* Xq, uint8_t* SFx, uint16_t* LAs,
                        void* ws, cudaStream_t s) {
  switch (r) {
    case 0:
      if (QUANT) return launch_qa<0, true, MX>(d, X, M, K, inv_s, gs_x, L1fT, lr_scale, Xq, SFx, LAs, ws, s);
      return SVDQ_ERR_INVALID_ARG;
    case 16: return launch_qa<16, QUANT, MX>(d, X, M, K, inv_s, gs_x, L1fT, lr_scale, Xq, SFx, LAs, ws, s);
    case 32: return launch_qa<32, QUANT, MX>(d, X, M, K, inv_s, gs_x, L1fT, lr_scale, Xq, SFx, LAs, ws, s);
    case 48: return launch_qa<48, QUANT, MX>(d, X, M, K, inv_s, gs_x, L1fT, lr_scale, Xq, SFx, LAs, ws, s);
    case 64: return launch_qa<64, QUANT, MX>(d, X, M, K, inv_s, gs_x, L1fT, lr_scale, Xq, SFx, LAs, ws, s);
    case 80: return launch_qa<80, QUANT, MX>(d, X, M, K, inv_s, gs_x, L1fT, lr_scale, Xq, SFx, LAs, ws, s);
    case 96: return launch_qa<96, QUANT, MX>(d, X, M, K, inv_s, gs_x, L1fT, lr_scale, Xq, SFx, LAs, ws, s);
    case 112: return launch_qa<112, QUANT, MX>(d, X, M, K, inv_s, gs_x, L1fT, lr_scale, Xq, SFx, LAs, ws, s);
    case 128: return launch_qa<128, QUANT, MX>(d, X, M, K, inv_s, gs_x, L1fT, lr_scale, Xq, SFx, LAs, ws, s);
    default: return SVDQ_ERR_UNSUPPORTED_SHAPE;
  }
}

// The next layer's quantization done in the GEMM epilogue (svdq_linear_gelu_quantize).
struct GqArgs {
  const float* inv_s2;
  float gs_x2;
  const uint16_t* L1fT2;
  int r2;
  float lr_scale2;
  uint8_t* Xq2;
  uint8_t* SFx2;
  uint16_t* LAs2;
  float* part;
};

size_t gq_workspace_bytes(int64_t M, int64_t N, int r2) {
  if (r2 <= 0) return 0;
  return (size_t)((N + LN_BN - 1) / LN_BN) * (size_t)pad128(M) * (size_t)r2 * sizeof(float);
}

svdq_status linear_impl(const uint8_t* Xq, const uint8_t* SFx, float gs_x, const uint8_t* Wq, const uint8_t* SFw,
                        float gs_w, const uint16_t* LAs, const uint16_t* L2p, int r, const uint16_t* bias, void* Y,
                        int y_fp32, int64_t M, int64_t N, int64_t K, int debug, uint64_t timeout_ns,
                        cudaStream_t s, int y_accum = 0, bool mx = false, const GqArgs* gq = nullptr) {
  // y_accum: the rank-only mode (no 4-bit operands, K = 0) that adds the up-projection into Y.
  // gq: no Y; the epilogue writes the next layer's quantized activations instead.
  svdq_status st = check_shape(M, N, y_accum ? 64 : K, r);
  if (st != SVDQ_OK) return st;
  if (mx && K % 128 != 0) return SVDQ_ERR_UNSUPPORTED_SHAPE;
  if (M == 0) return (y_accum && r == 0) ? SVDQ_ERR_INVALID_ARG : SVDQ_OK;   // an empty batch: nothing to launch
  if (y_accum ? (r == 0 || !LAs || !L2p || !Y || bias)
              : (!Xq || !SFx || !Wq || !SFw || (!gq && !Y) || (r > 0 && (!LAs || !L2p))))
    return SVDQ_ERR_INVALID_ARG;
  if (y_fp32 != 0 && y_fp32 != 1) return SVDQ_ERR_INVALID_ARG;
  if ((!y_accum && (!aligned16(Xq) || !aligned16(SFx) || !aligned16(Wq) || !aligned16(SFw))) ||
      (!gq && !aligned16(Y)) || (bias && !aligned16(bias)) || (r > 0 && (!aligned16(LAs) || !aligned16(L2p))))
    return SVDQ_ERR_MISALIGNED;
  if (gq) {
    if (N % 64 != 0 || (gq->r2 != 0 && gq->r2 != 16 && gq->r2 != 32)) return SVDQ_ERR_UNSUPPORTED_SHAPE;
    if (!gq->inv_s2 || !gq->Xq2 || !gq->SFx2 || !(gq->gs_x2 > 0.0f) || !std::isfinite(gq->gs_x2) ||
        (gq->r2 > 0 && (!gq->L1fT2 || !gq->LAs2 || !gq->part)))
      return SVDQ_ERR_INVALID_ARG;
    if (!aligned16(gq->inv_s2) || !aligned16(gq->Xq2) || !aligned16(gq->SFx2) ||
        (gq->r2 > 0 && (!aligned16(gq->L1fT2) || !aligned16(gq->LAs2) || !aligned16(gq->part))))
      return SVDQ_ERR_MISALIGNED;
  }
  int dev;
  DevInfo* d;
  if ((st = current_device(&dev, &d)) != SVDQ_OK) return st;

  CUtensorMap tm_xq, tm_wq, tm_las, tm_l2p;
  if (!y_accum &&
      (!make_map_2d(&tm_xq, CU_TENSOR_MAP_DATA_TYPE_UINT8, Xq, (uint64_t)K / 2, (uint64_t)M, (uint64_t)K / 2, 128,
                    LN_BM) ||
       !make_map_2d(&tm_wq, CU_TENSOR_MAP_DATA_TYPE_UINT8, Wq, (uint64_t)K / 2, (uint64_t)N, (uint64_t)K / 2, 128,
                    LN_BN / 2)))
    return SVDQ_ERR_CUDA;
  if (r > 0) {
    if (!make_map_2d(&tm_las, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, LAs, (uint64_t)2 * r, (uint64_t)M,
                     (uint64_t)4 * r, 64, LN_BM) ||
        !make_map_2d(&tm_l2p, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, L2p, (uint64_t)r, (uint64_t)N,
                     (uint64_t)2 * r, 32, LN_BN / 2, CU_TENSOR_MAP_SWIZZLE_64B))
      return SVDQ_ERR_CUDA;
  } else {
    tm_las = tm_xq;
    tm_l2p = tm_wq;
  }
  if (y_accum) {                 // no K tiles: the 4-bit maps are never used
    tm_xq = tm_las;
    tm_wq = tm_l2p;
  }
  const int variant = gq ? 2 : mx ? 1 : 0;
  auto kernel = gq ? k_linear<false, true> : mx ? k_linear<true, false> : k_linear<false, false>;
  const int smem_bytes = gq ? LN_SMEM_GQ : LN_SMEM;
  if (!d->linear_attr[variant]) {
    if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_bytes) != cudaSuccess)
      return SVDQ_ERR_CUDA;
    d->linear_attr[variant] = true;
  }
  LinearArgs a;
  a.SFx = SFx;
  a.SFw = SFw;
  a.bias = bias;
  a.Y = Y;
  a.y_fp32 = y_fp32;
  a.y_vec32 = (reinterpret_cast<uintptr_t>(Y) & 31u) == 0 ? 1 : 0;
  a.y_accum = y_accum;
  a.M = (int)M;
  a.N = (int)N;
  a.K = y_accum ? 0 : (int)K;
  a.r = r;
  a.gs = gs_x * gs_w;
  a.debug = debug;
  a.timeout_ns = timeout_ns ? timeout_ns : LN_DEFAULT_TIMEOUT_NS;
  a.inv_s2 = gq ? gq->inv_s2 : nullptr;
  a.gs_x2 = gq ? gq->gs_x2 : 1.0f;
  a.L1fT2 = gq ? gq->L1fT2 : nullptr;
  a.r2 = gq ? gq->r2 : 0;
  a.Mpad = (int)pad128(M);
  a.Xq2 = gq ? gq->Xq2 : nullptr;
  a.SFx2 = gq ? gq->SFx2 : nullptr;
  a.part = gq ? gq->part : nullptr;
  const int64_t tiles = ((M + LN_BM - 1) / LN_BM) * ((N + LN_BN - 1) / LN_BN);
  const int grid = (int)(tiles < d->sms ? tiles : d->sms);
  if (launch_pdl(kernel, dim3(grid), dim3(LN_THREADS), (size_t)smem_bytes, s, 1, tm_xq, tm_wq, tm_las, tm_l2p, a) !=
      cudaSuccess)
    return SVDQ_ERR_CUDA;
  if (gq && gq->r2 > 0) {
    const int items = (int)M * (gq->r2 / 4);
    if (launch_pdl(k_lowrank_finalize, dim3((items + 255) / 256), dim3(256), 0, s, 1, (const float*)gq->part,
                   (int)((N + LN_BN - 1) / LN_BN), (int)M, (int)pad128(M), gq->r2, gq->lr_scale2, gq->LAs2) !=
        cudaSuccess)
      return SVDQ_ERR_CUDA;
  }
  return launch_status();
}

}  // namespace

extern "C" {

const char* svdq_status_string(int status) {
  switch (status) {
    case SVDQ_OK: return "SVDQ_OK";
    case SVDQ_ERR_INVALID_ARG: return "SVDQ_ERR_INVALID_ARG";
    case SVDQ_ERR_UNSUPPORTED_SHAPE: return "SVDQ_ERR_UNSUPPORTED_SHAPE";
    case SVDQ_ERR_MISALIGNED: return "SVDQ_ERR_MISALIGNED";
    case SVDQ_ERR_CUDA: return "SVDQ_ERR_CUDA";
    case SVDQ_ERR_TIMEOUT: return "SVDQ_ERR_TIMEOUT";
    case SVDQ_ERR_DEVICE: return "SVDQ_ERR_DEVICE";
    case SVDQ_ERR_SCRATCH: return "SVDQ_ERR_SCRATCH";
    case SVDQ_ERR_CHECK: return "SVDQ_ERR_CHECK";
    default: return "SVDQ_ERR_UNKNOWN";
  }
}

int svdq_version(void) { return 100; }

size_t svdq_sf_bytes(int64_t rows, int64_t K) {
  if (rows < 0 || K < 0 || K % 64 != 0) return 0;
  return (size_t)pad128(rows) * (size_t)(K / 16);
}

svdq_status svdq_pack_weight(const float* R, const uint16_t* L2b, int64_t K, int64_t N, int r, uint8_t* Wq,
                             uint8_t* SFw, float* gs_w, float* gs_w_host, uint16_t* L2p, svdq_stream_t stream) {
  svdq_status st = check_shape(1, N, K, r);
  if (st != SVDQ_OK) return st;
  if (!R || !Wq || !SFw || !gs_w || (r > 0 && (!L2b || !L2p))) return SVDQ_ERR_INVALID_ARG;
  if (!aligned16(R) || !aligned16(Wq) || !aligned16(SFw) || (r > 0 && (!aligned16(L2b) || !aligned16(L2p))))
    return SVDQ_ERR_MISALIGNED;
  int dev;
  DevInfo* d;
  if ((st = current_device(&dev, &d)) != SVDQ_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  unsigned int* bits = reinterpret_cast<unsigned int*>(gs_w);
  k_zero_u32<<<1, 1, 0, s>>>(bits);
  const int64_t n = K * N;
  int64_t blocks = (n / 4 + 255) / 256;
  if (blocks > 4 * (int64_t)d->sms) blocks = 4 * (int64_t)d->sms;
  if (blocks < 1) blocks = 1;
  k_absmax_f32<<<(unsigned)blocks, 256, 0, s>>>(R, n, bits);
  k_global_scale<<<1, 1, 0, s>>>(gs_w);
  const int64_t Npad = pad128(N);
  k_pack_weight<<<dim3((unsigned)(Npad / 128), (unsigned)(K / 64)), 128, 0, s>>>(R, (int)K, (int)N, (int)Npad, gs_w,
                                                                                  Wq, SFw);
  if (r > 0) k_layout_l2<<<(unsigned)((N + 127) / 128), 128, 0, s>>>(L2b, (int)N, r, L2p);
  if ((st = launch_status()) != SVDQ_OK) return st;
  if (gs_w_host) {
    if (cudaMemcpyAsync(gs_w_host, gs_w, sizeof(float), cudaMemcpyDeviceToHost, s) != cudaSuccess ||
        cudaStreamSynchronize(s) != cudaSuccess)
      return SVDQ_ERR_CUDA;
  }
  return SVDQ_OK;
}

size_t svdq_mx_sf_bytes(int64_t rows, int64_t K) {
  if (rows < 0 || K < 0 || K % 128 != 0) return 0;
  return (size_t)pad128(rows) * (size_t)(K / 32);
}

svdq_status svdq_pack_weight_mx(const float* R, const uint16_t* L2b, int64_t K, int64_t N, int r, uint8_t* Wq,
                                uint8_t* SFw, uint16_t* L2p, svdq_stream_t stream) {
  svdq_status st = check_shape(1, N, K, r);
  if (st != SVDQ_OK) return st;
  if (K % 128 != 0) return SVDQ_ERR_UNSUPPORTED_SHAPE;
  if (!R || !Wq || !SFw || (r > 0 && (!L2b || !L2p))) return SVDQ_ERR_INVALID_ARG;
  if (!aligned16(R) || !aligned16(Wq) || !aligned16(SFw) || (r > 0 && (!aligned16(L2b) || !aligned16(L2p))))
    return SVDQ_ERR_MISALIGNED;
  int dev;
  DevInfo* d;
  if ((st = current_device(&dev, &d)) != SVDQ_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const int64_t Npad = pad128(N);
  k_pack_weight_mx<<<dim3((unsigned)(Npad / 128), (unsigned)(K / 128)), 128, 0, s>>>(R, (int)K, (int)N, (int)Npad,
                                                                                     Wq, SFw);
  if (r > 0) k_layout_l2<<<(unsigned)((N + 127) / 128), 128, 0, s>>>(L2b, (int)N, r, L2p);
  return launch_status();
}

svdq_status svdq_quantize_act_mx(const uint16_t* X, int64_t M, int64_t K, const float* inv_s, const uint16_t* L1fT,
                                 int r, float lr_scale, uint8_t* Xq, uint8_t* SFx, uint16_t* LAs, void* workspace,
                                 size_t workspace_bytes, svdq_stream_t stream) {
  svdq_status st = check_shape(M, 16, K, r);
  if (st != SVDQ_OK) return st;
  if (K % 128 != 0) return SVDQ_ERR_UNSUPPORTED_SHAPE;
  if (M == 0) return SVDQ_OK;                 // an empty batch: nothing to launch
  if (!X || !inv_s || !Xq || !SFx || (r > 0 && (!L1fT || !LAs))) return SVDQ_ERR_INVALID_ARG;
  if (r > 0 && (!workspace || workspace_bytes < qa_workspace_bytes(M, r))) return SVDQ_ERR_INVALID_ARG;
  if (!aligned16(X) || !aligned16(inv_s) || !aligned16(Xq) || !aligned16(SFx) ||
      (r > 0 && (!aligned16(L1fT) || !aligned16(LAs) || !aligned16(workspace))))
    return SVDQ_ERR_MISALIGNED;
  int dev;
  DevInfo* d;
  if ((st = current_device(&dev, &d)) != SVDQ_OK) return st;
  return dispatch_qa<true, true>(d, r, X, M, K, inv_s, 1.0f, L1fT, lr_scale, Xq, SFx, LAs, workspace,
                                 reinterpret_cast<cudaStream_t>(stream));
}

svdq_status svdq_linear_mx(const uint8_t* Xq, const uint8_t* SFx, const uint8_t* Wq, const uint8_t* SFw,
                           const uint16_t* LAs, const uint16_t* L2p, int r, const uint16_t* bias, void* Y, int y_fp32,
                           int64_t M, int64_t N, int64_t K, svdq_stream_t stream) {
  return linear_impl(Xq, SFx, 1.0f, Wq, SFw, 1.0f, LAs, L2p, r, bias, Y, y_fp32, M, N, K, 0, 0,
                     reinterpret_cast<cudaStream_t>(stream), 0, true);
}

size_t svdq_linear_gelu_quantize_workspace_bytes(int64_t M, int64_t N, int r2) {
  if (M < 1 || N < 1 || r2 < 0) return 0;
  return gq_workspace_bytes(M, N, r2);
}

svdq_status svdq_linear_gelu_quantize(const uint8_t* Xq, const uint8_t* SFx, float gs_x, const uint8_t* Wq,
                                      const uint8_t* SFw, float gs_w, const uint16_t* LAs, const uint16_t* L2p, int r,
                                      const uint16_t* bias, int64_t M, int64_t N, int64_t K, const float* inv_s2,
                                      float gs_x2, const uint16_t* L1fT2, int r2, float lr_scale2, uint8_t* Xq2,
                                      uint8_t* SFx2, uint16_t* LAs2, void* workspace, size_t workspace_bytes,
                                      svdq_stream_t stream) {
  svdq_status st = check_shape(M, N, K, r);
  if (st != SVDQ_OK) return st;
  if (N % 64 != 0 || (r2 != 0 && r2 != 16 && r2 != 32)) return SVDQ_ERR_UNSUPPORTED_SHAPE;
  if (M == 0) return SVDQ_OK;                 // an empty batch: nothing to launch
  if (r2 > 0 && workspace_bytes < gq_workspace_bytes(M, N, r2)) return SVDQ_ERR_INVALID_ARG;
  GqArgs g;
  g.inv_s2 = inv_s2;
  g.gs_x2 = gs_x2;
  g.L1fT2 = L1fT2;
  g.r2 = r2;
  g.lr_scale2 = lr_scale2;
  g.Xq2 = Xq2;
  g.SFx2 = SFx2;
  g.LAs2 = LAs2;
  g.part = static_cast<float*>(workspace);
  return linear_impl(Xq, SFx, gs_x, Wq, SFw, gs_w, LAs, L2p, r, bias, nullptr, 0, M, N, K, 0, 0,
                     reinterpret_cast<cudaStream_t>(stream), 0, false, &g);
}

svdq_status svdq_gelu_bf16(const uint16_t* X, int64_t n, uint16_t* Y, svdq_stream_t stream) {
  if (n < 0 || (n > 0 && (!X || !Y))) return SVDQ_ERR_INVALID_ARG;
  if (n == 0) return SVDQ_OK;
  if (!aligned16(X) || !aligned16(Y)) return SVDQ_ERR_MISALIGNED;
  int dev;
  DevInfo* d;
  svdq_status st;
  if ((st = current_device(&dev, &d)) != SVDQ_OK) return st;
  const int64_t nv = (n + 7) / 8;
  const int64_t cap = (int64_t)d->sms * 8;                   // 8 blocks of 256 threads per SM
  const int blocks = (int)std::max<int64_t>(1, std::min<int64_t>((nv + 4 * 256 - 1) / (4 * 256), cap));
  if (launch_pdl(k_gelu_bf16, dim3(blocks), dim3(256), 0, reinterpret_cast<cudaStream_t>(stream), 1, X, n, Y) !=
      cudaSuccess)
    return SVDQ_ERR_CUDA;
  return launch_status();
}

svdq_status svdq_calib_absmax_cols(const uint16_t* X, int64_t M, int64_t K, float* amax_x, int accumulate,
                                   svdq_stream_t stream) {
  if (M < 0 || K < 8 || K % 8 != 0 || K >= (int64_t(1) << 31) || !amax_x || (M > 0 && !X) ||
      (accumulate != 0 && accumulate != 1))
    return SVDQ_ERR_INVALID_ARG;
  if ((M > 0 && !aligned16(X)) || (reinterpret_cast<uintptr_t>(amax_x) & 3u)) return SVDQ_ERR_MISALIGNED;
  int dev;
  DevInfo* d;
  svdq_status st;
  if ((st = current_device(&dev, &d)) != SVDQ_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (!accumulate && cudaMemsetAsync(amax_x, 0, (size_t)K * sizeof(float), s) != cudaSuccess) return SVDQ_ERR_CUDA;
  if (M == 0) return launch_status();
  const int gx = (int)((K + 255) / 256);
  // enough row slices for about four blocks per SM
  const int64_t want = std::max<int64_t>(1, (int64_t)d->sms * 4 / gx);
  const int slices = (int)std::min<int64_t>(want, (M + 63) / 64);
  const int rows = (int)((M + slices - 1) / slices);
  k_absmax_cols<<<dim3(gx, (unsigned)((M + rows - 1) / rows)), 256, 0, s>>>(X, M, (int)K, rows, amax_x);
  return launch_status();
}

svdq_status svdq_calib_absmax_rows(const double* W, int64_t K, int64_t N, double* amax_w, svdq_stream_t stream) {
  if (K < 1 || N < 1 || K >= (int64_t(1) << 31) || !W || !amax_w) return SVDQ_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(W) | reinterpret_cast<uintptr_t>(amax_w)) & 7u) return SVDQ_ERR_MISALIGNED;
  int dev;
  DevInfo* d;
  svdq_status st;
  if ((st = current_device(&dev, &d)) != SVDQ_OK) return st;
  k_absmax_rows<<<(unsigned)K, 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(W, N, amax_w);
  return launch_status();
}

svdq_status svdq_calib_smooth(const float* amax_x, const double* amax_w, int64_t K, double alpha, double* s,
                              float* inv_s, svdq_stream_t stream) {
  if (K < 1 || K >= (int64_t(1) << 31) || !amax_x || !amax_w || !s || !inv_s || !(alpha >= 0.0 && alpha <= 1.0))
    return SVDQ_ERR_INVALID_ARG;
  int dev;
  DevInfo* d;
  svdq_status st;
  if ((st = current_device(&dev, &d)) != SVDQ_OK) return st;
  k_smooth<<<(unsigned)((K + 255) / 256), 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(amax_x, amax_w, (int)K,
                                                                                           alpha, s, inv_s);
  return launch_status();
}

svdq_status svdq_calib_scale_rows(const double* W, const double* s, int64_t K, int64_t N, double* W_hat,
                                  svdq_stream_t stream) {
  if (K < 1 || N < 1 || !W || !s || !W_hat) return SVDQ_ERR_INVALID_ARG;
  int dev;
  DevInfo* d;
  svdq_status st;
  if ((st = current_device(&dev, &d)) != SVDQ_OK) return st;
  const int64_t blocks = std::min<int64_t>((K * N + 255) / 256, (int64_t)d->sms * 16);
  k_scale_rows<<<(unsigned)blocks, 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(W, s, K, N, W_hat);
  return launch_status();
}

svdq_status svdq_calib_act_amax(const uint16_t* X, int64_t M, int64_t K, const float* inv_s, float* amax,
                                int accumulate, svdq_stream_t stream) {
  if (M < 0 || K < 8 || K % 8 != 0 || K >= (int64_t(1) << 31) || !inv_s || !amax || (M > 0 && !X) ||
      (accumulate != 0 && accumulate != 1))
    return SVDQ_ERR_INVALID_ARG;
  if ((M > 0 && !aligned16(X)) || !aligned16(inv_s) || (reinterpret_cast<uintptr_t>(amax) & 3u))
    return SVDQ_ERR_MISALIGNED;
  int dev;
  DevInfo* d;
  svdq_status st;
  if ((st = current_device(&dev, &d)) != SVDQ_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (!accumulate && cudaMemsetAsync(amax, 0, sizeof(float), s) != cudaSuccess) return SVDQ_ERR_CUDA;
  if (M == 0) return launch_status();
  const int64_t blocks = std::max<int64_t>(1, std::min<int64_t>((M * (K / 8) + 255) / 256, (int64_t)d->sms * 8));
  k_act_amax<<<(unsigned)blocks, 256, 0, s>>>(X, M, (int)K, inv_s, amax);
  return launch_status();
}

void svdq_map_cache_stats(uint64_t* hits, uint64_t* misses) {
  std::lock_guard<std::mutex> lk(g_map_mu);
  if (hits) *hits = g_map_hits;
  if (misses) *misses = g_map_misses;
}

svdq_status svdq_dequant_weight(const uint8_t* Wq, const uint8_t* SFw, const float* gs_w, int64_t K, int64_t N,
                                float* Rq, svdq_stream_t stream) {
  svdq_status st = check_shape(1, N, K, 0);
  if (st != SVDQ_OK) return st;
  if (!Wq || !SFw || !gs_w || !Rq) return SVDQ_ERR_INVALID_ARG;
  if (!aligned16(Wq) || !aligned16(SFw) || !aligned16(Rq)) return SVDQ_ERR_MISALIGNED;
  int dev;
  DevInfo* d;
  if ((st = current_device(&dev, &d)) != SVDQ_OK) return st;
  k_dequant_weight<<<dim3((unsigned)((N + 127) / 128), (unsigned)(K / 64)), 128, 0,
                     reinterpret_cast<cudaStream_t>(stream)>>>(Wq, SFw, gs_w, (int)K, (int)N, Rq);
  return launch_status();
}

size_t svdq_quantize_act_workspace_bytes(int64_t M, int64_t K, int r) {
  if (M < 1 || K < 64 || K % 64 != 0 || r < 0 || r % 16 != 0 || r > 128) return 0;
  return qa_workspace_bytes(M, r);
}

svdq_status svdq_quantize_act(const uint16_t* X, int64_t M, int64_t K, const float* inv_s, float gs_x,
                              const uint16_t* L1fT, int r, float lr_scale, uint8_t* Xq, uint8_t* SFx, uint16_t* LAs,
                              void* workspace, size_t workspace_bytes, svdq_stream_t stream) {
  svdq_status st = check_shape(M, 16, K, r);
  if (st != SVDQ_OK) return st;
  if (M == 0) return SVDQ_OK;                 // an empty batch: nothing to launch
  if (!X || !inv_s || !Xq || !SFx || (r > 0 && (!L1fT || !LAs))) return SVDQ_ERR_INVALID_ARG;
  if (r > 0 && (!workspace || workspace_bytes < qa_workspace_bytes(M, r))) return SVDQ_ERR_INVALID_ARG;
  if (!aligned16(X) || !aligned16(inv_s) || !aligned16(Xq) || !aligned16(SFx) ||
      (r > 0 && (!aligned16(L1fT) || !aligned16(LAs) || !aligned16(workspace))))
    return SVDQ_ERR_MISALIGNED;
  int dev;
  DevInfo* d;
  if ((st = current_device(&dev, &d)) != SVDQ_OK) return st;
  return dispatch_qa<true>(d, r, X, M, K, inv_s, gs_x, L1fT, lr_scale, Xq, SFx, LAs, workspace,
                           reinterpret_cast<cudaStream_t>(stream));
}

svdq_status svdq_quantize_act_noalloc(const uint16_t* X, int64_t M, int64_t K, const float* inv_s, float gs_x,
                                      const uint16_t* L1fT, int r, float lr_scale, uint8_t* Xq, uint8_t* SFx,
                                      uint16_t* LAs, svdq_stream_t stream) {
  svdq_status st = check_shape(M, 16, K, r);
  if (st != SVDQ_OK) return st;
  if (M == 0) return SVDQ_OK;                 // an empty batch: nothing to launch
  if (!X || !inv_s || !Xq || !SFx || (r > 0 && (!L1fT || !LAs))) return SVDQ_ERR_INVALID_ARG;
  if (!aligned16(X) || !aligned16(inv_s) || !aligned16(Xq) || !aligned16(SFx) ||
      (r > 0 && (!aligned16(L1fT) || !aligned16(LAs))))
    return SVDQ_ERR_MISALIGNED;
  int dev;
  DevInfo* d;
  if ((st = current_device(&dev, &d)) != SVDQ_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  void* ws = nullptr;
  if (r > 0) {
    if (noalloc_scratch_need(M, K, r, d->sms) > kNoAllocScratchBytes) return SVDQ_ERR_SCRATCH;
    if ((st = noalloc_scratch(dev, d, &ws)) != SVDQ_OK) return st;
    // the row-block counters start at 0 (a call that ran out of time can leave them set)
    if (cudaMemsetAsync(ws, 0, qa_ticket_bytes(M), s) != cudaSuccess) return SVDQ_ERR_CUDA;
  }
  return dispatch_qa<true>(d, r, X, M, K, inv_s, gs_x, L1fT, lr_scale, Xq, SFx, LAs, ws, s);
}

svdq_status svdq_lowrank_down(const uint16_t* X, int64_t M, int64_t K, const uint16_t* L1fT, int r, float lr_scale,
                              uint16_t* LAs, void* workspace, size_t workspace_bytes, svdq_stream_t stream) {
  svdq_status st = check_shape(M, 16, K, r);
  if (st != SVDQ_OK) return st;
  if (M == 0) return r == 0 ? SVDQ_ERR_INVALID_ARG : SVDQ_OK;   // an empty batch: nothing to launch
  if (r == 0 || !X || !L1fT || !LAs || !workspace || workspace_bytes < qa_workspace_bytes(M, r))
    return SVDQ_ERR_INVALID_ARG;
  if (!aligned16(X) || !aligned16(L1fT) || !aligned16(LAs) || !aligned16(workspace)) return SVDQ_ERR_MISALIGNED;
  int dev;
  DevInfo* d;
  if ((st = current_device(&dev, &d)) != SVDQ_OK) return st;
  return dispatch_qa<false>(d, r, X, M, K, nullptr, 1.0f, L1fT, lr_scale, nullptr, nullptr, LAs, workspace,
                            reinterpret_cast<cudaStream_t>(stream));
}

svdq_status svdq_lowrank_up(const uint16_t* LAs, const uint16_t* L2p, int r, float gs, void* Y, int y_fp32,
                            int64_t M, int64_t N, svdq_stream_t stream) {
  return linear_impl(nullptr, nullptr, 1.0f, nullptr, nullptr, gs, LAs, L2p, r, nullptr, Y, y_fp32, M, N, 0, 0, 0,
                     reinterpret_cast<cudaStream_t>(stream), 1);
}

svdq_status svdq_linear(const uint8_t* Xq, const uint8_t* SFx, float gs_x, const uint8_t* Wq, const uint8_t* SFw,
                        float gs_w, const uint16_t* LAs, const uint16_t* L2p, int r, const uint16_t* bias, void* Y,
                        int y_fp32, int64_t M, int64_t N, int64_t K, svdq_stream_t stream) {
  return linear_impl(Xq, SFx, gs_x, Wq, SFw, gs_w, LAs, L2p, r, bias, Y, y_fp32, M, N, K, 0, 0,
                     reinterpret_cast<cudaStream_t>(stream));
}

svdq_status svdq_linear_debug(const uint8_t* Xq, const uint8_t* SFx, float gs_x, const uint8_t* Wq,
                              const uint8_t* SFw, float gs_w, const uint16_t* LAs, const uint16_t* L2p, int r,
                              const uint16_t* bias, void* Y, int y_fp32, int64_t M, int64_t N, int64_t K,
                              int debug_flags, uint64_t timeout_ns, svdq_stream_t stream) {
#ifdef SVDQ_CHECK
  if (debug_flags & ~(LN_DBG_NO_LOADS | LN_DBG_MISALIGN)) return SVDQ_ERR_INVALID_ARG;
#else
  if (debug_flags & ~LN_DBG_NO_LOADS) return SVDQ_ERR_INVALID_ARG;   // the misaligned box only where checked
#endif
  return linear_impl(Xq, SFx, gs_x, Wq, SFw, gs_w, LAs, L2p, r, bias, Y, y_fp32, M, N, K, debug_flags, timeout_ns,
                     reinterpret_cast<cudaStream_t>(stream));
}

svdq_status svdq_get_device_error(svdq_stream_t stream, int* site) {
  if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess) return SVDQ_ERR_CUDA;
  unsigned int flags = 0, where = 0, zero = 0;
  if (cudaMemcpyFromSymbol(&flags, svdq::g_err_flags, sizeof(flags)) != cudaSuccess ||
      cudaMemcpyFromSymbol(&where, svdq::g_err_site, sizeof(where)) != cudaSuccess ||
      cudaMemcpyToSymbol(svdq::g_err_flags, &zero, sizeof(zero)) != cudaSuccess ||
      cudaMemcpyToSymbol(svdq::g_err_site, &zero, sizeof(zero)) != cudaSuccess)
    return SVDQ_ERR_CUDA;
  if (site) *site = (int)where;
  if (flags & svdq::ERR_CHECK) return SVDQ_ERR_CHECK;
  return (flags & svdq::ERR_TIMEOUT) ? SVDQ_ERR_TIMEOUT : SVDQ_OK;
}

int svdq_build_flags(void) {
#ifdef SVDQ_CHECK
  return 1;
#else
  return 0;
#endif
}

}  // extern "C"
