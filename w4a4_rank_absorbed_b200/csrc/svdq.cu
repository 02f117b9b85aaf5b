// C ABI of the SVDQuant W4A4 linear layer (declared in include/svdq.h):
// argument checks, TMA descriptor encoding and kernel launches.
// All kernels live in this one translation unit so they share one device
// error word.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <cstring>
#include <mutex>

#include "../../include/svdq.h"
#include "common.cuh"
#include "linear.cuh"
#include "linear_pair.cuh"
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
  bool linear_attr = false;
  bool linear_pair_attr = false;
  bool qa_attr[9] = {};
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

// 2-D row-major tensor (rows x inner elements, row pitch in bytes), box (box_inner x box_rows), 128B swizzle.
bool make_map_2d(CUtensorMap* m, CUtensorMapDataType dt, const void* base, uint64_t inner, uint64_t rows,
                 uint64_t pitch_bytes, uint32_t box_inner, uint32_t box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {inner, rows};
  cuuint64_t strides[1] = {pitch_bytes};
  cuuint32_t box[2] = {box_inner, box_rows};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, dt, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
            CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// ------------------------------------------------------------- checks -------
bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

constexpr int64_t kMaxDim = (int64_t(1) << 31) - 1;

svdq_status check_shape(int64_t M, int64_t N, int64_t K, int r) {
  if (M < 1 || N < 1 || K < 1 || r < 0) return SVDQ_ERR_INVALID_ARG;
  if (M > kMaxDim || N > kMaxDim || K > kMaxDim) return SVDQ_ERR_UNSUPPORTED_SHAPE;
  if (K % 64 != 0 || N % 16 != 0 || r % 16 != 0 || r > 128) return SVDQ_ERR_UNSUPPORTED_SHAPE;
  return SVDQ_OK;
}

svdq_status launch_status() {
  return cudaGetLastError() == cudaSuccess ? SVDQ_OK : SVDQ_ERR_CUDA;
}

int64_t pad128(int64_t v) { return (v + 127) / 128 * 128; }

// --------------------------------------------------------- quantize_act -----
template <int R>
svdq_status launch_qa(DevInfo* d, int slot, const uint16_t* X, int64_t M, int64_t K, const float* inv_s,
                      float gs_x, const uint16_t* L1fT, float lr_scale, uint8_t* Xq, uint8_t* SFx, uint16_t* LAs,
                      cudaStream_t s) {
  using Cfg = QaCfg<R>;
  CUtensorMap tm_x, tm_l1;
  if (!make_map_2d(&tm_x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, X, (uint64_t)K, (uint64_t)M, (uint64_t)K * 2, 64, 32))
    return SVDQ_ERR_CUDA;
  if (R > 0) {
    if (!make_map_2d(&tm_l1, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, L1fT, (uint64_t)K, (uint64_t)R, (uint64_t)K * 2, 64,
                     R > 0 ? R : 1))
      return SVDQ_ERR_CUDA;
  } else {
    tm_l1 = tm_x;
  }
  if (!d->qa_attr[slot]) {
    if (cudaFuncSetAttribute(k_quantize_act<R>, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::kSmem) !=
        cudaSuccess)
      return SVDQ_ERR_CUDA;
    d->qa_attr[slot] = true;
  }
  const int64_t Mpad = pad128(M);
  const dim3 grid((unsigned)(Mpad / QA_ROWS));
  k_quantize_act<R><<<grid, QA_THREADS, Cfg::kSmem, s>>>(tm_x, tm_l1, inv_s, gs_x, lr_scale, (int)M, (int)K,
                                                         (int)Mpad, Xq, SFx, LAs, LN_DEFAULT_TIMEOUT_NS);
  return launch_status();
}

svdq_status linear_impl(const uint8_t* Xq, const uint8_t* SFx, float gs_x, const uint8_t* Wq, const uint8_t* SFw,
                        float gs_w, const uint16_t* LAs, const uint16_t* L2p, int r, const uint16_t* bias, void* Y,
                        int y_fp32, int64_t M, int64_t N, int64_t K, int debug, uint64_t timeout_ns,
                        cudaStream_t s) {
  svdq_status st = check_shape(M, N, K, r);
  if (st != SVDQ_OK) return st;
  if (!Xq || !SFx || !Wq || !SFw || !Y || (r > 0 && (!LAs || !L2p)) || (y_fp32 != 0 && y_fp32 != 1))
    return SVDQ_ERR_INVALID_ARG;
  if (!aligned16(Xq) || !aligned16(SFx) || !aligned16(Wq) || !aligned16(SFw) || !aligned16(Y) ||
      (bias && !aligned16(bias)) || (r > 0 && (!aligned16(LAs) || !aligned16(L2p))))
    return SVDQ_ERR_MISALIGNED;
  int dev;
  DevInfo* d;
  if ((st = current_device(&dev, &d)) != SVDQ_OK) return st;

  CUtensorMap tm_xq, tm_wq, tm_las, tm_l2p;
  if (!make_map_2d(&tm_xq, CU_TENSOR_MAP_DATA_TYPE_UINT8, Xq, (uint64_t)K / 2, (uint64_t)M, (uint64_t)K / 2, 128,
                   LN_BM) ||
      !make_map_2d(&tm_wq, CU_TENSOR_MAP_DATA_TYPE_UINT8, Wq, (uint64_t)K / 2, (uint64_t)N, (uint64_t)K / 2, 128,
                   LN_BN / 2))
    return SVDQ_ERR_CUDA;
  if (r > 0) {
    if (!make_map_2d(&tm_las, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, LAs, (uint64_t)2 * r, (uint64_t)M,
                     (uint64_t)4 * r, 64, LN_BM) ||
        !make_map_2d(&tm_l2p, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, L2p, (uint64_t)2 * r, (uint64_t)N,
                     (uint64_t)4 * r, 64, LN_BN / 2))
      return SVDQ_ERR_CUDA;
  } else {
    tm_las = tm_xq;
    tm_l2p = tm_wq;
  }
  // The single-CTA kernel by default.  The CTA-pair kernel (256 x 256 tiles, half of B per CTA)
  // gives the same results but measured slower on B200 (0.118 against 0.075 ms on the QKV layer):
  // the signals between the two CTAs sit on every stage's critical path.  Debug bit 2 selects it.
  const bool pair = (debug & LN_DBG_FORCE_PAIR) != 0;
  if (pair && !d->linear_pair_attr) {
    if (cudaFuncSetAttribute(k_linear_pair, cudaFuncAttributeMaxDynamicSharedMemorySize, LP_SMEM) != cudaSuccess)
      return SVDQ_ERR_CUDA;
    d->linear_pair_attr = true;
  }
  if (!pair && !d->linear_attr) {
    if (cudaFuncSetAttribute(k_linear, cudaFuncAttributeMaxDynamicSharedMemorySize, LN_SMEM) != cudaSuccess)
      return SVDQ_ERR_CUDA;
    d->linear_attr = true;
  }
  LinearArgs a;
  a.SFx = SFx;
  a.SFw = SFw;
  a.bias = bias;
  a.Y = Y;
  a.y_fp32 = y_fp32;
  a.y_vec32 = (reinterpret_cast<uintptr_t>(Y) & 31u) == 0 ? 1 : 0;
  a.M = (int)M;
  a.N = (int)N;
  a.K = (int)K;
  a.r = r;
  a.gs = gs_x * gs_w;
  a.debug = debug;
  a.timeout_ns = timeout_ns ? timeout_ns : LN_DEFAULT_TIMEOUT_NS;
  if (pair) {
    const int64_t tiles = ((M + LP_BM - 1) / LP_BM) * ((N + LP_BN - 1) / LP_BN);
    const int64_t pairs = tiles < d->sms / 2 ? tiles : d->sms / 2;
    k_linear_pair<<<(int)(2 * pairs), LP_THREADS, LP_SMEM, s>>>(tm_xq, tm_wq, tm_las, tm_l2p, a);
  } else {
    const int64_t tiles = ((M + LN_BM - 1) / LN_BM) * ((N + LN_BN - 1) / LN_BN);
    const int grid = (int)(tiles < d->sms ? tiles : d->sms);
    k_linear<<<grid, LN_THREADS, LN_SMEM, s>>>(tm_xq, tm_wq, tm_las, tm_l2p, a);
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
    default: return "SVDQ_ERR_UNKNOWN";
  }
}

int svdq_version(void) { return 100; }

size_t svdq_sf_bytes(int64_t rows, int64_t K) {
  if (rows < 0 || K < 0 || K % 64 != 0) return 0;
  return (size_t)pad128(rows) * (size_t)(K / 16);
}

svdq_status svdq_pack_weight(const float* R, const uint16_t* L2b, int64_t K, int64_t N, int r, uint8_t* Wq,
                             uint8_t* SFw, float* gs_w, uint16_t* L2p, svdq_stream_t stream) {
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
  return launch_status();
}

svdq_status svdq_quantize_act(const uint16_t* X, int64_t M, int64_t K, const float* inv_s, float gs_x,
                              const uint16_t* L1fT, int r, float lr_scale, uint8_t* Xq, uint8_t* SFx, uint16_t* LAs,
                              svdq_stream_t stream) {
  svdq_status st = check_shape(M, 16, K, r);
  if (st != SVDQ_OK) return st;
  if (!X || !inv_s || !Xq || !SFx || (r > 0 && (!L1fT || !LAs))) return SVDQ_ERR_INVALID_ARG;
  if (!aligned16(X) || !aligned16(inv_s) || !aligned16(Xq) || !aligned16(SFx) ||
      (r > 0 && (!aligned16(L1fT) || !aligned16(LAs))))
    return SVDQ_ERR_MISALIGNED;
  int dev;
  DevInfo* d;
  if ((st = current_device(&dev, &d)) != SVDQ_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  switch (r) {
    case 0: return launch_qa<0>(d, 0, X, M, K, inv_s, gs_x, L1fT, lr_scale, Xq, SFx, LAs, s);
    case 16: return launch_qa<16>(d, 1, X, M, K, inv_s, gs_x, L1fT, lr_scale, Xq, SFx, LAs, s);
    case 32: return launch_qa<32>(d, 2, X, M, K, inv_s, gs_x, L1fT, lr_scale, Xq, SFx, LAs, s);
    case 48: return launch_qa<48>(d, 3, X, M, K, inv_s, gs_x, L1fT, lr_scale, Xq, SFx, LAs, s);
    case 64: return launch_qa<64>(d, 4, X, M, K, inv_s, gs_x, L1fT, lr_scale, Xq, SFx, LAs, s);
    case 80: return launch_qa<80>(d, 5, X, M, K, inv_s, gs_x, L1fT, lr_scale, Xq, SFx, LAs, s);
    case 96: return launch_qa<96>(d, 6, X, M, K, inv_s, gs_x, L1fT, lr_scale, Xq, SFx, LAs, s);
    case 112: return launch_qa<112>(d, 7, X, M, K, inv_s, gs_x, L1fT, lr_scale, Xq, SFx, LAs, s);
    case 128: return launch_qa<128>(d, 8, X, M, K, inv_s, gs_x, L1fT, lr_scale, Xq, SFx, LAs, s);
    default: return SVDQ_ERR_UNSUPPORTED_SHAPE;
  }
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
  if ((debug_flags & ~(LN_DBG_NO_LOADS | LN_DBG_FORCE_SINGLE | LN_DBG_FORCE_PAIR)) ||
      ((debug_flags & LN_DBG_FORCE_SINGLE) && (debug_flags & LN_DBG_FORCE_PAIR)))
    return SVDQ_ERR_INVALID_ARG;
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
  return (flags & svdq::ERR_TIMEOUT) ? SVDQ_ERR_TIMEOUT : SVDQ_OK;
}

}  // extern "C"
