/*
 * svdq.h -- C ABI of the B200 (sm_100a) SVDQuant W4A4 linear layer.
 *
 * The layer (SVDQuant review, §4.2, low-rank decomposition equation):
 *
 *     Y = Q(X_hat) Q(R)  +  (X_hat L1) L2  +  bias,     X_hat = X diag(s)^-1
 *
 * with the low-rank branch fused into the 4-bit branch as in §4.3 (Nunchaku):
 * the down-projection X_hat L1 is computed inside the activation-quantization
 * kernel and the up-projection (X_hat L1) L2 inside the 4-bit GEMM.
 * The offline decomposition (smoothing factors s, L1, L2, residual R) is
 * computed by the caller and passed in as data ("From SmoothQuant to
 * SVDQuant", section quantization scheme: weight-side quantities are static).
 *
 * Number formats (NVFP4, "From SmoothQuant to SVDQuant", section Personal view:
 * groups of 16 with a two-level scale; SVDQuant review §3: q_max = 6):
 *   - 4-bit codes are FP4 E2M1, two per byte along K, element 2j in the low
 *     nibble of byte j.  An M x K operand is stored as M rows of K/2 bytes.
 *   - one UE4M3 (unsigned E4M3) scale per 16 consecutive values along K,
 *     stored in the "MMA scale order" below; one float32 global scale per
 *     tensor, gs = amax / 2688 (1 when amax = 0).
 *   - per group: sb = UE4M3_rne_sat(amax_group * f32(1 / f32(6 gs))),
 *     d = f32(dec(sb) * gs), code = E2M1_rne_sat(x * f32(1/d)), all codes 0
 *     when sb = 0.  Every step is one correctly rounded float32 operation.
 *   - 16-bit tensors (X, L1f, L2, LAs, L2p, bias, bf16 Y) are bfloat16,
 *     passed as uint16_t bit patterns.
 *
 * MMA scale order (the byte order the block-scaled tcgen05 MMA consumes):
 * for an operand with `rows` rows and KS = K/16 scales per row, the buffer
 * has svdq_sf_bytes(rows, K) = ceil(rows/128)*128*KS bytes; scale (r, kk)
 * is at byte  ((r/128)*(KS/4) + kk/4)*512 + (r%32)*16 + ((r/32)%4)*4 + kk%4.
 * Bytes of padding rows (rows..ceil(rows/128)*128-1) are written as 0 by
 * the kernels that produce the buffer.
 *
 * Conventions for every call:
 *   - Pointers are device pointers unless stated; the caller owns and
 *     allocates every buffer, workspaces included; the library allocates no
 *     device memory.
 *   - Calls are asynchronous on `stream` (a cudaStream_t; NULL = legacy
 *     default stream).  Argument errors are returned before any launch;
 *     a launch failure returns SVDQ_ERR_CUDA.  Kernel-side faults that do not
 *     stop the kernel (a bounded wait that ran out) are reported by
 *     svdq_get_device_error().
 *   - Pointers must be 16-byte aligned (svdq_linear stores Y 32 bytes at a time
 *     when Y is 32-byte aligned, 16 bytes otherwise).  Shapes: K % 64 == 0,
 *     N % 16 == 0, r % 16 == 0 with 0 <= r <= 128, 1 <= K, N < 2^31, 0 <= M < 2^31.
 *     M = 0 (an empty batch) is a valid call of every per-forward entry point: it
 *     launches nothing and returns SVDQ_OK (buffer pointers may then be NULL).
 *   - Buffer sizes cannot be checked from pointers: every buffer must hold the
 *     shape the call states (a larger r than LAs / L2p were sized for makes the
 *     kernels read past them).
 *   - One device per call: the current device of the calling thread.
 *     Requires compute capability 10.0 (B200, sm_100a).
 */
#ifndef SVDQ_H_
#define SVDQ_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define SVDQ_API __attribute__((visibility("default")))
#else
#define SVDQ_API
#endif

typedef struct CUstream_st* svdq_stream_t;   /* same type as cudaStream_t */

typedef enum {
    SVDQ_OK = 0,
    SVDQ_ERR_INVALID_ARG = 1,        /* null pointer, negative size, bad flag          */
    SVDQ_ERR_UNSUPPORTED_SHAPE = 2,  /* K % 64, N % 16, r % 16, r > 128, size overflow */
    SVDQ_ERR_MISALIGNED = 3,         /* a pointer not 16-byte aligned                  */
    SVDQ_ERR_CUDA = 4,               /* a CUDA runtime/driver call or launch failed    */
    SVDQ_ERR_TIMEOUT = 5,            /* a kernel's bounded wait ran out (device error) */
    SVDQ_ERR_DEVICE = 6,             /* current device is not compute capability 10.x  */
    SVDQ_ERR_SCRATCH = 7,            /* shape needs more than the library's own scratch */
    SVDQ_ERR_CHECK = 8               /* debug build: a copy failed its bounds/alignment check */
} svdq_status;

/* Human-readable name of a status code (static string). */
SVDQ_API const char* svdq_status_string(int status);

/* Library ABI version (major * 100 + minor). */
SVDQ_API int svdq_version(void);

/* Bytes of a scale-factor buffer for a rows x K operand in MMA scale order
 * (0 if rows < 0 or K % 64 != 0). */
SVDQ_API size_t svdq_sf_bytes(int64_t rows, int64_t K);

/*
 * svdq_pack_weight -- static NVFP4 quantization of the residual weight
 * (SVDQuant review, §4.2: only the residual R is quantized to 4 bits;
 * "From SmoothQuant to SVDQuant", quantization scheme item 1: done offline).
 *
 *   R    [in]  float32, K x N row-major (N contiguous), finite values.
 *   L2b  [in]  bf16, r x N row-major: the up-projection factor L2 (may be
 *              NULL when r == 0).
 *   Wq   [out] uint8, N x K/2: E2M1 codes of R^T (row n holds column n of R).
 *   SFw  [out] uint8, svdq_sf_bytes(N, K): UE4M3 scales in MMA scale order.
 *   gs_w [out] float32 (one device float): the weight global scale,
 *              amax(|R|) / 2688; also used as the amax accumulator while the
 *              call runs, so it must not alias anything else.
 *   gs_w_host [out] HOST float or NULL.  When given, the call copies gs_w to
 *              it and synchronises `stream` before returning (the caller
 *              needs the value to form lr_scale for svdq_quantize_act and the
 *              scale argument of svdq_linear).  When NULL the call is
 *              asynchronous like the others.
 *   L2p  [out] bf16, N x r row-major: row n = L2b[:, n], the up-projection
 *              laid out K-major for the GEMM (NULL when r == 0).
 * Five launches (zero, amax, scale, encode, L2 layout).
 */
SVDQ_API svdq_status svdq_pack_weight(const float* R, const uint16_t* L2b, int64_t K, int64_t N, int r,
                             uint8_t* Wq, uint8_t* SFw, float* gs_w, float* gs_w_host, uint16_t* L2p,
                             svdq_stream_t stream);

/*
 * svdq_dequant_weight -- the value of a packed weight, Q(R), for the offline
 * refinement of the decomposition (SVDQuant review, §4.2: R is optimized
 * repeatedly to minimize the quantization error, which needs Q(R) itself).
 *
 *   Wq, SFw, gs_w [in] from svdq_pack_weight (gs_w the device float).
 *   Rq   [out] float32, K x N row-major:
 *              Rq[k, n] = f32(e2m1(code) * f32(dec(sb) * gs_w)), sign from the code.
 */
SVDQ_API svdq_status svdq_dequant_weight(const uint8_t* Wq, const uint8_t* SFw, const float* gs_w, int64_t K,
                                int64_t N, float* Rq, svdq_stream_t stream);

/*
 * MXFP4 form of the layer.  The pages name MXFP4 beside NVFP4 as a 4-bit
 * format the decomposition serves (WUSH summary page, format compatibility
 * and the MXFP4 / NVFP4 evaluations; "From SmoothQuant to SVDQuant", personal
 * view, on group sizes) without defining it; the reading taken is the
 * Microscaling (MX) FP4 format of its public specification:
 *   - blocks of 32 consecutive values along K, one E8M0 scale byte e per
 *     block standing for 2^(e - 127); no per-tensor scale;
 *   - X = floor(log2(amax_block)) - 2 clamped to [-127, 127], e = X + 127;
 *     code = E2M1_rne_sat(x * 2^-X) (the product is exact); a block whose
 *     values are all zero gets e = 0 and codes 0.
 * Codes are packed as for NVFP4.  Scales use the MMA scale order of the
 * NVFP4 header text with KS = K/32 scales per row (4 per 32-bit word, so an
 * atom of 512 bytes covers 128 rows x 128 values of K):
 *   svdq_mx_sf_bytes(rows, K) = ceil(rows/128)*128*(K/32) bytes.
 * Every MX call requires K % 128 == 0 (SVDQ_ERR_UNSUPPORTED_SHAPE otherwise).
 */
SVDQ_API size_t svdq_mx_sf_bytes(int64_t rows, int64_t K);

/*
 * svdq_pack_weight_mx -- MXFP4 quantization of the residual weight R
 * (K x N float32, N contiguous) into Wq (N x K/2 codes of R^T) and SFw
 * (svdq_mx_sf_bytes(N, K) bytes), plus the L2 layout of svdq_pack_weight
 * (L2b r x N -> L2p N x r; both NULL when r == 0).  Two launches; no
 * reduction over R (there is no global scale).
 */
SVDQ_API svdq_status svdq_pack_weight_mx(const float* R, const uint16_t* L2b, int64_t K, int64_t N, int r,
                                         uint8_t* Wq, uint8_t* SFw, uint16_t* L2p, svdq_stream_t stream);

/*
 * svdq_quantize_act_mx -- svdq_quantize_act with the MXFP4 codec: X_hat =
 * f32(X * inv_s) quantized in blocks of 32 to Xq (M x K/2) and SFx
 * (svdq_mx_sf_bytes(M, K)); the fused down-projection, LAs and the workspace
 * are exactly those of svdq_quantize_act (lr_scale is usually 1, since no
 * global scale multiplies the product).
 */
SVDQ_API svdq_status svdq_quantize_act_mx(const uint16_t* X, int64_t M, int64_t K, const float* inv_s,
                                          const uint16_t* L1fT, int r, float lr_scale, uint8_t* Xq,
                                          uint8_t* SFx, uint16_t* LAs, void* workspace, size_t workspace_bytes,
                                          svdq_stream_t stream);

/*
 * svdq_linear_mx -- svdq_linear on MXFP4 operands (the tcgen05 MMA of kind
 * mxf4 with E8M0 block scales, one scale per 32 values):
 *   Y = sum_k dec(Xq) dec(SFx) dec(Wq) dec(SFw) + LAs . L2p^T + bias,
 * rounded once to bf16 (y_fp32 == 0) or float32.  Arguments as svdq_linear
 * without the global scales.
 */
SVDQ_API svdq_status svdq_linear_mx(const uint8_t* Xq, const uint8_t* SFx, const uint8_t* Wq, const uint8_t* SFw,
                                    const uint16_t* LAs, const uint16_t* L2p, int r, const uint16_t* bias, void* Y,
                                    int y_fp32, int64_t M, int64_t N, int64_t K, svdq_stream_t stream);

/*
 * svdq_quantize_act -- activation kernel with the fused down-projection
 * (SVDQuant review, §4.3: the down-projection is merged into the
 * quantization kernel so the activations are read once).
 *
 *   X        [in]  bf16, M x K row-major (read from HBM exactly once).
 *   inv_s    [in]  float32, K: reciprocal smoothing factors 1/s_j;
 *                  X_hat = f32(X * inv_s) (the smoothing divide).
 *   gs_x     [in]  host float: static activation global scale (calibration).
 *   L1fT     [in]  bf16, r x K row-major (K contiguous): (diag(s)^-1 L1)^T,
 *                  the down factor with the smoothing folded in, so that
 *                  X_hat L1 = X L1f.  May be NULL when r == 0.
 *   lr_scale [in]  host float: f32(1 / (gs_x * gs_w)); the low-rank output
 *                  is pre-scaled by it so the GEMM can add both branches in
 *                  one accumulator and scale once by gs_x * gs_w.
 *   Xq       [out] uint8, M x K/2: E2M1 codes of X_hat.
 *   SFx      [out] uint8, svdq_sf_bytes(M, K): UE4M3 scales, MMA scale order.
 *   workspace [in/out] device memory of at least
 *                  svdq_quantize_act_workspace_bytes(M, K, r) bytes (NULL and 0
 *                  when r == 0).  When a row block's 128 rows are too few to
 *                  fill the GPU, up to 8 CTAs share the block's K axis and add
 *                  their partial down-projections here; the first bytes are one
 *                  counter per row block that the kernel leaves at 0.  Zero the
 *                  whole workspace once after allocating it (and again after a
 *                  call that reported SVDQ_ERR_TIMEOUT); calls on streams that
 *                  may overlap need workspaces of their own.
 *   LAs      [out] bf16, M x 2r: the hi/lo pair of
 *                  v = f32(lr_scale * (X L1f)[m, :]) (fp32 accumulation),
 *                  hi = bf16_rne(v), lo = bf16_rne(v - hi), interleaved by 16
 *                  columns: LAs[m, 32j + t] = hi(v[16j + t]) and
 *                  LAs[m, 32j + 16 + t] = lo(v[16j + t]) for t < 16 (the order
 *                  svdq_linear's rank stage reads).  NULL when r == 0.
 * Launched as a programmatic dependent of the previous kernel on the stream
 * (its set-up overlaps that kernel's tail; it reads X only after that kernel
 * has finished).
 */
SVDQ_API svdq_status svdq_quantize_act(const uint16_t* X, int64_t M, int64_t K, const float* inv_s,
                              float gs_x, const uint16_t* L1fT, int r, float lr_scale,
                              uint8_t* Xq, uint8_t* SFx, uint16_t* LAs,
                              void* workspace, size_t workspace_bytes, svdq_stream_t stream);

/* Bytes of the workspace svdq_quantize_act and svdq_lowrank_down need for M rows of K columns at
 * rank r (0 when r == 0; 0 for a shape the calls reject).  Independent of the device. */
SVDQ_API size_t svdq_quantize_act_workspace_bytes(int64_t M, int64_t K, int r);

/*
 * svdq_quantize_act_noalloc -- svdq_quantize_act for callers that cannot
 * allocate device memory.  (The pages have no counterpart: this is an entry
 * point of the library, not a step of the method.)
 *
 * Some callers have no way to obtain a workspace: a host application whose
 * memory pool owns all of the device memory and forbids other allocations, or
 * a runtime that must not allocate once it is running (cudaMalloc can
 * synchronise the device and takes an unbounded time).  This entry point takes
 * the same arguments as svdq_quantize_act minus the workspace and allocates
 * nothing: the partial sums of the K-split down-projection live in a scratch
 * array the library declares in device memory, SVDQ_NOALLOC_SCRATCH_BYTES
 * (8 MiB) on every GPU that loads the library, held until the process exits.
 *
 *   - A shape whose K-split needs more than that (about 8 MiB of partial sums
 *     plus one counter per 128 rows; e.g. M = 4608, r = 32 needs 2.4 MiB) is
 *     refused with SVDQ_ERR_SCRATCH before anything is launched.
 *   - The first call on a device looks up the array's device address
 *     (cudaGetSymbolAddress) with that device current; make that first call
 *     before any stream capture on the device.
 *   - Every call on a device shares the one array.  Each call clears the
 *     counters it needs (an asynchronous memset on `stream`); calls whose
 *     kernels overlap on the GPU (different streams, or graphs replayed
 *     concurrently) race on the array and give undefined LAs.
 *   - Results are identical to svdq_quantize_act's.
 */
#define SVDQ_NOALLOC_SCRATCH_BYTES (8u << 20)
SVDQ_API svdq_status svdq_quantize_act_noalloc(const uint16_t* X, int64_t M, int64_t K, const float* inv_s,
                              float gs_x, const uint16_t* L1fT, int r, float lr_scale,
                              uint8_t* Xq, uint8_t* SFx, uint16_t* LAs, svdq_stream_t stream);

/*
 * svdq_linear -- block-scaled NVFP4 GEMM on the tcgen05 tensor cores with the
 * up-projection fused into the same TMEM accumulator (SVDQuant review, §4.3:
 * the up-projection is merged into the 4-bit GEMM kernel):
 *
 *   acc  = sum_k dec(Xq) dec(SFx) dec(Wq) dec(SFw)  +  LAs . L2p^T
 *   Y    = f32(gs_x * gs_w) * acc + bias             (rounded once to bf16, or fp32)
 *
 *   Xq, SFx     [in] from svdq_quantize_act;  Wq, SFw, L2p [in] from svdq_pack_weight.
 *   gs_x, gs_w  [in] host floats.
 *   LAs, L2p    [in] may be NULL when r == 0 (plain NVFP4 GEMM).
 *   bias        [in] bf16, N, or NULL.
 *   Y           [out] M x N row-major: bf16 when y_fp32 == 0, float32 when 1.
 * Persistent, warp-specialised kernel: one CTA per SM, 128 x 256 output tiles,
 * launched as a programmatic dependent of the previous kernel on the stream
 * (set-up overlaps that kernel's tail; inputs are read and Y written only
 * after it has finished).
 */
SVDQ_API svdq_status svdq_linear(const uint8_t* Xq, const uint8_t* SFx, float gs_x,
                        const uint8_t* Wq, const uint8_t* SFw, float gs_w,
                        const uint16_t* LAs, const uint16_t* L2p, int r,
                        const uint16_t* bias, void* Y, int y_fp32,
                        int64_t M, int64_t N, int64_t K, svdq_stream_t stream);

/*
 * svdq_linear_gelu_quantize -- the first layer of an MLP pair with the next
 * layer's input preparation fused into its epilogue.  The pages fuse each
 * layer's low-rank down-projection into its activation quantization so that
 * the 16-bit activations are read from memory once (SVDQuant review, §4.3
 * Nunchaku); between two layers of a diffusion transformer's MLP (FLUX.1,
 * "SVDQuant: Absorbing Outliers by Low-Rank Components for 4-Bit Diffusion
 * Models", abstract) the same reasoning removes the write and re-read of the
 * intermediate activations altogether.  The pages define neither the
 * activation nor this fusion; the readings taken:
 *   - the activation is GELU in its tanh form, on the bf16-rounded output of
 *     this layer, with its result rounded to bf16 (what an unfused pair writes
 *     and reads): y = bf16(f32(gs_x gs_w acc + bias)), x2 = bf16(GELU(y));
 *   - GELU(y) is the fixed binary32 sequence
 *       t = C2 (y + C1 y^3) (products and sums each rounded: y2 = y*y, y3 = y2*y,
 *       w = C1*y3, inner = y + w, t = C2*inner), e = exp(-|t|), q = 1/(1 + e),
 *       GELU = y * (t >= 0 ? q : e*q),
 *     C1 = f32(0.044715), C2 = f32(2 sqrt(2/pi)), exp by Cody-Waite reduction
 *     and its degree-7 Taylor polynomial (0 below -80), so that its value is
 *     reproducible bit for bit;
 *   - the next layer then sees exactly what svdq_quantize_act would produce
 *     from x2: codes and scales of f32(x2 * inv_s2) with global scale gs_x2,
 *     and LAs2 = hi/lo of f32(lr_scale2 * x2 L1f2).
 *
 * Arguments as svdq_linear (this layer: Xq, SFx, gs_x, Wq, SFw, gs_w, LAs, L2p,
 * r, bias, M, N, K; no Y), plus the next layer's constants and outputs:
 *   inv_s2  [in]  float32, N: the next layer's smoothing factors 1/s.
 *   gs_x2   [in]  host float > 0: the next layer's activation global scale.
 *   L1fT2   [in]  bf16, r2 x N: the next layer's down factor (NULL if r2 == 0).
 *   r2, lr_scale2: the next layer's rank (0, 16 or 32) and LAs pre-scale.
 *   Xq2     [out] uint8, M x N/2;  SFx2 [out] uint8, svdq_sf_bytes(M, N).
 *   LAs2    [out] bf16, M x 2 r2 (NULL if r2 == 0).
 *   workspace [scratch] svdq_linear_gelu_quantize_workspace_bytes(M, N, r2)
 *           bytes (float32 partial sums, one M x r2 slice per 256 output
 *           columns; no initial contents needed; NULL if r2 == 0).
 * Requires N % 64 == 0 (N is the next layer's K).  Two launches: the GEMM
 * (its epilogue computes GELU, the next layer's codes and scales and its
 * down-projection over each 256-column tile) and a reduction of the slices
 * in a fixed order into LAs2.
 */
SVDQ_API size_t svdq_linear_gelu_quantize_workspace_bytes(int64_t M, int64_t N, int r2);
SVDQ_API svdq_status svdq_linear_gelu_quantize(const uint8_t* Xq, const uint8_t* SFx, float gs_x, const uint8_t* Wq,
                                               const uint8_t* SFw, float gs_w, const uint16_t* LAs,
                                               const uint16_t* L2p, int r, const uint16_t* bias, int64_t M,
                                               int64_t N, int64_t K, const float* inv_s2, float gs_x2,
                                               const uint16_t* L1fT2, int r2, float lr_scale2, uint8_t* Xq2,
                                               uint8_t* SFx2, uint16_t* LAs2, void* workspace,
                                               size_t workspace_bytes, svdq_stream_t stream);

/*
 * svdq_gelu_bf16 -- Y = bf16(GELU(X)) element-wise on n bf16 values, with the
 * GELU of svdq_linear_gelu_quantize: the activation of the unfused MLP pair
 * (svdq_linear writes the first layer's Y, this kernel applies GELU, and
 * svdq_quantize_act reads the result).  X and Y 16-byte aligned; n >= 0.
 */
SVDQ_API svdq_status svdq_gelu_bf16(const uint16_t* X, int64_t n, uint16_t* Y, svdq_stream_t stream);

/*
 * Calibration on the GPU ("From SmoothQuant to SVDQuant", quantization scheme:
 * the smoothing factors, the low-rank split and the activation global scale are
 * fixed offline from calibration data; section Smooth Quant (W8A8): the
 * per-channel factor s_j = max|X_j|^alpha / max|W_j|^(1 - alpha)).  These calls
 * compute the statistics and the smoothing; the truncated SVD of W_hat is done
 * by the caller (the Python layer uses a randomized range finder on the GPU).
 * Every maximum is exact (maxima merge by an order-independent atomic max).
 *
 * svdq_calib_absmax_cols: amax_x[j] = max over rows of |X[m, j]|, X bf16 M x K
 *   (K % 8 == 0, X 16-byte aligned).  accumulate = 1 merges into amax_x (max with
 *   its contents: several calibration batches in turn), 0 starts from zero.
 * svdq_calib_absmax_rows: amax_w[j] = max over n of |W[j, n]|, W float64 K x N.
 * svdq_calib_smooth: s_j = amax_x[j]^alpha / amax_w[j]^(1 - alpha) in float64
 *   (1 where either maximum is 0), inv_s[j] = f32(1 / s_j); 0 <= alpha <= 1.
 * svdq_calib_scale_rows: W_hat = diag(s) W, float64 K x N (one rounding each).
 * svdq_calib_act_amax: amax = max |f32(X * inv_s)| over a bf16 M x K X (the
 *   activation global scale is f32(amax / 2688)); accumulate as above.
 */
SVDQ_API svdq_status svdq_calib_absmax_cols(const uint16_t* X, int64_t M, int64_t K, float* amax_x, int accumulate,
                                            svdq_stream_t stream);
SVDQ_API svdq_status svdq_calib_absmax_rows(const double* W, int64_t K, int64_t N, double* amax_w,
                                            svdq_stream_t stream);
SVDQ_API svdq_status svdq_calib_smooth(const float* amax_x, const double* amax_w, int64_t K, double alpha,
                                       double* s, float* inv_s, svdq_stream_t stream);
SVDQ_API svdq_status svdq_calib_scale_rows(const double* W, const double* s, int64_t K, int64_t N, double* W_hat,
                                           svdq_stream_t stream);
SVDQ_API svdq_status svdq_calib_act_amax(const uint16_t* X, int64_t M, int64_t K, const float* inv_s, float* amax,
                                         int accumulate, svdq_stream_t stream);

/*
 * svdq_lowrank_down -- the low-rank down-projection as a kernel of its own: the
 * unfused form of the branch (SVDQuant review, §4.3: without fusion the branch
 * re-reads the 16-bit activations from memory, which is what the fused
 * svdq_quantize_act avoids).  Kept to measure what the fusion buys.
 *
 *   X, M, K, L1fT, r, lr_scale, workspace: as in svdq_quantize_act (r >= 16).
 *   LAs [out] bf16, M x 2r, the same layout and values as svdq_quantize_act's
 *       LAs for the same inputs (the two kernels share the down-projection
 *       code; this one skips the quantization).
 */
SVDQ_API svdq_status svdq_lowrank_down(const uint16_t* X, int64_t M, int64_t K, const uint16_t* L1fT, int r,
                              float lr_scale, uint16_t* LAs, void* workspace, size_t workspace_bytes,
                              svdq_stream_t stream);

/*
 * svdq_lowrank_up -- the low-rank up-projection as a kernel of its own, adding
 * into an existing output (the unfused form of the branch, SVDQuant review,
 * §4.3: without fusion the branch reads and rewrites the output):
 *
 *   Y[m, n] = round(gs * sum_t (hi + lo)(LAs)[m, t] * L2p[n, t] + Y[m, n])
 *
 *   LAs  [in]  bf16, M x 2r, the layout of svdq_quantize_act / svdq_lowrank_down.
 *   L2p  [in]  bf16, N x r, from svdq_pack_weight (r >= 16).
 *   gs   [in]  host float: the scale of the product (gs_x * gs_w when LAs was
 *              pre-scaled by lr_scale = 1 / (gs_x * gs_w); 1 when it was not).
 *   Y    [in/out] M x N row-major, bf16 (y_fp32 = 0) or float32 (y_fp32 = 1),
 *              read and rewritten; rounded once to its own type.
 * The tcgen05 GEMM kernel of svdq_linear with no 4-bit tiles, only the rank
 * tiles, and an epilogue that reads Y instead of the bias.
 */
SVDQ_API svdq_status svdq_lowrank_up(const uint16_t* LAs, const uint16_t* L2p, int r, float gs, void* Y, int y_fp32,
                            int64_t M, int64_t N, svdq_stream_t stream);

/*
 * svdq_map_cache_stats -- counters of the library's host cache of TMA tensor
 * maps (64 entries, keyed by address, element type, shape, strides, box and
 * swizzle; least recently used replaced): a call whose buffers and shapes were
 * seen before reuses the encoded maps instead of encoding them again.  The
 * pages have no counterpart (it is host-side launch cost).  hits / misses may
 * be NULL.
 */
SVDQ_API void svdq_map_cache_stats(uint64_t* hits, uint64_t* misses);

/*
 * svdq_get_device_error -- synchronises `stream`, then reads and clears the
 * library's device error word on the current device.  Returns SVDQ_OK, or
 * SVDQ_ERR_TIMEOUT when a kernel's bounded wait on a barrier ran out (the
 * kernel then stopped early; its outputs are undefined), or SVDQ_ERR_CUDA.
 * If `site` is not NULL it receives an identifier of the wait that ran out.
 */
SVDQ_API svdq_status svdq_get_device_error(svdq_stream_t stream, int* site);

/*
 * svdq_build_flags -- bit 0 set in the debug build (libsvdq_check.so, compiled
 * with -DSVDQ_CHECK): every TMA / bulk copy of the kernels is checked before it
 * is issued (innermost coordinate aligned to 16 bytes, coordinates and sources
 * inside their tensors, destination inside the launch's shared memory); a
 * failed check skips the copy and records SVDQ_ERR_CHECK with the check's site
 * (read by svdq_get_device_error; the kernel's bounded waits then end it).
 * The pages have no counterpart (it is a debugging aid).
 */
SVDQ_API int svdq_build_flags(void);

/*
 * svdq_linear_debug -- svdq_linear with test hooks, for the fault-path tests.
 *   debug_flags bit 0: the load warp issues no loads, so the MMA warp's first
 *                      wait can never complete and must run out.
 *               bit 1: (debug build only) the first A box of every tile is
 *                      requested at a misaligned innermost coordinate; the
 *                      build's copy check skips it and records SVDQ_ERR_CHECK.
 *                      SVDQ_ERR_INVALID_ARG in the regular build.
 *   Any other bit is SVDQ_ERR_INVALID_ARG.
 *   timeout_ns: bound of every barrier wait (0 = the default of 2 s).
 * Otherwise identical to svdq_linear.
 */
SVDQ_API svdq_status svdq_linear_debug(const uint8_t* Xq, const uint8_t* SFx, float gs_x,
                              const uint8_t* Wq, const uint8_t* SFw, float gs_w,
                              const uint16_t* LAs, const uint16_t* L2p, int r,
                              const uint16_t* bias, void* Y, int y_fp32,
                              int64_t M, int64_t N, int64_t K,
                              int debug_flags, uint64_t timeout_ns, svdq_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* SVDQ_H_ */
