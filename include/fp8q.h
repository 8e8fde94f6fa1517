/*
 * fp8q.h -- C ABI of the B200 (sm_100a) FP8 W8A8 linear layer library, libfp8q.so.
 *
 * The layer is the one Llama-3.x "FP8-Dynamic" and "FP8-Block" checkpoints use:
 *
 *   - Weights are E4M3 codes with one scale per output channel, taken from a
 *     minmax observer ("Llama-3.1-8B-Instruct-FP8-Dynamic" explainer, FP8 动态量化
 *     table, weights row; "Llama-3.1-70B-FP8-Dynamic" explainer, section 1.2), or
 *     one scale per 128 x 128 block ("Llama-3.2-3B-Instruct-FP8-Block" explainer,
 *     quantization_config table, block_structure [128, 128]).
 *   - Activations are quantized at run time, one dynamic scale per token (the
 *     FP8-Dynamic table's input_activations row; 70B explainer FAQ Q2), or one
 *     per group of 128 input features (FP8-Block table, input activations row).
 *   - E4M3 has 4 exponent and 3 mantissa bits and tops out at 448 ("Llama 3 精读实录",
 *     section 2.1).  Codes are the E4M3FN bit patterns (no infinities; 0x7F and
 *     0xFF are NaN and never produced for finite input).
 *   - lm_head stays in high precision: it is not passed to this library (same
 *     tables, ignore row).
 *
 * Arithmetic, identical on every path:
 *   amax  = max |x| over the unit (row, 128-group or 128x128 block), exact in fp32
 *   scale = amax / 448 as one IEEE fp32 division; 1.0 when amax == 0
 *   code  = E4M3(x / scale): IEEE fp32 quotient, then round to nearest even,
 *           saturating to +-448, sign kept (-0 is 0x80)
 *   Y[m,n] = bf16_rne( acc[m,n] * x_scale[m] * w_scale[n] ),
 *           acc = fp32 sum over k of E4M3(xq[m,k]) * E4M3(wq[n,k]) (channel mode)
 *   Y[m,n] = bf16_rne( sum_kb  x_scale[m,kb] * w_scale[n/128,kb] * acc_kb[m,n] )
 *           with acc_kb the fp32 sum over the 128-wide K slice kb (block mode)
 *
 * Conventions for every entry point:
 *   - All data pointers are DEVICE pointers owned by the caller.  The library
 *     never allocates, frees or synchronizes; work is enqueued on `stream`
 *     (a cudaStream_t passed as void*; NULL is the legacy default stream).
 *   - Matrices are row-major; ld* arguments are row strides in ELEMENTS.
 *   - Arguments are checked before anything is launched.  A bad argument
 *     returns an error status and launches nothing.  A launch failure returns
 *     FP8Q_ERR_CUDA.  Errors that happen later on the device surface at the
 *     caller's next synchronization; a kernel whose internal wait runs out
 *     (about 4 s, which only a broken machine reaches) sets a device-side
 *     error word that fp8q_device_error() reads.
 *   - The calls are thread-safe; they keep no state between calls other than
 *     the device error word and a cached device-attribute table.
 */
#ifndef FP8Q_H_
#define FP8Q_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define FP8Q_API __attribute__((visibility("default")))
#else
#define FP8Q_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    FP8Q_OK = 0,
    FP8Q_ERR_INVALID_ARG = 1,     /* null pointer, negative size, bad mode, ...        */
    FP8Q_ERR_UNSUPPORTED = 2,     /* valid but outside what the kernels cover          */
    FP8Q_ERR_MISALIGNED = 3,      /* pointer or stride breaks a 16-byte requirement     */
    FP8Q_ERR_CUDA = 4,            /* a CUDA runtime/driver call failed                  */
    FP8Q_ERR_DEVICE_TIMEOUT = 5   /* a kernel gave up waiting (see fp8q_device_error)   */
} fp8q_status;

typedef enum {
    FP8Q_CHANNEL_TOKEN = 0,       /* W: one scale per output channel; X: one per token  */
    FP8Q_BLOCK128 = 1,            /* W: one per 128x128 block;  X: one per 128-group     */
    /* Option, OR'ed into the mode of fp8_quant_weight / fp8_quant_act: round
     * every scale to bf16 before the codes are computed (the FP8 checkpoints
     * store bf16 scales), so the codes are those a bf16-scale checkpoint holds.
     * A scale that rounds to zero becomes 1.  fp8_linear accepts and ignores it. */
    FP8Q_SCALE_BF16 = 0x10
} fp8q_mode;

/*
 * fp8_quant_weight -- quantize a bf16 weight W[N, K] (nn.Linear layout, out x in).
 *
 *   W_bf16   [N, ldw] bf16, read-only.  ldw >= K, (ldw * 2) % 16 == 0, 16-byte aligned.
 *   Wq       [N, ldwq] uint8 E4M3 codes, written.  ldwq >= K, ldwq % 16 == 0, 16-byte aligned.
 *   w_scale  fp32, written:  [N]                              (FP8Q_CHANNEL_TOKEN)
 *                            [ceil(N/128), K/128] row-major   (FP8Q_BLOCK128)
 *   Requirements: N >= 0, K > 0, K % 16 == 0; K % 128 == 0 in block mode.
 *   In block mode the last row-block may hold fewer than 128 rows; its amax
 *   covers the rows that exist.
 */
FP8Q_API fp8q_status fp8_quant_weight(const void* W_bf16, int64_t N, int64_t K, int64_t ldw, int mode,
                             uint8_t* Wq, int64_t ldwq, float* w_scale, void* stream);

/*
 * fp8_quant_act -- quantize bf16 activations X[M, K] (one row per token).
 *
 *   X_bf16   [M, ldx] bf16, read-only.  Same stride/alignment rules as W.
 *   Xq       [M, ldxq] uint8 codes, written.
 *   x_scale  fp32, written:  [M]                  (FP8Q_CHANNEL_TOKEN, per token)
 *                            [M, K/128] row-major (FP8Q_BLOCK128, per 128-group)
 *   Requirements: M >= 0 (M == 0 is a no-op), K > 0, K % 16 == 0;
 *   K % 128 == 0 in block mode.
 */
FP8Q_API fp8q_status fp8_quant_act(const void* X_bf16, int64_t M, int64_t K, int64_t ldx, int mode,
                          uint8_t* Xq, int64_t ldxq, float* x_scale, void* stream);

/*
 * fp8_quant_act_static -- quantize bf16 activations with one fixed scale.
 *
 * The static alternative to the dynamic per-token scheme: "Llama 3 精读实录"
 * section 2 calibrates each tensor offline from percentiles of a calibration
 * set (its 0.1% and 99.9% quantiles as the range, not min/max).  Every element
 * is coded as E4M3(fl32(x / scale)), saturating beyond the range.
 *   X_bf16, Xq  as fp8_quant_act.
 *   scale       > 0, finite: the calibrated scale (range / 448).
 *   x_scale     [M] fp32, written with `scale` when not NULL, so that
 *               fp8_linear in FP8Q_CHANNEL_TOKEN mode consumes Xq unchanged.
 *   Requirements: M >= 0 (M == 0 is a no-op), K > 0, K % 16 == 0.
 */
FP8Q_API fp8q_status fp8_quant_act_static(const void* X_bf16, int64_t M, int64_t K, int64_t ldx, float scale,
                                          uint8_t* Xq, int64_t ldxq, float* x_scale, void* stream);

/*
 * fp8_calibrate_static_scale -- the static scale fp8_quant_act_static takes,
 * from a calibration tensor: "Llama 3 精读实录" section 2 uses its 0.1% and
 * 99.9% quantiles as the range instead of min / max.  Offline, once per tensor.
 *   q(p)   = v[i] + (v[j] - v[i]) * (p (n-1) - i),  i = floor(p (n-1)),
 *            j = min(i + 1, n - 1), v the n = M*K values sorted ascending (double)
 *   amax   = max(|q(lo)|, |q(hi)|);   scale = fl32(fl32(amax) / 448), 1 when amax == 0
 * The order statistics are exact: the kernels count the 65536 bf16 bit patterns.
 *   X_bf16  [M, ldx] bf16, read-only, 16-byte aligned, ldx >= K, ldx % 8 == 0.
 *   lo, hi  quantile levels in [0, 1] (0.001 and 0.999 for the pages' range).
 *   hist    device workspace of 65536 uint32 counts (262144 bytes), 4-byte
 *           aligned, zero-filled before its first use; every completed call
 *           leaves it all zero.  Not shared by concurrent calls.
 *   scale   one fp32 in device memory, written.
 * Requirements: M >= 1, K >= 1, K % 8 == 0, M * K < 2^32 (FP8Q_ERR_UNSUPPORTED
 * above).  Values must be finite.
 */
FP8Q_API fp8q_status fp8_calibrate_static_scale(const void* X_bf16, int64_t M, int64_t K, int64_t ldx, double lo,
                                                double hi, uint32_t* hist, float* scale, void* stream);

/*
 * fp8_rmsnorm_quant_act -- RMSNorm of bf16 activations, then per-token E4M3
 * quantization of the result, in one pass (the normalised bf16 rows are not
 * written).  Llama 3 normalises with RMSNorm (eps 1e-5) before attention and
 * before the MLP and keeps it in BF16 ("Llama 3 精读实录", sections 1.3 and 5),
 * so this produces exactly the codes and scales that fp8_quant_act in
 * FP8Q_CHANNEL_TOKEN mode gives for the bf16 RMSNorm output.
 *
 *   X_bf16     [M, ldx] bf16 hidden states, read-only (rules as fp8_quant_act).
 *   gamma_bf16 [K] bf16 RMSNorm weight, 16-byte aligned.
 *   eps        >= 0, finite (1e-5 for Llama 3).
 *   Xq, x_scale as fp8_quant_act in FP8Q_CHANNEL_TOKEN mode ([M] scales).
 *   rstd       [M] fp32, written when not NULL: the row's 1 / sqrt(ms + eps).
 *   Per row:  ms   = the mean over the row of x^2, rounded once to fp32
 *             rstd = 1 / sqrt(fl32(ms + eps)), correctly rounded fp32
 *             y    = bf16(gamma * bf16(x * rstd))           (fp32 products)
 *             codes and scale of y as fp8_quant_act.
 *   The squares are exact in fp64 and summed in fp64, so ms is the exactly
 *   rounded mean except for a mean within a few fp64 roundings of an fp32
 *   rounding boundary (then it may be one fp32 step off, and rstd with it).
 *   Everything after rstd is exact, so rstd determines y and the codes.  Rows
 *   whose mean of squares overflows fp32 are outside the contract.
 *   Requirements: M >= 0 (M == 0 is a no-op), K > 0, K % 16 == 0, and
 *   K <= 65536 (FP8Q_ERR_UNSUPPORTED above).
 */
FP8Q_API fp8q_status fp8_rmsnorm_quant_act(const void* X_bf16, const void* gamma_bf16, int64_t M, int64_t K,
                                           int64_t ldx, float eps, uint8_t* Xq, int64_t ldxq, float* x_scale,
                                           float* rstd, void* stream);

/*
 * fp8_linear -- Y[M, N] = dequant(Xq) . dequant(Wq)^T in bf16, on tcgen05 tensor cores.
 *
 *   Xq        [M, K] uint8 codes, contiguous (row stride K), 16-byte aligned.
 *   x_scale   [M] or [M, K/128] fp32 (as written by fp8_quant_act in `mode`).
 *   Wq        [N, K] uint8 codes, contiguous, 16-byte aligned.
 *   w_scale   [N] or [ceil(N/128), K/128] fp32 (as written by fp8_quant_weight).
 *   Y_bf16    [M, ldy] bf16, written.  ldy >= N, (ldy * 2) % 16 == 0, 16-byte aligned.
 *   workspace device scratch of at least fp8_linear_workspace_size(M, N, K, mode)
 *             bytes, 16-byte aligned (may be NULL when that size is 0).  For
 *             M <= 64 it is required: a NULL or misaligned one is refused
 *             before anything touches the device.  For M > 64 it is optional:
 *             a nonzero size means the stream-K prefill schedule is switched
 *             on (environment FP8Q_PREFILL_STREAMK=1; off by default) for this
 *             shape (channel mode, few 256 x 256 tiles per CTA pair) and runs
 *             when the workspace is given; without it (NULL, or shorter) the
 *             data-parallel schedule runs, with the same result up to the
 *             order of the fp32 sums.  It holds
 *             the split-K arrival counters and fp32 partial sums of the small-M
 *             (decode) path.  It must be zero-filled before its first use; every
 *             completed call leaves it all zero again, so one zeroed buffer
 *             serves any sequence of calls (of any shape) on one stream.  After
 *             a call that failed on the device (fp8q_device_error nonzero), zero
 *             it again.  Two calls that run concurrently must not share one
 *             workspace.
 *   Requirements: M >= 0 (M == 0 is a no-op), N > 0, K > 0, K % 16 == 0,
 *   N % 16 == 0; K % 128 == 0 in block mode.  The mode must be the one both
 *   operands were quantized with.
 *   Dispatch: M <= 64 takes the decode kernel (weights streamed once, swap-AB,
 *   stream-K split over all SMs; the last warp to finish a weight tile's
 *   channels adds its partial sums in a fixed order, so results are
 *   deterministic; small block-scaled problems split each weight tile's K over
 *   the CTAs of one thread-block cluster instead, summed in distributed shared
 *   memory, and leave the workspace untouched); larger M takes the
 *   persistent warp-specialised prefill kernels, with 256 x 256 tiles per CTA
 *   pair, data-parallel or stream-K
 *   (parts of a tile summed in a fixed order by the last pair to finish it).
 */
FP8Q_API fp8q_status fp8_linear(const uint8_t* Xq, const float* x_scale, const uint8_t* Wq,
                       const float* w_scale, int64_t M, int64_t N, int64_t K, int mode,
                       void* Y_bf16, int64_t ldy, void* workspace, size_t workspace_bytes,
                       void* stream);

/*
 * fp8_linear_swiglu -- the Llama MLP's gate and up projections and their
 * SwiGLU combination in one kernel ("Llama 3 精读实录" section 1.3: gate and up
 * computed separately, then silu(gate) * up):
 *   g = bf16(Xq . Wq_gate^T scaled),  u = bf16(Xq . Wq_up^T scaled)   (as fp8_linear)
 *   Y = bf16( bf16(silu(g)) * u ),   silu(v) = v / (1 + e^-v)
 * Only Y ([M, N], the down projection's input) is written.
 *   Xq, x_scale      as fp8_linear, FP8Q_CHANNEL_TOKEN scales ([M]).
 *   Wq_gate, Wq_up   [N, K] codes of the two weights (contiguous, 16-byte aligned);
 *   w_scale_gate/up  [N] fp32 per-channel scales.
 *   Y_bf16           [M, ldy] bf16, written (rules as fp8_linear).
 * Requirements as fp8_linear in channel mode.  Any M >= 1 runs the CTA-pair
 * prefill schedule (256 tokens x 128 channels per pair).  silu uses the fast
 * exponential; g and u match fp8_linear's outputs.  No workspace.
 */
FP8Q_API fp8q_status fp8_linear_swiglu(const uint8_t* Xq, const float* x_scale, const uint8_t* Wq_gate,
                                       const float* w_scale_gate, const uint8_t* Wq_up, const float* w_scale_up,
                                       int64_t M, int64_t N, int64_t K, void* Y_bf16, int64_t ldy, void* stream);

/*
 * fp8_linear_w8a16 -- weight-only FP8: the layer as GPUs without FP8 tensor
 * cores run these checkpoints ("Llama-3.1-70B-FP8-Dynamic" explainer, section
 * 三's GPU choice list and FAQ Q1: the FP8 weights are dequantized at compute
 * time).  The activations stay bf16:
 *   Y[m, n] = bf16( w_scale[n] * sum_k X[m, k] * E4M3(Wq[n, k]) ),
 * products and sums in fp32 (any order).
 *   X_bf16   [M, ldx] bf16 activations, 16-byte aligned, ldx >= K, ldx % 8 == 0.
 *   Wq       [N, K] uint8 codes, contiguous, 16-byte aligned (fp8_quant_weight,
 *            FP8Q_CHANNEL_TOKEN).
 *   w_scale  [N] fp32 per-channel scales.
 *   Y_bf16   [M, ldy] bf16, written; ldy >= N, 2-byte aligned.
 *   workspace  device scratch of fp8_linear_w8a16_workspace_size(M, N, K)
 *            bytes (NULL when that is 0), 16-byte aligned, with fp8_linear's
 *            contract: zero-filled before its first use, left all zero by
 *            every completed call; not shared by concurrent calls.
 * Requirements: 0 <= M <= 64 (M == 0 is a no-op; larger M returns
 * FP8Q_ERR_UNSUPPORTED: quantize the activations and call fp8_linear),
 * N > 0, K > 0, K % 16 == 0.
 * Dispatch: one token runs a CUDA-core kernel that streams the weights through
 * shared memory (no workspace); 2..64 tokens run the decode kernel's schedule
 * on the tensor cores with the weight tiles widened to bf16 in shared memory
 * (exactly: every E4M3 value is a bf16 value) and bf16 MMAs.
 */
FP8Q_API size_t fp8_linear_w8a16_workspace_size(int64_t M, int64_t N, int64_t K);
FP8Q_API fp8q_status fp8_linear_w8a16(const void* X_bf16, int64_t ldx, const uint8_t* Wq, const float* w_scale,
                                      int64_t M, int64_t N, int64_t K, void* Y_bf16, int64_t ldy,
                                      void* workspace, size_t workspace_bytes, void* stream);

/* Bytes of workspace fp8_linear needs for this problem on the current device
 * (0 for the prefill path).  Returns 0 for invalid arguments as well. */
FP8Q_API size_t fp8_linear_workspace_size(int64_t M, int64_t N, int64_t K, int mode);

/* Human-readable name of a status code (static string, never NULL). */
FP8Q_API const char* fp8q_status_string(int status);

/* Reads the device-side error word of the current device: 0 when no kernel
 * has given up waiting, otherwise a nonzero code naming the wait site.  It
 * synchronizes the device.  clear != 0 resets the word to 0 afterwards and,
 * when it was nonzero, also zeroes fp8_linear_noalloc's in-library scratch on
 * this device.  Returns -1 when a CUDA call fails. */
FP8Q_API int fp8q_device_error(int clear);

/*
 * fp8_linear_noalloc -- fp8_linear for M <= 64 without a caller-supplied workspace.
 *
 * The pages have no counterpart to this entry point; it exists for callers that
 * cannot allocate device memory at the moment they call: plugin or enqueue
 * interfaces that hand over inputs and outputs but no scratch, code that must
 * not pay cudaMalloc's implicit device synchronisation on its critical path,
 * and programs whose device-memory budget is fixed before they run.
 *
 * Same arguments, requirements and result as fp8_linear, minus the workspace.
 * The split-K scratch is instead a fixed array of 16 MiB (16777216 bytes)
 * compiled into the library: every GPU that loads libfp8q.so holds it until the
 * process exits.  This call allocates nothing (no cudaMalloc,
 * cudaFree or allocating library routine).
 *   - M > 64 returns FP8Q_ERR_UNSUPPORTED: call fp8_linear with a NULL workspace
 *     there, which needs no scratch and allocates nothing either.
 *   - A problem whose scratch would exceed the array (the size
 *     fp8_linear_workspace_size reports) returns FP8Q_ERR_UNSUPPORTED.
 *   - The first call on each device looks up the array's device address
 *     (cudaGetSymbolAddress, with that device current); make that first call
 *     before any stream capture.  With CUDA's lazy module loading (the default)
 *     the array is reserved on a device when the library's device code is
 *     first loaded there: by that first call, or by any earlier call of this
 *     library on the device.  A caller whose memory budget is fixed should
 *     therefore make one call at setup time.
 *   - Every call on a device shares the one array, which keeps whatever the last
 *     call left in it: zero-filled when the library is loaded, and every
 *     completed call leaves it all zero again.  Calls whose kernels overlap on the GPU
 *     (different streams, or different host threads) race on the array and give
 *     wrong results; serialise them.
 *   - A call whose kernel gave up waiting (fp8q_device_error nonzero) can leave
 *     counters and partial sums in the array.  fp8q_device_error(1) then zeroes
 *     the current device's array as well as the error word (cudaMemset, which
 *     allocates nothing); call it before the next fp8_linear_noalloc.
 */
FP8Q_API fp8q_status fp8_linear_noalloc(const uint8_t* Xq, const float* x_scale, const uint8_t* Wq,
                                        const float* w_scale, int64_t M, int64_t N, int64_t K, int mode,
                                        void* Y_bf16, int64_t ldy, void* stream);

/* Library version: major * 10000 + minor * 100 + patch. */
FP8Q_API int fp8q_version(void);

#ifdef __cplusplus
}
#endif

#endif /* FP8Q_H_ */
