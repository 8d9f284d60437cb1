/*
 * mxq.h -- C ABI of libmxq: the MXFP4 quantized linear layer on NVIDIA B200 (sm_100a).
 *
 * The layer, as the pages state the problem:
 *   - weights are quantised offline to OCP MXFP4 for both W4A4 and W4A8;
 *   - activations are quantised dynamically to MXFP4 (W4A4) or statically to
 *     FP8 E4M3 with one per-tensor scale (W4A8);
 *     [AMD Quark adds native W4A8 mixed-precision for Wan2.2 video generation on
 *      MI350 -- "Quark quantization pipeline and mixed-precision selection",
 *      bullets "MXFP4 formats and precision levels" and "Native execution paths"]
 *   - the GEMM consumes the MX operands directly, with no dequantisation phase and
 *     no conversion to FP16/BF16 in between;
 *     [AMD Quark ... FLUX.1-dev MXFP4 on MI350 -- "AMD Instinctプラットフォーム上の
 *      拡散モデル向けMXFP4量子化", and "MXFP4とは何か": 32-element blocks share one
 *      scale factor]
 *   - an optional fixed (parameter-free) Hadamard rotation precedes quantisation;
 *     [Wan2.2 page above -- "Fixed rotation selector"]
 *   - the block scale can follow the stock OCP rule or the data-free UOS boundary
 *     Qmax = 7.25.  [MXAttention: Data-Free Optimal Scaling and Pre-Normalization
 *     Quantization for MXFP4 Attention -- TL;DR, "What it actually does"]
 *
 * Conventions common to every call
 *   - Every pointer argument is a DEVICE pointer (cudaMalloc'd or equivalent) on the
 *     current CUDA device, at least 16-byte aligned.  The caller allocates and owns
 *     every buffer; the library allocates no device memory and keeps no per-call
 *     state (it reads its own static device status word, see mxq_debug_poll).
 *   - Every call is asynchronous on `stream` (a cudaStream_t; NULL = legacy default
 *     stream) and never synchronises it.  Calls are thread-safe.
 *   - Calls work on the current CUDA device, and one process may drive several devices.
 *     The first call that launches a given kernel on a device does that device's one-time
 *     set-up (the kernel's shared-memory opt-in, its occupancy, the static scratch address);
 *     make that first call outside stream capture.  A set-up that fails returns
 *     MXQ_ERR_CUDA and is tried again on the next call.  The set-up is kept for the life of
 *     the process: after cudaDeviceReset the library must not be used on that device again.
 *   - Stream order holds as for any kernel, with one refinement: the GEMM kernels
 *     (mxq_gemm_*, mxq_linear_*) are launched with programmatic stream
 *     serialisation.  If the kernel before them in the stream lets dependents start
 *     early (the activation quantisers of this library do), a GEMM may begin its
 *     set-up and prefetch its weight tiles into L2 while that kernel runs; it reads
 *     no operand and writes no output before the earlier kernel has completed and
 *     its writes are visible.  After any other kernel, or a copy, it starts as usual.
 *   - Arguments are validated on the host before anything is launched; on any
 *     error nothing is launched and a status other than MXQ_OK is returned.  A
 *     launch failure returns MXQ_ERR_CUDA.  No C++ exception crosses this ABI.
 *   - Matrices are row-major.  X[M][K] activations (BF16), W[N][K] weights (BF16,
 *     nn.Linear convention, K-major), D[M][N] output (BF16).
 *
 * Data layouts (a reading: the pages do not fix them)
 *   - MXFP4 codes: [rows][K/2] bytes, row stride exactly K/2.  Element k sits in
 *     byte k/2, low nibble when k is even.  Nibble = sign<<3 | index, index 0..7 <->
 *     magnitudes {0, 0.5, 1, 1.5, 2, 3, 4, 6} (OCP MX v1.0 E2M1).
 *   - Scale factors (E8M0, byte = e + 127, value 2^e): one byte per (row, 32-block).
 *     Physical buffer of mxq_sf_bytes(rows, K) bytes: rows padded to R = 128*ceil(rows/128),
 *     scale columns to C = 4*ceil((K/32)/4); the scale of (row r, block c) is at byte
 *       ((r/128)*(C/4) + c/4)*512 + (r%32)*16 + ((r%128)/32)*4 + (c%4)
 *     (512-byte atoms of 128 rows x 4 blocks, the tcgen05 block-scale operand layout).
 *     Padding bytes are written as 0x00.
 *   - FP8 activations: [M][K] E4M3 bytes, row stride exactly K.
 */
#ifndef MXQ_H_
#define MXQ_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define MXQ_API __attribute__((visibility("default")))
#else
#define MXQ_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

struct CUstream_st;
/* Identical to cudaStream_t / CUstream. */
typedef struct CUstream_st* mxq_stream_t;

typedef enum {
  MXQ_OK = 0,
  MXQ_ERR_INVALID_ARG = 1, /* null pointer, bad enum, non-finite / non-positive scale  */
  MXQ_ERR_SHAPE = 2,       /* dimension out of range or not a required multiple         */
  MXQ_ERR_ALIGN = 3,       /* pointer or leading dimension misaligned                   */
  MXQ_ERR_UNSUPPORTED = 4, /* no sm_100 device current, or configuration not built      */
  MXQ_ERR_CUDA = 5,        /* a CUDA runtime / driver call failed                       */
  MXQ_ERR_TIMEOUT = 6      /* a kernel gave up a bounded wait (reported by mxq_debug_poll) */
} mxq_status;

typedef enum {
  MXQ_SCALE_OCP = 0, /* e = floor(log2 amax) - 2: smallest e with amax/2^e <  8    */
  MXQ_SCALE_UOS = 1  /* smallest e with amax/2^e <= 7.25 (Qmax of the UOS boundary) */
} mxq_scale_rule;

typedef enum {
  MXQ_ACT_MXFP4 = 0,   /* dynamic MXFP4 activations (W4A4)            */
  MXQ_ACT_FP8_E4M3 = 1 /* static per-tensor FP8 E4M3 activations (W4A8) */
} mxq_act_format;

typedef enum {
  MXQ_PREC_W4A4 = 0,           /* plain MXFP4 weights and activations                  */
  MXQ_PREC_W4A4_TRANSFORM = 1, /* W4A4 with the fixed rotation + SmoothQuant            */
  MXQ_PREC_W4A8 = 2,           /* promotion: MXFP4 weights, static FP8 E4M3 activations */
  MXQ_PREC_BF16 = 3            /* fallback: the layer stays in BF16                     */
} mxq_precision;

/* Human-readable name of a status code (static string, never NULL). */
MXQ_API const char* mxq_status_string(mxq_status status);

/* Size in bytes of the padded, swizzled scale-factor buffer for a [rows][K]
 * MXFP4 tensor (K a multiple of 32).  Returns -1 for invalid sizes. */
MXQ_API int64_t mxq_sf_bytes(int64_t rows, int64_t K);

/*
 * mxq_quantize_act -- dynamic activation quantisation, one pass over X.
 *
 * MXFP4 (fmt = MXQ_ACT_MXFP4): for each row and each 32-element block along K:
 *   optional y = x * H128/sqrt(128) per 128-element chunk (hadamard128 != 0; fixed
 *   butterfly order, FP32), amax = max |y| over the block, exponent e by `rule`
 *   (clamped to [-127, 127], amax = 0 -> e = -127), codes = E2M1 round-to-nearest-
 *   even of y * 2^-e with saturation at 6 and the sign bit kept; scale byte e + 127.
 *   Writes q_out ([M][K/2] codes) and sf_out (mxq_sf_bytes(M, K) bytes, padding 0).
 *   `act_scale` is ignored.
 * FP8 (fmt = MXQ_ACT_FP8_E4M3): q = E4M3_RNE_satfinite(fl32(x * fl32(1/act_scale)))
 *   for the static per-tensor scale act_scale > 0 (dequantised value = q * act_scale).
 *   Writes q_out ([M][K] bytes); sf_out must be NULL; rule and hadamard128 must be
 *   MXQ_SCALE_OCP and 0.
 *
 * x_bf16: device [M][ldx] BF16, 16-byte aligned; 1 <= M <= 8388480 (65535 tiles of 128
 * rows; FP8 mode allows up to 2^31); 32 <= K <= 2^22 with K % 32 == 0 (K % 128 == 0 when
 * hadamard128); ldx >= K and ldx % 8 == 0 (16-byte aligned rows; rows that are 32-byte
 * aligned are read with 32-byte loads, the others with pairs of 16-byte loads).
 * Errors: MXQ_ERR_INVALID_ARG, MXQ_ERR_SHAPE, MXQ_ERR_ALIGN, MXQ_ERR_CUDA.
 */
MXQ_API mxq_status mxq_quantize_act(const void* x_bf16, int64_t M, int64_t K, int64_t ldx,
                            mxq_act_format fmt, mxq_scale_rule rule, int hadamard128,
                            float act_scale, void* q_out, void* sf_out, mxq_stream_t stream);

/*
 * mxq_pack_weight -- offline MXFP4 weight quantisation (run once, not on the hot path).
 *
 * Same per-block arithmetic as the MXFP4 activation quantiser, on W[N][K] rows:
 * codes_out [N][K/2], sf_out mxq_sf_bytes(N, K) bytes.  Use rule = MXQ_SCALE_OCP for
 * "OCP MXFP4 weights"; hadamard128 must equal the activation side's setting (the
 * library cannot check this: X R (W R)^T = X W^T only when both sides rotate).
 * w_bf16: device [N][ldw] BF16, 16-byte aligned, 1 <= N <= 8388480, 32 <= K <= 2^22,
 * K % 32 == 0 (K % 128 == 0 when hadamard128), ldw >= K, ldw % 8 == 0.
 */
MXQ_API mxq_status mxq_pack_weight(const void* w_bf16, int64_t N, int64_t K, int64_t ldw,
                           mxq_scale_rule rule, int hadamard128, void* codes_out, void* sf_out,
                           mxq_stream_t stream);

/*
 * mxq_gemm_w4a4 -- D[M][N] = bf16_rne(alpha * sum_k deqA[m][k] * deqB[n][k] + bias[n])
 * with deq = E2M1 value * 2^(scale byte - 127), accumulated in FP32 on the tensor
 * cores (tcgen05.mma kind::mxf4 block_scale) without dequantising either operand.
 *
 * a_codes [M][K/2] + a_sf (mxq_sf_bytes(M, K)); b_codes [N][K/2] + b_sf
 * (mxq_sf_bytes(N, K)), both as written by the quantiser / packer.
 * bias_bf16: NULL or [N] BF16.  d_bf16: [M][ldd] BF16, ldd >= N, ldd % 8 == 0.
 * 1 <= M, N <= 2^30 (any value: ragged tiles are handled); 128 <= K <= 2^22, K % 128 == 0.
 * alpha must be finite.
 */
MXQ_API mxq_status mxq_gemm_w4a4(const void* a_codes, const void* a_sf, const void* b_codes,
                         const void* b_sf, int64_t M, int64_t N, int64_t K, float alpha,
                         const void* bias_bf16, void* d_bf16, int64_t ldd, mxq_stream_t stream);

/*
 * mxq_gemm_w4a8 -- D[M][N] = bf16_rne(act_scale * sum_k e4m3(A[m][k]) * deqB[n][k] + bias[n])
 * on the tensor cores (tcgen05.mma kind::mxf8f6f4 block_scale: A = E4M3 with unit
 * block scales, B = E2M1 with its E8M0 block scales); the per-tensor activation
 * scale is applied in the FP32 epilogue.
 *
 * a_e4m3 [M][K] as written by mxq_quantize_act(fmt = MXQ_ACT_FP8_E4M3, same act_scale);
 * b_codes/b_sf as for W4A4 (b_codes must be 32-byte aligned).  Shapes as for W4A4.
 */
MXQ_API mxq_status mxq_gemm_w4a8(const void* a_e4m3, float act_scale, const void* b_codes,
                         const void* b_sf, int64_t M, int64_t N, int64_t K, const void* bias_bf16,
                         void* d_bf16, int64_t ldd, mxq_stream_t stream);

/*
 * mxq_linear_w4a4 -- the quantized linear layer in one call:
 *   D[M][N] = bf16_rne(alpha * sum_k deq(Q(X))[m][k] * deqW[n][k] + bias[n]),
 * Q = the dynamic MXFP4 activation quantiser of mxq_quantize_act (rule `rule`, no rotation),
 * run into the caller's workspace, then the block-scaled GEMM of mxq_gemm_w4a4 (two launches
 * on `stream`).  [the layer: AMD Quark adds native W4A8 ... Wan2.2 -- "MXFP4 formats and
 * precision levels"; FLUX.1-dev MXFP4 page -- the GEMM takes the MX operands directly]
 *
 * x_bf16: [M][ldx] BF16, 16-byte aligned, ldx >= K, ldx % 8 == 0.  w_codes / w_sf: from
 * mxq_pack_weight (N rows).  bias_bf16, d_bf16, ldd and the shape limits as for mxq_gemm_w4a4
 * (K % 128 == 0), and M <= 8388480.
 * workspace: device, 16-byte aligned, at least mxq_linear_workspace_bytes(M, K) bytes, owned
 * by the caller.  After the call it holds the quantised activations: codes at offset 0
 * ([M][K/2], as mxq_quantize_act writes them), scales at offset ceil(M*K/2 / 1024) * 1024
 * (mxq_sf_bytes(M, K) bytes).  Calls that share a workspace must not overlap (issue them on
 * one stream).
 */
MXQ_API int64_t mxq_linear_workspace_bytes(int64_t M, int64_t K);

MXQ_API mxq_status mxq_linear_w4a4(const void* x_bf16, int64_t M, int64_t K, int64_t ldx,
                                   mxq_scale_rule rule, const void* w_codes, const void* w_sf,
                                   int64_t N, float alpha, const void* bias_bf16, void* workspace,
                                   int64_t workspace_bytes, void* d_bf16, int64_t ldd,
                                   mxq_stream_t stream);

/*
 * mxq_linear_w4a4_static -- mxq_linear_w4a4 without a caller workspace, allocating nothing:
 * the quantised activations go to a fixed buffer inside the library (one per device, a
 * file-scope device array of MXQ_STATIC_SCRATCH_BYTES = 16 MiB, whose address is looked up
 * by the first call on each device, with that device current; make that first call outside
 * stream capture).  The pages have no counterpart of this call; it serves callers that
 * cannot hand out device memory.  Returns MXQ_ERR_SHAPE when mxq_linear_workspace_bytes(M, K)
 * exceeds the buffer (for K = 5120 about 6100 rows).  Nothing in the buffer needs to start at
 * zero.  The buffer is shared by every call on the device: calls that overlap in time
 * (different streams or host threads) race on it and must be serialised by the caller.
 * Other arguments, limits and errors as for mxq_linear_w4a4.
 */
#define MXQ_STATIC_SCRATCH_BYTES (16ll << 20)

MXQ_API mxq_status mxq_linear_w4a4_static(const void* x_bf16, int64_t M, int64_t K, int64_t ldx,
                                          mxq_scale_rule rule, const void* w_codes, const void* w_sf,
                                          int64_t N, float alpha, const void* bias_bf16, void* d_bf16,
                                          int64_t ldd, mxq_stream_t stream);

/*
 * mxq_dequant_mxfp4 -- out[r][k] = bf16(E2M1 value of code (r, k) * 2^(scale byte - 127)):
 * the MXFP4 -> BF16 expansion of a tensor in the layout above (weights from
 * mxq_pack_weight or activations from mxq_quantize_act).  Every product is a power of
 * two times an E2M1 value, so it is exact in BF16 (or +-Inf past the BF16 range).
 * Not on the W4A4 / W4A8 path (the GEMMs consume the MX operands directly); it serves
 * layers kept in higher precision and checks of stored weights.
 * [MXFP4 block structure and E8M0 scale: "MXFP4とは何か", AMD Instinct FP4 diffusion page]
 *
 * codes [rows][K/2] (16-byte aligned); sf as written by the quantiser
 * (mxq_sf_bytes(rows, K) bytes; scale byte 0xFF, the E8M0 NaN, is outside the domain and
 * its outputs are unspecified); out_bf16 [rows][ldo], 16-byte aligned, ldo >= K,
 * ldo % 8 == 0, not overlapping the inputs.  1 <= rows <= 2^31, 32 <= K <= 2^22, K % 32 == 0.
 */
MXQ_API mxq_status mxq_dequant_mxfp4(const void* codes, const void* sf, int64_t rows, int64_t K,
                                     void* out_bf16, int64_t ldo, mxq_stream_t stream);

/*
 * mxq_qdq_act -- quantise-dequantise ("fake quantisation") of activations in one pass:
 * out = bf16(dequant(quant(x))) with exactly the arithmetic of mxq_quantize_act for the
 * same (fmt, rule, hadamard128, act_scale), so that a BF16 layer fed `out` sees the values
 * the W4A4 / W4A8 GEMM sees.  With hadamard128 the output stays in the rotated basis
 * (x H/sqrt(128) quantised), as the GEMM's operand does.  FP8: out =
 * bf16(fl32(E4M3 value * act_scale)).
 * [Mixed-precision selection evaluates candidate precisions layer by layer: Wan2.2 page,
 *  "Quark quantization pipeline and mixed-precision selection"]
 *
 * Arguments and limits as for mxq_quantize_act; out_bf16 [M][ldo], 16-byte aligned,
 * ldo >= K, ldo % 8 == 0, not overlapping x.
 */
MXQ_API mxq_status mxq_qdq_act(const void* x_bf16, int64_t M, int64_t K, int64_t ldx,
                               mxq_act_format fmt, mxq_scale_rule rule, int hadamard128,
                               float act_scale, void* out_bf16, int64_t ldo, mxq_stream_t stream);

/*
 * SmoothQuant after the fixed rotation.  The selection transform on the Wan2.2 page is
 * a fixed Hadamard rotation followed by SmoothQuant (no learned parameters):
 * [AMD Quark adds native W4A8 ... Wan2.2 -- "Fixed rotation selector" and "Block-level
 *  SQNR calibration"].  Per channel k of the (rotated) values, activations are
 * multiplied by 1/lambda_k and weight rows by lambda_k, so X W^T is unchanged while
 * activation outliers migrate into the weights.  The pages give no formula for lambda;
 * mxq_smooth_factors uses the published SmoothQuant one (migration strength alpha).
 *
 * mxq_channel_absmax -- calibration statistic: amax_out[k] = max over rows of |y[r][k]|
 * with y = x, or y = x H/sqrt(128) per 128-column chunk when hadamard128 (the rotation
 * of mxq_quantize_act).  accumulate = 0: amax_out is cleared first (on `stream`);
 * accumulate != 0: the maxima merge into amax_out's current values (non-negative
 * FP32), so several calibration batches can be folded in.
 * x_bf16 / rows / K / ldx as for mxq_quantize_act; amax_out: device [K] FP32, 16-byte
 * aligned.
 */
MXQ_API mxq_status mxq_channel_absmax(const void* x_bf16, int64_t rows, int64_t K, int64_t ldx,
                                      int hadamard128, int accumulate, float* amax_out,
                                      mxq_stream_t stream);

/*
 * mxq_smooth_factors -- lambda[k] = max(amax_x[k]^alpha / max(amax_w[k], 1e-5)^(1-alpha), 1e-5)
 * in FP32 (powf), inv_lambda[k] = 1 / lambda[k] (IEEE division), for 0 <= alpha <= 1.
 * amax_x / amax_w: device [K] FP32 channel maxima of the calibration activations and of the
 * weights (both from mxq_channel_absmax with the same hadamard128).  1 <= K <= 2^22.
 */
MXQ_API mxq_status mxq_smooth_factors(const float* amax_x, const float* amax_w, int64_t K, float alpha,
                                      float* lambda_out, float* inv_lambda_out, mxq_stream_t stream);

/*
 * mxq_quantize_smooth -- the MXFP4 quantiser of mxq_quantize_act / mxq_pack_weight with one
 * FP32 multiply per value by chan_scale[k] after the optional rotation and before the
 * block maximum: codes of (x R)[r][k] * chan_scale[k].  Pass inv_lambda for activations
 * (every call) and lambda for the weights (offline packing); the W4A4 GEMM then runs
 * unchanged on the two outputs.  chan_scale: device [K] FP32, 16-byte aligned, finite.
 * Other arguments, layouts and limits as for mxq_quantize_act (MXFP4).
 */
MXQ_API mxq_status mxq_quantize_smooth(const void* x_bf16, int64_t rows, int64_t K, int64_t ldx,
                                       mxq_scale_rule rule, int hadamard128, const float* chan_scale,
                                       void* codes_out, void* sf_out, mxq_stream_t stream);

/*
 * Per-layer precision selection.  The Wan2.2 page selects each block's precision from its
 * whole-block output SQNR against BF16, measured with plain MXFP4 and with the transform
 * (fixed rotation + SmoothQuant), through tiered thresholds: plain W4A4, W4A8 promotion,
 * transform-enabled W4A4 or BF16 fallback.  [AMD Quark adds native W4A8 ... Wan2.2 --
 * "Block-level SQNR calibration"]  The threshold values are not on the pages: they are
 * parameters.
 *
 * mxq_sqnr_accumulate -- acc[0] += sum ref^2, acc[1] += sum (y - ref)^2 over M x N BF16
 * values (y: the quantised layer's output, ref: the BF16 layer's), in FP64 on the device.
 * accumulate = 0 clears acc first (on `stream`); != 0 adds to it, so the layers of a block
 * sum into one SQNR.  y_bf16 / ref_bf16: device [M][ldy] / [M][ldr], 16-byte aligned,
 * ldy, ldr >= N and multiples of 8; acc: device double[2].  The FP64 addition order varies
 * between runs (atomics), so the sums do in their last bits.
 */
MXQ_API mxq_status mxq_sqnr_accumulate(const void* y_bf16, int64_t ldy, const void* ref_bf16,
                                       int64_t ldr, int64_t M, int64_t N, int accumulate, double* acc,
                                       mxq_stream_t stream);

/* 10 log10(signal / noise) dB; +HUGE_VAL when noise == 0, -HUGE_VAL when signal == 0.
 * Host-only (no device access). */
MXQ_API double mxq_sqnr_db(double signal, double noise);

/* The tier decision, host-only: plain >= high_db -> MXQ_PREC_W4A4; else transform >= high_db
 * -> MXQ_PREC_W4A4_TRANSFORM; else max(plain, transform) >= low_db -> MXQ_PREC_W4A8; else
 * MXQ_PREC_BF16 (SQNRs in dB, ties pass). */
MXQ_API mxq_precision mxq_select_precision(double sqnr_plain_db, double sqnr_transform_db,
                                           double high_db, double low_db);

/*
 * MXFP4 attention with UOS and pre-normalisation quantisation (PNQ).
 * [MXAttention: Data-Free Optimal Scaling and Pre-Normalization Quantization for MXFP4
 *  Attention -- TL;DR, "Architecture", "What it actually does"]
 * Per head h (columns [h d, (h+1) d) of the [S][H d] activations):
 *   S = deq(Q) deq(K)^T, t = fl32(S * fl32(log2(e) / sqrt(d))),
 *   P = MXFP4(2^(t - c)) in 32-key blocks -- the unnormalised numerators quantised BEFORE
 *       the row sum, with the block-scale rule `rule` (UOS: Qmax = 7.25),
 *   l = sum_j deq(P)_j,  O = deq(P) deq(V) / l.
 * c is an integer offset (at least the row maximum of t minus 8); since E8M0 block scaling
 * is exactly equivariant under powers of two, the codes of P do not depend on which such c
 * is used.  The codes of P are those of the exact exponential 2^(t - c): a block's E8M0
 * exponent follows from its largest score by integer arithmetic (floor(t_max - c) - 2, plus
 * one under UOS when the fraction of t_max - c exceeds log2(1.8125)), and each element code
 * from a cubic q(g) in g = t - rint(t) (FP32 Horner, the last step rounded up; coefficients
 * from mxq_attn_code_poly) whose FP32 values cross the four E2M1 decision levels 0.75,
 * 0.875, 1 and 1.25 at exactly the FP32 g where 2^g crosses them.  Scores must satisfy
 * |t| < 2^22.  Numerators below 2^-118 of a row's largest one may be kept or flushed to 0
 * (the kernel's offset is raised lazily); they are below the FP32 resolution of l.
 *
 * mxq_attn_code_poly -- writes {1, a1, a2, a3}, the FP32 coefficients of that cubic, to
 * coeffs[0..3] (host only, no device access; for checking the decision property above).
 *
 * mxq_attn_padded_keys -- Sp = S_kv rounded up to the kernel's 256-key tile (-1 if S_kv is
 * outside [1, 2^23]).
 *
 * mxq_quantize_vt -- V [S][ldv] BF16 -> V^T in MXFP4 with 32-key blocks (the layout the P V
 * product consumes): codes_out [HD][Sp/2] (keys in [S, Sp) are zero), sf_out
 * mxq_sf_bytes(HD, Sp) bytes in the layout of the other scale buffers (rows = channels).
 * HD % 128 == 0, HD <= 2^16, ldv >= HD, ldv % 8 == 0, v 16-byte aligned.
 *
 * mxq_attention_mxfp4 -- q_codes / q_sf: Q [S_q][H d] quantised by mxq_quantize_act (MXFP4,
 * the same rule, no rotation); k_codes / k_sf: K [S_kv][H d] likewise; vt_codes / vt_sf:
 * from mxq_quantize_vt.  out_bf16: O [S_q][ldo] BF16 (head h in columns [h d, (h+1) d)),
 * ldo >= H d, ldo % 8 == 0.  d must be 128 (MXQ_ERR_UNSUPPORTED otherwise); H d <= 2^16;
 * 1 <= S_q <= 8388480; all buffers 16-byte aligned.  One sequence per call.
 */
MXQ_API int64_t mxq_attn_padded_keys(int64_t S_kv);

MXQ_API void mxq_attn_code_poly(float coeffs[4]);

MXQ_API mxq_status mxq_quantize_vt(const void* v_bf16, int64_t S, int64_t HD, int64_t ldv,
                                   mxq_scale_rule rule, void* codes_out, void* sf_out,
                                   mxq_stream_t stream);

MXQ_API mxq_status mxq_attention_mxfp4(const void* q_codes, const void* q_sf, const void* k_codes,
                                       const void* k_sf, const void* vt_codes, const void* vt_sf,
                                       int64_t S_q, int64_t S_kv, int64_t H, int64_t d,
                                       mxq_scale_rule rule, void* out_bf16, int64_t ldo,
                                       mxq_stream_t stream);

/*
 * mxq_debug_poll -- reads and clears the library's device status word, written by a
 * kernel that gave up one of its bounded waits (each wait on a barrier or a copy is
 * capped at about a second, after which the kernel records MXQ_ERR_TIMEOUT, drains
 * its own copies in flight, releases its tensor memory and returns).  Synchronises
 * the current device.  Returns MXQ_OK when no kernel has reported anything.
 */
MXQ_API mxq_status mxq_debug_poll(void);

/*
 * mxq_selftest_wait_timeout -- diagnostic of the failure path above: launches on `stream`
 * a one-thread kernel that waits, with the same bounded wait as every kernel of the
 * library, on a barrier nothing arrives on.  After about a second the wait gives up and
 * records MXQ_ERR_TIMEOUT, and the kernel returns: the next mxq_debug_poll returns
 * MXQ_ERR_TIMEOUT (and clears it), and the device stays usable.  While the status word
 * is set, waits in other kernels of the library give up at once, so nothing else should
 * run between this call and that poll.  Returns MXQ_ERR_UNSUPPORTED off B200.
 */
MXQ_API mxq_status mxq_selftest_wait_timeout(mxq_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* MXQ_H_ */
