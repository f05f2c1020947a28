/*
 * segquant.h -- C ABI of the B200 (sm_100a) SegQuant quantized-linear library:
 * DualScale polarity-split W8A8 GEMM with SegLinear segment-wise quantization.
 *
 * The method (SegQuant, arXiv 2507.14811), as described on the pages this
 * library follows:
 *  - "SegQuant" (papernotes.org notes), section "DualScale": the activation is
 *    split by polarity, X+ = max(X,0) and X- = min(X,0); each part has its own
 *    static step, s- = |min(x)|/q_min and s+ = max(x)/q_max; the layer output is
 *    rebuilt as Y ~= s+ s_w (X^+ W^) + s- s_w (X^- W^).  The two integer
 *    products run as one batched GEMM with a fused epilogue and no zero point.
 *  - same page, section "SegLinear": an output-segmented layer splits W by
 *    columns, Y^ = [X^W^_1, ..., X^W^_N]; an input-segmented layer splits X by
 *    columns and W by rows, Y^ = sum_i X^_i W^_i; every segment is quantized
 *    with its own parameters.
 *  - "SegQuant" author page (hliangzhao.me), section 3: the case-wise
 *    quantizer Q_dual(x) = round(x/s-) for x < 0, round(x/s+) for x >= 0.
 *
 * Readings taken where the pages are open (q_min magnitude 128, round half to
 * even, saturation, SmoothQuant divisor folded as x/d and w*d, fp32 epilogue
 * order) are spelled out per entry point below.
 *
 * Conventions for every call:
 *  - Every pointer is a DEVICE pointer unless marked "host".  The caller owns
 *    all buffers, workspaces included; the library allocates no device memory
 *    in any call.  (The one exception to caller-owned memory is the fixed
 *    scratch array of sq_dualscale_seglinear_host_noalloc, which is part of
 *    the library's device image.)
 *  - Calls are asynchronous on `stream` (0 = legacy default stream).  A return
 *    of SQ_OK means the arguments were valid and the kernels were launched;
 *    launch failures return SQ_ERR_CUDA.  Faults inside a kernel surface at
 *    the caller's next synchronisation, as with any CUDA call.
 *  - Arguments are validated on the host before anything is launched; an
 *    invalid call launches nothing and leaves every output untouched.
 *  - bf16 tensors are raw bfloat16 bit patterns (uint16) in row-major order.
 *  - Layout of the stacked activation planes ("planes"): int8 [G][2][M][K],
 *    row-major, K contiguous; plane [g][0] is X^+ (codes 0..127) and plane
 *    [g][1] is X^- (codes -128..0) of activation group g.
 */
#ifndef SEGQUANT_H
#define SEGQUANT_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Exported symbols (the library is built with hidden default visibility). */
#if defined(__GNUC__)
#define SQ_API __attribute__((visibility("default")))
#else
#define SQ_API
#endif

/* cudaStream_t without pulling in the CUDA headers. */
typedef struct CUstream_st *sq_stream_t;

typedef enum {
  SQ_OK = 0,
  SQ_ERR_INVALID_ARG = -1,   /* null pointer, bad size, bad segment table     */
  SQ_ERR_UNSUPPORTED = -2,   /* valid request the library does not implement  */
  SQ_ERR_ALIGNMENT = -3,     /* pointer / leading dimension misaligned       */
  SQ_ERR_OVERFLOW = -4,      /* a K-segment could overflow the int32 sum     */
  SQ_ERR_CUDA = -5,          /* a CUDA runtime call failed                    */
  SQ_ERR_DEVICE_TIMEOUT = -6,/* a kernel gave up waiting (see status call)    */
  SQ_ERR_NO_DEVICE = -7,     /* no sm_100 device is current                   */
  SQ_ERR_TOO_LARGE = -8,     /* one row does not fit a fixed-size scratch     */
  SQ_ERR_DEVICE_BOUNDS = -9  /* debug build: a kernel skipped a store outside
                                its buffer (see sq_debug_bounds_checks)      */
} sq_status;

typedef enum {
  SQ_SEG_NONE = 0,   /* one segment over K and N                           */
  SQ_SEG_OUTPUT = 1, /* segments over N (columns of the pages' W)          */
  SQ_SEG_INPUT = 2   /* segments over K (rows of the pages' W)             */
} sq_seg_mode;

typedef enum { SQ_OUT_BF16 = 0, SQ_OUT_F32 = 1 } sq_out_dtype;

/* Most segments a layer may have. */
#define SQ_MAX_SEGMENTS 64

/*
 * Flags of a segment table.  SQ_FLAG_SINGLE_SCALE selects the single-scale
 * (non-DualScale) path for a layer, for the adaptive use the papernotes page
 * proposes under "Limitations" (DualScale only where activations are strongly
 * polarity-asymmetric): one step s per group and K-segment serves both signs,
 * s = max(max u, -min u)/127; the code is the DualScale code with s+ = s- = s,
 * so X^+ and X^- collapse into one plane q = X^+ + X^- in [-128, 127]; the GEMM
 * runs one integer product per k-step instead of two, y = sum_i s_w s f(A_i) + b.
 * Layouts become planes [G][1][M][K] and accumulators [S][1][M][N]; s_act keeps
 * its [G][S][2] shape with both entries equal.
 */
#define SQ_FLAG_SINGLE_SCALE 1

/*
 * SQ_FLAG_W4: the layer's weights are W4A8 codes ("SegQuant-4", the W4A8 rows
 * of the results tables and the deployment-cost table of the papernotes.org
 * and author pages; the pages give no formula, the reading is the W8 rule with
 * q_max = 7).  They are stored packed (sq_quantize_weight_w4) and expanded by
 * sq_unpack_weight_w4 into the int8 GEMM operand holding 16*q (the code in the
 * high nibble of each byte).  With this flag sq_dualscale_seglinear_gemm
 * multiplies s+ and s- by 2^-4 when it loads them, which is exact, so the
 * result equals the W4A8 definition with codes q bit for bit.  The flag has no
 * effect on the activation calls.
 */
#define SQ_FLAG_W4 2

/*
 * SQ_FLAG_FP8: the FP8 variant (the "W8A8(fp)" rows of the results table for
 * SDXL, which the pages do not define).  Reading: every code is FP8 E4M3 (1
 * sign, 4 exponent bits with bias 7, 3 mantissa bits, largest finite 448, no
 * infinities, 0x7F/0xFF NaN), stored as its bit pattern in the int8 buffers.
 * Calibration: s+ = max/448 and s- = |min|/448 (single scale: the larger side
 * / 448).  Quantization, with u = fl(x / d) as for int8: x >= 0 -> X^+ =
 * e4m3(fl(u / s+)), X^- = 0x00; x < 0 -> X^- = e4m3(fl(u / s-)), X^+ = 0x00;
 * NaN -> both 0x00; e4m3() rounds half to even and saturates finite values to
 * +-448.  Weights: s_w = amax/448,
 * W^ = e4m3(fl(w'/s_w)).  GEMM: tcgen05 kind::f8f6f4 with fp32 accumulation
 * (exact products; sums in the tensor core's fp32, order unspecified), the
 * W8A8 epilogue on the fp32 sums.  Not combinable with SQ_FLAG_W4.
 */
#define SQ_FLAG_FP8 4

/*
 * Segment table (SegLinear).  `offsets` is a HOST array of n_seg + 1 strictly
 * increasing int32 values from 0 to the segmented extent (N for SQ_SEG_OUTPUT,
 * K for SQ_SEG_INPUT).  SQ_SEG_NONE takes n_seg = 1 and offsets may be NULL.
 * n_groups (G) is the number of activation groups: 1, or, for SQ_SEG_OUTPUT
 * only, n_seg, so that every output segment has its own SmoothQuant divisor,
 * s+/s- and activation planes.  S, the number of K-segments, is n_seg for
 * SQ_SEG_INPUT and 1 otherwise.
 * Restrictions of this library version: input-segment widths are multiples of 32 (the
 * int8 MMA K step) and at most 132104 (so 128*127*width < 2^31); with G > 1
 * output-segment widths are multiples of 128.
 */
typedef struct {
  int32_t mode;            /* sq_seg_mode                        */
  int32_t n_seg;           /* number of segments, 1..SQ_MAX_SEGMENTS */
  const int32_t *offsets;  /* host, n_seg + 1 entries            */
  int32_t n_groups;        /* G                                  */
  int32_t flags;           /* 0 or SQ_FLAG_SINGLE_SCALE, | SQ_FLAG_W4 or SQ_FLAG_FP8 */
} sq_segments;

/*
 * sq_calibrate_act -- static AMax calibration of the two activation steps.
 * Pages: papernotes.org "SegQuant", section DualScale (s- = |min|/q_min,
 * s+ = max/q_max) and section "Loss function / training strategy" (AMax).
 * For group g and K-segment i, over rows 0..M-1 and the channels c of segment
 * i: u = x[m][c] / d[g][c] (fp32, IEEE division); hi = max(0, max u),
 * lo = min(0, min u); s+ = hi/127 (1 if hi == 0), s- = -lo/128 (1 if lo == 0).
 * NaN inputs are ignored.
 *   x      bf16 [M][ldx]; M >= 1, K >= 16, K % 16 == 0, ldx >= K, ldx % 8 == 0,
 *          M * ldx <= 2^44, x 16-byte aligned
 *   d      fp32 [G][K] divisor (> 0, finite) or NULL for d = 1
 *   s_act  fp32 [G][S][2] output, {s+, s-} per group and K-segment
 * With SQ_FLAG_SINGLE_SCALE: s+ = s- = max(hi, -lo)/127 (1 if both are 0).
 * Launches three small kernels; no workspace.
 */
SQ_API sq_status sq_calibrate_act(const void *x, int64_t M, int64_t K, int64_t ldx,
                           const float *d, const sq_segments *seg,
                           float *s_act, sq_stream_t stream);

/*
 * sq_quantize_act -- DualScale activation quantization (the HBM-bound step).
 * Pages: author page section 3 (Q_dual), papernotes.org section DualScale.
 * For every element x (bf16, exact in fp32) of channel c in K-segment i and
 * every group g, with the smoothed activation u = fl(x / d[g][c]) (u = x when
 * d is NULL) and the quotients rounded to fp32 (IEEE division):
 *   x >= 0: X^+ = rne(min(fl(u / s+[g][i]), 127)),  X^- = 0
 *   x <  0: X^- = rne(max(fl(u / s-[g][i]), -128)), X^+ = 0
 *   NaN   : both 0.   (-0.0 counts as x >= 0; rne = round half to even, so a
 *   quotient that is itself a half-integer goes to the even code.)
 * The kernel forms each quotient from the rounded reciprocal with one FMA
 * correction, which gives the IEEE quotient exactly under these bounds:
 *   x      bf16 [M][ldx], constraints as in sq_calibrate_act
 *   d      fp32 [G][K] or NULL;  s_act fp32 [G][S][2]; every d and s finite
 *          and within [2^-40, 2^40] (codes are unspecified otherwise)
 *   planes int8 [G][2][M][K] output, 16-byte aligned
 * With SQ_FLAG_SINGLE_SCALE the two codes of an element are written as their
 * sum, one plane per group: planes int8 [G][1][M][K].
 * M == 0 is a valid no-op.
 */
SQ_API sq_status sq_quantize_act(const void *x, int64_t M, int64_t K, int64_t ldx,
                          const float *d, const float *s_act,
                          const sq_segments *seg, int8_t *planes,
                          sq_stream_t stream);

/*
 * sq_quantize_act_plan -- for layers with SmoothQuant divisors: decides, per
 * activation group and channel, whether the quantizer may form that channel's
 * codes without either quotient's correction (u = RN(x * fl(1/d)), then the
 * code of RN(u * fl(1/s)) -- one product each) and still produce exactly the
 * codes of sq_quantize_act for every bf16 input.  (A speed-up of the same
 * Q_dual; the pages define only the codes.)  Both forms lie within 2^-22 of
 * x / (d s), so they can differ only for x next to a rounding boundary
 * (h + 1/2) s d, h = 0 .. 127; the plan evaluates both forms on the bf16
 * neighbours of each boundary (768 inputs per channel) with the kernels' own
 * operations.  Call it once per layer after sq_calibrate_act (it depends on
 * d, the steps and the segment table only).
 *   d      fp32 [G][K] device (required);  s_act fp32 [G][S][2] device
 *   plan   uint32 [G][ceil(K / 32)] device output, 4-byte aligned: bit c % 32
 *          of word [g][c / 32] set when channel c of group g qualifies
 *          (also set for the padding channels past K)
 * All buffers are the caller's; the call is asynchronous on `stream` and
 * allocates nothing.  Errors: SQ_ERR_INVALID_ARG (a NULL buffer, K < 16 or
 * K % 16 != 0, a bad segment table), SQ_ERR_ALIGNMENT, SQ_ERR_UNSUPPORTED
 * with SQ_FLAG_FP8 (int8 codes only), SQ_ERR_CUDA.
 */
SQ_API sq_status sq_quantize_act_plan(const float *d, int64_t K, const float *s_act,
                                      const sq_segments *seg, uint32_t *plan,
                                      sq_stream_t stream);

/*
 * sq_quantize_act_planned -- sq_quantize_act with a plan of
 * sq_quantize_act_plan made from the same d, s_act and segment table (a plan
 * made from other steps or divisors gives wrong codes; nothing checks it).
 * A 256-channel block in which at most 16 channels do not qualify takes the
 * codes without the corrections and then rewrites those channels' codes with
 * the exact form; a block with more is quantized as by sq_quantize_act.  The
 * planes are bit for bit those of sq_quantize_act.  plan NULL: exactly
 * sq_quantize_act.  Arguments and errors as sq_quantize_act's, and: a plan
 * without d is SQ_ERR_INVALID_ARG, a plan with SQ_FLAG_FP8 SQ_ERR_UNSUPPORTED,
 * a plan not 4-byte aligned SQ_ERR_ALIGNMENT.
 */
SQ_API sq_status sq_quantize_act_planned(const void *x, int64_t M, int64_t K, int64_t ldx,
                                         const float *d, const float *s_act,
                                         const sq_segments *seg, const uint32_t *plan,
                                         int8_t *planes, sq_stream_t stream);

/*
 * sq_quantize_weight_seg -- segment-wise symmetric AMax weight quantization
 * (offline, once per layer).  Pages: papernotes.org section SegLinear (each
 * segment of W quantized independently) and AMax calibrator.
 * w is the nn.Linear weight [N][K] (the pages' W transposed).  For output
 * channel n in output segment j (group g = j when G > 1, else 0) and K-segment
 * i:  w' = w[n][k]*d[g][k];  s_w[i][n] = max_k |w'| / 127 (1 if that is 0);
 * W^[n][k] = rne(clamp(w'/s_w[i][n], -127, 127)).  Weights must be finite.
 *   w   bf16 [N][K] (K % 16 == 0, 16-byte aligned);  d fp32 [G][K] or NULL
 *   wq  int8 [N][K] output (16-byte aligned);  s_w fp32 [S][N] output
 */
SQ_API sq_status sq_quantize_weight_seg(const void *w, int64_t N, int64_t K,
                                 const float *d, const sq_segments *seg,
                                 int8_t *wq, float *s_w, sq_stream_t stream);

/*
 * sq_quantize_weight_w4 -- W4A8 weight quantization (offline): the rule of
 * sq_quantize_weight_seg with q_max = 7, s_w[i][n] = max_k |w'| / 7 (1 if 0),
 * q = rne(clamp(w'/s_w, -7, 7)), stored two codes per byte: byte [n][j] holds
 * channel 2j in its low nibble and 2j + 1 in its high nibble, 4-bit two's
 * complement.
 *   w    bf16 [N][K] (K % 16 == 0, 16-byte aligned);  d fp32 [G][K] or NULL
 *   wq4  uint8 [N][K/2] output (16-byte aligned);  s_w fp32 [S][N] output
 */
SQ_API sq_status sq_quantize_weight_w4(const void *w, int64_t N, int64_t K,
                                const float *d, const sq_segments *seg,
                                uint8_t *wq4, float *s_w, sq_stream_t stream);

/*
 * sq_unpack_weight_w4 -- expands packed W4 codes into the int8 GEMM operand:
 * wq[n][k] = 16 * q[n][k] (in [-112, 112]).  An HBM-bound pass over N*K/2 +
 * N*K bytes, run before a GEMM with SQ_FLAG_W4; the caller owns both buffers,
 * so one wq buffer can serve every W4 layer in turn.
 *   wq4 uint8 [N][K/2], wq int8 [N][K], both 16-byte aligned, K % 16 == 0.
 */
SQ_API sq_status sq_unpack_weight_w4(const uint8_t *wq4, int64_t N, int64_t K, int8_t *wq,
                              sq_stream_t stream);

/*
 * sq_dualscale_seglinear_gemm -- the batched int8 GEMM with the fused DualScale
 * reconstruction.  Pages: papernotes.org section DualScale (one BatchedGEMM
 * launch over X^+ and X^-, results merged in a fused epilogue) and section
 * SegLinear (output concatenation / input sum).
 * Integer products, exact in int32, on the tensor cores (tcgen05 kind::i8):
 *   A+_i[m][n] = sum_{k in segment i} X^+[g(n)][m][k] * W^[n][k]   (same for -)
 * Epilogue in fp32, never leaving the chip:
 *   y[m][n] = sum_i s_w[i][n] * (s+[g][i]*f(A+_i) + s-[g][i]*f(A-_i)) + bias[n]
 * with f = int32 -> fp32 round-to-nearest, evaluated in one fixed fp32 order
 * for every segment mode: c+- = fl(s_w[i][n] * s+-[g][i]); y = 0; for each
 * segment i ascending y = fma(c+, f(A+_i), y), then y = fma(c-, f(A-_i), y);
 * finally y = y + bias[n].  The result is therefore a deterministic function
 * of the inputs, independent of tiling.  Output rounds to bf16 (RN) or stays
 * fp32.
 *   planes int8 [G][P][M][K] from sq_quantize_act (P = 1 with
 *          SQ_FLAG_SINGLE_SCALE: one product, y = sum_i s_w[i][n] s[g][i] f(A_i)
 *          + bias, s = s_act[g][i][0]); wq int8 [N][K]
 *   s_w fp32 [S][N]; s_act fp32 [G][S][2]; bias bf16 [N] or NULL
 *   y      bf16 or fp32 [M][ldy] output, ldy >= N, ldy*elem % 16 == 0,
 *          16-byte aligned
 *   K % 16 == 0, K >= 16; N >= 1; M * N <= 2^44; M == 0 is a valid no-op.
 * With SQ_FLAG_W4, wq is the output of sq_unpack_weight_w4 (16 q) and the
 * result is that of the codes q (see SQ_FLAG_W4).
 * Returns SQ_ERR_OVERFLOW when a K-segment is wider than 132104.
 */
SQ_API sq_status sq_dualscale_seglinear_gemm(const int8_t *planes, const int8_t *wq,
                                      const float *s_w, const float *s_act,
                                      const void *bias, void *y,
                                      sq_out_dtype out_dtype, int64_t M,
                                      int64_t N, int64_t K, int64_t ldy,
                                      const sq_segments *seg,
                                      sq_stream_t stream);

/*
 * sq_dualscale_seglinear_gemm_ws -- sq_dualscale_seglinear_gemm with a
 * workspace that lets one-segment layers (SQ_SEG_NONE and SQ_SEG_OUTPUT)
 * balance their last wave of tiles.  The GEMM runs one persistent CTA per SM
 * over 128-row tiles; when the tile count is not a multiple of the SM count,
 * the last, partial wave would leave SMs idle.  With the workspace, every SM
 * takes whole tiles for the full waves and an equal share of the k-blocks of
 * the last wave's tiles: an SM whose share starts inside a tile writes its
 * int32 partial products to the workspace, and the SM holding the tile's
 * first k-block adds them (exact integer addition) before the same fp32
 * epilogue, so every output is bit for bit that of sq_dualscale_seglinear_gemm.
 * Arguments as sq_dualscale_seglinear_gemm, plus:
 *   workspace        device memory of at least sq_gemm_workspace_bytes()
 *                    bytes, 256-byte aligned, owned by the caller; zero-filled
 *                    once before its first use (every call that completes
 *                    leaves it as it must be for the next).  NULL, or fewer
 *                    bytes, gives the whole-tile schedule.
 *   workspace_bytes  its size.
 * Calls that use one workspace must not overlap on the GPU (order them on one
 * stream).  After an SQ_ERR_DEVICE_TIMEOUT report, zero-fill it again.
 * Input-segmented layers and the fused producer take whole tiles.
 * Cost: a split tile's partial sums are 128 KB per accumulator plane and SM,
 * written and read back through memory; on the SD3.5 FFN layers that traffic
 * costs more than the idle SMs of the last wave, so the plain entry point
 * (whole tiles) is the faster one there.
 */
SQ_API sq_status sq_dualscale_seglinear_gemm_ws(const int8_t *planes, const int8_t *wq,
                                                const float *s_w, const float *s_act,
                                                const void *bias, void *y,
                                                sq_out_dtype out_dtype, int64_t M, int64_t N,
                                                int64_t K, int64_t ldy, const sq_segments *seg,
                                                void *workspace, size_t workspace_bytes,
                                                sq_stream_t stream);

/* Workspace bytes for sq_dualscale_seglinear_gemm_ws and sq_debug_gemm_s32_ws
 * on the current device (one slot of partial sums per SM, plus flags); 0 if
 * no sm_100 device is current. */
SQ_API size_t sq_gemm_workspace_bytes(void);

/*
 * sq_dualscale_seglinear_gemm_gelu_quant -- the fused producer of an FFN's
 * second linear: the same GEMM and epilogue as sq_dualscale_seglinear_gemm,
 * but instead of y it writes the next layer's DualScale activation planes of
 *   x2 = bf16(gelu(bf16(y)))
 * (pages: papernotes.org section DualScale, whose polarity table measures the
 * FFN's GELU output, the next layer's input; the pages give no GELU formula,
 * the models use the tanh approximation
 *   gelu(x) = x/2 (1 + tanh(sqrt(2/pi) (x + 0.044715 x^3))),
 * evaluated here as one fixed sequence of fp32 operations: tanh from e^(2|u|)
 * by Cody and Waite's reduction and a degree-7 Taylor series, 1 for |u| >= 9).
 * The next layer's codes follow sq_quantize_act with d = 1 and its steps
 * s_act_next = {s+, s-}: x2 >= 0: q+ = rne(min(fl(x2 / s+), 127)),
 * x2 < 0: q- = rne(max(fl(x2 / s-), -128)).  Its planes never round-trip
 * through a bf16 activation in HBM.
 *   planes, wq, s_w, s_act, bias, M, N, K, seg: as in
 *          sq_dualscale_seglinear_gemm; seg must be SQ_SEG_NONE (one K-segment,
 *          one group) and not SQ_FLAG_FP8 (SQ_ERR_UNSUPPORTED otherwise)
 *   s_act_next fp32 [2] device {s+, s-} of the next layer (one group, one
 *          K-segment, no SmoothQuant divisor), within [2^-40, 2^40]
 *   flags_next 0 (DualScale: planes_next int8 [2][M][N]) or
 *          SQ_FLAG_SINGLE_SCALE (one merged plane [1][M][N])
 *   planes_next int8 output, 16-byte aligned; N % 16 == 0 (it is the next
 *          layer's K)
 * y is finite whenever the scales and the bias are; the codes of a
 * non-finite y are unspecified.
 */
SQ_API sq_status sq_dualscale_seglinear_gemm_gelu_quant(const int8_t *planes, const int8_t *wq,
                                                       const float *s_w, const float *s_act,
                                                       const void *bias, int64_t M, int64_t N,
                                                       int64_t K, const sq_segments *seg,
                                                       const float *s_act_next,
                                                       int32_t flags_next, int8_t *planes_next,
                                                       sq_stream_t stream);

/*
 * sq_debug_gemm_s32 -- the same tensor-core kernel, storing the raw int32
 * accumulators instead of the epilogue, for bit-exact checks.
 *   acc int32 [S][P][M][N] output (16-byte aligned), polarity 0 = A+, 1 = A-;
 *   P = 1 (one product of the merged plane) with SQ_FLAG_SINGLE_SCALE.
 */
SQ_API sq_status sq_debug_gemm_s32(const int8_t *planes, const int8_t *wq, int64_t M,
                            int64_t N, int64_t K, const sq_segments *seg,
                            int32_t *acc, sq_stream_t stream);

/* sq_debug_gemm_s32 with the workspace of sq_dualscale_seglinear_gemm_ws: the
 * accumulators of split last-wave tiles are the sums of their pieces. */
SQ_API sq_status sq_debug_gemm_s32_ws(const int8_t *planes, const int8_t *wq, int64_t M,
                                      int64_t N, int64_t K, const sq_segments *seg,
                                      int32_t *acc, void *workspace, size_t workspace_bytes,
                                      sq_stream_t stream);

/*
 * Host-to-host execution of one layer with overlapped transfers.
 *
 * A pipeline owns three CUDA streams and a few events (host-side resources)
 * and uses a caller-provided device workspace of two slots, each holding one
 * chunk of `chunk_rows` activation rows (bf16), its planes and its output rows.
 * sq_dualscale_seglinear_host copies the rows of x_host to the device chunk by
 * chunk, runs sq_quantize_act and sq_dualscale_seglinear_gemm on each chunk and
 * copies the output rows back, so that the host-to-device copy of chunk c + 1,
 * the kernels of chunk c and the device-to-host copy of chunk c - 1 overlap.
 * The result is that of the device calls on the whole layer, bit for bit: rows
 * are independent in both kernels.  (The pages measure a single GPU's kernels;
 * this is serving plumbing around them, not part of the method.)
 *
 * sq_host_pipeline_workspace_bytes -- workspace size for layers with K <= max_K,
 * N <= max_N, G <= max_G and P <= max_P (P = 2 for DualScale, 1 single scale);
 * 0 for invalid sizes, including chunk_rows * max_K or chunk_rows * max_N above
 * 2^44 elements.
 *
 * sq_host_pipeline_create -- chunk_rows >= 1; workspace: device memory of at
 * least sq_host_pipeline_workspace_bytes(...) bytes, 256-byte aligned, owned by
 * the caller and untouched by anything else while the pipeline is in use.
 * Creates the streams and events on the current device.
 *
 * sq_host_pipeline_destroy -- waits for the pipeline's work, then releases its
 * streams and events (not the workspace).  NULL is a no-op.
 *
 * If sq_dualscale_seglinear_host fails after it has enqueued work, it waits for
 * the pipeline's streams before returning the error.
 *
 * sq_dualscale_seglinear_host -- arguments as in sq_quantize_act and
 * sq_dualscale_seglinear_gemm, except that x_host (bf16 [M][ldx]) and y_host
 * ([M][ldy], bf16 or fp32) are HOST pointers; page-locked memory is needed
 * for the copies to overlap (pageable memory works, serialised).  The work is
 * ordered after everything already enqueued on `stream`, and work enqueued on
 * `stream` afterwards (e.g. cudaStreamSynchronize) waits for the whole layer.
 * A pipeline serves one host thread at a time.
 */
typedef struct sq_host_pipeline sq_host_pipeline;

SQ_API size_t sq_host_pipeline_workspace_bytes(int64_t chunk_rows, int64_t max_K, int64_t max_N,
                                        int32_t max_G, int32_t max_P);
SQ_API sq_status sq_host_pipeline_create(int64_t chunk_rows, int64_t max_K, int64_t max_N,
                                  int32_t max_G, int32_t max_P, void *workspace,
                                  size_t workspace_bytes, sq_host_pipeline **out);
SQ_API sq_status sq_host_pipeline_destroy(sq_host_pipeline *pl);
SQ_API sq_status sq_dualscale_seglinear_host(sq_host_pipeline *pl, const void *x_host,
                                      int64_t M, int64_t K, int64_t ldx, const float *d,
                                      const float *s_act, const int8_t *wq,
                                      const float *s_w, const void *bias, void *y_host,
                                      sq_out_dtype out_dtype, int64_t N, int64_t ldy,
                                      const sq_segments *seg, sq_stream_t stream);

/*
 * sq_dualscale_seglinear_host_noalloc -- the host-to-host layer of
 * sq_dualscale_seglinear_host for callers that cannot allocate device memory.
 * (The pages have no counterpart: this is deployment plumbing, not part of the
 * method.)
 *
 * Who needs it: a library that is loaded into a host application which owns
 * the device-memory budget (a plug-in of an inference server, an embedded
 * runtime) is often not allowed to call cudaMalloc at all; a latency-critical
 * loop cannot afford cudaMalloc and cudaFree, which may synchronise the whole
 * device and stall every other stream; and a process already at the edge of
 * the device's memory cannot count on an allocation succeeding in the middle
 * of its work.  Such callers cannot provide the workspace that
 * sq_host_pipeline_create needs.
 *
 * This call needs none.  Its device scratch is one fixed array of
 * SQ_NOALLOC_SCRATCH_BYTES (32 MiB) inside the library's device image: every
 * GPU on which the library is loaded holds it until the process exits.  The
 * call itself calls no cudaMalloc, cudaFree or other allocating routine, and
 * it creates no streams or events.
 *
 * Arguments and results are those of sq_dualscale_seglinear_host without the
 * pipeline: x_host (bf16 [M][ldx]) and y_host ([M][ldy], bf16 or fp32) are
 * HOST pointers (page-locked or pageable), the other pointers are device
 * buffers the caller owns, and the output equals the device calls
 * sq_quantize_act + sq_dualscale_seglinear_gemm on the whole layer bit for
 * bit.  Rows are processed in chunks as large as the scratch allows (a
 * multiple of 128 rows when at least 128 fit), all on `stream`, one after the
 * other: copy in, quantize, GEMM, copy out.  Nothing overlaps, so it is slower
 * than a pipeline, and work enqueued on `stream` afterwards waits for the
 * whole layer.
 *
 * Limit: one row's x (2K bytes), planes (G*P*K bytes) and output (4 bytes per
 * column, N rounded up to a multiple of 8), each region rounded up to 256
 * bytes, must fit in SQ_NOALLOC_SCRATCH_BYTES; otherwise the call returns
 * SQ_ERR_TOO_LARGE and enqueues nothing.  Other errors as in
 * sq_dualscale_seglinear_host; after a failure past the first enqueue the call
 * waits for `stream` before it returns.
 *
 * Sharing: every call on a device uses the same scratch, and the scratch keeps
 * whatever the last call left in it.  Nothing in it has to start at zero:
 * each chunk's rows, planes and output are written in full before they are
 * read.  Calls that can overlap on the GPU -- calls on different streams, or
 * from several host threads, without an ordering between them -- race on the
 * scratch and corrupt each other's results; order them on one stream (or with
 * events).
 *
 * First call: the first call on each device looks up the scratch's device
 * address (cudaGetSymbolAddress), which may load the library's device code on
 * that device.  Make that first call before any stream capture begins.
 */
#define SQ_NOALLOC_SCRATCH_BYTES (32u * 1024u * 1024u)

SQ_API sq_status sq_dualscale_seglinear_host_noalloc(const void *x_host, int64_t M, int64_t K,
                                                     int64_t ldx, const float *d,
                                                     const float *s_act, const int8_t *wq,
                                                     const float *s_w, const void *bias,
                                                     void *y_host, sq_out_dtype out_dtype,
                                                     int64_t N, int64_t ldy,
                                                     const sq_segments *seg,
                                                     sq_stream_t stream);

/*
 * sq_debug_timeout_probe -- test only: launches one small kernel that waits on
 * a barrier nothing ever signals, with the library's bounded wait and a limit
 * of `limit_us` microseconds (1..100000), so that the wait runs out and the
 * kernel records SQ_ERR_DEVICE_TIMEOUT in the device error word, exactly as a
 * stalled GEMM or quantize kernel would.  Nothing faults or hangs; the
 * context stays usable.  Read the result with sq_get_device_status().  (A
 * verification aid for the failure reporting; it has no counterpart in the
 * pages.)
 */
SQ_API sq_status sq_debug_timeout_probe(uint32_t limit_us, sq_stream_t stream);

/*
 * sq_debug_bounds_checks -- 1 if this library is the bounds-checked debug
 * build (libsegquant_debug.so, compiled with SQ_DEBUG_BOUNDS), 0 for the
 * release build.  In the debug build every plain global store of every kernel
 * first tests its index against its buffer's logical extent (the sizes and
 * leading dimensions of the call); a store that fails the test is skipped and
 * the kernel records SQ_ERR_DEVICE_BOUNDS in the device error word (the first
 * report of a launch wins), read with sq_get_device_status().  Tensor stores
 * (TMA) are clipped to their tensor maps by the hardware and need no test.
 * The debug build computes the same results as the release build; it exists
 * to run the test suite with the checks in place.
 */
SQ_API int32_t sq_debug_bounds_checks(void);

/*
 * sq_debug_bounds_probe -- test only: launches one thread that stores through
 * the checked path into element n of `buf` while telling the check that the
 * buffer holds n elements.  buf: device int32 [n + 1] (the extra element is a
 * guard, so that even an unchecked store stays inside the allocation);
 * n >= 1.  The debug build skips the store and records SQ_ERR_DEVICE_BOUNDS;
 * the release build launches nothing and returns SQ_ERR_UNSUPPORTED.
 */
SQ_API sq_status sq_debug_bounds_probe(int32_t *buf, int64_t n, sq_stream_t stream);

/*
 * sq_get_device_status -- waits for the work enqueued on `stream`, then
 * returns the library's device-side error word and clears it: SQ_OK, or
 * SQ_ERR_DEVICE_TIMEOUT if a kernel's bounded wait on a barrier ran out (the
 * kernel then abandoned its tile and left its outputs incomplete), or, in the
 * debug build only, SQ_ERR_DEVICE_BOUNDS.
 * The word is one per device, shared by every stream and every caller of the
 * library in the process: a report set by a kernel on another stream is seen
 * (and cleared) by whichever caller reads first, and a report set between
 * this call's read and its clear is lost.  Callers that launch on several
 * streams should synchronise those streams, or serialise their status checks,
 * before relying on the result.  Synchronises only `stream` (0: the legacy
 * default stream, which also waits for the other blocking streams).
 * After a timeout a kernel waits, again with a limit, for its own copies and
 * tensor-core operations to finish before it releases its tensor memory and
 * exits.  If that wait runs out too, those operations were still pending when
 * the memory was released: treat the CUDA context as unusable and end the
 * process (a healthy GPU completes them in microseconds).
 */
SQ_API sq_status sq_get_device_status(sq_stream_t stream);

/*
 * sq_choose_single_scale -- the adaptive DualScale policy, on the host: decides
 * whether a layer should use the single-scale path (SQ_FLAG_SINGLE_SCALE).
 * Pages: papernotes.org "SegQuant", section "Limitations" (DualScale doubles
 * the integer work; enable it only where activations are strongly
 * polarity-asymmetric).  The pages fix no test; the reading taken: for every
 * group and K-segment recover the calibrated max = s+ * 127 and
 * |min| = s- * 128 (FP8: both * 448) from the DualScale steps; the layer
 * switches to single scale when, in every group and K-segment, the larger side
 * is below threshold times the smaller (fp32 arithmetic).  A side that was
 * empty in calibration has step 1 and so counts as a large side: such layers
 * keep DualScale.  After a decision of 1 the caller re-runs sq_calibrate_act
 * with SQ_FLAG_SINGLE_SCALE and uses that flag on every call of the layer.
 *   s_act    HOST fp32 [n_steps][2] {s+, s-}: the steps of sq_calibrate_act
 *            without SQ_FLAG_SINGLE_SCALE, copied to the host; positive, finite
 *   n_steps  G * S, 1..SQ_MAX_SEGMENTS^2
 *   flags    0 or SQ_FLAG_FP8 (which code range the steps belong to)
 *   threshold > 1 (2 in the library's own layer helper)
 *   single   HOST int32 output: 1 (use single scale) or 0 (keep DualScale)
 * Touches no device and launches nothing.
 */
SQ_API sq_status sq_choose_single_scale(const float *s_act, int32_t n_steps, int32_t flags,
                                        float threshold, int32_t *single);

/* Static, human-readable name of a status code (never NULL). */
SQ_API const char *sq_status_string(sq_status status);

/* Library ABI version (major * 100 + minor). */
SQ_API int32_t sq_version(void);

#ifdef __cplusplus
}
#endif
#endif /* SEGQUANT_H */
