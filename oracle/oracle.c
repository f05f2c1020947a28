/*
 * oracle.c -- plain CPU oracle for the SegQuant quantized linear layer
 * (DualScale polarity split + SegLinear segmentation, W8A8).
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the library's product path may call,
 * link or load this file; only the tests, the smoke check and the benchmark's
 * CPU-baseline leg do.  It shares no code, header, table or helper with the
 * CUDA path (w8a8_gemm_b200/csrc): its own structs, its own bf16 decoding, its
 * own loops.  Every step is written the slow, obvious way so that it can be
 * checked against the pages by eye.
 *
 * Sources (page title, section, formula):
 *  - "SegQuant: A Semantics-Aware and Generalizable Quantization Framework for
 *    Diffusion Models" (papernotes.org notes), section "DualScale":
 *    X+ = max(X,0), X- = min(X,0); s- = |min(x)|/q_min, s+ = max(x)/q_max;
 *    Y ~= s+ s_w (X^+ W^) + s- s_w (X^- W^).
 *  - same page, section "SegLinear": output-segmented Y^ = [X^W^_1, ..., X^W^_N]
 *    (W split by columns); input-segmented Y^ = sum_i X^_i W^_i (W split by rows).
 *  - "SegQuant" author page (hliangzhao.me), section 3 "DualScale": the
 *    case-wise quantizer Q_dual(x) = round(x/s-) for x < 0, round(x/s+) for
 *    x >= 0, and the two-product reconstruction.
 *  - papernotes.org page, "Loss function / training strategy": AMax (max-abs)
 *    calibration is one of the two calibrators.
 *
 * Readings where the pages are silent or ambiguous (all stated again in the
 * design notes):
 *  - q_min: the pages divide |min| by q_min; with signed int8 q_min = -128 that
 *    would give a negative step, so the magnitude 128 is used: s- = |min|/128,
 *    s+ = max/127.  X^- lies in [-128, 0], X^+ in [0, 127].
 *  - "round" is round-half-to-even, in fp32.
 *  - The SmoothQuant divisor d (per group, per input channel, > 0) is an input.
 *    Activations are quantized as x / d, weights as w * d.  The quantizer is
 *    the pages' round(u / s) evaluated in fp32 with IEEE divisions: the
 *    smoothed activation u = fl(x / d) (u = x when there is no divisor), the
 *    quotient v = fl(u / s+-), then q = rne(clamp(v)).  Where v itself lands
 *    on a half-integer, the tie goes to the even code, even if the exact
 *    quotient u / s lay on one side of it.
 *  - Out-of-range values saturate: q+ <= 127, q- >= -128.  NaN goes to 0 in
 *    both planes (neither x < 0 nor x >= 0 holds); -0.0 goes to the + plane.
 *  - Degenerate calibration: max <= 0 gives s+ = 1, min >= 0 gives s- = 1; an
 *    all-zero weight column segment gives s_w = 1.
 *  - Weights: symmetric AMax per output channel and per K-segment,
 *    s_w = amax / 127, q = rne(clamp(w' / s_w, -127, 127)).
 *  - W4A8 (the papernotes page's and the author page's "SegQuant-4" / W4A8
 *    rows in the results and deployment tables; the pages give no formula):
 *    the same symmetric AMax rule with q_max = 7, s_w = amax / 7,
 *    q = rne(clamp(w' / s_w, -7, 7)); activations stay DualScale int8 and the
 *    integer product and epilogue are unchanged.  Storage: two codes per byte,
 *    4-bit two's complement, channel 2j in the low nibble and 2j + 1 in the
 *    high nibble (orc_pack_w4).
 *  - Output-segmented layers may carry their own activation parameters per
 *    output segment (a "group" g: its own d and s+/s-, hence its own planes).
 *    G = 1 is the pages' formula with one shared X^.
 *  - Single-scale mode (the adaptive variant the papernotes page names under
 *    "Limitations": DualScale only on polarity-asymmetric layers): one step
 *    s = max(max u, -min u) / 127 for both signs, i.e. the DualScale quantizer
 *    with s+ = s-, whose two planes are then one: q = q+ + q- in [-128, 127],
 *    and one integer product A = sum q w.  Planes [G][1][M][K].
 *  - Epilogue in fp32, fixed order (the pages fix none), read left to right
 *    as the reconstruction formula is written: y starts at 0; for each
 *    K-segment i in ascending order, with the folded coefficients
 *    c+_i = fl(s_w[i][n] * s+_i), c-_i = fl(s_w[i][n] * s-_i) of the products
 *    s+ s_w and s- s_w the formula shows, y = fma(c+_i, f(A+_i), y), then
 *    y = fma(c-_i, f(A-_i), y) (single scale: y = fma(c_i, f(A_i), y)); the
 *    bias is added last.  f is int32 -> fp32 round-to-nearest; fma rounds
 *    once.
 *
 * Layouts (row-major, innermost last):
 *  x      bf16 bits [M][ldx]          activations (nn.Linear input)
 *  w      bf16 bits [N][K]            nn.Linear weight (the pages' W^T)
 *  d      fp32 [G][K] or NULL (=1)    SmoothQuant divisor per group
 *  s_act  fp32 [G][S][2]              {s+, s-} per group and K-segment
 *  planes int8 [G][P][M][K]           P = 2: plane 0 = X^+, plane 1 = X^-;
 *                                     P = 1 (single scale): q = X^+ + X^-
 *  wq     int8 [N][K]                 quantized weight
 *  s_w    fp32 [S][N]                 weight scale per K-segment, per column
 *  acc    int32 [S][P][M][N]          raw accumulators per segment, polarity
 *  y      fp32 [rows][N]              layer output (fp32 epilogue)
 *
 * Segment description: mode 0 = none, 1 = output-segmented (offsets over N),
 * 2 = input-segmented (offsets over K).  offsets has n_seg + 1 ascending
 * entries from 0 to N (or K).  S = n_seg in input mode, else 1.  G is 1 or, in
 * output mode, n_seg.
 *
 * Build: gcc -O2 -fopenmp -ffp-contract=off -fno-fast-math (no -ffast-math:
 * the rounding of every fp32 operation is part of the definition).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORC_MODE_NONE 0
#define ORC_MODE_OUTPUT 1
#define ORC_MODE_INPUT 2

static float orc_bf16(uint16_t h) {
  uint32_t u = ((uint32_t)h) << 16;
  float f;
  memcpy(&f, &u, sizeof f);
  return f;
}

/* index i with off[i] <= p < off[i+1] */
static int orc_seg_index(const int32_t *off, int n_seg, int64_t p) {
  for (int i = 0; i < n_seg; ++i)
    if (p < off[i + 1]) return i;
  return n_seg - 1;
}

static int orc_check_seg(int mode, int n_seg, const int32_t *off, int G,
                         int64_t N, int64_t K) {
  if (mode == ORC_MODE_NONE) return (n_seg == 1 && G == 1) ? 0 : -1;
  if (n_seg < 1 || off == NULL) return -1;
  int64_t extent = (mode == ORC_MODE_OUTPUT) ? N : K;
  if (off[0] != 0 || off[n_seg] != extent) return -1;
  for (int i = 0; i < n_seg; ++i)
    if (off[i + 1] <= off[i]) return -1;
  if (mode == ORC_MODE_INPUT && G != 1) return -1;
  if (mode == ORC_MODE_OUTPUT && G != 1 && G != n_seg) return -1;
  return 0;
}

int orc_num_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

/* ---------------------------------------------------------------------------
 * AMax calibration of the two activation scales (static, offline).
 * For group g and K-segment i, over the calibration rows and the channels c of
 * segment i: u = x / d[g][c]; hi = max(0, max u); lo = min(0, min u);
 * s+ = hi / 127 (1 if hi == 0), s- = -lo / 128 (1 if lo == 0).
 * In output mode N is unused; pass the layer's N anyway for the check.
 * ------------------------------------------------------------------------- */
int orc_calibrate_act(const uint16_t *x, int64_t M, int64_t K, int64_t ldx,
                      const float *d, int mode, int n_seg,
                      const int32_t *offsets, int G, int64_t N, int single,
                      float *s_act) {
  if (orc_check_seg(mode, n_seg, offsets, G, N, K)) return -1;
  int S = (mode == ORC_MODE_INPUT) ? n_seg : 1;
  for (int g = 0; g < G; ++g) {
    for (int i = 0; i < S; ++i) {
      int64_t c0 = (S == 1) ? 0 : offsets[i];
      int64_t c1 = (S == 1) ? K : offsets[i + 1];
      float hi = 0.0f, lo = 0.0f;
      for (int64_t m = 0; m < M; ++m) {
        for (int64_t c = c0; c < c1; ++c) {
          float xv = orc_bf16(x[m * ldx + c]);
          float dv = d ? d[(int64_t)g * K + c] : 1.0f;
          float u = xv / dv;
          if (u > hi) hi = u; /* NaN compares false: ignored */
          if (u < lo) lo = u;
        }
      }
      float sp = (hi > 0.0f) ? hi / 127.0f : 1.0f;
      float sm = (lo < 0.0f) ? (-lo) / 128.0f : 1.0f;
      if (single) { /* one symmetric step: the larger side over 127 */
        float amax = (hi > -lo) ? hi : -lo;
        sp = (amax > 0.0f) ? amax / 127.0f : 1.0f;
        sm = sp;
      }
      s_act[((int64_t)g * S + i) * 2 + 0] = sp;
      s_act[((int64_t)g * S + i) * 2 + 1] = sm;
    }
  }
  return 0;
}

/* ---------------------------------------------------------------------------
 * DualScale activation quantization (Q_dual) with SmoothQuant divisor:
 * author page section 3, Q_dual(x) = round(x/s-) for x < 0 and round(x/s+)
 * for x >= 0, applied to the smoothed activation u = x / d.  Both quotients
 * are fp32 IEEE divisions; the clamps are the int8 code range.
 * ------------------------------------------------------------------------- */
int orc_quantize_act(const uint16_t *x, int64_t M, int64_t K, int64_t ldx,
                     const float *d, const float *s_act, int mode, int n_seg,
                     const int32_t *offsets, int G, int64_t N, int single,
                     int8_t *planes) {
  if (orc_check_seg(mode, n_seg, offsets, G, N, K)) return -1;
  int S = (mode == ORC_MODE_INPUT) ? n_seg : 1;
  int P = single ? 1 : 2;
  for (int g = 0; g < G; ++g) {
    int8_t *plus = planes + ((int64_t)g * P + 0) * M * K;
    int8_t *minus = single ? plus : planes + ((int64_t)g * P + 1) * M * K;
    for (int64_t m = 0; m < M; ++m) {
      for (int64_t c = 0; c < K; ++c) {
        int i = (S == 1) ? 0 : orc_seg_index(offsets, n_seg, c);
        float sp = s_act[((int64_t)g * S + i) * 2 + 0];
        float sm = s_act[((int64_t)g * S + i) * 2 + 1];
        float xv = orc_bf16(x[m * ldx + c]);
        float u = d ? xv / d[(int64_t)g * K + c] : xv; /* smoothed activation */
        int qp = 0, qm = 0;
        if (xv < 0.0f) { /* X- branch: round(u / s-) */
          float v = u / sm;
          if (v < -128.0f) v = -128.0f;
          qm = (int)rintf(v);
        } else if (xv >= 0.0f) { /* X+ branch: round(u / s+) */
          float v = u / sp;
          if (v > 127.0f) v = 127.0f;
          qp = (int)rintf(v);
        }
        if (single) {
          plus[m * K + c] = (int8_t)(qp + qm); /* one of the two is 0 */
        } else {
          plus[m * K + c] = (int8_t)qp;
          minus[m * K + c] = (int8_t)qm;
        }
      }
    }
  }
  return 0;
}

/* ---------------------------------------------------------------------------
 * Segment-wise symmetric AMax weight quantization.
 * Column n of the pages' W (row n of the nn.Linear weight) is quantized
 * independently on every K-segment i; in output mode each output segment j
 * folds its own group's divisor d[j] when G > 1.
 * ------------------------------------------------------------------------- */
int orc_quantize_weight_q(const uint16_t *w, int64_t N, int64_t K, const float *d,
                          int mode, int n_seg, const int32_t *offsets, int G,
                          int qmax, int8_t *wq, float *s_w) {
  if (orc_check_seg(mode, n_seg, offsets, G, N, K)) return -1;
  if (qmax != 127 && qmax != 7) return -1;
  float fq = (float)qmax;
  int S = (mode == ORC_MODE_INPUT) ? n_seg : 1;
  for (int64_t n = 0; n < N; ++n) {
    int g = (mode == ORC_MODE_OUTPUT && G > 1)
                ? orc_seg_index(offsets, n_seg, n) : 0;
    for (int i = 0; i < S; ++i) {
      int64_t k0 = (S == 1) ? 0 : offsets[i];
      int64_t k1 = (S == 1) ? K : offsets[i + 1];
      float amax = 0.0f;
      for (int64_t k = k0; k < k1; ++k) {
        float dv = d ? d[(int64_t)g * K + k] : 1.0f;
        float wv = orc_bf16(w[n * K + k]) * dv;
        float a = fabsf(wv);
        if (a > amax) amax = a;
      }
      float s = (amax > 0.0f) ? amax / fq : 1.0f;
      s_w[(int64_t)i * N + n] = s;
      for (int64_t k = k0; k < k1; ++k) {
        float dv = d ? d[(int64_t)g * K + k] : 1.0f;
        float v = (orc_bf16(w[n * K + k]) * dv) / s;
        if (v > fq) v = fq;
        if (v < -fq) v = -fq;
        wq[n * K + k] = (int8_t)(int)rintf(v);
      }
    }
  }
  return 0;
}

int orc_quantize_weight(const uint16_t *w, int64_t N, int64_t K, const float *d,
                        int mode, int n_seg, const int32_t *offsets, int G,
                        int8_t *wq, float *s_w) {
  return orc_quantize_weight_q(w, N, K, d, mode, n_seg, offsets, G, 127, wq, s_w);
}

/* 4-bit storage of codes in [-8, 7]: byte [n][j] holds channel 2j in its low
 * nibble and channel 2j + 1 in its high nibble, each as 4-bit two's complement.
 * K must be even. */
int orc_pack_w4(const int8_t *wq, int64_t N, int64_t K, uint8_t *packed) {
  if (K % 2 != 0) return -1;
  for (int64_t n = 0; n < N; ++n)
    for (int64_t j = 0; j < K / 2; ++j) {
      int lo = wq[n * K + 2 * j], hi = wq[n * K + 2 * j + 1];
      if (lo < -8 || lo > 7 || hi < -8 || hi > 7) return -1;
      packed[n * (K / 2) + j] = (uint8_t)((lo & 0xF) | ((hi & 0xF) << 4));
    }
  return 0;
}

/* ---------------------------------------------------------------------------
 * Integer products: A+-_i[m][n] = sum_{k in segment i} X^+-[g(n)][m][k] * W^[n][k]
 * accumulated in int32 (the pages' fixed-width integer GEMM).  rows == NULL
 * means all M rows; otherwise acc row r holds row rows[r].
 * acc layout [S][2][n_rows][N].
 * ------------------------------------------------------------------------- */
int orc_gemm_s32(const int8_t *planes, const int8_t *wq, int64_t M, int64_t N,
                 int64_t K, int mode, int n_seg, const int32_t *offsets, int G,
                 int P, const int64_t *rows, int64_t n_rows, int32_t *acc,
                 int n_threads) {
  if (orc_check_seg(mode, n_seg, offsets, G, N, K)) return -1;
  if (P != 1 && P != 2) return -1;
  int S = (mode == ORC_MODE_INPUT) ? n_seg : 1;
  if (rows == NULL) n_rows = M;
#ifdef _OPENMP
  if (n_threads < 1) n_threads = 1;
#pragma omp parallel for schedule(dynamic, 1) num_threads(n_threads)
#endif
  for (int64_t r = 0; r < n_rows; ++r) {
    int64_t m = rows ? rows[r] : r;
    for (int64_t n = 0; n < N; ++n) {
      int g = (mode == ORC_MODE_OUTPUT && G > 1)
                  ? orc_seg_index(offsets, n_seg, n) : 0;
      const int8_t *wn = wq + n * K;
      for (int i = 0; i < S; ++i) {
        int64_t k0 = (S == 1) ? 0 : offsets[i];
        int64_t k1 = (S == 1) ? K : offsets[i + 1];
        for (int pl = 0; pl < P; ++pl) {
          const int8_t *xq = planes + (((int64_t)g * P + pl) * M + m) * K;
          int32_t a = 0;
          for (int64_t k = k0; k < k1; ++k) a += (int32_t)xq[k] * (int32_t)wn[k];
          acc[(((int64_t)i * P + pl) * n_rows + r) * N + n] = a;
        }
      }
    }
  }
  return 0;
}

/* ---------------------------------------------------------------------------
 * Full layer: integer products, then the DualScale reconstruction in fp32
 *   y[m][n] = sum_i (s_w[i][n] s+_i) f(A+_i) + (s_w[i][n] s-_i) f(A-_i) + bias[n]
 * with one fused multiply-add per term, segments in ascending order, + before
 * -, and the bias added last.  bias: bf16 bits [N] or NULL.  y [n_rows][N].
 * ------------------------------------------------------------------------- */
int orc_gemm(const int8_t *planes, const int8_t *wq, const float *s_w,
             const float *s_act, const uint16_t *bias, int64_t M, int64_t N,
             int64_t K, int mode, int n_seg, const int32_t *offsets, int G,
             int P, const int64_t *rows, int64_t n_rows, float *y,
             int n_threads) {
  if (orc_check_seg(mode, n_seg, offsets, G, N, K)) return -1;
  if (P != 1 && P != 2) return -1;
  int S = (mode == ORC_MODE_INPUT) ? n_seg : 1;
  if (rows == NULL) n_rows = M;
#ifdef _OPENMP
  if (n_threads < 1) n_threads = 1;
#pragma omp parallel for schedule(dynamic, 1) num_threads(n_threads)
#endif
  for (int64_t r = 0; r < n_rows; ++r) {
    int64_t m = rows ? rows[r] : r;
    for (int64_t n = 0; n < N; ++n) {
      int g = (mode == ORC_MODE_OUTPUT && G > 1)
                  ? orc_seg_index(offsets, n_seg, n) : 0;
      const int8_t *xp = planes + (((int64_t)g * P + 0) * M + m) * K;
      const int8_t *xm = planes + (((int64_t)g * P + (P - 1)) * M + m) * K;
      const int8_t *wn = wq + n * K;
      float yv = 0.0f;
      for (int i = 0; i < S; ++i) {
        int64_t k0 = (S == 1) ? 0 : offsets[i];
        int64_t k1 = (S == 1) ? K : offsets[i + 1];
        float sw = s_w[(int64_t)i * N + n];
        float cp = sw * s_act[((int64_t)g * S + i) * 2 + 0]; /* c+ = s_w s+ */
        float cm = sw * s_act[((int64_t)g * S + i) * 2 + 1]; /* c- = s_w s- */
        if (P == 2) { /* DualScale: + term, then - term */
          int32_t ap = 0, am = 0;
          for (int64_t k = k0; k < k1; ++k) {
            ap += (int32_t)xp[k] * (int32_t)wn[k];
            am += (int32_t)xm[k] * (int32_t)wn[k];
          }
          yv = fmaf(cp, (float)ap, yv);
          yv = fmaf(cm, (float)am, yv);
        } else { /* single scale: one term */
          int32_t a = 0;
          for (int64_t k = k0; k < k1; ++k) a += (int32_t)xp[k] * (int32_t)wn[k];
          yv = fmaf(cp, (float)a, yv);
        }
      }
      if (bias) yv = yv + orc_bf16(bias[n]);
      y[r * N + n] = yv;
    }
  }
  return 0;
}

/* ===========================================================================
 * FP8 variant (the pages' "W8A8(fp)" rows for SDXL in the results table,
 * which they do not define).  Reading: both operands are FP8 E4M3 codes (the
 * OCP "E4M3FN" format: 1 sign, 4 exponent bits with bias 7, 3 mantissa bits,
 * no infinities, S.1111.111 is NaN, largest finite 448 = 1.75 * 2^8, smallest
 * normal 2^-6, subnormals m * 2^-9).  DualScale steps become s+ = max/448 and
 * s- = |min|/448 (single scale: the larger side / 448), weights
 * s_w = amax/448; every code is e4m3(fl(v)) with round-half-to-even and
 * finite saturation to +-448.  The products of two E4M3 values are exact; the
 * oracle sums them exactly (in double, whose 53 bits hold every such sum for
 * K < 2^15) and rounds the sum once to fp32; the epilogue is the W8A8 one.
 * ========================================================================= */

static float orc_e4m3_value(uint8_t b) {
  int s = b >> 7, e = (b >> 3) & 0xF, m = b & 7;
  float v;
  if (e == 0xF && m == 7) return NAN;
  if (e == 0)
    v = ldexpf((float)m, -9); /* subnormal: m * 2^-9 */
  else
    v = ldexpf((float)(8 + m), e - 10); /* (1 + m/8) * 2^(e-7) */
  return s ? -v : v;
}

/* fp32 -> E4M3 code, round half to even, |v| beyond 448 (infinities
 * included) saturates to 448; NaN gives 0x7F. */
static uint8_t orc_e4m3_code(float v) {
  if (isnan(v)) return 0x7F;
  uint8_t sign = signbit(v) ? 0x80 : 0x00;
  float a = fabsf(v);
  if (a >= 448.0f) return sign | 0x7E;
  /* quantum of the binade of a: 2^(e-3) for normals (e >= -6), 2^-9 below */
  int e;
  frexpf(a, &e);         /* a = f * 2^e, f in [0.5, 1): binade exponent e - 1 */
  int be = e - 1;
  if (be < -6) be = -6;  /* subnormal range shares the quantum 2^-9 */
  float q = ldexpf(1.0f, be - 3);
  float n = rintf(a / q); /* exact division by a power of two, then RNE */
  float r = n * q;        /* exact; may step into the next binade */
  if (r > 448.0f) r = 448.0f;
  /* encode r */
  if (r == 0.0f) return sign;
  int re;
  frexpf(r, &re);
  int rb = re - 1;
  if (rb < -6) { /* subnormal: r = m * 2^-9 */
    int m = (int)ldexpf(r, 9);
    return sign | (uint8_t)m;
  }
  int m = (int)(ldexpf(r, -rb) * 8.0f) - 8;
  return sign | (uint8_t)(((rb + 7) << 3) | m);
}

int orc_e4m3_encode(const float *v, int64_t n, uint8_t *out) {
  for (int64_t i = 0; i < n; ++i) out[i] = orc_e4m3_code(v[i]);
  return 0;
}

int orc_e4m3_decode(const uint8_t *b, int64_t n, float *out) {
  for (int64_t i = 0; i < n; ++i) out[i] = orc_e4m3_value(b[i]);
  return 0;
}

int orc_calibrate_act_fp8(const uint16_t *x, int64_t M, int64_t K, int64_t ldx,
                          const float *d, int mode, int n_seg, const int32_t *offsets,
                          int G, int64_t N, int single, float *s_act) {
  if (orc_check_seg(mode, n_seg, offsets, G, N, K)) return -1;
  int S = (mode == ORC_MODE_INPUT) ? n_seg : 1;
  for (int g = 0; g < G; ++g) {
    for (int i = 0; i < S; ++i) {
      int64_t c0 = (S == 1) ? 0 : offsets[i];
      int64_t c1 = (S == 1) ? K : offsets[i + 1];
      float hi = 0.0f, lo = 0.0f;
      for (int64_t m = 0; m < M; ++m)
        for (int64_t c = c0; c < c1; ++c) {
          float dv = d ? d[(int64_t)g * K + c] : 1.0f;
          float u = orc_bf16(x[m * ldx + c]) / dv;
          if (u > hi) hi = u;
          if (u < lo) lo = u;
        }
      float sp = (hi > 0.0f) ? hi / 448.0f : 1.0f;
      float sm = (lo < 0.0f) ? (-lo) / 448.0f : 1.0f;
      if (single) {
        float amax = (hi > -lo) ? hi : -lo;
        sp = (amax > 0.0f) ? amax / 448.0f : 1.0f;
        sm = sp;
      }
      s_act[((int64_t)g * S + i) * 2 + 0] = sp;
      s_act[((int64_t)g * S + i) * 2 + 1] = sm;
    }
  }
  return 0;
}

/* Planes of E4M3 codes [G][P][M][K], with u = fl(x / d) and fp32 IEEE
 * divisions as in orc_quantize_act.  x >= 0 (-0.0 included): the + plane
 * holds e4m3(fl(u / s+)) and the - plane 0x00; x < 0: the - plane holds
 * e4m3(fl(u / s-)) and the + plane 0x00; NaN: both 0x00.  Single scale: one
 * plane holding the code of whichever branch applies. */
int orc_quantize_act_fp8(const uint16_t *x, int64_t M, int64_t K, int64_t ldx,
                         const float *d, const float *s_act, int mode, int n_seg,
                         const int32_t *offsets, int G, int64_t N, int single,
                         uint8_t *planes) {
  if (orc_check_seg(mode, n_seg, offsets, G, N, K)) return -1;
  int S = (mode == ORC_MODE_INPUT) ? n_seg : 1;
  int P = single ? 1 : 2;
  for (int g = 0; g < G; ++g) {
    uint8_t *plus = planes + ((int64_t)g * P + 0) * M * K;
    uint8_t *minus = planes + ((int64_t)g * P + (P - 1)) * M * K;
    for (int64_t m = 0; m < M; ++m)
      for (int64_t c = 0; c < K; ++c) {
        int i = (S == 1) ? 0 : orc_seg_index(offsets, n_seg, c);
        float sp = s_act[((int64_t)g * S + i) * 2 + 0];
        float sm = s_act[((int64_t)g * S + i) * 2 + 1];
        float xv = orc_bf16(x[m * ldx + c]);
        float u = d ? xv / d[(int64_t)g * K + c] : xv;
        uint8_t qp = 0, qm = 0;
        if (xv < 0.0f)
          qm = orc_e4m3_code(u / sm);
        else if (xv >= 0.0f)
          qp = orc_e4m3_code(u / sp);
        if (single) {
          plus[m * K + c] = (xv < 0.0f) ? qm : qp;
        } else {
          plus[m * K + c] = qp;
          minus[m * K + c] = qm;
        }
      }
  }
  return 0;
}

int orc_quantize_weight_fp8(const uint16_t *w, int64_t N, int64_t K, const float *d,
                            int mode, int n_seg, const int32_t *offsets, int G,
                            uint8_t *wq, float *s_w) {
  if (orc_check_seg(mode, n_seg, offsets, G, N, K)) return -1;
  int S = (mode == ORC_MODE_INPUT) ? n_seg : 1;
  for (int64_t n = 0; n < N; ++n) {
    int g = (mode == ORC_MODE_OUTPUT && G > 1) ? orc_seg_index(offsets, n_seg, n) : 0;
    for (int i = 0; i < S; ++i) {
      int64_t k0 = (S == 1) ? 0 : offsets[i];
      int64_t k1 = (S == 1) ? K : offsets[i + 1];
      float amax = 0.0f;
      for (int64_t k = k0; k < k1; ++k) {
        float dv = d ? d[(int64_t)g * K + k] : 1.0f;
        float a = fabsf(orc_bf16(w[n * K + k]) * dv);
        if (a > amax) amax = a;
      }
      float s = (amax > 0.0f) ? amax / 448.0f : 1.0f;
      s_w[(int64_t)i * N + n] = s;
      for (int64_t k = k0; k < k1; ++k) {
        float dv = d ? d[(int64_t)g * K + k] : 1.0f;
        wq[n * K + k] = orc_e4m3_code((orc_bf16(w[n * K + k]) * dv) / s);
      }
    }
  }
  return 0;
}

/* Exact per-segment products of E4M3 codes, rounded once to fp32:
 * acc layout [S][P][n_rows][N] (fp32). */
int orc_gemm_fp8_acc(const uint8_t *planes, const uint8_t *wq, int64_t M, int64_t N,
                     int64_t K, int mode, int n_seg, const int32_t *offsets, int G,
                     int P, const int64_t *rows, int64_t n_rows, float *acc,
                     int n_threads) {
  if (orc_check_seg(mode, n_seg, offsets, G, N, K)) return -1;
  if (P != 1 && P != 2) return -1;
  int S = (mode == ORC_MODE_INPUT) ? n_seg : 1;
  if (rows == NULL) n_rows = M;
#ifdef _OPENMP
  if (n_threads < 1) n_threads = 1;
#pragma omp parallel for schedule(dynamic, 1) num_threads(n_threads)
#endif
  for (int64_t r = 0; r < n_rows; ++r) {
    int64_t m = rows ? rows[r] : r;
    for (int64_t n = 0; n < N; ++n) {
      int g = (mode == ORC_MODE_OUTPUT && G > 1) ? orc_seg_index(offsets, n_seg, n) : 0;
      const uint8_t *wn = wq + n * K;
      for (int i = 0; i < S; ++i) {
        int64_t k0 = (S == 1) ? 0 : offsets[i];
        int64_t k1 = (S == 1) ? K : offsets[i + 1];
        for (int pl = 0; pl < P; ++pl) {
          const uint8_t *xq = planes + (((int64_t)g * P + pl) * M + m) * K;
          double a = 0.0;
          for (int64_t k = k0; k < k1; ++k)
            a += (double)orc_e4m3_value(xq[k]) * (double)orc_e4m3_value(wn[k]);
          acc[(((int64_t)i * P + pl) * n_rows + r) * N + n] = (float)a;
        }
      }
    }
  }
  return 0;
}

/* Full FP8 layer: the W8A8 epilogue with f(A) replaced by the fp32 sums. */
int orc_gemm_fp8(const uint8_t *planes, const uint8_t *wq, const float *s_w,
                 const float *s_act, const uint16_t *bias, int64_t M, int64_t N,
                 int64_t K, int mode, int n_seg, const int32_t *offsets, int G, int P,
                 const int64_t *rows, int64_t n_rows, float *y, int n_threads) {
  if (orc_check_seg(mode, n_seg, offsets, G, N, K)) return -1;
  if (P != 1 && P != 2) return -1;
  int S = (mode == ORC_MODE_INPUT) ? n_seg : 1;
  if (rows == NULL) n_rows = M;
  float *acc = (float *)malloc(sizeof(float) * (size_t)S * P * n_rows * N);
  if (!acc) return -2;
  int rc = orc_gemm_fp8_acc(planes, wq, M, N, K, mode, n_seg, offsets, G, P, rows, n_rows,
                            acc, n_threads);
  if (rc) {
    free(acc);
    return rc;
  }
  for (int64_t r = 0; r < n_rows; ++r)
    for (int64_t n = 0; n < N; ++n) {
      int g = (mode == ORC_MODE_OUTPUT && G > 1) ? orc_seg_index(offsets, n_seg, n) : 0;
      float yv = 0.0f;
      for (int i = 0; i < S; ++i) {
        float sw = s_w[(int64_t)i * N + n];
        float cp = sw * s_act[((int64_t)g * S + i) * 2 + 0];
        float cm = sw * s_act[((int64_t)g * S + i) * 2 + 1];
        yv = fmaf(cp, acc[(((int64_t)i * P + 0) * n_rows + r) * N + n], yv);
        if (P == 2) yv = fmaf(cm, acc[(((int64_t)i * P + 1) * n_rows + r) * N + n], yv);
      }
      if (bias) yv = yv + orc_bf16(bias[n]);
      y[r * N + n] = yv;
    }
  free(acc);
  return 0;
}


/* ------------------------------------------------------------------------
 * FFN activation between the two linears (the input of fc2 is GELU of fc1's
 * output; "SegQuant" papernotes.org, section DualScale, polarity table row
 * "FFN (DiT)"), for the fused producer.  The pages name the activation but
 * give no formula; the models' FFNs use the tanh approximation
 *   gelu(x) = x/2 * (1 + tanh(sqrt(2/pi) * (x + 0.044715 x^3))).
 * It is written out here as a fixed sequence of fp32 operations, each rounded
 * once (this file is built with -ffp-contract=off), so that a GPU running the
 * same sequence gets the same bits:
 *   tanh(u) = 1 - 2 / (e^(2|u|) + 1), sign of u; 1 for |u| >= 9 (the fp32
 *             value of tanh there is 1);
 *   e^z     (0 <= z <= 18): z = n ln2 + f with n = rint(z / ln2), |f| <= ln2/2
 *             (Cody and Waite's reduction, ln2 split into a head exact in
 *             n * head and a tail), e^f by its Taylor series to degree 7
 *             (remainder below 2^-27), times 2^n (exact).
 * The values are rounded to bf16 before and after (the models' activation
 * type), round half to even.
 * ------------------------------------------------------------------------ */
static uint16_t orc_bf16_rne(float v) {
  uint32_t u;
  memcpy(&u, &v, sizeof u);
  if ((u & 0x7fffffffu) > 0x7f800000u) return (uint16_t)((u >> 16) | 0x40u);  /* NaN stays NaN */
  u += 0x7fffu + ((u >> 16) & 1u);
  return (uint16_t)(u >> 16);
}

static float orc_exp_0_18(float z) {
  const float inv_ln2 = 0x1.715476p+0f;   /* fp32(1/ln 2) */
  const float ln2_hi = 0x1.62e4p-1f;      /* 17 significant bits: n * ln2_hi is exact */
  const float ln2_lo = 0x1.7f7d1cp-20f;   /* fp32(ln 2 - ln2_hi) */
  const float n = rintf(z * inv_ln2);
  float f = fmaf(-n, ln2_hi, z);
  f = fmaf(-n, ln2_lo, f);
  float p = 0x1.a01a02p-13f;              /* 1/7! */
  p = fmaf(p, f, 0x1.6c16c2p-10f);        /* 1/6! */
  p = fmaf(p, f, 0x1.111112p-7f);         /* 1/5! */
  p = fmaf(p, f, 0x1.555556p-5f);         /* 1/4! */
  p = fmaf(p, f, 0x1.555556p-3f);         /* 1/3! */
  p = fmaf(p, f, 0.5f);
  p = fmaf(p, f, 1.0f);
  p = fmaf(p, f, 1.0f);
  return p * ldexpf(1.0f, (int)n);
}

static float orc_tanh(float u) {
  const float a = fabsf(u);
  float t = 1.0f;
  if (a < 9.0f) {
    const float e = orc_exp_0_18(2.0f * a);
    t = 1.0f - 2.0f / (e + 1.0f);
  }
  return u < 0.0f ? -t : t;
}

static float orc_gelu_tanh(float x) {
  const float k0 = 0x1.988454p-1f;   /* fp32(sqrt(2/pi)) */
  const float k1 = 0x1.6e4e26p-5f;   /* fp32(0.044715) */
  const float x3 = (x * x) * x;
  const float u = k0 * fmaf(k1, x3, x);
  const float t = orc_tanh(u);
  return (0.5f * x) * (1.0f + t);
}

/* bf16(gelu(bf16(y))) for n fp32 values, as bf16 bit patterns. */
int orc_gelu_bf16(const float *y, int64_t n, uint16_t *out) {
  if (n < 0 || (n > 0 && (y == NULL || out == NULL))) return -1;
  for (int64_t i = 0; i < n; ++i) out[i] = orc_bf16_rne(orc_gelu_tanh(orc_bf16(orc_bf16_rne(y[i]))));
  return 0;
}

/* The pieces, for the pins: bf16 rounding, e^z on [0, 18], tanh and gelu. */
int orc_gelu_parts(const float *x, int64_t n, float *exp_out, float *tanh_out, float *gelu_out,
                   uint16_t *bf16_out) {
  for (int64_t i = 0; i < n; ++i) {
    if (exp_out) exp_out[i] = orc_exp_0_18(x[i]);
    if (tanh_out) tanh_out[i] = orc_tanh(x[i]);
    if (gelu_out) gelu_out[i] = orc_gelu_tanh(x[i]);
    if (bf16_out) bf16_out[i] = orc_bf16_rne(x[i]);
  }
  return 0;
}
