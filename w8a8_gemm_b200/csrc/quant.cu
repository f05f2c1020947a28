// quant.cu -- the element-wise, HBM-bound kernels of the SegQuant path:
//  * DualScale activation quantization (Q_dual on X / d, two int8 planes per
//    activation group) -- "SegQuant" author page, section 3; papernotes.org
//    "SegQuant", section DualScale;
//  * static AMax calibration of s+ / s- (same section; AMax calibrator);
//  * segment-wise symmetric AMax weight quantization (section SegLinear).
// Every fp32 operation that decides an integer code is written with an explicit
// round-to-nearest intrinsic so that no contraction or approximation changes it.
#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <type_traits>

#include "sm100.cuh"
#include "sq_internal.h"

namespace sq {
namespace {

constexpr int kColsPerThread = 8;                     // one 16-byte bf16 load
constexpr int kWarpCols = 32 * kColsPerThread;        // 256 channels per warp row
constexpr int kRowsPerBlock = 8;                      // warps per block
constexpr int kQRows = 32;                            // rows per staged tile
constexpr int kQStages = 4;                           // tiles in flight per block
constexpr int kQTileBytes = kQRows * kWarpCols * 2;   // 16 KB of bf16
constexpr int kFixMax = 16;                           // channels a column block may patch
constexpr int kFixOffset = kQStages * kQTileBytes + 64;  // the warps' lists, after the barriers
constexpr uint64_t kQuantWaitNs = 2000000000ull;      // bounded wait on a tile: 2 s

__device__ __forceinline__ float bf16_bits_to_f32(uint32_t h) {
  return __uint_as_float(h << 16);
}

__device__ __forceinline__ void unpack8(const uint4 &v, float (&x)[8]) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    x[2 * j] = bf16_bits_to_f32(w[j] & 0xFFFFu);
    x[2 * j + 1] = bf16_bits_to_f32(w[j] >> 16);
  }
}

// ------------------------------------------------------------- calibration
// Pass 1: per-thread max of u = x / d and of -u over its rows, combined across
// the lanes of one K-segment, then atomicMax into s_act, which holds the raw
// maxima until pass 2 (non-negative floats order like their bit patterns).
__global__ void __launch_bounds__(256) calib_reduce_kernel(const uint16_t *__restrict__ x,
                                                           int64_t M, int64_t K, int64_t ldx,
                                                           const float *__restrict__ d,
                                                           SegParams seg, float *s_act,
                                                           int *status) {
  const int g = blockIdx.z;
  const int64_t c0 = (static_cast<int64_t>(blockIdx.x) * 32 + threadIdx.x) * kColsPerThread;
  if (c0 >= K) return;
  const int i = (seg.mode == SQ_SEG_INPUT) ? seg_index(seg.off, seg.n_seg, c0) : 0;
  float dv[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) dv[j] = d ? d[g * K + c0 + j] : 1.0f;
  float hi = 0.0f, nlo = 0.0f;
  for (int64_t r = static_cast<int64_t>(blockIdx.y) * kRowsPerBlock + threadIdx.y; r < M;
       r += static_cast<int64_t>(gridDim.y) * kRowsPerBlock) {
    const uint4 v = *reinterpret_cast<const uint4 *>(x + r * ldx + c0);
    float xv[8];
    unpack8(v, xv);
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const float u = d ? __fdiv_rn(xv[j], dv[j]) : xv[j];
      if (u > hi) hi = u;      // NaN compares false and is ignored
      if (-u > nlo) nlo = -u;
    }
  }
  // Lanes of one K-segment combine their maxima first; the lowest lane of
  // each segment group then issues the two atomics.
  const unsigned group = __match_any_sync(__activemask(), i);
  const unsigned hib = __reduce_max_sync(group, __float_as_uint(hi));
  const unsigned nlob = __reduce_max_sync(group, __float_as_uint(nlo));
  if ((threadIdx.x & 31) == __ffs(group) - 1 &&
      store_ok(status, g < seg.G && i < seg.S)) {  // s_act: [G][S][2]
    unsigned int *slot = reinterpret_cast<unsigned int *>(s_act + (g * seg.S + i) * 2);
    if (hib) atomicMax(slot, hib);
    if (nlob) atomicMax(slot + 1, nlob);
  }
}

// Pass 2: s+ = max / 127, s- = |min| / 128; an empty side gets step 1.  In
// single-scale mode both take max(max, |min|) / 127.  FP8 (E4M3): both
// divisors are 448.
__global__ void calib_finalize_kernel(float *s_act, int n, int single, int fp8, int *status) {
  const float qp = fp8 ? 448.0f : 127.0f, qm = fp8 ? 448.0f : 128.0f;
  for (int t = threadIdx.x; t < n; t += blockDim.x) {
    if (!store_ok(status, 2 * t + 1 < 2 * n)) continue;
    const float hi = s_act[2 * t], nlo = s_act[2 * t + 1];
    if (single) {
      const float amax = hi > nlo ? hi : nlo;
      const float s = amax > 0.0f ? __fdiv_rn(amax, qp) : 1.0f;
      s_act[2 * t] = s;
      s_act[2 * t + 1] = s;
    } else {
      s_act[2 * t] = hi > 0.0f ? __fdiv_rn(hi, qp) : 1.0f;
      s_act[2 * t + 1] = nlo > 0.0f ? __fdiv_rn(nlo, qm) : 1.0f;
    }
  }
}

// ---------------------------------------------------- activation quantize
// The codes are round(u / s) with u = fl(x / d) and the quotients rounded to
// fp32 first (IEEE division), then to an integer (half to even).  A quotient
// a / b is formed without a divide: with r = fl(1/b), q0 = fl(a r) is within
// an ulp of a / b, the residual a - q0 b is exact in one FMA, and
// fl(q0 + (a - q0 b) r) is the correctly rounded quotient (Markstein's
// correction, "Computation of elementary functions on the IBM RISC System/6000
// processor", IBM J. Res. Dev. 34(1), 1990).  The identity holds for every
// bf16 dividend and every fp32 divisor significand (checked exhaustively on
// the CPU) and for fp32 dividends (sampled); it needs dividend, divisor and
// residual away from the ends of the fp32 range, hence the bounds on d and s
// in the library's header.

// sat(a * b) clamped to [0, 1]; NaN gives +0.
__device__ __forceinline__ float mul_sat(float a, float b) {
  float r;
  asm("fma.rn.sat.f32 %0, %1, %2, 0f00000000;" : "=f"(r) : "f"(a), "f"(b));
  return r;
}
__device__ __forceinline__ float fma_sat(float a, float b, float c) {
  float r;
  asm("fma.rn.sat.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}
__device__ __forceinline__ uint64_t pack2(float a, float b) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
  return r;
}
__device__ __forceinline__ void unpack2(uint64_t v, float &a, float &b) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(a), "=f"(b) : "l"(v));
}
__device__ __forceinline__ uint64_t ffma2(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ uint64_t fmul2(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
// min / max that keep a NaN operand (the plain forms return the other one)
__device__ __forceinline__ float min_nan(float a, float b) {
  float r;
  asm("min.NaN.f32 %0, %1, %2;" : "=f"(r) : "f"(a), "f"(b));
  return r;
}
__device__ __forceinline__ float max_nan(float a, float b) {
  float r;
  asm("max.NaN.f32 %0, %1, %2;" : "=f"(r) : "f"(a), "f"(b));
  return r;
}

// Lowers every byte equal to 128 to 127 in a word of + codes (bytes 0 .. 128):
// bit 7 of a byte moved to its bit 0 and subtracted, with no borrow between
// bytes.
__device__ __forceinline__ uint32_t cap127(uint32_t w) { return w - ((w >> 7) & 0x01010101u); }

// Packs the low bytes of four words into one word (byte j = low byte of word j).
__device__ __forceinline__ uint32_t pack4_lo(uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  return __byte_perm(__byte_perm(a, b, 0x0040), __byte_perm(c, d, 0x0040), 0x5410);
}

// Bit patterns of fl(1.5 * 2^23 + k * u0) and fl(1.5 * 2^23 + k * u1), one packed
// FMA (f32x2) for both; the low byte of each is rne(k * u) for |k u| <= 128.
__device__ __forceinline__ void round2(float u0, float u1, float k, uint32_t &r0, uint32_t &r1) {
  const uint64_t d = ffma2(pack2(u0, u1), pack2(k, k), pack2(12582912.0f, 12582912.0f));
  asm("mov.b64 {%0, %1}, %2;" : "=r"(r0), "=r"(r1) : "l"(d));
}

// Per-thread constants of the current (group, column block): the thread's
// eight channels share one K-segment (segment widths are multiples of 32), so
// one step pair serves them all; the divisors are per channel.
//   int8: r7p = fl(1/s+)/128, m128p = -128 s+; r7m = -fl(1/s-)/128, m128m = 128 s-
//   FP8:  r7p = fl(1/s+), m128p = -s+, lim_p = 1024 s+; the same with s-.
//   nd = -d, rd = fl(1/d), ld = the overflow clamp min(FLT_MAX/2 * d, FLT_MAX)
//   (HAS_D only).
struct StepConsts {
  float r7p, m128p, r7m, m128m, lim_p, lim_m;
  float nd[8], rd[8], ld[8];
};

// u = fl(x / d) for eight channels (HAS_D), Markstein's correction in packed
// FMAs.  x is first clamped to +-min(FLT_MAX/2 * d, FLT_MAX) so that no step
// overflows (the clamp keeps NaN; a clamped value's code saturates, like the
// value's own).
__device__ __forceinline__ void smooth8(float (&x)[8], const StepConsts &k) {
#pragma unroll
  for (int j = 0; j < 8; j += 2) {
    const float x0 = max_nan(min_nan(x[j], k.ld[j]), -k.ld[j]);
    const float x1 = max_nan(min_nan(x[j + 1], k.ld[j + 1]), -k.ld[j + 1]);
    const uint64_t xx = pack2(x0, x1), rd = pack2(k.rd[j], k.rd[j + 1]);
    const uint64_t q0 = fmul2(xx, rd);
    const uint64_t e = ffma2(q0, pack2(k.nd[j], k.nd[j + 1]), xx);  // x - q0 d, exact
    unpack2(ffma2(e, rd, q0), x[j], x[j + 1]);
  }
}

// u = RN(x fl(1/d)) for eight channels, without the correction and the clamp:
// for channels whose codes a quantize plan shows to be the same as with both
// corrections (an overflowing product saturates its code like the clamped
// quotient, and NaN stays NaN).
__device__ __forceinline__ void scale8(float (&x)[8], const StepConsts &k) {
#pragma unroll
  for (int j = 0; j < 8; j += 2)
    unpack2(fmul2(pack2(x[j], x[j + 1]), pack2(k.rd[j], k.rd[j + 1])), x[j], x[j + 1]);
}

// sat(fl(u / s) / 128) for two channels of one polarity, everything scaled by
// 2^-7 (exact) so that .sat clamps to the code range: q0 = sat(u fl(1/s)/128)
// (x on the other side of zero, NaN and overflow all clamp), the residual
// u - q0 * 128 s in one packed FMA, then v = sat(q0 + e fl(1/s)/128).  For the
// - plane r7 and the residual's factor carry the other sign, so that v is
// sat(fl(-u / s-) / 128) for u < 0 and 0 otherwise.
__device__ __forceinline__ void quot2_sat(float u0, float u1, float r7, float m128, float &v0,
                                          float &v1) {
  const float a0 = mul_sat(u0, r7), a1 = mul_sat(u1, r7);
  float e0, e1;
  unpack2(ffma2(pack2(a0, a1), pack2(m128, m128), pack2(u0, u1)), e0, e1);
  v0 = fma_sat(e0, r7, a0);
  v1 = fma_sat(e1, r7, a1);
}

// Eight channels u of one row -> X^+ and X^- codes, 8 bytes each:
//   q+ = rne(128 v+), v+ = sat(fl(u / s+) / 128): the FP add of 1.5 * 2^23
//        rounds to nearest even and the code is the low byte of the sum's
//        bits; 128 is then lowered to 127 (cap127, four codes at a time);
//   q- = -rne(128 v-), v- = sat(fl(-u / s-) / 128), codes in [-128, 0].
// This is the case-wise Q_dual with the reference's clamps: u >= 0 (including
// -0.0) gives a code in [0, 127] and none in X^-, u < 0 the reverse, NaN 0.
__device__ __forceinline__ void dualscale8(const float (&u)[8], const StepConsts &k,
                                           uint2 &plus, uint2 &minus) {
  uint32_t qp[8], qm[8];
#pragma unroll
  for (int j = 0; j < 8; j += 2) {
    float vp0, vp1, vm0, vm1;
    quot2_sat(u[j], u[j + 1], k.r7p, k.m128p, vp0, vp1);
    quot2_sat(u[j], u[j + 1], k.r7m, k.m128m, vm0, vm1);
    round2(vp0, vp1, 128.0f, qp[j], qp[j + 1]);
    round2(vm0, vm1, -128.0f, qm[j], qm[j + 1]);
  }
  plus = make_uint2(cap127(pack4_lo(qp[0], qp[1], qp[2], qp[3])),
                    cap127(pack4_lo(qp[4], qp[5], qp[6], qp[7])));
  minus = make_uint2(pack4_lo(qm[0], qm[1], qm[2], qm[3]), pack4_lo(qm[4], qm[5], qm[6], qm[7]));
}

// The same codes without the quotient's correction, for step pairs where that
// provably changes none: q+ = rne(128 sat(RN(u fl(1/s+)) / 128)), and q- the
// same with s-.  RN(u fl(1/s)) and fl(u / s) both lie within 2^-23 relative of
// u / s, so their integer roundings can differ only for u next to a rounding
// boundary (h + 1/2) s, h = 0 .. 127; correction_changes_a_code() tests
// exactly those inputs (for every step pair of a column block) before a block
// uses this form.  NaN, overflow
// and the other polarity saturate as in dualscale8.
__device__ __forceinline__ void dualscale8_fast(const float (&u)[8], const StepConsts &k,
                                                uint2 &plus, uint2 &minus) {
  uint32_t qp[8], qm[8];
#pragma unroll
  for (int j = 0; j < 8; j += 2) {
    round2(mul_sat(u[j], k.r7p), mul_sat(u[j + 1], k.r7p), 128.0f, qp[j], qp[j + 1]);
    round2(mul_sat(u[j], k.r7m), mul_sat(u[j + 1], k.r7m), -128.0f, qm[j], qm[j + 1]);
  }
  plus = make_uint2(cap127(pack4_lo(qp[0], qp[1], qp[2], qp[3])),
                    cap127(pack4_lo(qp[4], qp[5], qp[6], qp[7])));
  minus = make_uint2(pack4_lo(qm[0], qm[1], qm[2], qm[3]), pack4_lo(qm[4], qm[5], qm[6], qm[7]));
}

// This thread's share of the test whether dualscale8_fast gives dualscale8's
// codes for every bf16 input at the step pair of `k` (int8 codes, no
// divisor); returns true if one of its inputs differs, and the block combines
// the threads' answers.  The two roundings of u / s are within
// 2^-23 relative of it, so a difference needs a boundary b = h + 1/2 within
// 2^-23 relative of u / s, i.e. u within that distance of b s.  bf16 values
// are 2^-8 relative apart, so such a u is a bf16 neighbour of fl(b s) (itself
// within 2^-24 of b s): the candidates are fl(b s) truncated to bf16 and the
// bf16 values just below and above it, for b = 1/2 .. 127 + 1/2 and both
// polarities (768 inputs).  Beyond 127.5 both forms saturate alike.
__device__ bool correction_changes_a_code(const StepConsts &k, float s_plus, float s_minus) {
  int bad = 0;
  for (int j = threadIdx.x; j < 768; j += blockDim.x) {
    const int pol = j / 384, rem = j - pol * 384;
    const float b = static_cast<float>(rem / 3) + 0.5f;
    const uint32_t t = __float_as_uint(__fmul_rn(b, pol ? s_minus : s_plus)) & 0xFFFF0000u;
    const float x = __uint_as_float(t + static_cast<uint32_t>(rem % 3 - 1) * 0x10000u);
    // One element of dualscale8 and of dualscale8_fast, on the candidate's
    // own plane (the other plane's code is 0 in both forms).
    const float u = pol ? -x : x;
    const float r7 = pol ? k.r7m : k.r7p, m128 = pol ? k.m128m : k.m128p;
    const float scale = pol ? -128.0f : 128.0f;
    const float a = mul_sat(u, r7);
    const float v = fma_sat(__fmaf_rn(a, m128, u), r7, a);
    uint32_t q_exact = __float_as_uint(__fmaf_rn(v, scale, 12582912.0f)) & 0xFFu;
    uint32_t q_fast = __float_as_uint(__fmaf_rn(a, scale, 12582912.0f)) & 0xFFu;
    if (!pol) {  // the + plane's codes are lowered to 127
      q_exact = min(q_exact, 127u);
      q_fast = min(q_fast, 127u);
    }
    bad |= q_exact != q_fast;
  }
  return bad != 0;
}

// FP8 (E4M3) codes of eight channels: v = fl(u / s) by the same correction
// (unscaled), code = e4m3(v), round half to even with saturation to +-448 (the
// CUDA conversion intrinsics).  u is clamped to 1024 s on its own side first
// (beyond that the code saturates anyway), which keeps every step finite.
// x >= 0 (-0.0 included) fills the + plane, x < 0 the - plane, NaN neither;
// the branch that does not apply converts +0.0, whose code is 0x00.  The
// quotient takes the sign of x, which the correction loses for x = -0.0.
__device__ __forceinline__ uint32_t e4m3x4(float a, float b, float c, float d) {
  const uint32_t lo = __nv_cvt_float2_to_fp8x2(make_float2(a, b), __NV_SATFINITE, __NV_E4M3);
  const uint32_t hi = __nv_cvt_float2_to_fp8x2(make_float2(c, d), __NV_SATFINITE, __NV_E4M3);
  return lo | (hi << 16);
}

__device__ __forceinline__ float quot_fp8(float u, float x, float r, float ms) {
  const float q0 = __fmul_rn(u, r);
  const float v = __fmaf_rn(__fmaf_rn(q0, ms, u), r, q0);
  return __int_as_float(__float_as_int(v) | (__float_as_int(x) & 0x80000000));
}

__device__ __forceinline__ void dualscale8_fp8(const float (&x)[8], const float (&u)[8],
                                               const StepConsts &k, uint2 &plus, uint2 &minus) {
  float vp[8], vm[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    vp[j] = x[j] >= 0.0f ? quot_fp8(min_nan(u[j], k.lim_p), x[j], k.r7p, k.m128p) : 0.0f;
    vm[j] = x[j] < 0.0f ? quot_fp8(max_nan(u[j], -k.lim_m), x[j], k.r7m, k.m128m) : 0.0f;
  }
  plus = make_uint2(e4m3x4(vp[0], vp[1], vp[2], vp[3]), e4m3x4(vp[4], vp[5], vp[6], vp[7]));
  minus = make_uint2(e4m3x4(vm[0], vm[1], vm[2], vm[3]), e4m3x4(vm[4], vm[5], vm[6], vm[7]));
}

// Work unit = one activation group g and one tile of 32 rows x 256 channels.
// Units are numbered group-major, then column block, then row tile, and every
// block takes one contiguous range of them: the grid is balanced to within one
// unit, and a block changes (group, column block) -- and recomputes its
// constants (StepConsts) -- at most a few times.  With G > 1 every group
// re-reads the same X tiles, which stay resident in L2 between the passes.
// Thread 0 keeps kQStages tiles in flight with 2D TMA copies into shared
// memory; every warp then takes whole rows of the staged tile (lane = 8
// channels, one conflict-free 16-byte shared load) and writes 8 bytes per plane
// per row, 256 contiguous bytes per warp.
// fetch_scales reads the inputs of one (group, column block) into registers
// (s+, s- in sc[0..1], the eight divisors in dv) and fold_consts turns them
// into StepConsts, so that the reads can be issued ahead of the first tile
// copies.
template <bool HAS_D>
__device__ __forceinline__ void fetch_scales(int g, int64_t c0, int64_t K, const float *d,
                                             const float *s_act, const SegParams &seg,
                                             float (&sc)[2], float (&dv)[8]) {
  if (c0 >= K) return;
  const int i = (seg.mode == SQ_SEG_INPUT) ? seg_index(seg.off, seg.n_seg, c0) : 0;
  sc[0] = s_act[(g * seg.S + i) * 2 + 0];
  sc[1] = s_act[(g * seg.S + i) * 2 + 1];
  if constexpr (HAS_D) {
#pragma unroll
    for (int j = 0; j < 8; ++j) dv[j] = d[g * K + c0 + j];
  }
}
// The quantize plan's bits for one thread's eight channels c0 .. c0 + 7 of
// group g (0xFF when all may skip the corrections; channels past K count as
// set; 0 without a plan), read beside the scales for the same reason.
__device__ __forceinline__ uint32_t plan_bits8(const uint32_t *plan, int g, int64_t c0,
                                               int64_t K) {
  if (plan == nullptr) return 0u;
  if (c0 >= K) return 0xFFu;
  const int64_t words = (K + 31) / 32;
  return (plan[g * words + c0 / 32] >> (c0 & 31)) & 0xFFu;
}
template <bool FP8, bool HAS_D>
__device__ __forceinline__ void fold_consts(int64_t c0, int64_t K, const float (&sc)[2],
                                            const float (&dv)[8], StepConsts &k) {
  if (c0 >= K) return;
  const float rp = __frcp_rn(sc[0]), rm = __frcp_rn(sc[1]);
  if constexpr (FP8) {
    k.r7p = rp;
    k.m128p = -sc[0];
    k.r7m = rm;
    k.m128m = -sc[1];
    k.lim_p = 1024.0f * sc[0];
    k.lim_m = 1024.0f * sc[1];
  } else {
    k.r7p = rp * 0.0078125f;
    k.m128p = -128.0f * sc[0];
    k.r7m = rm * -0.0078125f;
    k.m128m = 128.0f * sc[1];
  }
  if constexpr (HAS_D) {
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      k.nd[j] = -dv[j];
      k.rd[j] = __frcp_rn(dv[j]);
      // min(FLT_MAX / 2 * d, FLT_MAX): no overflow in x fl(1/d), +-inf clamped
      k.ld[j] = fminf(__fmul_rn(1.7014117e38f, dv[j]), 3.4028235e38f);
    }
  }
}

// Position of a work unit: group, column block, row tile (row tiles vary fastest).
struct UnitCursor {
  int g, cb, rt;
  __device__ void set(int64_t u, int n_cb, int n_rt) {
    const int64_t per_group = static_cast<int64_t>(n_cb) * n_rt;
    g = static_cast<int>(u / per_group);
    const int64_t rem = u - g * per_group;
    cb = static_cast<int>(rem / n_rt);
    rt = static_cast<int>(rem - static_cast<int64_t>(cb) * n_rt);
  }
  __device__ void next(int n_cb, int n_rt) {
    if (++rt == n_rt) {
      rt = 0;
      if (++cb == n_cb) {
        cb = 0;
        ++g;
      }
    }
  }
};

// With divisors and a quantize plan, a column block whose plan leaves out a
// few channels still takes the uncorrected codes, and each warp then rewrites
// the codes of those channels in its rows with the exact form (patch_codes).
// build_fix_list puts the left-out channels of this thread's column block --
// enumerated by bit of the lanes' eight plan bits, then by lane -- with their
// constants (folded exactly as fold_consts does) into the warp's list: entry i
// = {channel offset in the block, fl(1/d), -d, the clamp} and {r7p, m128p,
// r7m, m128m}.  Returns the number of channels, which exceeds kFixMax (and
// leaves the list unused) when there are more than the list holds.
__device__ __noinline__ int build_fix_list(uint32_t pbits, const float (&sc)[2], const float (&dv)[8],
                              int lane, float4 *list) {
  const uint32_t out = ~pbits & 0xFFu;
  int total = 0, my_bit = 0, my_src = 0;
  for (int b = 0; b < 8; ++b) {
    const uint32_t m = __ballot_sync(0xFFFFFFFFu, (out >> b) & 1u);
    const int n = __popc(m);
    if (lane >= total && lane < total + n) {
      uint32_t mm = m;
      for (int i = 0; i < lane - total; ++i) mm &= mm - 1;  // drop the lower set bits
      my_bit = b;
      my_src = __ffs(mm) - 1;
    }
    total += n;
  }
  if (total > kFixMax) return total;
  const float s2[2] = {__shfl_sync(0xFFFFFFFFu, sc[0], my_src),
                       __shfl_sync(0xFFFFFFFFu, sc[1], my_src)};
  float d1 = 1.0f;
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const float t = __shfl_sync(0xFFFFFFFFu, dv[j], my_src);
    if (j == my_bit) d1 = t;
  }
  if (lane < total) {
    float d8[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) d8[j] = d1;
    StepConsts k;
    fold_consts<false, true>(0, 1, s2, d8, k);
    list[2 * lane] = make_float4(__int_as_float(my_src * kColsPerThread + my_bit), k.rd[0],
                                 k.nd[0], k.ld[0]);
    list[2 * lane + 1] = make_float4(k.r7p, k.m128p, k.r7m, k.m128m);
  }
  __syncwarp();
  return total;
}

// The exact codes (smooth8, then dualscale8, on one element) of the listed
// channels in this warp's rows of the staged tile (rows warp, warp + 8, ...),
// written over the uncorrected ones.  blk = the group's first plane at the
// column block's first channel c_blk.
template <bool P2>
__device__ __noinline__ void patch_codes(const uint16_t *tile, const float4 *list, int nfix, int warp,
                            int lane, int rows_here, int64_t r_base, int8_t *blk,
                            int8_t *planes, int64_t plane_stride, int64_t K, int64_t c_blk,
                            const SegParams &seg, int *status) {
  const int n_rows = (rows_here - warp + 7) / 8;
  for (int e = lane; e < n_rows * nfix; e += 32) {
    const int t = e / nfix, f = e - t * nfix;
    const int rr = warp + 8 * t;
    const float4 a = list[2 * f], b = list[2 * f + 1];
    const int co = __float_as_int(a.x);
    const float x = __uint_as_float(static_cast<uint32_t>(tile[rr * kWarpCols + co]) << 16);
    const float xc = max_nan(min_nan(x, a.w), -a.w);
    const float q0 = __fmul_rn(xc, a.y);
    const float u = __fmaf_rn(__fmaf_rn(q0, a.z, xc), a.y, q0);
    const float ap = mul_sat(u, b.x), am = mul_sat(u, b.z);
    const float vp = fma_sat(__fmaf_rn(ap, b.y, u), b.x, ap);
    const float vm = fma_sat(__fmaf_rn(am, b.w, u), b.z, am);
    const uint32_t qp = min(__float_as_uint(__fmaf_rn(vp, 128.0f, 12582912.0f)) & 0xFFu, 127u);
    const uint32_t qm = __float_as_uint(__fmaf_rn(vm, -128.0f, 12582912.0f)) & 0xFFu;
    const int64_t r = r_base + rr;
    const int64_t at = (blk - planes) + r * K + co;
    if (!store_ok(status, at >= 0 && c_blk + co < K &&
                              at + (P2 ? plane_stride : 0) <
                                  static_cast<int64_t>(seg.G) * seg.P * plane_stride))
      continue;
    if constexpr (P2) {
      blk[r * K + co] = static_cast<int8_t>(qp);
      blk[plane_stride + r * K + co] = static_cast<int8_t>(qm);
    } else {
      blk[r * K + co] = static_cast<int8_t>(qp | qm);
    }
  }
}

template <bool FP8, bool HAS_D>
__global__ void __launch_bounds__(256, 3) quant_act_kernel(const __grid_constant__ CUtensorMap tmX,
                                                           int64_t M, int64_t K,
                                                           const float *__restrict__ d,
                                                           const float *__restrict__ s_act,
                                                           SegParams seg,
                                                           int8_t *__restrict__ planes,
                                                           const uint32_t *__restrict__ plan,
                                                           int *status) {
  extern __shared__ __align__(128) uint8_t qsmem[];
  uint64_t *full = reinterpret_cast<uint64_t *>(qsmem + kQStages * kQTileBytes);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int n_rt = static_cast<int>((M + kQRows - 1) / kQRows);      // row tiles
  const int n_cb = static_cast<int>((K + kWarpCols - 1) / kWarpCols);  // column blocks
  const int64_t n_units = static_cast<int64_t>(n_rt) * n_cb * seg.G;
  const int64_t u_begin = n_units * blockIdx.x / gridDim.x;
  const int64_t u_end = n_units * (blockIdx.x + 1) / gridDim.x;
  const int n_mine = static_cast<int>(u_end - u_begin);

  UnitCursor fetch;  // next unit to bring in (thread 0 only)
  if (tid == 0) {
    for (int st = 0; st < kQStages; ++st) mbar_init(&full[st], 1);
    fence_mbar_init();
    prefetch_tmap(&tmX);
  }
  grid_dependency_wait();  // nothing above touches global memory
  // The first unit's scales are requested before the tile copies, so that
  // these small reads do not queue behind the whole grid's tile traffic.
  UnitCursor cur;
  cur.set(u_begin, n_cb, n_rt);
  float sc[2] = {1.0f, 1.0f}, dv[8] = {1.0f, 1.0f, 1.0f, 1.0f, 1.0f, 1.0f, 1.0f, 1.0f};
  StepConsts kc;
  uint32_t pbits = 0;  // plan bits of this thread's channels (with divisors)
  int nfix = 0;        // channels the current column block patches
  float4 *fix_list = reinterpret_cast<float4 *>(qsmem + kFixOffset) + warp * 2 * kFixMax;
  if (n_mine > 0) {
    const int64_t c0 = static_cast<int64_t>(cur.cb) * kWarpCols + lane * kColsPerThread;
    fetch_scales<HAS_D>(cur.g, c0, K, d, s_act, seg, sc, dv);
    if constexpr (HAS_D && !FP8) pbits = plan_bits8(plan, cur.g, c0, K);
  }
  if (tid == 0) {
    fetch.set(u_begin, n_cb, n_rt);
    for (int st = 0; st < kQStages && st < n_mine; ++st) {
      mbar_arrive_expect_tx(&full[st], kQTileBytes);
      tma_load_2d(qsmem + st * kQTileBytes, &tmX, &full[st], fetch.cb * kWarpCols,
                  fetch.rt * kQRows);
      fetch.next(n_cb, n_rt);
    }
  }
  __syncthreads();  // barriers initialised
  if (n_mine > 0)
    fold_consts<FP8, HAS_D>(static_cast<int64_t>(cur.cb) * kWarpCols + lane * kColsPerThread, K,
                            sc, dv, kc);
  // Whether the block's current (group, column block) may take the codes
  // without the quotients' corrections (block-uniform), for int8 codes:
  // without a divisor, when the block-wide test passed for the step pair of
  // every K-segment that meets the column block; with divisors, when a
  // quantize plan is given and leaves out at most kFixMax of the 256 channels
  // (each warp sees the same 256 and lists them for patch_codes).
  const auto correction_free = [&](int g, int cb) -> bool {
    if constexpr (FP8) {
      return false;
    } else if constexpr (HAS_D) {
      if (plan == nullptr) return false;
      nfix = build_fix_list(pbits, sc, dv, lane, fix_list);
      return nfix <= kFixMax;
    } else {
      const int64_t first = static_cast<int64_t>(cb) * kWarpCols;
      const int64_t last = (first + kWarpCols < K ? first + kWarpCols : K) - 1;
      int i0 = 0, i1 = 0;
      if (seg.mode == SQ_SEG_INPUT) {
        i0 = seg_index(seg.off, seg.n_seg, first);
        i1 = seg_index(seg.off, seg.n_seg, last);
      }
      bool bad = false;
      for (int i = i0; i <= i1; ++i) {
        const float pair[2] = {s_act[(g * seg.S + i) * 2 + 0], s_act[(g * seg.S + i) * 2 + 1]};
        StepConsts k;
        fold_consts<false, false>(0, 1, pair, dv, k);
        bad |= correction_changes_a_code(k, pair[0], pair[1]);
      }
      return __syncthreads_or(bad) == 0;
    }
  };
  bool fast = n_mine > 0 ? correction_free(cur.g, cur.cb) : false;
  int key_g = cur.g, key_cb = cur.cb;  // (group, column block) of the constants held
  const int64_t plane_stride = M * K;
  for (int it = 0; it < n_mine; ++it, cur.next(n_cb, n_rt)) {
    const int64_t c0 = static_cast<int64_t>(cur.cb) * kWarpCols + lane * kColsPerThread;
    if (cur.g != key_g || cur.cb != key_cb) {
      key_g = cur.g;
      key_cb = cur.cb;
      fetch_scales<HAS_D>(cur.g, c0, K, d, s_act, seg, sc, dv);
      if constexpr (HAS_D && !FP8) pbits = plan_bits8(plan, cur.g, c0, K);
      fold_consts<FP8, HAS_D>(c0, K, sc, dv, kc);
      fast = correction_free(cur.g, cur.cb);
    }
    const int st = it % kQStages;
    if (!mbar_wait(&full[st], (it / kQStages) & 1, kQuantWaitNs)) {
      atomicExch(status, static_cast<int>(SQ_ERR_DEVICE_TIMEOUT));
      return;
    }
    const uint16_t *tile = reinterpret_cast<const uint16_t *>(qsmem + st * kQTileBytes);
    const int64_t r_base = static_cast<int64_t>(cur.rt) * kQRows;
    const int rows_here = static_cast<int>(M - r_base < kQRows ? M - r_base : kQRows);
    const auto rows = [&](auto fast_form, auto two_planes) {
      // (the uncorrected codes exist for int8 codes only)
      constexpr bool FAST = decltype(fast_form)::value && !FP8;
      constexpr bool P2 = decltype(two_planes)::value;
      int8_t *plus = planes + static_cast<int64_t>(cur.g) * (P2 ? 2 : 1) * plane_stride + c0;
#pragma unroll 4
      for (int rr = warp; rr < rows_here; rr += 8) {
        const int64_t r = r_base + rr;
        const uint4 v = *reinterpret_cast<const uint4 *>(tile + rr * kWarpCols + lane * kColsPerThread);
        float xv[8];
        unpack8(v, xv);
        uint2 pk, nk;
        if constexpr (FAST) {
          if constexpr (HAS_D) scale8(xv, kc);  // u = RN(x fl(1/d)), the sign of x kept
          dualscale8_fast(xv, kc, pk, nk);
        } else if constexpr (FP8) {
          float uv[8];
#pragma unroll
          for (int j = 0; j < 8; ++j) uv[j] = xv[j];
          if constexpr (HAS_D) smooth8(uv, kc);
          dualscale8_fp8(xv, uv, kc, pk, nk);
        } else {
          if constexpr (HAS_D) smooth8(xv, kc);  // the sign of x survives in u
          dualscale8(xv, kc, pk, nk);
        }
        // planes: [G][P][M][K]; this row's 8 codes of each plane
        const int64_t at = (plus - planes) + r * K;
        if (!store_ok(status, at >= 0 && r < M && c0 + 8 <= K &&
                                  at + (P2 ? plane_stride : 0) + 8 <=
                                      static_cast<int64_t>(seg.G) * seg.P * plane_stride))
          continue;
        if constexpr (P2) {
          *reinterpret_cast<uint2 *>(plus + r * K) = pk;
          *reinterpret_cast<uint2 *>(plus + plane_stride + r * K) = nk;
        } else {
          // single scale: at most one of the two codes of an element is
          // non-zero (int8: the OR is their sum; FP8: the branch's code)
          *reinterpret_cast<uint2 *>(plus + r * K) = make_uint2(pk.x | nk.x, pk.y | nk.y);
        }
      }
    };
    if (c0 < K) {
      if (seg.P == 2) {
        if (!FP8 && fast)
          rows(std::true_type{}, std::true_type{});
        else
          rows(std::false_type{}, std::true_type{});
      } else {
        if (!FP8 && fast)
          rows(std::true_type{}, std::false_type{});
        else
          rows(std::false_type{}, std::false_type{});
      }
    }
    if constexpr (HAS_D && !FP8) {
      // every lane, including those past K in a ragged block (fast and nfix
      // are block-uniform)
      if (fast && nfix > 0) {
        __syncwarp();  // the warp's row stores come before the patches
        int8_t *blk = planes + static_cast<int64_t>(cur.g) * seg.P * plane_stride +
                      static_cast<int64_t>(cur.cb) * kWarpCols;
        if (seg.P == 2)
          patch_codes<true>(tile, fix_list, nfix, warp, lane, rows_here, r_base, blk, planes,
                            plane_stride, K, static_cast<int64_t>(cur.cb) * kWarpCols, seg,
                            status);
        else
          patch_codes<false>(tile, fix_list, nfix, warp, lane, rows_here, r_base, blk, planes,
                             plane_stride, K, static_cast<int64_t>(cur.cb) * kWarpCols, seg,
                             status);
      }
    }
    __syncthreads();  // every warp is done with stage st
    if (tid == 0 && it + kQStages < n_mine) {
      mbar_arrive_expect_tx(&full[st], kQTileBytes);
      tma_load_2d(qsmem + st * kQTileBytes, &tmX, &full[st], fetch.cb * kWarpCols,
                  fetch.rt * kQRows);
      fetch.next(n_cb, n_rt);
    }
  }
}

// ------------------------------------------------------------ quantize plan
// For every activation group g and channel c (with a divisor d[g][c]): whether
// the codes formed without either correction -- u = RN(x fl(1/d)), then
// q = rne(128 sat(RN(u fl(1/s)) / 128)) -- equal the quantizer's exact codes
// (u = fl(x/d), then fl(u/s)) for every bf16 input x, at the calibrated step
// pair of c's K-segment.  Both forms lie within 2^-22 (relative) of
// x / (d s), so they can differ only for x within that distance of a rounding
// boundary (h + 1/2) s d; bf16 inputs are 2^-8 apart, so such an x is a bf16
// neighbour of fl(fl((h + 1/2) s) d) (itself within 2^-23 of the boundary).
// One thread per channel evaluates both forms on those neighbours -- the
// truncation to bf16 and the values just below and above, h = 0 .. 127, both
// polarities: 768 inputs -- with exactly the kernels' operations.  Bit c % 32
// of word [g][c / 32] is set when all agree (and for channels past K).
__global__ void __launch_bounds__(256) quant_plan_kernel(const float *__restrict__ d, int64_t K,
                                                         const float *__restrict__ s_act,
                                                         SegParams seg, uint32_t *plan,
                                                         int *status) {
  const int g = blockIdx.y;
  const int64_t c = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  bool ok = true;
  if (c < K) {
    const int i = (seg.mode == SQ_SEG_INPUT) ? seg_index(seg.off, seg.n_seg, c) : 0;
    const float sc[2] = {s_act[(g * seg.S + i) * 2 + 0], s_act[(g * seg.S + i) * 2 + 1]};
    const float dc = d[g * K + c];
    StepConsts k;
    float dv[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) dv[j] = dc;
    fold_consts<false, true>(0, 1, sc, dv, k);
    for (int pol = 0; pol < 2; ++pol) {
      const float s = sc[pol];
      const float r7 = pol ? k.r7m : k.r7p, m128 = pol ? k.m128m : k.m128p;
      const float scale = pol ? -128.0f : 128.0f;
      for (int h = 0; h < 128; ++h) {
        const float b = static_cast<float>(h) + 0.5f;
        const uint32_t t = __float_as_uint(__fmul_rn(__fmul_rn(b, s), dc)) & 0xFFFF0000u;
        for (int e = -1; e <= 1; ++e) {
          const float xm = __uint_as_float(t + static_cast<uint32_t>(e) * 0x10000u);
          const float x = pol ? -xm : xm;
          // exact: smooth8's quotient, then dualscale8's
          const float xc = max_nan(min_nan(x, k.ld[0]), -k.ld[0]);
          const float q0 = __fmul_rn(xc, k.rd[0]);
          const float u = __fmaf_rn(__fmaf_rn(q0, k.nd[0], xc), k.rd[0], q0);
          const float a = mul_sat(u, r7);
          const float v = fma_sat(__fmaf_rn(a, m128, u), r7, a);
          uint32_t q_exact = __float_as_uint(__fmaf_rn(v, scale, 12582912.0f)) & 0xFFu;
          // uncorrected: scale8, then dualscale8_fast
          const float uf = __fmul_rn(x, k.rd[0]);
          uint32_t q_fast =
              __float_as_uint(__fmaf_rn(mul_sat(uf, r7), scale, 12582912.0f)) & 0xFFu;
          if (!pol) {  // the + plane's codes are lowered to 127
            q_exact = min(q_exact, 127u);
            q_fast = min(q_fast, 127u);
          }
          ok = ok && q_exact == q_fast;
        }
      }
    }
  }
  const unsigned bits = __ballot_sync(0xFFFFFFFFu, ok);
  const int64_t words = (K + 31) / 32;
  // plan: [G][words]
  if ((threadIdx.x & 31) == 0 && c / 32 < words && store_ok(status, g < seg.G))
    plan[g * words + c / 32] = bits;
}

// -------------------------------------------------------- weight quantize
// One block per output channel n (a row of the nn.Linear weight); for every
// K-segment: block-wide AMax of w * d, then the codes.
__device__ __forceinline__ float block_max(float v, float *red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xFFFFFFFFu, v, o));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  __syncthreads();  // red[] may still be read from the previous call
  if (lane == 0) red[warp] = v;
  __syncthreads();
  float r = 0.0f;
  for (int w = 0; w < (blockDim.x >> 5); ++w) r = fmaxf(r, red[w]);
  return r;
}

// QMAX = 127 (W8) or 7 (W4A8, "SegQuant-4"); with QMAX = 7 the codes are
// stored two per byte (channel 2j in the low nibble, 2j + 1 in the high one,
// 4-bit two's complement), each thread handling channel pairs.  QMAX = 448:
// FP8 E4M3 codes e4m3(fl(w'/s_w)) (round half to even, saturating).
__device__ __forceinline__ int weight_code(float wv, float s, float qmax) {
  const float v = fminf(fmaxf(__fdiv_rn(wv, s), -qmax), qmax);
  return __float2int_rn(v);
}

template <int QMAX>
__global__ void __launch_bounds__(256) quant_weight_kernel(const uint16_t *__restrict__ w,
                                                           int64_t N, int64_t K,
                                                           const float *__restrict__ d,
                                                           SegParams seg,
                                                           int8_t *__restrict__ wq,
                                                           float *__restrict__ s_w,
                                                           int *status) {
  constexpr float kQ = static_cast<float>(QMAX);
  __shared__ float red[32];
  const int64_t n = blockIdx.x;
  const int g = (seg.mode == SQ_SEG_OUTPUT && seg.G > 1) ? seg_index(seg.off, seg.n_seg, n) : 0;
  const uint16_t *row = w + n * K;
  const float *dg = d ? d + g * K : nullptr;
  for (int i = 0; i < seg.S; ++i) {
    const int64_t k0 = (seg.S == 1) ? 0 : seg.off[i];
    const int64_t k1 = (seg.S == 1) ? K : seg.off[i + 1];
    float amax = 0.0f;
    for (int64_t k = k0 + threadIdx.x; k < k1; k += blockDim.x) {
      const float wv = dg ? __fmul_rn(bf16_bits_to_f32(row[k]), dg[k]) : bf16_bits_to_f32(row[k]);
      amax = fmaxf(amax, fabsf(wv));
    }
    amax = block_max(amax, red);
    const float s = amax > 0.0f ? __fdiv_rn(amax, kQ) : 1.0f;
    if (threadIdx.x == 0 && store_ok(status, i < seg.S && n < N)) s_w[i * N + n] = s;  // [S][N]
    const auto wval = [&](int64_t k) {
      return dg ? __fmul_rn(bf16_bits_to_f32(row[k]), dg[k]) : bf16_bits_to_f32(row[k]);
    };
    // wq: [N][K] (int8 and FP8 codes) or [N][K / 2] (packed W4 pairs)
    if constexpr (QMAX == 127) {
      for (int64_t k = k0 + threadIdx.x; k < k1; k += blockDim.x)
        if (store_ok(status, n < N && k < K))
          wq[n * K + k] = static_cast<int8_t>(weight_code(wval(k), s, kQ));
    } else if constexpr (QMAX == 448) {
      for (int64_t k = k0 + threadIdx.x; k < k1; k += blockDim.x)
        if (store_ok(status, n < N && k < K))
          wq[n * K + k] = static_cast<int8_t>(
              __nv_cvt_float_to_fp8(__fdiv_rn(wval(k), s), __NV_SATFINITE, __NV_E4M3));
    } else {
      // segment bounds are even (multiples of 32), so pairs never straddle one
      uint8_t *packed = reinterpret_cast<uint8_t *>(wq) + n * (K / 2);
      for (int64_t j = k0 / 2 + threadIdx.x; j < k1 / 2; j += blockDim.x) {
        const int lo = weight_code(wval(2 * j), s, kQ), hi = weight_code(wval(2 * j + 1), s, kQ);
        if (store_ok(status, n < N && 2 * j + 1 < K))
          packed[j] = static_cast<uint8_t>((lo & 0xF) | ((hi & 0xF) << 4));
      }
    }
  }
}

// Packed W4 codes -> the int8 GEMM operand 16 q: each code moves into the high
// nibble of its own byte (low nibble 0), so no sign extension is needed.  One
// thread per 8 packed bytes (16 codes); a grid-stride loop over N*K/16 units.
__global__ void __launch_bounds__(256) unpack_w4_kernel(const uint2 *__restrict__ src,
                                                        uint4 *__restrict__ dst, int64_t units,
                                                        int *status) {
  for (int64_t u = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; u < units;
       u += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    if (!store_ok(status, u >= 0 && u < units)) continue;  // dst: [N * K / 16] uint4
    const uint2 v = src[u];
    const uint32_t e0 = (v.x & 0x0F0F0F0Fu) << 4, o0 = v.x & 0xF0F0F0F0u;  // channels 2j, 2j+1
    const uint32_t e1 = (v.y & 0x0F0F0F0Fu) << 4, o1 = v.y & 0xF0F0F0F0u;
    dst[u] = make_uint4(__byte_perm(e0, o0, 0x5140), __byte_perm(e0, o0, 0x7362),
                        __byte_perm(e1, o1, 0x5140), __byte_perm(e1, o1, 0x7362));
  }
}

int num_sms() {
  static int sms = 0;
  if (sms == 0) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (sms <= 0) sms = 148;
  }
  return sms;
}

}  // namespace

cudaError_t launch_calibrate_act(const uint16_t *x, int64_t M, int64_t K, int64_t ldx,
                                 const float *d, const SegParams &seg, float *s_act,
                                 int *status, cudaStream_t stream) {
  const int n = seg.G * seg.S;
  cudaError_t e = cudaMemsetAsync(s_act, 0, sizeof(float) * 2 * n, stream);
  if (e != cudaSuccess) return e;
  if (M > 0) {
    const int gx = static_cast<int>((K + kWarpCols - 1) / kWarpCols);
    int gy = static_cast<int>((M + kRowsPerBlock - 1) / kRowsPerBlock);
    const int cap = (num_sms() * 4 + gx * seg.G - 1) / (gx * seg.G);
    if (gy > cap) gy = cap < 1 ? 1 : cap;
    calib_reduce_kernel<<<dim3(gx, gy, seg.G), dim3(32, kRowsPerBlock), 0, stream>>>(
        x, M, K, ldx, d, seg, s_act, status);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  calib_finalize_kernel<<<1, 256, 0, stream>>>(s_act, n, seg.P == 1 ? 1 : 0, seg.fp8, status);
  return cudaGetLastError();
}

sq_status launch_quantize_act(const uint16_t *x, int64_t M, int64_t K, int64_t ldx,
                              const float *d, const float *s_act, const SegParams &seg,
                              int8_t *planes, const uint32_t *plan, int *status,
                              cudaStream_t stream) {
  if (M == 0) return SQ_OK;
  EncodeTiledFn enc = tensor_map_encoder();
  if (enc == nullptr) return SQ_ERR_CUDA;
  CUtensorMap tmX;
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(K), static_cast<cuuint64_t>(M)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(ldx) * 2};
  const cuuint32_t box[2] = {kWarpCols, kQRows};
  const cuuint32_t estr[2] = {1, 1};
  if (enc(&tmX, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<uint16_t *>(x), dims, strides,
          box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return SQ_ERR_CUDA;
  const int64_t n_units =
      ((M + kQRows - 1) / kQRows) * ((K + kWarpCols - 1) / kWarpCols) * seg.G;
  // Three resident blocks per SM, each keeping kQStages tiles in flight; the
  // units are split evenly over exactly that many blocks.
  int64_t nblk = static_cast<int64_t>(num_sms()) * 3;
  if (nblk > n_units) nblk = n_units;
  const size_t smem = kFixOffset + (d != nullptr && plan != nullptr && !seg.fp8
                                         ? 8 * 2 * kFixMax * sizeof(float4)
                                         : 0);
  auto kernel = seg.fp8 ? (d ? quant_act_kernel<true, true> : quant_act_kernel<true, false>)
                        : (d ? quant_act_kernel<false, true> : quant_act_kernel<false, false>);
  if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(smem)) != cudaSuccess)
    return SQ_ERR_CUDA;
  // Programmatic dependent launch: the blocks may start their prologue while
  // the preceding kernel finishes; they wait for it before touching memory.
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(nblk));
  cfg.blockDim = dim3(256);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, kernel, tmX, M, K, d, s_act, seg, planes, plan, status) !=
      cudaSuccess)
    return SQ_ERR_CUDA;
  return cudaGetLastError() == cudaSuccess ? SQ_OK : SQ_ERR_CUDA;
}

cudaError_t launch_quantize_plan(const float *d, int64_t K, const float *s_act,
                                 const SegParams &seg, uint32_t *plan, int *status,
                                 cudaStream_t stream) {
  const dim3 grid(static_cast<unsigned>((K + 255) / 256), static_cast<unsigned>(seg.G));
  quant_plan_kernel<<<grid, 256, 0, stream>>>(d, K, s_act, seg, plan, status);
  return cudaGetLastError();
}

cudaError_t launch_quantize_weight(const uint16_t *w, int64_t N, int64_t K, const float *d,
                                   const SegParams &seg, int8_t *wq, float *s_w, int *status,
                                   cudaStream_t stream) {
  if (N == 0) return cudaSuccess;
  if (seg.fp8)
    quant_weight_kernel<448><<<static_cast<unsigned>(N), 256, 0, stream>>>(w, N, K, d, seg, wq,
                                                                          s_w, status);
  else
    quant_weight_kernel<127><<<static_cast<unsigned>(N), 256, 0, stream>>>(w, N, K, d, seg, wq,
                                                                          s_w, status);
  return cudaGetLastError();
}

cudaError_t launch_quantize_weight_w4(const uint16_t *w, int64_t N, int64_t K, const float *d,
                                      const SegParams &seg, uint8_t *wq4, float *s_w,
                                      int *status, cudaStream_t stream) {
  if (N == 0) return cudaSuccess;
  quant_weight_kernel<7><<<static_cast<unsigned>(N), 256, 0, stream>>>(
      w, N, K, d, seg, reinterpret_cast<int8_t *>(wq4), s_w, status);
  return cudaGetLastError();
}

cudaError_t launch_unpack_w4(const uint8_t *wq4, int64_t N, int64_t K, int8_t *wq, int *status,
                             cudaStream_t stream) {
  const int64_t units = N * K / 16;  // K % 16 == 0
  if (units == 0) return cudaSuccess;
  int64_t blocks = (units + 255) / 256;
  const int64_t cap = static_cast<int64_t>(num_sms()) * 8;
  if (blocks > cap) blocks = cap;
  unpack_w4_kernel<<<static_cast<unsigned>(blocks), 256, 0, stream>>>(
      reinterpret_cast<const uint2 *>(wq4), reinterpret_cast<uint4 *>(wq), units, status);
  return cudaGetLastError();
}

}  // namespace sq
