// gemm.cu -- DualScale + SegLinear W8A8 GEMM for sm_100a.
//
// What it computes ("SegQuant", papernotes.org, sections DualScale and
// SegLinear): for every output element
//   y[m][n] = sum_i s_w[i][n] * (s+_i * A+_i[m][n] + s-_i * A-_i[m][n]) + bias[n]
// where A+-_i are the exact int32 products of the X^+ / X^- planes with the
// shared int8 weight over K-segment i.  The pages run the two products as one
// batched GEMM with a fused epilogue; here both polarities of a 128-row tile
// share every weight tile staged in shared memory and accumulate side by side
// in tensor memory, so the X^- product never reaches HBM.
//
// Structure (one persistent CTA per SM; 320 threads, 576 for input-segmented
// layers):
//   warp 0      TMA producer: per 128-byte k-block, one 3D box {128 B, 128
//               rows, 2 planes} of [X^+; X^-] and one box {128 B, BN rows} of
//               W^, into a STAGES-deep ring guarded by mbarriers;
//   warp 1      TMEM owner and MMA issuer (one thread): tcgen05.mma kind::i8,
//               M = 128, N = BN, K = 32, two per k-step (X^+ and X^-);
//   warps 2-    epilogue (8 warps, 16 for input-segmented layers): tcgen05.ld
//               of both accumulators in the 16x256b pattern, fp32
//               reconstruction, bias, bf16/fp32 stores.  Input-segmented
//               layers drain one accumulator pair per K-segment into fp32
//               running sums held in registers while the MMA warp fills the
//               other TMEM buffer.
// TMEM holds 512 columns: BN = 256 gives one buffer (+ and - of 256 columns);
// BN = 128 gives two, so drains overlap the next segment's MMAs.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <cstring>
#include <mutex>

#include "sm100.cuh"
#include "sq_internal.h"

namespace sq {
namespace {

// Column tile of one-segment layers: 256 (one TMEM buffer, the epilogue runs
// between tiles) or 128 (two buffers, the epilogue overlaps the next tile).
#ifndef SQ_GEMM_BN_ONE_SEG
#define SQ_GEMM_BN_ONE_SEG 256
#endif

constexpr int BM = 128;              // rows of M per tile (TMEM lanes)
constexpr int BK = 128;              // int8 K elements per stage = one 128-B swizzle row
constexpr int MMA_K = 32;            // K of one kind::i8 MMA
// Epilogue warps: 8 for one-segment layers (register-heavy final epilogue), 16
// for input-segmented layers (latency-bound per-segment drains).
constexpr int threads_for(int epi_warps) { return 64 + 32 * epi_warps; }
constexpr uint64_t kWaitLimitNs = 2000000000ull;   // 2 s: far above any tile's latency

struct GemmParams {
  int32_t M, N, K;
  int32_t num_n_tiles, num_tiles, num_kb;
  int32_t G, S;
  int32_t n_seg_out;                // output segments mapped to groups (G > 1)
  int32_t k_off[SQ_MAX_SEGMENTS + 1];
  int32_t n_off[SQ_MAX_SEGMENTS + 1];
  const float *s_w;
  const float *s_act;
  // Factor applied to s+ and s- as they are loaded: 1, or 2^-4 when the weight
  // operand holds 16 q of W4A8 codes q (exact: a power of two).
  float act_mul;
  const uint16_t *bias;
  void *y;
  int64_t ldy;
  int *status;
  const float *s_next;  // OUT_PLANES: the next layer's {s+, s-}
  int32_t p_next;       // OUT_PLANES: its planes (2, or 1 single scale)
  // Split tail (one K-segment only): the first sk_W waves of gridDim.x tiles
  // run whole, one tile per CTA and wave; the k-blocks of the last sk_R tiles
  // are shared out evenly over all CTAs.  A CTA whose share starts inside a
  // tile writes its int32 partial sums to its slot of sk_ws and raises its
  // epilogue warps' flags; the CTA holding the tile's first k-block adds the
  // partials before the epilogue.  sk_R == 0: every CTA takes whole tiles.
  int32_t sk_W, sk_R;
  int32_t *sk_ws;       // [gridDim.x][slot_words] int32 partial sums
  int32_t *sk_flags;    // [gridDim.x][EPI_WARPS], zero between calls
  int64_t sk_slot_words;
};

// A CTA's work, as pieces (tile, k-blocks [kb0, kb1), role), enumerated in the
// same order by the producer, the MMA issuer and the epilogue.
enum PieceRole { PIECE_FULL = 0, PIECE_PARTIAL = 1, PIECE_FINAL = 2 };
template <bool TAIL>  // false: whole tiles only (input-segmented and fused layers)
struct Pieces {
  int c, G, W, KB, num_tiles, j;
  int64_t U, u, u_end;
  __device__ void init(const GemmParams &p) {
    c = blockIdx.x;
    G = gridDim.x;
    KB = p.num_kb;
    num_tiles = p.num_tiles;
    j = 0;
    if (TAIL && p.sk_R > 0) {
      W = p.sk_W;
      U = static_cast<int64_t>(p.sk_R) * KB;
      u = U * c / G;
      u_end = U * (c + 1) / G;
    } else {
      W = (num_tiles + G - 1) / G;
      U = u = u_end = 0;
    }
  }
  __device__ bool next(int &tile, int &kb0, int &kb1, int &role) {
    if (j < W) {
      tile = c + j * G;
      ++j;
      if (tile >= num_tiles) return false;
      kb0 = 0;
      kb1 = KB;
      role = PIECE_FULL;
      return true;
    }
    if (!TAIL || u >= u_end) return false;
    const int tt = static_cast<int>(u / KB);
    kb0 = static_cast<int>(u - static_cast<int64_t>(tt) * KB);
    const int64_t left = u_end - u;
    kb1 = (left < KB - kb0) ? kb0 + static_cast<int>(left) : KB;
    tile = W * G + tt;
    role = kb0 > 0 ? PIECE_PARTIAL : (kb1 == KB ? PIECE_FULL : PIECE_FINAL);
    u += kb1 - kb0;
    return true;
  }
  // The CTA holding the last k-block of split tile `tile`: the contributors
  // of a PIECE_FINAL piece of CTA c are CTAs c + 1 .. that one.
  __device__ int last_holder(int tile) const {
    const int64_t v = static_cast<int64_t>(tile - W * G) * KB + KB - 1;
    int cc = static_cast<int>(v * G / U);
    while (cc + 1 < G && U * (cc + 1) / G <= v) ++cc;
    while (cc > 0 && U * cc / G > v) --cc;
    return cc;
  }
};

// Whole tiles only: tile = blockIdx.x, blockIdx.x + gridDim.x, ...
template <>
struct Pieces<false> {
  int tile_, num_tiles, KB;
  int64_t U = 1;
  int G = 1;
  __device__ void init(const GemmParams &p) {
    tile_ = static_cast<int>(blockIdx.x) - static_cast<int>(gridDim.x);
    num_tiles = p.num_tiles;
    KB = p.num_kb;
  }
  __device__ bool next(int &tile, int &kb0, int &kb1, int &role) {
    tile_ += gridDim.x;
    tile = tile_;
    kb0 = 0;
    kb1 = KB;
    role = PIECE_FULL;
    return tile_ < num_tiles;
  }
  __device__ int last_holder(int) const { return -1; }
};

// Partial sums: one 32-word run per thread, chunk and polarity.
// A run holds 32 words per lane of one warp, laid out [v4 group][lane][4]: each
// store or load instruction of the warp covers 512 contiguous bytes.  `run`
// points at the run's first word plus 4 * lane; g0 is the first v4 group.
// (p: the workspace's extent, gridDim.x slots of sk_slot_words, for the
// debug build's bound test)
template <int N>
__device__ __forceinline__ void sk_store(const GemmParams &p, int32_t *run, int g0,
                                         const uint32_t *v) {
#pragma unroll
  for (int i = 0; i < N; i += 4) {
    int32_t *at = run + (g0 + i / 4) * 128;
    if (store_ok(p.status, at >= p.sk_ws && at + 4 <= p.sk_ws + gridDim.x * p.sk_slot_words))
      __stcg(reinterpret_cast<uint4 *>(at), make_uint4(v[i], v[i + 1], v[i + 2], v[i + 3]));
  }
}
// Adds partial sums: int32 (exact) for integer codes, fp32 for FP8 codes.  The
// loads are plain L2 loads (after the flag's acquire), so the compiler can
// issue them all before the first add.
template <int N, bool F8>
__device__ __forceinline__ void sk_add(const int32_t *run, int g0, uint32_t *v) {
  uint4 a[N / 4];
#pragma unroll
  for (int i = 0; i < N / 4; ++i) a[i] = __ldcg(reinterpret_cast<const uint4 *>(run + (g0 + i) * 128));
#pragma unroll
  for (int i = 0; i < N / 4; ++i) {
    const uint32_t w[4] = {a[i].x, a[i].y, a[i].z, a[i].w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      if constexpr (F8)
        v[4 * i + e] = __float_as_uint(__fadd_rn(__uint_as_float(v[4 * i + e]), __uint_as_float(w[e])));
      else
        v[4 * i + e] += w[e];
    }
  }
}
__device__ __forceinline__ int ld_acquire(const int32_t *f) {
  int v;
  asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(f) : "memory");
  return v;
}
__device__ __forceinline__ void st_release(int32_t *f, int v) {
  asm volatile("st.release.gpu.global.b32 [%0], %1;" ::"l"(f), "r"(v) : "memory");
}

// POL = activation planes per group: 2 for DualScale (X^+ and X^-), 1 for the
// single-scale path (one merged plane).
template <int BN, int STAGES, int EPI_WARPS, int POL, bool SEGK, bool TMA_STORE>
struct Smem {
  static constexpr int A_BYTES = POL * BM * BK;  // X^+ tile, then X^- tile
  static constexpr int B_BYTES = BN * BK;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int NBUF = 512 / (POL * BN);  // TMEM accumulator buffers
  static constexpr int EPI_OFFSET = STAGES * STAGE_BYTES;  // per-warp column constants
  static constexpr int COLS = BN / (EPI_WARPS / 4);  // columns per epilogue warp
  // per warp: one K-segment: the folded c+ = fl(s_w s+), c- = fl(s_w s-)
  // and the bias (COLS floats each; c- unused with one plane); several
  // K-segments: c+ and c- double-buffered (the bias goes, at the end of a
  // tile, into the buffer the last K-segment did not use)
  static constexpr int CONST_FLOATS = (SEGK ? 4 : 3) * COLS;
  static constexpr int EPI_BYTES = EPI_WARPS * CONST_FLOATS * 4;
  // per-warp staging of one 32 x 32 bf16 output chunk for the tensor store
  static constexpr int STG_OFFSET = EPI_OFFSET + EPI_BYTES;
  static constexpr int STG_BYTES = TMA_STORE ? EPI_WARPS * 2048 : 0;
  static constexpr int BAR_OFFSET = STG_OFFSET + STG_BYTES;
  static_assert(STG_OFFSET % 1024 == 0, "staging must be aligned to the swizzle pattern");
  static constexpr int NUM_BARS = 2 * STAGES + 2 * NBUF + 1;
  static constexpr int BYTES = BAR_OFFSET + NUM_BARS * 8 + 16 + 1024;  // + 1 KB alignment slack
};

__device__ __forceinline__ int group_of_tile(const GemmParams &p, int nt, int BN) {
  if (p.G == 1) return 0;
  return seg_index(p.n_off, p.n_seg_out, static_cast<int64_t>(nt) * BN);
}

// Bounded wait that also gives up when another role has already aborted.
__device__ __forceinline__ bool wait_bar(uint64_t *bar, uint32_t parity, volatile int *abort_flag,
                                         int *status) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  while (true) {
    if (mbar_try_wait_sleep(bar, parity, kSleepHintNs)) return true;
    if (*abort_flag) return false;
    if (globaltimer_ns() - t0 > kWaitLimitNs) {
      *abort_flag = 1;
      atomicExch(status, static_cast<int>(SQ_ERR_DEVICE_TIMEOUT));
      return false;
    }
  }
}

// Packed pairs of fp32 (sm_100 f32x2 arithmetic): two lanes of work per instruction.
__device__ __forceinline__ uint64_t f2pack(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ void f2unpack(uint64_t v, float &lo, float &hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t ffma2(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ float bf16_to_f32(uint16_t h) {
  return __uint_as_float(static_cast<uint32_t>(h) << 16);
}

// ---- the FFN activation of the fused producer (OUT_PLANES) ----------------
// gelu(x) = x/2 (1 + tanh(sqrt(2/pi) (x + 0.044715 x^3))), the tanh
// approximation the models' FFNs use between the two linears, as one fixed
// sequence of fp32 operations, each rounded once:
//   tanh(u) = 1 - 2 / (e^(2|u|) + 1) with the sign of u; 1 for |u| >= 9;
//   e^z (0 <= z <= 18): z = n ln2 + f, n = rint(z / ln2) (Cody and Waite's
//   reduction with ln2 split into a head exact in n * head and a tail), e^f by
//   its Taylor series to degree 7, times 2^n.
__device__ __forceinline__ float exp_0_18(float z) {
  const float n = rintf(__fmul_rn(z, 0x1.715476p+0f));  // z / ln2
  float f = __fmaf_rn(-n, 0x1.62e4p-1f, z);             // ln2 head (17 bits)
  f = __fmaf_rn(-n, 0x1.7f7d1cp-20f, f);                // ln2 tail
  float q = 0x1.a01a02p-13f;                            // 1/7!
  q = __fmaf_rn(q, f, 0x1.6c16c2p-10f);                 // 1/6!
  q = __fmaf_rn(q, f, 0x1.111112p-7f);                  // 1/5!
  q = __fmaf_rn(q, f, 0x1.555556p-5f);                  // 1/4!
  q = __fmaf_rn(q, f, 0x1.555556p-3f);                  // 1/3!
  q = __fmaf_rn(q, f, 0.5f);
  q = __fmaf_rn(q, f, 1.0f);
  q = __fmaf_rn(q, f, 1.0f);
  // 2^n, 0 <= n <= 26: n as an integer from the bits of 1.5 * 2^23 + n (exact)
  const int ni = __float_as_int(__fadd_rn(n, 12582912.0f)) - 0x4B400000;
  return __fmul_rn(q, __int_as_float((ni + 127) << 23));
}

__device__ __forceinline__ float gelu_tanh(float x) {
  const float x3 = __fmul_rn(__fmul_rn(x, x), x);
  const float u = __fmul_rn(0x1.988454p-1f, __fmaf_rn(0x1.6e4e26p-5f, x3, x));
  // Branch-free: e^(2|u|) with |u| capped at 9, and 1 selected from 9 on.
  // 2 / d = 2 RN(1/d) exactly (d = e + 1 in [2, e^18 + 1]: no underflow).
  const float a = fabsf(u);
  const float e = exp_0_18(__fmul_rn(2.0f, fminf(a, 9.0f)));
  float t = __fsub_rn(1.0f, __fmul_rn(2.0f, __frcp_rn(__fadd_rn(e, 1.0f))));
  t = a < 9.0f ? t : 1.0f;
  if (u < 0.0f) t = -t;
  return __fmul_rn(__fmul_rn(0.5f, x), __fadd_rn(1.0f, t));
}

// DualScale codes of the next layer's input x2 = bf16(gelu(bf16(y))), the
// activation quantizer's rule with d = 1: x2 >= 0 gives q+ = rne(min(fl(x2/s+),
// 127)), x2 < 0 gives q- = rne(max(fl(x2/s-), -128)); the other code is 0.  The
// quotient is the correctly rounded one, formed from r = fl(1/s) by
// Markstein's correction: q0 = fl(x2 r), then fl(q0 + (x2 - q0 s) r).  Where
// x2 r overflows, the correction yields NaN, and fminf / fmaxf return the
// clamp bound: the saturated code.
__device__ __forceinline__ void gelu_codes(float y, float sp, float rp, float sm, float rm,
                                           int &qp, int &qm) {
  const float xb = __bfloat162float(__float2bfloat16_rn(y));
  const float x2 = __bfloat162float(__float2bfloat16_rn(gelu_tanh(xb)));
  // rne of a value in [-128, 127]: the integer part of the bits of
  // 1.5 * 2^23 + v, where the add rounds to the nearest integer, ties to even.
  const bool neg = x2 < 0.0f;
  const float s = neg ? sm : sp, r = neg ? rm : rp;
  const float q0 = __fmul_rn(x2, r);
  const float quot = __fmaf_rn(__fmaf_rn(-q0, s, x2), r, q0);
  const float v = neg ? fmaxf(quot, -128.0f) : fminf(quot, 127.0f);
  const int q = __float_as_int(__fadd_rn(v, 12582912.0f)) - 0x4B400000;
  qp = neg ? 0 : q;
  qm = neg ? q : 0;
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t *>(&v);
}

// Two adjacent output columns n, n + 1 of row m (n even; n + 1 may be >= N).
template <int OUT>
__device__ __forceinline__ void store_pair(const GemmParams &p, int64_t m, int64_t n, float y0,
                                           float y1) {
  if (n >= p.N) return;
  // y: [M][ldy], columns < N <= ldy
  if (!store_ok(p.status, m >= 0 && m < p.M && n >= 0 && n < p.ldy)) return;
  if (OUT == OUT_BF16) {
    uint16_t *row = reinterpret_cast<uint16_t *>(p.y) + m * p.ldy;
    if (n + 1 < p.N) {
      *reinterpret_cast<uint32_t *>(row + n) = pack_bf16x2(y0, y1);
    } else {
      const __nv_bfloat16 b = __float2bfloat16_rn(y0);
      row[n] = *reinterpret_cast<const uint16_t *>(&b);
    }
  } else {
    float *row = reinterpret_cast<float *>(p.y) + m * p.ldy;
    if (n + 1 < p.N)
      *reinterpret_cast<float2 *>(row + n) = make_float2(y0, y1);
    else
      row[n] = y0;
  }
}

// TMEM columns of one chunk: 16 or 32 per lane.
template <int CW>
__device__ __forceinline__ void tmem_ld_cols(uint32_t taddr, uint32_t (&r)[CW]) {
  if constexpr (CW == 32)
    tmem_ld_32x32b_x32(taddr, r);
  else
    tmem_ld_32x32b_x16(taddr, r);
}

// One CTA per SM (shared memory allows no more).  Its warps spread over the four
// 16K-register sub-partitions (10 warps: 3/3/2/2, a thread at most 168
// registers; 18 warps: 5/5/4/4, at most 96).
// accumulator word -> fp32: int32 (kind::i8, RN conversion) or the fp32 bits
// themselves (kind::f8f6f4).
template <bool F8>
__device__ __forceinline__ float acc_f32(uint32_t v) {
  if constexpr (F8)
    return __uint_as_float(v);
  else
    return __int2float_rn(static_cast<int32_t>(v));
}

// F8: E4M3 planes and weights (kind::f8f6f4, fp32 accumulators) instead of int8.
template <int BN, int STAGES, int OUT, bool SEGK, int EPI_WARPS, int POL, bool F8>
__global__ void __launch_bounds__(threads_for(EPI_WARPS), 1)
    dualscale_gemm_kernel(const __grid_constant__ CUtensorMap tmA,
                          const __grid_constant__ CUtensorMap tmB,
                          const __grid_constant__ CUtensorMap tmY,
                          const __grid_constant__ GemmParams p) {
  // One-segment bf16 output (and the next layer's planes) leave through
  // shared memory and TMA stores.
  constexpr bool TMA_STORE = (OUT == OUT_BF16 || OUT == OUT_PLANES) && !SEGK;
  // Split tail of the last wave: one-segment layers with a plain output.
  constexpr bool TAIL = !SEGK && OUT != OUT_PLANES;
  static_assert(OUT != OUT_PLANES || (!SEGK && !F8), "planes output: one K-segment, int8");
  using L = Smem<BN, STAGES, EPI_WARPS, POL, SEGK, TMA_STORE>;
  constexpr int NBUF = L::NBUF;
  constexpr int ACC_COLS = POL * BN;  // TMEM columns of one accumulator buffer
  constexpr int HALF = L::COLS;      // columns per epilogue warp
  // Column chunk of the one-segment epilogue (32) and of the raw-accumulator
  // output: 32 columns with 8 warps, 16 with 16 (a smaller register budget).
  constexpr int CW = EPI_WARPS >= 16 ? 16 : 32;
  static_assert(EPI_WARPS % 4 == 0 && HALF % 32 == 0, "epilogue split");
  static_assert(NBUF >= 1, "BN too large for TMEM");

  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t *full = reinterpret_cast<uint64_t *>(smem + L::BAR_OFFSET);
  uint64_t *empty = full + STAGES;
  uint64_t *acc_full = empty + STAGES;
  uint64_t *acc_empty = acc_full + NBUF;
  uint64_t *mma_done = acc_empty + NBUF;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(mma_done + 1);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < NBUF; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], EPI_WARPS);
    }
    mbar_init(mma_done, 1);
    *abort_flag = 0;
    fence_mbar_init();
    prefetch_tmap(&tmA);
    prefetch_tmap(&tmB);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  grid_dependency_wait();  // the prologue above touches no global memory

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      uint32_t armed = 0, armed_parity = 0;  // per stage: has a load, its phase
      Pieces<TAIL> pc;
      pc.init(p);
      int tile, kb0, kb1, role;
      while (pc.next(tile, kb0, kb1, role)) {
        const int mt = tile / p.num_n_tiles, nt = tile % p.num_n_tiles;
        const int g = group_of_tile(p, nt, BN);
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!wait_bar(&empty[stage], phase ^ 1, abort_flag, p.status)) goto producer_done;
          uint8_t *sa = smem + stage * L::STAGE_BYTES;
          mbar_arrive_expect_tx(&full[stage], L::STAGE_BYTES);
          tma_load_3d(sa, &tmA, &full[stage], kb * BK, mt * BM, POL * g);
          tma_load_2d(sa + L::A_BYTES, &tmB, &full[stage], kb * BK, nt * BN);
          armed |= 1u << stage;
          armed_parity = (armed_parity & ~(1u << stage)) | (phase << stage);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
    producer_done:
      // Never leave with a copy in flight into this CTA's shared memory.
      for (int s = 0; s < STAGES; ++s)
        if (armed & (1u << s)) mbar_wait(&full[s], (armed_parity >> s) & 1u, kWaitLimitNs);
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = F8 ? idesc_e4m3(BM, BN) : idesc_i8(BM, BN);
      int stage = 0;
      uint32_t phase = 0;
      uint32_t acc_iter = 0;
      Pieces<TAIL> pc;
      pc.init(p);
      int tile, kb0, kb1, role;
      while (pc.next(tile, kb0, kb1, role)) {
        int seg = 0;
        int seg_end = SEGK ? p.k_off[1] : p.K;
        uint32_t buf = acc_iter % NBUF;
        if (!wait_bar(&acc_empty[buf], ((acc_iter / NBUF) & 1) ^ 1, abort_flag, p.status))
          goto mma_exit;
        tc_fence_after();
        uint32_t d_plus = tmem_base + buf * ACC_COLS;
        uint32_t accumulate = 0;
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!wait_bar(&full[stage], phase, abort_flag, p.status)) goto mma_exit;
          tc_fence_after();
          const uint32_t sa = smem_u32(smem + stage * L::STAGE_BYTES);
          const uint32_t sb = sa + L::A_BYTES;
#pragma unroll
          for (int kk = 0; kk < BK / MMA_K; ++kk) {
            const int k = kb * BK + kk * MMA_K;
            if (k >= p.K) break;
            if (SEGK && k == seg_end) {
              // K-segment boundary: hand this accumulator pair to the epilogue
              // and continue in the next TMEM buffer.
              mma_commit(&acc_full[buf]);
              ++acc_iter;
              buf = acc_iter % NBUF;
              if (!wait_bar(&acc_empty[buf], ((acc_iter / NBUF) & 1) ^ 1, abort_flag, p.status))
                goto mma_exit;
              tc_fence_after();
              d_plus = tmem_base + buf * ACC_COLS;
              accumulate = 0;
              ++seg;
              seg_end = p.k_off[seg + 1];
            }
            const uint64_t b_desc = sdesc_kmajor_sw128(sb + kk * MMA_K);
            if constexpr (F8) {
              mma_e4m3(d_plus, sdesc_kmajor_sw128(sa + kk * MMA_K), b_desc, idesc, accumulate);
              if (POL == 2)
                mma_e4m3(d_plus + BN, sdesc_kmajor_sw128(sa + BM * BK + kk * MMA_K), b_desc,
                         idesc, accumulate);
            } else {
              mma_i8(d_plus, sdesc_kmajor_sw128(sa + kk * MMA_K), b_desc, idesc, accumulate);
              if (POL == 2)
                mma_i8(d_plus + BN, sdesc_kmajor_sw128(sa + BM * BK + kk * MMA_K), b_desc,
                       idesc, accumulate);
            }
            accumulate = 1;
          }
          mma_commit(&empty[stage]);  // frees the stage once these MMAs finish
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
        mma_commit(&acc_full[buf]);
        ++acc_iter;
      }
    mma_exit:
      // Wait for every MMA this thread issued before TMEM can be released.
      mma_commit(mma_done);
      mbar_wait(mma_done, 0, kWaitLimitNs);
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int ew = warp - 2;
    const int quarter = warp & 3;       // TMEM lanes this warp may read
    const int half = ew >> 2;           // which column part of the tile
    const int row = quarter * 32 + lane;
    const uint32_t lane_addr = static_cast<uint32_t>(quarter * 32) << 16;
    // Warp-private column constants in shared memory, read back as float2
    // pairs: with one K-segment c+ = fl(s_w s+), c- = fl(s_w s-) and the bias,
    // [HALF] floats each; with several, two buffers of c+ and c- (the bias
    // goes, at the end of a tile, into the buffer the last segment did not use).
    float *cst_base = reinterpret_cast<float *>(smem + L::EPI_OFFSET) + ew * L::CONST_FLOATS;
    uint8_t *stg = smem + L::STG_OFFSET + ew * 2048;  // used when TMA_STORE
    uint32_t acc_iter = 0;
    // OUT_PLANES: the next layer's steps s+- and their reciprocals fl(1/s+-).
    float sp_nx = 1.0f, rp_nx = 1.0f, sm_nx = 1.0f, rm_nx = 1.0f;
    if constexpr (OUT == OUT_PLANES) {
      sp_nx = p.s_next[0];
      sm_nx = p.s_next[1];
      rp_nx = __frcp_rn(sp_nx);
      rm_nx = __frcp_rn(sm_nx);
    }
    Pieces<TAIL> pc;
    pc.init(p);
    int tile, kb0, kb1, role;
    while (pc.next(tile, kb0, kb1, role)) {
      const int mt = tile / p.num_n_tiles, nt = tile % p.num_n_tiles;
      const int g = group_of_tile(p, nt, BN);
      const int64_t m = static_cast<int64_t>(mt) * BM + row;
      const int64_t nb = static_cast<int64_t>(nt) * BN + half * HALF;
      (void)kb0;
      (void)kb1;
      // Split tail: the partial sums of a PIECE_PARTIAL go to this CTA's slot;
      // a PIECE_FINAL adds those of CTAs blockIdx.x + 1 .. sk_last first.
      int sk_last = -1;
      if (TAIL && role == PIECE_FINAL) sk_last = pc.last_holder(tile);
      const auto slot_run = [&](int cta, int c, int pol) {
        return p.sk_ws + cta * p.sk_slot_words +
               ((static_cast<int64_t>(ew) * (HALF / 32) + c) * POL + pol) * 1024 + lane * 4;
      };
      if (TAIL && role == PIECE_FINAL) {
        // Wait (bounded) until every contributor has written its partials.
        bool ok = true;
        if (lane == 0) {
          const uint64_t t0 = globaltimer_ns();
          for (int cc = blockIdx.x + 1; cc <= sk_last && ok; ++cc) {
            if (pc.U * cc / pc.G == pc.U * (cc + 1) / pc.G) continue;  // holds no k-block
            const int32_t *f = p.sk_flags + cc * EPI_WARPS + ew;
            while (ld_acquire(f) == 0) {
              if (*abort_flag) {
                ok = false;
                break;
              }
              if (globaltimer_ns() - t0 > kWaitLimitNs) {
                *abort_flag = 1;
                atomicExch(p.status, static_cast<int>(SQ_ERR_DEVICE_TIMEOUT));
                ok = false;
                break;
              }
              __nanosleep(64);
            }
          }
        }
        ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
        if (!ok) goto epilogue_exit;
        for (int cc = blockIdx.x + 1; cc <= sk_last; ++cc)  // every lane acquires
          if (pc.U * cc / pc.G != pc.U * (cc + 1) / pc.G)
            (void)ld_acquire(p.sk_flags + cc * EPI_WARPS + ew);
      }
      if (!SEGK && OUT != OUT_S32 && !(TAIL && role == PIECE_PARTIAL)) {
        // The folded c+- = fl(s_w s+-) and the bias of this warp's columns,
        // staged while the MMAs run (one K-segment: s_act[g][0]).
        const float sp0 = __fmul_rn(p.s_act[g * 2 + 0], p.act_mul);
        const float sm0 = __fmul_rn(p.s_act[g * 2 + 1], p.act_mul);
        __syncwarp();
        for (int j = lane; j < HALF; j += 32) {
          const int64_t n = nb + j;
          const float w = n < p.N ? p.s_w[n] : 0.0f;
          cst_base[j] = __fmaf_rn(w, sp0, 0.0f);
          if constexpr (POL == 2) cst_base[HALF + j] = __fmaf_rn(w, sm0, 0.0f);
          cst_base[POL * HALF + j] =
              (p.bias != nullptr && n < p.N) ? bf16_to_f32(p.bias[n]) : 0.0f;
        }
        __syncwarp();
      }
      // Multi-segment state: packed running sums (column pairs) and the next
      // K-segment's weight and activation scales, loaded one segment ahead and
      // not used (not even scaled by act_mul) until that segment starts, so
      // that no instruction waits for a global load between two drains.
      uint64_t run2[SEGK ? HALF / 2 : 1];
      float sw_next[SEGK ? HALF / 32 : 1];
      float sp_next = 0.0f, sm_next = 0.0f;
      if constexpr (SEGK && OUT != OUT_S32) {
#pragma unroll
        for (int j = 0; j < HALF / 2; ++j) run2[j] = 0ull;
#pragma unroll
        for (int q = 0; q < HALF / 32; ++q) {
          const int64_t n = nb + q * 32 + lane;
          sw_next[q] = n < p.N ? p.s_w[n] : 0.0f;
        }
        sp_next = p.s_act[g * p.S * 2 + 0];
        sm_next = p.s_act[g * p.S * 2 + 1];
      }
      const int units = SEGK ? p.S : 1;
      for (int u = 0; u < units; ++u) {
        float *cst = cst_base;
        if constexpr (SEGK && OUT != OUT_S32) {
          // Folded coefficients of K-segment u: c+- = s_w[u][n] * s+-[u], into
          // buffer u & 1 (the other buffer may still be read by segment u - 1
          // only in program order of this warp, so no wait is needed).
          const float sp = __fmul_rn(sp_next, p.act_mul);
          const float sm = __fmul_rn(sm_next, p.act_mul);
          cst = cst_base + (u & 1) * 2 * HALF;
#pragma unroll
          for (int q = 0; q < HALF / 32; ++q) {
            cst[q * 32 + lane] = sw_next[q] * sp;
            cst[HALF + q * 32 + lane] = sw_next[q] * sm;
          }
          if (u + 1 < units) {
            const float *swn = p.s_w + static_cast<int64_t>(u + 1) * p.N;
#pragma unroll
            for (int q = 0; q < HALF / 32; ++q) {
              const int64_t n = nb + q * 32 + lane;
              sw_next[q] = n < p.N ? swn[n] : 0.0f;
            }
            sp_next = p.s_act[(g * p.S + u + 1) * 2 + 0];
            sm_next = p.s_act[(g * p.S + u + 1) * 2 + 1];
          }
          __syncwarp();
        }
        const uint32_t buf = acc_iter % NBUF;
        if (!wait_bar(&acc_full[buf], (acc_iter / NBUF) & 1, abort_flag, p.status))
          goto epilogue_exit;
        tc_fence_after();
        const uint32_t t_plus = tmem_base + lane_addr + buf * ACC_COLS + half * HALF;
#pragma unroll
        for (int c = 0; c < ((SEGK && OUT != OUT_S32) ? 0 : HALF / CW); ++c) {
          const int64_t n0 = nb + c * CW;
          if constexpr (OUT == OUT_S32) {
            uint32_t ap[CW], am[CW];
            tmem_ld_cols<CW>(t_plus + c * CW, ap);
            if constexpr (POL == 2) tmem_ld_cols<CW>(t_plus + BN + c * CW, am);
            tmem_ld_wait();
            if (TAIL && role == PIECE_PARTIAL) {
              sk_store<CW>(p, slot_run(blockIdx.x, c, 0), 0, ap);
              if constexpr (POL == 2) sk_store<CW>(p, slot_run(blockIdx.x, c, 1), 0, am);
              continue;
            }
            if (TAIL && role == PIECE_FINAL)
              for (int cc = blockIdx.x + 1; cc <= sk_last; ++cc)
                if (pc.U * cc / pc.G != pc.U * (cc + 1) / pc.G) {
                  sk_add<CW, F8>(slot_run(cc, c, 0), 0, ap);
                  if constexpr (POL == 2) sk_add<CW, F8>(slot_run(cc, c, 1), 0, am);
                }
            if (m < p.M) {
              int32_t *accp = reinterpret_cast<int32_t *>(p.y) +
                              ((static_cast<int64_t>(u) * POL) * p.M + m) * p.N;
              int32_t *accm = accp + static_cast<int64_t>(p.M) * p.N;
#pragma unroll
              for (int j = 0; j < CW; ++j)
                // acc: [units][POL][M][N]
                if (n0 + j < p.N &&
                    store_ok(p.status, u < (SEGK ? p.S : 1) && m < p.M && n0 + j >= 0)) {
                  accp[n0 + j] = static_cast<int32_t>(ap[j]);
                  if constexpr (POL == 2) accm[n0 + j] = static_cast<int32_t>(am[j]);
                }
            }
          } else if constexpr (!SEGK) {
            // One K-segment, in the reference order: y = fma(c-, f(A-),
            // fl(c+ f(A+))) + bias with the folded c+- = fl(s_w s+-) staged per
            // column, or y = fl(c f(A)) + bias for a single scale; each step one
            // rounding, two columns per packed instruction.  The 32-column
            // chunk is read in the 16x256b pattern: thread t holds rows
            // 16k + 8h + t/4 (k, h < 2) and the column pairs 8j + 2 (t % 4)
            // (j < 4), so it reads 4 float2 of each constant, not 8 float4.
            static_assert(CW == 32, "32-column chunks");
            constexpr uint32_t kLanes16 = 16u << 16;
            uint32_t pl[16], ph[16], ml[POL == 2 ? 16 : 1], mh[POL == 2 ? 16 : 1];
            tmem_ld_16x256b_x4(t_plus + c * 32, pl);
            tmem_ld_16x256b_x4(t_plus + c * 32 + kLanes16, ph);
            if constexpr (POL == 2) {
              tmem_ld_16x256b_x4(t_plus + BN + c * 32, ml);
              tmem_ld_16x256b_x4(t_plus + BN + c * 32 + kLanes16, mh);
            }
            tmem_ld_wait();
            if (TAIL && role == PIECE_PARTIAL) {
              sk_store<16>(p, slot_run(blockIdx.x, c, 0), 0, pl);
              sk_store<16>(p, slot_run(blockIdx.x, c, 0), 4, ph);
              if constexpr (POL == 2) {
                sk_store<16>(p, slot_run(blockIdx.x, c, 1), 0, ml);
                sk_store<16>(p, slot_run(blockIdx.x, c, 1), 4, mh);
              }
              continue;
            }
            if (TAIL && role == PIECE_FINAL)
              for (int cc = blockIdx.x + 1; cc <= sk_last; ++cc)
                if (pc.U * cc / pc.G != pc.U * (cc + 1) / pc.G) {
                  sk_add<16, F8>(slot_run(cc, c, 0), 0, pl);
                  sk_add<16, F8>(slot_run(cc, c, 0), 4, ph);
                  if constexpr (POL == 2) {
                    sk_add<16, F8>(slot_run(cc, c, 1), 0, ml);
                    sk_add<16, F8>(slot_run(cc, c, 1), 4, mh);
                  }
                }
            const int q = lane & 3;
            const float *cpc = cst + c * 32 + 2 * q;
            const float *cmc = cst + HALF + c * 32 + 2 * q;
            const float *bc = cst + POL * HALF + c * 32 + 2 * q;
            const uint64_t zero2 = f2pack(0.0f, 0.0f), one2 = f2pack(1.0f, 1.0f);
            if constexpr (TMA_STORE) {
              if (lane == 0) bulk_wait_read_all();  // the previous chunk is out
              __syncwarp();
            }
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              const uint64_t cp = *reinterpret_cast<const uint64_t *>(cpc + 8 * j);
              const uint64_t b = *reinterpret_cast<const uint64_t *>(bc + 8 * j);
              uint64_t cm = 0;
              if constexpr (POL == 2) cm = *reinterpret_cast<const uint64_t *>(cmc + 8 * j);
#pragma unroll
              for (int k = 0; k < 2; ++k)
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                  const int r = 4 * j + 2 * h;
                  const uint32_t a0 = k ? ph[r] : pl[r], a1 = k ? ph[r + 1] : pl[r + 1];
                  uint64_t y = ffma2(cp, f2pack(acc_f32<F8>(a0), acc_f32<F8>(a1)), zero2);
                  if constexpr (POL == 2) {
                    const uint32_t b0 = k ? mh[r] : ml[r], b1 = k ? mh[r + 1] : ml[r + 1];
                    y = ffma2(cm, f2pack(acc_f32<F8>(b0), acc_f32<F8>(b1)), y);
                  }
                  y = ffma2(one2, y, b);
                  float y0, y1;
                  f2unpack(y, y0, y1);
                  const int rr = 16 * k + 8 * h + (lane >> 2);  // row within the warp's 32
                  if constexpr (OUT == OUT_PLANES) {
                    // Two 32 x 32-byte staging blocks (X^+ then X^-), row-major:
                    // columns 8j + 2q and 8j + 2q + 1 as one 16-bit store each.
                    int qp0, qm0, qp1, qm1;
                    gelu_codes(y0, sp_nx, rp_nx, sm_nx, rm_nx, qp0, qm0);
                    gelu_codes(y1, sp_nx, rp_nx, sm_nx, rm_nx, qp1, qm1);
                    uint16_t *dst = reinterpret_cast<uint16_t *>(stg + rr * 32 + 8 * j + 2 * q);
                    if (p.p_next == 2) {
                      dst[0] = static_cast<uint16_t>((qp0 & 0xFF) | ((qp1 & 0xFF) << 8));
                      dst[512] = static_cast<uint16_t>((qm0 & 0xFF) | ((qm1 & 0xFF) << 8));
                    } else {  // single scale: one merged plane (one code is 0)
                      dst[0] = static_cast<uint16_t>(((qp0 + qm0) & 0xFF) |
                                                     (((qp1 + qm1) & 0xFF) << 8));
                    }
                  } else if constexpr (TMA_STORE) {
                    // Staging buffer in the tensor map's 64-byte swizzle:
                    // 16-byte piece j of row rr sits at piece j ^ ((rr / 2) % 4),
                    // so the 8 rows x 16 bytes of one store instruction fall
                    // into 8 distinct bank groups.
                    *reinterpret_cast<uint32_t *>(stg + rr * 64 + ((j ^ ((rr >> 1) & 3)) << 4) +
                                                  4 * q) = pack_bf16x2(y0, y1);
                  } else {
                    const int64_t mr = static_cast<int64_t>(mt) * BM + quarter * 32 + rr;
                    if (mr < p.M) store_pair<OUT>(p, mr, n0 + 8 * j + 2 * q, y0, y1);
                  }
                }
            }
            if constexpr (TMA_STORE) {
              // The warp's 32 rows x 32 columns leave in one tensor store per
              // plane, which writes whole lines and drops rows >= M and
              // columns >= N.
              fence_proxy_async_smem();
              __syncwarp();
              const int row0 = mt * BM + quarter * 32;
              if (lane == 0 && row0 < p.M && n0 < p.N) {
                if constexpr (OUT == OUT_PLANES) {
                  for (int pl = 0; pl < p.p_next; ++pl)
                    tma_store_3d(&tmY, stg + pl * 1024, static_cast<int32_t>(n0), row0, pl);
                } else {
                  tma_store_2d(&tmY, stg, static_cast<int32_t>(n0), row0);
                }
                bulk_commit_group();
              }
            }
          }
        }
        if constexpr (SEGK && OUT != OUT_S32) {
          // Several K-segments: y = fma(c-, f(A-), fma(c+, f(A+), y)) from
          // y = 0, two columns per packed instruction; the bias is added at
          // the end.  The accumulators are read in the 16x256b pattern: a
          // thread holds rows t/4 + {0, 8, 16, 24} of the warp's 32 and
          // columns 8j + 2 (t % 4) + {0, 1}, j < 4, so it needs 8 of the 32
          // column coefficients per polarity (4 float2 reads instead of 8
          // float4), which keeps the shared-memory pipe off the critical path.
          // run2[8k + 2j + h] holds row 16k + 8h + t/4, column pair j.  The
          // warp folds in A+, copies A- into registers and hands the TMEM
          // buffer back before folding A- in, so that the MMAs of the segment
          // after next overlap the rest of this segment's arithmetic.
          static_assert(HALF == 32, "one 32-column TMEM block per polarity and warp");
          const int q2 = 2 * (lane & 3);
          const auto cvt2 = [](uint32_t x, uint32_t y) {
            return f2pack(acc_f32<F8>(x), acc_f32<F8>(y));
          };
          const auto fold = [&](const uint32_t(&lo)[16], const uint32_t(&hi)[16],
                                const float *c) {
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              const uint64_t cj = *reinterpret_cast<const uint64_t *>(c + 8 * j + q2);
#pragma unroll
              for (int h = 0; h < 2; ++h) {
                const int r = 4 * j + 2 * h;
                run2[2 * j + h] = ffma2(cj, cvt2(lo[r], lo[r + 1]), run2[2 * j + h]);
                run2[8 + 2 * j + h] = ffma2(cj, cvt2(hi[r], hi[r + 1]), run2[8 + 2 * j + h]);
              }
            }
          };
          constexpr uint32_t kLanes16 = 16u << 16;
          uint32_t lo[16], hi[16];
          tmem_ld_16x256b_x4(t_plus, lo);
          tmem_ld_16x256b_x4(t_plus + kLanes16, hi);
          tmem_ld_wait();
          if constexpr (POL == 2) {
            fold(lo, hi, cst);
            tmem_ld_16x256b_x4(t_plus + BN, lo);
            tmem_ld_16x256b_x4(t_plus + BN + kLanes16, hi);
            tmem_ld_wait();
          }
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&acc_empty[buf]);
          fold(lo, hi, POL == 2 ? cst + HALF : cst);
        } else {
          if (TAIL && role == PIECE_PARTIAL) {
            // every lane's partials are visible before the flag is raised
            __threadfence();
            __syncwarp();
            if (lane == 0 && store_ok(p.status, ew < EPI_WARPS))  // flags: [gridDim.x][EPI_WARPS]
              st_release(p.sk_flags + blockIdx.x * EPI_WARPS + ew, 1);
          }
          if (TAIL && role == PIECE_FINAL) {
            // consumed: leave the flags at zero for the next call
            __syncwarp();
            if (lane == 0)
              for (int cc = blockIdx.x + 1; cc <= sk_last; ++cc)
                if (pc.U * cc / pc.G != pc.U * (cc + 1) / pc.G)
                  if (store_ok(p.status, cc < static_cast<int>(gridDim.x)))
                    p.sk_flags[cc * EPI_WARPS + ew] = 0;
          }
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&acc_empty[buf]);
        }
        ++acc_iter;
      }
      if constexpr (SEGK && OUT != OUT_S32) {
        float *bst = cst_base + (units & 1) * 2 * HALF;  // buffer not read by the last segment
        for (int j = lane; j < HALF; j += 32) {
          const int64_t n = nb + j;
          bst[j] = (p.bias != nullptr && n < p.N) ? bf16_to_f32(p.bias[n]) : 0.0f;
        }
        __syncwarp();
        // Rows and columns in the 16x256b pattern of the drains: thread t
        // holds, for each of its 4 rows, column pairs 8j + 2q (q = t % 4).
        const int q = lane & 3;
#pragma unroll
        for (int k = 0; k < 2; ++k)
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const int64_t mr =
                static_cast<int64_t>(mt) * BM + quarter * 32 + 16 * k + 8 * h + (lane >> 2);
            float y[8];  // pairs j = 0..3
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              const float2 b = *reinterpret_cast<const float2 *>(bst + 8 * j + 2 * q);
              f2unpack(run2[8 * k + 2 * j + h], y[2 * j], y[2 * j + 1]);
              y[2 * j] = __fadd_rn(y[2 * j], b.x);
              y[2 * j + 1] = __fadd_rn(y[2 * j + 1], b.y);
            }
            if constexpr (OUT == OUT_BF16) {
              // The 4 lanes of a row exchange bf16 pairs (a 4 x 4 transpose in
              // two xor rounds) so that lane q ends with columns 8q .. 8q + 7
              // and writes them with one 16-byte store.
              uint32_t w[4];
#pragma unroll
              for (int j = 0; j < 4; ++j) w[j] = pack_bf16x2(y[2 * j], y[2 * j + 1]);
              {
                const bool up = q & 2;  // swap the off-diagonal 2 x 2 blocks
                const uint32_t s0 = __shfl_xor_sync(0xffffffffu, up ? w[0] : w[2], 2);
                const uint32_t s1 = __shfl_xor_sync(0xffffffffu, up ? w[1] : w[3], 2);
                if (up) { w[0] = s0; w[1] = s1; } else { w[2] = s0; w[3] = s1; }
              }
              {
                const bool odd = q & 1;  // transpose each 2 x 2 block
                const uint32_t s0 = __shfl_xor_sync(0xffffffffu, odd ? w[0] : w[1], 1);
                const uint32_t s1 = __shfl_xor_sync(0xffffffffu, odd ? w[2] : w[3], 1);
                if (odd) { w[0] = s0; w[2] = s1; } else { w[1] = s0; w[3] = s1; }
              }
              const int64_t n0 = nb + 8 * q;
              // y: [M][ldy], columns < N <= ldy
              if (mr < p.M && n0 < p.N && store_ok(p.status, mr >= 0 && n0 >= 0 && n0 < p.ldy)) {
                uint16_t *row = reinterpret_cast<uint16_t *>(p.y) + mr * p.ldy;
                if (n0 + 8 <= p.N) {
                  *reinterpret_cast<uint4 *>(row + n0) = make_uint4(w[0], w[1], w[2], w[3]);
                } else {
#pragma unroll
                  for (int e = 0; e < 8; ++e)
                    if (n0 + e < p.N)
                      row[n0 + e] = static_cast<uint16_t>(w[e >> 1] >> (16 * (e & 1)));
                }
              }
            } else if (mr < p.M) {
#pragma unroll
              for (int j = 0; j < 4; ++j)
                store_pair<OUT>(p, mr, nb + 8 * j + 2 * q, y[2 * j], y[2 * j + 1]);
            }
          }
        __syncwarp();
      }
    }
  epilogue_exit:
    if constexpr (TMA_STORE) {
      if (lane == 0) bulk_wait_all();  // every tensor store of this warp is complete
      __syncwarp();
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, 512);
  }
}

// ------------------------------------------------------------------ host side
int device_sm_count() {
  int dev = 0, sms = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  return sms > 0 ? sms : 148;
}

template <int BN, int STAGES, int OUT, bool SEGK, int EPI_WARPS, int POL, bool F8>
sq_status run_gemm(const GemmRequest &r, const GemmParams &p, cudaStream_t stream) {
  using L = Smem<BN, STAGES, EPI_WARPS, POL, SEGK, (OUT == OUT_BF16 || OUT == OUT_PLANES) && !SEGK>;
  EncodeTiledFn enc = tensor_map_encoder();
  if (enc == nullptr) return SQ_ERR_CUDA;
  const int G = r.seg.G;
  CUtensorMap tmA, tmB;
  {
    // planes viewed as 3D: x = K (bytes), y = M rows, z = POL * G planes.
    const cuuint64_t dims[3] = {static_cast<cuuint64_t>(r.K), static_cast<cuuint64_t>(r.M),
                                static_cast<cuuint64_t>(POL * G)};
    const cuuint64_t strides[2] = {static_cast<cuuint64_t>(r.K),
                                   static_cast<cuuint64_t>(r.K) * static_cast<cuuint64_t>(r.M)};
    const cuuint32_t box[3] = {BK, BM, POL};
    const cuuint32_t estr[3] = {1, 1, 1};
    if (enc(&tmA, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<int8_t *>(r.planes), dims, strides,
            box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return SQ_ERR_CUDA;
  }
  {
    const cuuint64_t dims[2] = {static_cast<cuuint64_t>(r.K), static_cast<cuuint64_t>(r.N)};
    const cuuint64_t strides[1] = {static_cast<cuuint64_t>(r.K)};
    const cuuint32_t box[2] = {BK, BN};
    const cuuint32_t estr[2] = {1, 1};
    if (enc(&tmB, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<int8_t *>(r.wq), dims, strides,
            box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return SQ_ERR_CUDA;
  }
  CUtensorMap tmY;
  memset(&tmY, 0, sizeof tmY);
  if (OUT == OUT_PLANES) {
    // The next layer's planes as 3D int8: x = N columns, y = M rows, z = plane;
    // 32 x 32 boxes, one plane each.
    const cuuint64_t dims[3] = {static_cast<cuuint64_t>(r.N), static_cast<cuuint64_t>(r.M),
                                static_cast<cuuint64_t>(r.p_next)};
    const cuuint64_t strides[2] = {static_cast<cuuint64_t>(r.N),
                                   static_cast<cuuint64_t>(r.N) * static_cast<cuuint64_t>(r.M)};
    const cuuint32_t box[3] = {32, 32, 1};
    const cuuint32_t estr[3] = {1, 1, 1};
    if (enc(&tmY, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, r.y, dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
            CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return SQ_ERR_CUDA;
  }
  if (OUT == OUT_BF16 && !SEGK) {
    // Y viewed as 2D bf16: x = N columns, y = M rows; 32 x 32 boxes.
    const cuuint64_t dims[2] = {static_cast<cuuint64_t>(r.N), static_cast<cuuint64_t>(r.M)};
    const cuuint64_t strides[1] = {static_cast<cuuint64_t>(r.ldy) * 2};
    const cuuint32_t box[2] = {32, 32};
    const cuuint32_t estr[2] = {1, 1};
    if (enc(&tmY, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, r.y, dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B,
            CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return SQ_ERR_CUDA;
  }
  static_assert(L::BYTES <= 232448, "dynamic shared memory above the per-block limit");
  // Split tail of the last wave (one-segment layers, plain outputs): with a
  // workspace large enough, all SMs take a CTA and the k-blocks of the last,
  // partial wave's tiles are shared out evenly among them.
  GemmParams q = p;
  q.sk_W = q.sk_R = 0;
  q.sk_ws = nullptr;
  q.sk_flags = nullptr;
  q.sk_slot_words = 0;
  const int sms = device_sm_count();
  int grid = p.num_tiles < sms ? p.num_tiles : sms;
  if constexpr (!SEGK && OUT != OUT_PLANES) {
    const int64_t slot_words = static_cast<int64_t>(EPI_WARPS) * (L::COLS / 32) * POL * 1024;
    const size_t need = ((static_cast<size_t>(sms) * EPI_WARPS + 63) / 64) * 64 * 4 +
                        static_cast<size_t>(sms) * slot_words * 4;
    if (r.workspace != nullptr && r.workspace_bytes >= need && p.num_tiles > sms &&
        p.num_tiles % sms != 0) {
      q.sk_W = p.num_tiles / sms;
      q.sk_R = p.num_tiles % sms;
      q.sk_flags = static_cast<int32_t *>(r.workspace);
      q.sk_ws = q.sk_flags + ((static_cast<int64_t>(sms) * EPI_WARPS + 63) / 64) * 64;
      q.sk_slot_words = slot_words;
      grid = sms;
    }
  }
  auto kernel = dualscale_gemm_kernel<BN, STAGES, OUT, SEGK, EPI_WARPS, POL, F8>;
  static bool attr_set[64] = {};  // per instantiation and device
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) return SQ_ERR_CUDA;
  if (!attr_set[dev]) {
    if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, L::BYTES) !=
        cudaSuccess)
      return SQ_ERR_CUDA;
    attr_set[dev] = true;
  }
  // Programmatic dependent launch: CTAs may run their prologue (barriers,
  // TMEM allocation) while the preceding kernel finishes.
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(threads_for(EPI_WARPS));
  cfg.dynamicSmemBytes = L::BYTES;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, kernel, tmA, tmB, tmY, q) != cudaSuccess) return SQ_ERR_CUDA;
  return cudaGetLastError() == cudaSuccess ? SQ_OK : SQ_ERR_CUDA;
}

// Tile configurations.  DualScale, one segment: 128 x 256 tiles, the + and -
// accumulators fill TMEM (3 stages).  Single scale, one segment: 128 x 256
// tiles with two TMEM buffers (4 stages).  Input-segmented: 128 x 128 tiles
// with two TMEM buffers and 16 epilogue warps for the per-segment drains, which
// bound that path (int32 -> fp32 conversion and FMA per element and segment);
// narrower tiles give more buffers but cost more than they save (measured).
constexpr int kSegBN = 128;  // tile width of the input-segmented path

template <int OUT, int POL, bool F8>
sq_status dispatch(const GemmRequest &r, const GemmParams &p, bool segk, int BN,
                   cudaStream_t stream) {
  if constexpr (OUT == OUT_PLANES) {
    // one K-segment, one group (checked by the caller)
    return run_gemm<256, POL == 2 ? 3 : 4, OUT, false, 8, POL, false>(r, p, stream);
  } else {
  if (segk) return run_gemm<kSegBN, 4, OUT, true, 16, POL, F8>(r, p, stream);
  if (BN == 256) return run_gemm<256, POL == 2 ? 3 : 4, OUT, false, 8, POL, F8>(r, p, stream);
  return run_gemm<128, 4, OUT, false, 8, POL, F8>(r, p, stream);
  }
}

template <int OUT, int POL>
sq_status dispatch_kind(const GemmRequest &r, const GemmParams &p, bool segk, int BN,
                        cudaStream_t stream) {
  if constexpr (OUT == OUT_PLANES) return dispatch<OUT, POL, false>(r, p, segk, BN, stream);
  return r.seg.fp8 ? dispatch<OUT, POL, true>(r, p, segk, BN, stream)
                   : dispatch<OUT, POL, false>(r, p, segk, BN, stream);
}

}  // namespace

size_t gemm_workspace_bytes() {
  // flags (rounded up to 64 words) and one slot of partial sums per SM, for
  // the widest configuration: 8 epilogue warps x 128 columns x 2 planes
  const size_t sms = static_cast<size_t>(device_sm_count());
  return ((sms * 8 + 63) / 64) * 64 * 4 + sms * (8 * 4 * 2 * 1024 * 4);
}

sq_status launch_gemm(const GemmRequest &r, cudaStream_t stream) {
  if (r.M == 0) return SQ_OK;
  const bool segk = r.seg.mode == SQ_SEG_INPUT && r.seg.S > 1;
  int BN = segk ? kSegBN : SQ_GEMM_BN_ONE_SEG;
  if (r.seg.G > 1) {
    for (int j = 0; j < r.seg.n_seg; ++j)
      if ((r.seg.off[j + 1] - r.seg.off[j]) % 256 != 0) BN = 128;
  }
  // A layer with at most half as many 256-wide tiles as SMs (a few rows) is
  // bound by streaming its weights, not by the MMAs: 128-wide tiles put twice
  // as many SMs on that stream.  Measured: 256 x 1536 x 1536 GEMM 18.0 ->
  // 16.0 us, two rows x 3072 -> 18432 in six groups 27.0 -> 23.2 us; but with
  // one row tile and one activation group (every CTA reading the same two
  // activation rows) 26.8 -> 29.2 us, so that case keeps 256-wide tiles.
  const int64_t m_tiles = (r.M + BM - 1) / BM;
  if (!segk && BN == 256 && r.out_kind != OUT_PLANES && (m_tiles > 1 || r.seg.G > 1) &&
      2 * m_tiles * ((r.N + 255) / 256) <= device_sm_count())
    BN = 128;
  GemmParams p;
  p.M = static_cast<int32_t>(r.M);
  p.N = static_cast<int32_t>(r.N);
  p.K = static_cast<int32_t>(r.K);
  p.num_n_tiles = static_cast<int32_t>((r.N + BN - 1) / BN);
  const int32_t num_m_tiles = static_cast<int32_t>((r.M + BM - 1) / BM);
  p.num_tiles = num_m_tiles * p.num_n_tiles;
  p.num_kb = static_cast<int32_t>((r.K + BK - 1) / BK);
  p.G = r.seg.G;
  p.S = r.seg.S;
  p.n_seg_out = (r.seg.mode == SQ_SEG_OUTPUT) ? r.seg.n_seg : 1;
  for (int i = 0; i <= SQ_MAX_SEGMENTS; ++i) {
    p.k_off[i] = 0;
    p.n_off[i] = 0;
  }
  if (r.seg.mode == SQ_SEG_INPUT) {
    for (int i = 0; i <= r.seg.n_seg; ++i) p.k_off[i] = r.seg.off[i];
  } else {
    p.k_off[0] = 0;
    p.k_off[1] = p.K;
  }
  if (r.seg.mode == SQ_SEG_OUTPUT)
    for (int i = 0; i <= r.seg.n_seg; ++i) p.n_off[i] = r.seg.off[i];
  p.s_w = r.s_w;
  p.s_act = r.s_act;
  p.act_mul = r.seg.w4 ? 0.0625f : 1.0f;
  p.bias = r.bias;
  p.y = r.y;
  p.ldy = r.ldy;
  p.status = r.status;
  p.s_next = r.s_next;
  p.p_next = r.p_next;

  if (r.seg.P == 1) {
    switch (r.out_kind) {
      case OUT_S32: return dispatch_kind<OUT_S32, 1>(r, p, segk, BN, stream);
      case OUT_F32: return dispatch_kind<OUT_F32, 1>(r, p, segk, BN, stream);
      case OUT_PLANES: return dispatch_kind<OUT_PLANES, 1>(r, p, segk, BN, stream);
      default: return dispatch_kind<OUT_BF16, 1>(r, p, segk, BN, stream);
    }
  }
  switch (r.out_kind) {
    case OUT_S32: return dispatch_kind<OUT_S32, 2>(r, p, segk, BN, stream);
    case OUT_F32: return dispatch_kind<OUT_F32, 2>(r, p, segk, BN, stream);
    case OUT_PLANES: return dispatch_kind<OUT_PLANES, 2>(r, p, segk, BN, stream);
    default: return dispatch_kind<OUT_BF16, 2>(r, p, segk, BN, stream);
  }
}

}  // namespace sq
