// quant.cu -- the element-wise, HBM-bound kernels of the SegQuant path:
//  * DualScale activation quantization (Q_dual on X / d, two int8 planes per
//    activation group) -- "SegQuant" author page, section 3; papernotes.org
//    "SegQuant", section DualScale;
//  * static AMax calibration of s+ / s- (same section; AMax calibrator);
//  * segment-wise symmetric AMax weight quantization (section SegLinear).
// Every fp32 operation that decides an integer code is written with an explicit
// round-to-nearest intrinsic so that no contraction or approximation changes it.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "sq_internal.h"

namespace sq {
namespace {

constexpr int kColsPerThread = 8;                     // one 16-byte bf16 load
constexpr int kWarpCols = 32 * kColsPerThread;        // 256 channels per warp row
constexpr int kRowsPerBlock = 8;                      // warps per block
constexpr int kUnroll = 3;                            // rows in flight per thread

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
                                                           SegParams seg, float *s_act) {
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
  if ((threadIdx.x & 31) == __ffs(group) - 1) {
    unsigned int *slot = reinterpret_cast<unsigned int *>(s_act + (g * seg.S + i) * 2);
    if (hib) atomicMax(slot, hib);
    if (nlob) atomicMax(slot + 1, nlob);
  }
}

// Pass 2: s+ = max / 127, s- = |min| / 128; an empty side gets step 1.
__global__ void calib_finalize_kernel(float *s_act, int n) {
  for (int t = threadIdx.x; t < n; t += blockDim.x) {
    const float hi = s_act[2 * t], nlo = s_act[2 * t + 1];
    s_act[2 * t] = hi > 0.0f ? __fdiv_rn(hi, 127.0f) : 1.0f;
    s_act[2 * t + 1] = nlo > 0.0f ? __fdiv_rn(nlo, 128.0f) : 1.0f;
  }
}

// ---------------------------------------------------- activation quantize
// q = rne(v) saturated to [-128, 127] (cvt.rni.sat.s8.f32; NaN gives 0).
__device__ __forceinline__ uint32_t f2s8_rn_sat(float v) {
  uint32_t r;
  asm("cvt.rni.sat.s8.f32 %0, %1;" : "=r"(r) : "f"(v));
  return r;
}

// Packs the low bytes of four codes into one word (byte j = code j).
__device__ __forceinline__ uint32_t pack4(uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  return __byte_perm(__byte_perm(a, b, 0x0040), __byte_perm(c, d, 0x0040), 0x5410);
}

// Eight channels x of one row -> X^+ and X^- codes, 8 bytes each.  One signed
// code per element, q = sat(rne(x * (x >= 0 ? m+ : m-))): its sign is the
// sign of x, so X^+ = max(q, 0) and X^- = min(q, 0) byte-wise.  This is the
// case-wise Q_dual with the clamps of the reference: x >= 0 (including -0.0)
// gives a code in [0, 127], x < 0 a code in [-128, 0], NaN gives 0 in both.
__device__ __forceinline__ void dualscale8(const float (&x)[8], const float (&mp)[8],
                                           const float (&mm)[8], uint2 &plus, uint2 &minus) {
  uint32_t q[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) q[j] = f2s8_rn_sat(__fmul_rn(x[j], x[j] >= 0.0f ? mp[j] : mm[j]));
  const uint32_t w0 = pack4(q[0], q[1], q[2], q[3]);
  const uint32_t w1 = pack4(q[4], q[5], q[6], q[7]);
  plus = make_uint2(__vmaxs4(w0, 0u), __vmaxs4(w1, 0u));
  minus = make_uint2(__vmins4(w0, 0u), __vmins4(w1, 0u));
}

// Block: 32 x 8 threads.  blockIdx.x owns 256 consecutive channels; every
// warp streams whole rows of them (512 contiguous bytes per row), kUnroll rows
// in flight per thread.  With one activation group the folded multipliers
// m+- = 1/(d*s+-) of the thread's eight channels live in registers; with G
// groups they sit in shared memory, [G][2][256] floats.
template <bool kOneGroup>
__global__ void __launch_bounds__(256, 4) quant_act_kernel(const uint16_t *__restrict__ x,
                                                        int64_t M, int64_t K, int64_t ldx,
                                                        const float *__restrict__ d,
                                                        const float *__restrict__ s_act,
                                                        SegParams seg,
                                                        int8_t *__restrict__ planes) {
  extern __shared__ float mtab[];  // [G][2][kWarpCols] when G > 1
  const int G = kOneGroup ? 1 : seg.G;
  const int64_t cblk = static_cast<int64_t>(blockIdx.x) * kWarpCols;
  const int64_t c0 = cblk + threadIdx.x * kColsPerThread;
  float mp_r[8], mm_r[8];
  if (kOneGroup) {
    if (c0 < K) {
      const int i = (seg.mode == SQ_SEG_INPUT) ? seg_index(seg.off, seg.n_seg, c0) : 0;
      const float sp = s_act[i * 2 + 0], sm = s_act[i * 2 + 1];
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const float dv = d ? d[c0 + j] : 1.0f;
        mp_r[j] = __fdiv_rn(1.0f, __fmul_rn(dv, sp));
        mm_r[j] = __fdiv_rn(1.0f, __fmul_rn(dv, sm));
      }
    }
  } else {
    const int tid = threadIdx.y * 32 + threadIdx.x;
    for (int t = tid; t < G * kWarpCols; t += 256) {
      const int g = t / kWarpCols, cl = t % kWarpCols;
      const int64_t c = cblk + cl;
      float mp = 0.0f, mm = 0.0f;
      if (c < K) {
        const int i = (seg.mode == SQ_SEG_INPUT) ? seg_index(seg.off, seg.n_seg, c) : 0;
        const float dv = d ? d[g * K + c] : 1.0f;
        mp = __fdiv_rn(1.0f, __fmul_rn(dv, s_act[(g * seg.S + i) * 2 + 0]));
        mm = __fdiv_rn(1.0f, __fmul_rn(dv, s_act[(g * seg.S + i) * 2 + 1]));
      }
      mtab[(g * 2 + 0) * kWarpCols + cl] = mp;
      mtab[(g * 2 + 1) * kWarpCols + cl] = mm;
    }
    __syncthreads();
  }
  if (c0 >= K) return;
  const int64_t plane_stride = M * K;
  const int64_t row_step = static_cast<int64_t>(gridDim.y) * kRowsPerBlock * kUnroll;
  for (int64_t base = static_cast<int64_t>(blockIdx.y) * kRowsPerBlock * kUnroll + threadIdx.y;
       base < M; base += row_step) {
    uint4 v[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int64_t r = base + u * kRowsPerBlock;
      if (r < M) v[u] = __ldcs(reinterpret_cast<const uint4 *>(x + r * ldx + c0));
    }
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int64_t r = base + u * kRowsPerBlock;
      if (r >= M) break;
      float xv[8];
      unpack8(v[u], xv);
      for (int g = 0; g < G; ++g) {
        if (!kOneGroup) {
          const float4 *mp4 = reinterpret_cast<const float4 *>(
              mtab + (g * 2 + 0) * kWarpCols + threadIdx.x * kColsPerThread);
          const float4 *mm4 = reinterpret_cast<const float4 *>(
              mtab + (g * 2 + 1) * kWarpCols + threadIdx.x * kColsPerThread);
          const float4 a = mp4[0], b = mp4[1], c = mm4[0], e = mm4[1];
          mp_r[0] = a.x; mp_r[1] = a.y; mp_r[2] = a.z; mp_r[3] = a.w;
          mp_r[4] = b.x; mp_r[5] = b.y; mp_r[6] = b.z; mp_r[7] = b.w;
          mm_r[0] = c.x; mm_r[1] = c.y; mm_r[2] = c.z; mm_r[3] = c.w;
          mm_r[4] = e.x; mm_r[5] = e.y; mm_r[6] = e.z; mm_r[7] = e.w;
        }
        uint2 pk, nk;
        dualscale8(xv, mp_r, mm_r, pk, nk);
        int8_t *dst = planes + (static_cast<int64_t>(g) * 2) * plane_stride + r * K + c0;
        __stcs(reinterpret_cast<uint2 *>(dst), pk);
        __stcs(reinterpret_cast<uint2 *>(dst + plane_stride), nk);
      }
    }
  }
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

__global__ void __launch_bounds__(256) quant_weight_kernel(const uint16_t *__restrict__ w,
                                                           int64_t N, int64_t K,
                                                           const float *__restrict__ d,
                                                           SegParams seg,
                                                           int8_t *__restrict__ wq,
                                                           float *__restrict__ s_w) {
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
    const float s = amax > 0.0f ? __fdiv_rn(amax, 127.0f) : 1.0f;
    if (threadIdx.x == 0) s_w[i * N + n] = s;
    for (int64_t k = k0 + threadIdx.x; k < k1; k += blockDim.x) {
      const float wv = dg ? __fmul_rn(bf16_bits_to_f32(row[k]), dg[k]) : bf16_bits_to_f32(row[k]);
      const float v = fminf(fmaxf(__fdiv_rn(wv, s), -127.0f), 127.0f);
      wq[n * K + k] = static_cast<int8_t>(__float2int_rn(v));
    }
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
                                 cudaStream_t stream) {
  const int n = seg.G * seg.S;
  cudaError_t e = cudaMemsetAsync(s_act, 0, sizeof(float) * 2 * n, stream);
  if (e != cudaSuccess) return e;
  if (M > 0) {
    const int gx = static_cast<int>((K + kWarpCols - 1) / kWarpCols);
    int gy = static_cast<int>((M + kRowsPerBlock - 1) / kRowsPerBlock);
    const int cap = (num_sms() * 4 + gx * seg.G - 1) / (gx * seg.G);
    if (gy > cap) gy = cap < 1 ? 1 : cap;
    calib_reduce_kernel<<<dim3(gx, gy, seg.G), dim3(32, kRowsPerBlock), 0, stream>>>(
        x, M, K, ldx, d, seg, s_act);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  calib_finalize_kernel<<<1, 256, 0, stream>>>(s_act, n);
  return cudaGetLastError();
}

cudaError_t launch_quantize_act(const uint16_t *x, int64_t M, int64_t K, int64_t ldx,
                                const float *d, const float *s_act, const SegParams &seg,
                                int8_t *planes, cudaStream_t stream) {
  if (M == 0) return cudaSuccess;
  const int gx = static_cast<int>((K + kWarpCols - 1) / kWarpCols);
  const int64_t row_groups = (M + kRowsPerBlock * kUnroll - 1) / (kRowsPerBlock * kUnroll);
  // 8 resident blocks of 256 threads per SM fill its 2048 thread slots.
  int64_t gy = (static_cast<int64_t>(num_sms()) * 8 + gx - 1) / gx;
  if (gy > row_groups) gy = row_groups;
  if (gy < 1) gy = 1;
  const dim3 grid(gx, static_cast<unsigned>(gy)), block(32, kRowsPerBlock);
  if (seg.G == 1) {
    quant_act_kernel<true><<<grid, block, 0, stream>>>(x, M, K, ldx, d, s_act, seg, planes);
    return cudaGetLastError();
  }
  const size_t smem = sizeof(float) * 2 * kWarpCols * seg.G;
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(quant_act_kernel<false>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
  }
  quant_act_kernel<false><<<grid, block, smem, stream>>>(x, M, K, ldx, d, s_act, seg, planes);
  return cudaGetLastError();
}

cudaError_t launch_quantize_weight(const uint16_t *w, int64_t N, int64_t K, const float *d,
                                   const SegParams &seg, int8_t *wq, float *s_w,
                                   cudaStream_t stream) {
  if (N == 0) return cudaSuccess;
  quant_weight_kernel<<<static_cast<unsigned>(N), 256, 0, stream>>>(w, N, K, d, seg, wq, s_w);
  return cudaGetLastError();
}

}  // namespace sq
