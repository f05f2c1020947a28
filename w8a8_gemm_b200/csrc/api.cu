// api.cu -- the C ABI declared in include/segquant.h: argument validation on
// the host, the device error word, and dispatch to the kernels.  Nothing here
// allocates device memory.
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>

#include "sq_internal.h"

namespace sq {
namespace {

// Error word written by kernels whose bounded waits ran out.
__device__ int g_device_status = 0;

constexpr int64_t kMaxSegWidth = 132104;   // 128 * 127 * 132104 < 2^31
constexpr int kMaxDevices = 64;

bool aligned(const void *p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// Current device must be sm_100 (the kernels are built for sm_100a only).
sq_status check_device() {
  static int checked[kMaxDevices] = {};  // 0 unknown, 1 ok, -1 unsupported
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    cudaGetLastError();
    return SQ_ERR_NO_DEVICE;
  }
  if (checked[dev] == 0) {
    int major = 0, minor = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess) {
      cudaGetLastError();
      return SQ_ERR_NO_DEVICE;
    }
    checked[dev] = (major == 10 && minor == 0) ? 1 : -1;
  }
  return checked[dev] == 1 ? SQ_OK : SQ_ERR_NO_DEVICE;
}

// Validates a segment table.  extent_n < 0 means N is not known to the call
// (activation-side calls), in which case the output offsets end is not checked.
sq_status parse_segments(const sq_segments *seg, int64_t K, int64_t extent_n, SegParams *out) {
  SegParams p{};
  if (seg == nullptr) {
    p.mode = SQ_SEG_NONE;
    p.n_seg = 1;
    p.G = 1;
    p.S = 1;
    p.P = 2;
    p.off[0] = 0;
    p.off[1] = static_cast<int32_t>(K);
    *out = p;
    return SQ_OK;
  }
  if (seg->mode < SQ_SEG_NONE || seg->mode > SQ_SEG_INPUT) return SQ_ERR_INVALID_ARG;
  if (seg->n_seg < 1 || seg->n_seg > SQ_MAX_SEGMENTS || seg->n_groups < 1)
    return SQ_ERR_INVALID_ARG;
  if ((seg->flags & ~(SQ_FLAG_SINGLE_SCALE | SQ_FLAG_W4 | SQ_FLAG_FP8)) != 0)
    return SQ_ERR_INVALID_ARG;
  if ((seg->flags & SQ_FLAG_W4) && (seg->flags & SQ_FLAG_FP8)) return SQ_ERR_INVALID_ARG;
  p.P = (seg->flags & SQ_FLAG_SINGLE_SCALE) ? 1 : 2;
  p.w4 = (seg->flags & SQ_FLAG_W4) ? 1 : 0;
  p.fp8 = (seg->flags & SQ_FLAG_FP8) ? 1 : 0;
  p.mode = seg->mode;
  p.n_seg = seg->n_seg;
  p.G = seg->n_groups;
  if (seg->mode == SQ_SEG_NONE) {
    if (seg->n_seg != 1 || seg->n_groups != 1) return SQ_ERR_INVALID_ARG;
    p.S = 1;
    p.off[0] = 0;
    p.off[1] = static_cast<int32_t>(K);
    *out = p;
    return SQ_OK;
  }
  if (seg->offsets == nullptr || seg->offsets[0] != 0) return SQ_ERR_INVALID_ARG;
  for (int i = 0; i < seg->n_seg; ++i) {
    if (seg->offsets[i + 1] <= seg->offsets[i]) return SQ_ERR_INVALID_ARG;
    p.off[i] = seg->offsets[i];
  }
  p.off[seg->n_seg] = seg->offsets[seg->n_seg];
  if (seg->mode == SQ_SEG_INPUT) {
    if (seg->n_groups != 1) return SQ_ERR_INVALID_ARG;
    if (p.off[p.n_seg] != K) return SQ_ERR_INVALID_ARG;
    for (int i = 0; i < p.n_seg; ++i) {
      const int64_t w = p.off[i + 1] - p.off[i];
      if (w % 32 != 0) return SQ_ERR_UNSUPPORTED;
      if (w > kMaxSegWidth) return SQ_ERR_OVERFLOW;
    }
    p.S = p.n_seg;
  } else {
    if (seg->n_groups != 1 && seg->n_groups != seg->n_seg) return SQ_ERR_INVALID_ARG;
    if (extent_n >= 0 && p.off[p.n_seg] != extent_n) return SQ_ERR_INVALID_ARG;
    if (seg->n_groups > 1)
      for (int i = 0; i < p.n_seg; ++i)
        if ((p.off[i + 1] - p.off[i]) % 128 != 0) return SQ_ERR_UNSUPPORTED;
    p.S = 1;
  }
  *out = p;
  return SQ_OK;
}

sq_status check_k(int64_t K) {
  if (K < 16 || K % 16 != 0 || K > INT32_MAX) return SQ_ERR_INVALID_ARG;
  return SQ_OK;
}

sq_status check_act(const void *x, int64_t M, int64_t K, int64_t ldx) {
  if (M < 0 || M > INT32_MAX) return SQ_ERR_INVALID_ARG;
  sq_status st = check_k(K);
  if (st != SQ_OK) return st;
  if (ldx < K) return SQ_ERR_INVALID_ARG;
  // More than 2^44 input elements fit no device; the bound keeps the
  // quantizer's work-unit arithmetic far inside int64.
  if (M > 0 && ldx > (int64_t(1) << 44) / M) return SQ_ERR_INVALID_ARG;
  if (M > 0 && x == nullptr) return SQ_ERR_INVALID_ARG;
  if (ldx % 8 != 0 || !aligned(x, 16)) return SQ_ERR_ALIGNMENT;
  return SQ_OK;
}

sq_status from_cuda(cudaError_t e) { return e == cudaSuccess ? SQ_OK : SQ_ERR_CUDA; }

#define SQ_TRY(expr)               \
  do {                             \
    const sq_status _s = (expr);   \
    if (_s != SQ_OK) return _s;    \
  } while (0)

sq_status gemm_common(const int8_t *planes, const int8_t *wq, const float *s_w,
                      const float *s_act, const void *bias, void *y, int out_kind, int64_t M,
                      int64_t N, int64_t K, int64_t ldy, const sq_segments *seg,
                      cudaStream_t stream, bool launch = true, const float *s_next = nullptr,
                      int p_next = 0, void *workspace = nullptr, size_t workspace_bytes = 0) {
  if (M < 0 || M > INT32_MAX || N < 1 || N > INT32_MAX) return SQ_ERR_INVALID_ARG;
  // An output of more than 2^44 elements fits no device; the bound keeps the
  // kernel's tile count (at most 2^30 tiles of 128 x 128) inside int32.
  if (M * N > (int64_t(1) << 44)) return SQ_ERR_INVALID_ARG;
  SQ_TRY(check_k(K));
  SegParams sp;
  SQ_TRY(parse_segments(seg, K, N, &sp));
  if (sp.S == 1 && K > kMaxSegWidth) return SQ_ERR_OVERFLOW;
  if (M == 0) return SQ_OK;
  if (planes == nullptr || wq == nullptr || y == nullptr) return SQ_ERR_INVALID_ARG;
  if (out_kind != OUT_S32 && (s_w == nullptr || s_act == nullptr)) return SQ_ERR_INVALID_ARG;
  if (!aligned(planes, 16) || !aligned(wq, 16) || !aligned(y, 16)) return SQ_ERR_ALIGNMENT;
  if (s_w && !aligned(s_w, 4)) return SQ_ERR_ALIGNMENT;
  if (s_act && !aligned(s_act, 4)) return SQ_ERR_ALIGNMENT;
  if (bias && !aligned(bias, 2)) return SQ_ERR_ALIGNMENT;
  if (out_kind == OUT_PLANES) {
    // the fused producer: this layer one K-segment and one group, int8 codes;
    // the next layer's planes [p_next][M][N] (N is its K)
    if (sp.mode != SQ_SEG_NONE || sp.fp8) return SQ_ERR_UNSUPPORTED;
    if (s_next == nullptr || (p_next != 1 && p_next != 2) || ldy != N)
      return SQ_ERR_INVALID_ARG;
    if (!aligned(s_next, 4) || N % 16 != 0) return SQ_ERR_ALIGNMENT;
  } else if (out_kind != OUT_S32) {
    const int64_t elem = (out_kind == OUT_BF16) ? 2 : 4;
    if (ldy < N) return SQ_ERR_INVALID_ARG;
    if ((ldy * elem) % 16 != 0) return SQ_ERR_ALIGNMENT;
  }
  if (workspace != nullptr && !aligned(workspace, 256)) return SQ_ERR_ALIGNMENT;
  SQ_TRY(check_device());
  if (!launch) return SQ_OK;
  GemmRequest r;
  r.planes = planes;
  r.wq = wq;
  r.s_w = s_w;
  r.s_act = s_act;
  r.bias = static_cast<const uint16_t *>(bias);
  r.y = y;
  r.ldy = ldy;
  r.out_kind = out_kind;
  r.M = M;
  r.N = N;
  r.K = K;
  r.seg = sp;
  r.s_next = s_next;
  r.p_next = p_next;
  r.workspace = workspace;
  r.workspace_bytes = workspace_bytes;
  r.status = device_status_word();
  if (r.status == nullptr) return SQ_ERR_CUDA;
  return launch_gemm(r, stream);
}

sq_status quantize_common(const void *x, int64_t M, int64_t K, int64_t ldx, const float *d,
                          const float *s_act, const sq_segments *seg, int8_t *planes,
                          cudaStream_t stream, bool launch = true,
                          const uint32_t *plan = nullptr) {
  SQ_TRY(check_act(x, M, K, ldx));
  SegParams sp;
  SQ_TRY(parse_segments(seg, K, -1, &sp));
  if (plan != nullptr && d == nullptr) return SQ_ERR_INVALID_ARG;  // a plan is per divisor
  if (plan != nullptr && sp.fp8) return SQ_ERR_UNSUPPORTED;      // it covers int8 codes
  if (M == 0) return SQ_OK;
  if (s_act == nullptr || planes == nullptr) return SQ_ERR_INVALID_ARG;
  if (!aligned(s_act, 4) || (d && !aligned(d, 4)) || !aligned(planes, 16) ||
      (plan && !aligned(plan, 4)))
    return SQ_ERR_ALIGNMENT;
  SQ_TRY(check_device());
  if (!launch) return SQ_OK;
  int *status = device_status_word();
  if (status == nullptr) return SQ_ERR_CUDA;
  return launch_quantize_act(static_cast<const uint16_t *>(x), M, K, ldx, d, s_act, sp, planes,
                             plan, status, stream);
}

}  // namespace

sq_status validate_quantize_act(const void *x, int64_t M, int64_t K, int64_t ldx, const float *d,
                                const float *s_act, const sq_segments *seg, int8_t *planes) {
  return quantize_common(x, M, K, ldx, d, s_act, seg, planes, nullptr, false);
}

sq_status validate_gemm(const int8_t *planes, const int8_t *wq, const float *s_w,
                        const float *s_act, const void *bias, void *y, int out_kind, int64_t M,
                        int64_t N, int64_t K, int64_t ldy, const sq_segments *seg) {
  return gemm_common(planes, wq, s_w, s_act, bias, y, out_kind, M, N, K, ldy, seg, nullptr,
                     false);
}

EncodeTiledFn tensor_map_encoder() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  });
  return fn;
}

int *device_status_word() {
  static int *addr[kMaxDevices] = {};
  static std::mutex mu;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lock(mu);
  if (addr[dev] == nullptr) {
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_device_status) != cudaSuccess) {
      cudaGetLastError();
      return nullptr;
    }
    addr[dev] = static_cast<int *>(p);
  }
  return addr[dev];
}

}  // namespace sq

using namespace sq;

extern "C" {

sq_status sq_calibrate_act(const void *x, int64_t M, int64_t K, int64_t ldx, const float *d,
                           const sq_segments *seg, float *s_act, sq_stream_t stream) {
  if (M < 1) return SQ_ERR_INVALID_ARG;
  SQ_TRY(check_act(x, M, K, ldx));
  SegParams sp;
  SQ_TRY(parse_segments(seg, K, -1, &sp));
  if (s_act == nullptr || !aligned(s_act, 4)) return SQ_ERR_INVALID_ARG;
  if (d && !aligned(d, 4)) return SQ_ERR_ALIGNMENT;
  SQ_TRY(check_device());
  int *status = device_status_word();
  if (status == nullptr) return SQ_ERR_CUDA;
  return from_cuda(launch_calibrate_act(static_cast<const uint16_t *>(x), M, K, ldx, d, sp,
                                        s_act, status, reinterpret_cast<cudaStream_t>(stream)));
}

sq_status sq_quantize_act(const void *x, int64_t M, int64_t K, int64_t ldx, const float *d,
                          const float *s_act, const sq_segments *seg, int8_t *planes,
                          sq_stream_t stream) {
  return quantize_common(x, M, K, ldx, d, s_act, seg, planes,
                         reinterpret_cast<cudaStream_t>(stream));
}

sq_status sq_quantize_act_plan(const float *d, int64_t K, const float *s_act,
                               const sq_segments *seg, uint32_t *plan, sq_stream_t stream) {
  SQ_TRY(check_k(K));
  SegParams sp;
  SQ_TRY(parse_segments(seg, K, -1, &sp));
  if (d == nullptr || s_act == nullptr || plan == nullptr) return SQ_ERR_INVALID_ARG;
  if (sp.fp8) return SQ_ERR_UNSUPPORTED;
  if (!aligned(d, 4) || !aligned(s_act, 4) || !aligned(plan, 4)) return SQ_ERR_ALIGNMENT;
  SQ_TRY(check_device());
  int *status = device_status_word();
  if (status == nullptr) return SQ_ERR_CUDA;
  return from_cuda(
      launch_quantize_plan(d, K, s_act, sp, plan, status, reinterpret_cast<cudaStream_t>(stream)));
}

sq_status sq_quantize_act_planned(const void *x, int64_t M, int64_t K, int64_t ldx,
                                  const float *d, const float *s_act, const sq_segments *seg,
                                  const uint32_t *plan, int8_t *planes, sq_stream_t stream) {
  return quantize_common(x, M, K, ldx, d, s_act, seg, planes,
                         reinterpret_cast<cudaStream_t>(stream), true, plan);
}

sq_status sq_quantize_weight_seg(const void *w, int64_t N, int64_t K, const float *d,
                                 const sq_segments *seg, int8_t *wq, float *s_w,
                                 sq_stream_t stream) {
  if (N < 1 || N > INT32_MAX) return SQ_ERR_INVALID_ARG;
  SQ_TRY(check_k(K));
  SegParams sp;
  SQ_TRY(parse_segments(seg, K, N, &sp));
  if (w == nullptr || wq == nullptr || s_w == nullptr) return SQ_ERR_INVALID_ARG;
  if (!aligned(w, 16) || !aligned(wq, 16) || !aligned(s_w, 4) || (d && !aligned(d, 4)))
    return SQ_ERR_ALIGNMENT;
  SQ_TRY(check_device());
  int *status = device_status_word();
  if (status == nullptr) return SQ_ERR_CUDA;
  return from_cuda(launch_quantize_weight(static_cast<const uint16_t *>(w), N, K, d, sp, wq, s_w,
                                          status, reinterpret_cast<cudaStream_t>(stream)));
}

sq_status sq_quantize_weight_w4(const void *w, int64_t N, int64_t K, const float *d,
                                const sq_segments *seg, uint8_t *wq4, float *s_w,
                                sq_stream_t stream) {
  if (N < 1 || N > INT32_MAX) return SQ_ERR_INVALID_ARG;
  SQ_TRY(check_k(K));
  SegParams sp;
  SQ_TRY(parse_segments(seg, K, N, &sp));
  if (w == nullptr || wq4 == nullptr || s_w == nullptr || sp.fp8) return SQ_ERR_INVALID_ARG;
  if (!aligned(w, 16) || !aligned(wq4, 16) || !aligned(s_w, 4) || (d && !aligned(d, 4)))
    return SQ_ERR_ALIGNMENT;
  SQ_TRY(check_device());
  int *status = device_status_word();
  if (status == nullptr) return SQ_ERR_CUDA;
  return from_cuda(launch_quantize_weight_w4(static_cast<const uint16_t *>(w), N, K, d, sp, wq4,
                                             s_w, status, reinterpret_cast<cudaStream_t>(stream)));
}

sq_status sq_unpack_weight_w4(const uint8_t *wq4, int64_t N, int64_t K, int8_t *wq,
                              sq_stream_t stream) {
  if (N < 1 || N > INT32_MAX) return SQ_ERR_INVALID_ARG;
  SQ_TRY(check_k(K));
  if (wq4 == nullptr || wq == nullptr) return SQ_ERR_INVALID_ARG;
  if (!aligned(wq4, 16) || !aligned(wq, 16)) return SQ_ERR_ALIGNMENT;
  SQ_TRY(check_device());
  int *status = device_status_word();
  if (status == nullptr) return SQ_ERR_CUDA;
  return from_cuda(
      launch_unpack_w4(wq4, N, K, wq, status, reinterpret_cast<cudaStream_t>(stream)));
}

sq_status sq_dualscale_seglinear_gemm(const int8_t *planes, const int8_t *wq, const float *s_w,
                                      const float *s_act, const void *bias, void *y,
                                      sq_out_dtype out_dtype, int64_t M, int64_t N, int64_t K,
                                      int64_t ldy, const sq_segments *seg, sq_stream_t stream) {
  if (out_dtype != SQ_OUT_BF16 && out_dtype != SQ_OUT_F32) return SQ_ERR_INVALID_ARG;
  return gemm_common(planes, wq, s_w, s_act, bias, y,
                     out_dtype == SQ_OUT_BF16 ? OUT_BF16 : OUT_F32, M, N, K, ldy, seg,
                     reinterpret_cast<cudaStream_t>(stream));
}

sq_status sq_dualscale_seglinear_gemm_ws(const int8_t *planes, const int8_t *wq,
                                         const float *s_w, const float *s_act, const void *bias,
                                         void *y, sq_out_dtype out_dtype, int64_t M, int64_t N,
                                         int64_t K, int64_t ldy, const sq_segments *seg,
                                         void *workspace, size_t workspace_bytes,
                                         sq_stream_t stream) {
  if (out_dtype != SQ_OUT_BF16 && out_dtype != SQ_OUT_F32) return SQ_ERR_INVALID_ARG;
  return gemm_common(planes, wq, s_w, s_act, bias, y,
                     out_dtype == SQ_OUT_BF16 ? OUT_BF16 : OUT_F32, M, N, K, ldy, seg,
                     reinterpret_cast<cudaStream_t>(stream), true, nullptr, 0, workspace,
                     workspace_bytes);
}

size_t sq_gemm_workspace_bytes(void) {
  if (check_device() != SQ_OK) return 0;
  return gemm_workspace_bytes();
}

sq_status sq_dualscale_seglinear_gemm_gelu_quant(const int8_t *planes, const int8_t *wq,
                                                const float *s_w, const float *s_act,
                                                const void *bias, int64_t M, int64_t N, int64_t K,
                                                const sq_segments *seg, const float *s_act_next,
                                                int32_t flags_next, int8_t *planes_next,
                                                sq_stream_t stream) {
  if (flags_next != 0 && flags_next != SQ_FLAG_SINGLE_SCALE) return SQ_ERR_INVALID_ARG;
  const int p_next = (flags_next & SQ_FLAG_SINGLE_SCALE) ? 1 : 2;
  return gemm_common(planes, wq, s_w, s_act, bias, planes_next, OUT_PLANES, M, N, K, N, seg,
                     reinterpret_cast<cudaStream_t>(stream), true, s_act_next, p_next);
}

sq_status sq_debug_gemm_s32(const int8_t *planes, const int8_t *wq, int64_t M, int64_t N,
                            int64_t K, const sq_segments *seg, int32_t *acc,
                            sq_stream_t stream) {
  return gemm_common(planes, wq, nullptr, nullptr, nullptr, acc, OUT_S32, M, N, K, N, seg,
                     reinterpret_cast<cudaStream_t>(stream));
}

sq_status sq_debug_gemm_s32_ws(const int8_t *planes, const int8_t *wq, int64_t M, int64_t N,
                               int64_t K, const sq_segments *seg, int32_t *acc, void *workspace,
                               size_t workspace_bytes, sq_stream_t stream) {
  return gemm_common(planes, wq, nullptr, nullptr, nullptr, acc, OUT_S32, M, N, K, N, seg,
                     reinterpret_cast<cudaStream_t>(stream), true, nullptr, 0, workspace,
                     workspace_bytes);
}

sq_status sq_debug_timeout_probe(uint32_t limit_us, sq_stream_t stream) {
  if (limit_us < 1 || limit_us > 100000) return SQ_ERR_INVALID_ARG;
  SQ_TRY(check_device());
  int *status = device_status_word();
  if (status == nullptr) return SQ_ERR_CUDA;
  return from_cuda(launch_timeout_probe(limit_us, status, reinterpret_cast<cudaStream_t>(stream)));
}

int32_t sq_debug_bounds_checks(void) {
#ifdef SQ_DEBUG_BOUNDS
  return 1;
#else
  return 0;
#endif
}

sq_status sq_debug_bounds_probe(int32_t *buf, int64_t n, sq_stream_t stream) {
  if (buf == nullptr || n < 1) return SQ_ERR_INVALID_ARG;
  if (!aligned(buf, 4)) return SQ_ERR_ALIGNMENT;
  if (!sq_debug_bounds_checks()) return SQ_ERR_UNSUPPORTED;
  SQ_TRY(check_device());
  int *status = device_status_word();
  if (status == nullptr) return SQ_ERR_CUDA;
  return from_cuda(launch_bounds_probe(buf, n, status, reinterpret_cast<cudaStream_t>(stream)));
}

sq_status sq_get_device_status(sq_stream_t stream) {
  SQ_TRY(check_device());
  int *word = device_status_word();
  if (word == nullptr) return SQ_ERR_CUDA;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  // Everything enqueued on `stream` before this call finishes first; the word
  // is then read, and cleared only if it was set.
  int v = 0;
  if (cudaMemcpyAsync(&v, word, sizeof v, cudaMemcpyDeviceToHost, st) != cudaSuccess ||
      cudaStreamSynchronize(st) != cudaSuccess)
    return SQ_ERR_CUDA;
  if (v != 0 && (cudaMemsetAsync(word, 0, sizeof v, st) != cudaSuccess ||
                 cudaStreamSynchronize(st) != cudaSuccess))
    return SQ_ERR_CUDA;
  return v == 0 ? SQ_OK : static_cast<sq_status>(v);
}

sq_status sq_choose_single_scale(const float *s_act, int32_t n_steps, int32_t flags,
                                 float threshold, int32_t *single) {
  if (s_act == nullptr || single == nullptr) return SQ_ERR_INVALID_ARG;
  if (n_steps < 1 || n_steps > SQ_MAX_SEGMENTS * SQ_MAX_SEGMENTS) return SQ_ERR_INVALID_ARG;
  if ((flags & ~SQ_FLAG_FP8) != 0) return SQ_ERR_INVALID_ARG;
  if (!(threshold > 1.0f) || !(threshold < 3.4e38f)) return SQ_ERR_INVALID_ARG;
  const float qp = (flags & SQ_FLAG_FP8) ? 448.0f : 127.0f;
  const float qm = (flags & SQ_FLAG_FP8) ? 448.0f : 128.0f;
  int32_t all_close = 1;
  for (int32_t t = 0; t < n_steps; ++t) {
    const float sp = s_act[2 * t], sm = s_act[2 * t + 1];
    if (!(sp > 0.0f) || !(sm > 0.0f) || !(sp < 3.4e38f) || !(sm < 3.4e38f))
      return SQ_ERR_INVALID_ARG;
    const float hi = sp * qp, lo = sm * qm;  // the calibrated max and |min|
    const float big = hi > lo ? hi : lo, small = hi > lo ? lo : hi;
    if (!(big < threshold * small)) all_close = 0;
  }
  *single = all_close;
  return SQ_OK;
}

const char *sq_status_string(sq_status s) {
  switch (s) {
    case SQ_OK: return "SQ_OK";
    case SQ_ERR_INVALID_ARG: return "SQ_ERR_INVALID_ARG: invalid argument";
    case SQ_ERR_UNSUPPORTED: return "SQ_ERR_UNSUPPORTED: valid request the library does not implement";
    case SQ_ERR_ALIGNMENT: return "SQ_ERR_ALIGNMENT: pointer or leading dimension misaligned";
    case SQ_ERR_OVERFLOW: return "SQ_ERR_OVERFLOW: K-segment too wide for int32 accumulation";
    case SQ_ERR_CUDA: return "SQ_ERR_CUDA: a CUDA runtime call failed";
    case SQ_ERR_DEVICE_TIMEOUT: return "SQ_ERR_DEVICE_TIMEOUT: a kernel gave up waiting on a barrier";
    case SQ_ERR_NO_DEVICE: return "SQ_ERR_NO_DEVICE: no sm_100 device is current";
    case SQ_ERR_TOO_LARGE: return "SQ_ERR_TOO_LARGE: one row does not fit the fixed scratch";
    case SQ_ERR_DEVICE_BOUNDS:
      return "SQ_ERR_DEVICE_BOUNDS: a kernel skipped a store outside its buffer (debug build)";
  }
  return "unknown sq_status";
}

int32_t sq_version(void) { return 201; }

}  // extern "C"
