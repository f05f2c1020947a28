// sq_internal.h -- declarations shared by the library's own translation units
// (kernels and the C-ABI layer).  Not installed; not used by anything else.
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/segquant.h"

namespace sq {

// Segment table as the kernels see it (passed by value as a kernel argument).
struct SegParams {
  int32_t mode;   // sq_seg_mode
  int32_t n_seg;  // segments
  int32_t G;      // activation groups
  int32_t S;      // K-segments (n_seg in input mode, else 1)
  int32_t P;      // activation planes per group: 2 (DualScale) or 1 (single scale)
  int32_t w4;     // 1: the weight operand holds 16 q of W4A8 codes q (SQ_FLAG_W4)
  int32_t fp8;    // 1: codes are FP8 E4M3 bit patterns (SQ_FLAG_FP8)
  int32_t off[SQ_MAX_SEGMENTS + 1];
};

// Guard of a plain global store: `ok` is the test of the store's index against
// its buffer's logical extent.  In the bounds-checked debug build
// (SQ_DEBUG_BOUNDS) a failed test records SQ_ERR_DEVICE_BOUNDS in `status`
// (first report wins) and the caller skips the store; in the release build the
// guard is always true and costs nothing.
__device__ __forceinline__ bool store_ok(int *status, bool ok) {
#ifdef SQ_DEBUG_BOUNDS
  if (!ok) atomicCAS(status, 0, static_cast<int>(SQ_ERR_DEVICE_BOUNDS));
  return ok;
#else
  (void)status;
  (void)ok;
  return true;
#endif
}

// Index i with off[i] <= p < off[i + 1] (tables are short: a linear scan).
__host__ __device__ inline int seg_index(const int32_t *off, int n_seg, int64_t p) {
  int i = 0;
  while (i + 1 < n_seg && p >= off[i + 1]) ++i;
  return i;
}

// ---- launchers (quant.cu) --------------------------------------------------
cudaError_t launch_calibrate_act(const uint16_t *x, int64_t M, int64_t K, int64_t ldx,
                                 const float *d, const SegParams &seg, float *s_act,
                                 int *status, cudaStream_t stream);
sq_status launch_quantize_act(const uint16_t *x, int64_t M, int64_t K, int64_t ldx,
                              const float *d, const float *s_act, const SegParams &seg,
                              int8_t *planes, const uint32_t *plan, int *status,
                              cudaStream_t stream);
// Quantize plan: bits [G][ceil(K/32)] (see quant_plan_kernel).
cudaError_t launch_quantize_plan(const float *d, int64_t K, const float *s_act,
                                 const SegParams &seg, uint32_t *plan, int *status,
                                 cudaStream_t stream);
cudaError_t launch_quantize_weight(const uint16_t *w, int64_t N, int64_t K, const float *d,
                                   const SegParams &seg, int8_t *wq, float *s_w, int *status,
                                   cudaStream_t stream);
cudaError_t launch_quantize_weight_w4(const uint16_t *w, int64_t N, int64_t K, const float *d,
                                      const SegParams &seg, uint8_t *wq4, float *s_w,
                                      int *status, cudaStream_t stream);
cudaError_t launch_unpack_w4(const uint8_t *wq4, int64_t N, int64_t K, int8_t *wq, int *status,
                             cudaStream_t stream);

// ---- launcher (gemm.cu) ----------------------------------------------------
// OUT_PLANES: the next layer's int8 activation planes, from bf16(gelu(bf16(y)))
// (the fused producer of an FFN's second linear).
enum OutKind { OUT_BF16 = 0, OUT_F32 = 1, OUT_S32 = 2, OUT_PLANES = 3 };

struct GemmRequest {
  const int8_t *planes;
  const int8_t *wq;
  const float *s_w;
  const float *s_act;
  const uint16_t *bias;
  void *y;
  int64_t ldy;
  int out_kind;
  int64_t M, N, K;
  SegParams seg;
  int *status;  // device error word
  // OUT_PLANES: the next layer's steps {s+, s-} (fp32 [2], device) and its
  // planes per group (2 DualScale, 1 single scale); y is int8 [p_next][M][N].
  const float *s_next = nullptr;
  int p_next = 0;
  // Optional workspace for the split last wave (zero-filled before its first
  // use; every call leaves its flags at zero): nullptr = whole tiles only.
  void *workspace = nullptr;
  size_t workspace_bytes = 0;
};

sq_status launch_gemm(const GemmRequest &req, cudaStream_t stream);
// Workspace bytes that let any one-segment GEMM split its last wave on the
// current device.
size_t gemm_workspace_bytes();

// ---- test-only probes (probe.cu) -------------------------------------------
cudaError_t launch_timeout_probe(uint32_t limit_us, int *status, cudaStream_t stream);
// Debug build only: one checked store to element n of a buffer said to hold n.
cudaError_t launch_bounds_probe(int32_t *buf, int64_t n, int *status, cudaStream_t stream);

// Host-side validation of a quantize / GEMM call without launching anything
// (the checks of sq_quantize_act and sq_dualscale_seglinear_gemm).
sq_status validate_quantize_act(const void *x, int64_t M, int64_t K, int64_t ldx, const float *d,
                                const float *s_act, const sq_segments *seg, int8_t *planes);
sq_status validate_gemm(const int8_t *planes, const int8_t *wq, const float *s_w,
                        const float *s_act, const void *bias, void *y, int out_kind, int64_t M,
                        int64_t N, int64_t K, int64_t ldy, const sq_segments *seg);

// Device address of the library's error word on the current device.
int *device_status_word();

// cuTensorMapEncodeTiled, resolved through the runtime (no link-time libcuda).
typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion,
                                  CUtensorMapFloatOOBfill);
EncodeTiledFn tensor_map_encoder();  // nullptr if the driver lacks it

}  // namespace sq
