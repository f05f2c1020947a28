// host.cu -- host-to-host execution of one quantized linear layer with the
// transfers overlapped: rows move to the device in chunks, every chunk runs
// the activation quantizer and the GEMM, and its output rows move back, on
// three streams with two workspace slots.  Only the library's own entry points
// launch kernels; this file only orders copies and launches.
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>
#include <new>

#include "sq_internal.h"

struct sq_host_pipeline {
  int device;
  int64_t chunk_rows, max_K, max_N;
  int32_t max_G, max_P;
  uint8_t *slot[2];  // each: x chunk | planes chunk | y chunk
  size_t x_off, planes_off, y_off, slot_bytes;
  cudaStream_t s_in, s_comp, s_out;
  cudaEvent_t ev_start, ev_done, ev_in[2], ev_comp[2], ev_out[2];
};

namespace sq {
namespace {

constexpr size_t kAlign = 256;

size_t round_up(size_t v) { return (v + kAlign - 1) / kAlign * kAlign; }

// Slot layout for a pipeline's maximum sizes; false if a size is invalid.
bool slot_layout(int64_t chunk, int64_t K, int64_t N, int32_t G, int32_t P, size_t *x_off,
                 size_t *planes_off, size_t *y_off, size_t *slot_bytes) {
  if (chunk < 1 || chunk > INT32_MAX || K < 16 || K % 16 != 0 || K > INT32_MAX || N < 1 ||
      N > INT32_MAX || G < 1 || G > SQ_MAX_SEGMENTS || P < 1 || P > 2)
    return false;
  const int64_t n_pad = (N + 7) / 8 * 8;  // output rows 16-byte aligned for bf16 and fp32
  // Every product below then stays far inside 64 bits.
  constexpr int64_t kMaxElems = int64_t(1) << 44;
  if (chunk > kMaxElems / K || chunk > kMaxElems / n_pad) return false;
  const size_t x_bytes = static_cast<size_t>(chunk) * K * 2;
  const size_t planes_bytes = static_cast<size_t>(G) * P * chunk * K;
  const size_t y_bytes = static_cast<size_t>(chunk) * n_pad * 4;
  *x_off = 0;
  *planes_off = round_up(x_bytes);
  *y_off = *planes_off + round_up(planes_bytes);
  *slot_bytes = *y_off + round_up(y_bytes);
  return true;
}

void release(sq_host_pipeline *pl) {
  cudaEvent_t *evs[] = {&pl->ev_start, &pl->ev_done, &pl->ev_in[0], &pl->ev_in[1],
                        &pl->ev_comp[0], &pl->ev_comp[1], &pl->ev_out[0], &pl->ev_out[1]};
  for (cudaEvent_t *e : evs)
    if (*e) cudaEventDestroy(*e);
  cudaStream_t *ss[] = {&pl->s_in, &pl->s_comp, &pl->s_out};
  for (cudaStream_t *st : ss)
    if (*st) cudaStreamDestroy(*st);
  delete pl;
}

// ---- fixed scratch of sq_dualscale_seglinear_host_noalloc -----------------
// One statically sized buffer in the library's device image: every device that
// loads the library holds it until the process exits, and every call of the
// no-allocation entry point on that device shares it.  Host code must not use
// the symbol itself as a pointer (on the host it names a stand-in, not device
// memory); its device address is looked up once per device.
__device__ __align__(256) uint8_t g_noalloc_scratch[SQ_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;

// Device address of g_noalloc_scratch on the current device, or nullptr.
uint8_t *noalloc_scratch() {
  static uint8_t *addr[kMaxDevices] = {};
  static std::mutex mu;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    cudaGetLastError();
    return nullptr;
  }
  std::lock_guard<std::mutex> lock(mu);
  if (addr[dev] == nullptr) {
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) {
      cudaGetLastError();
      return nullptr;
    }
    addr[dev] = static_cast<uint8_t *>(p);
  }
  return addr[dev];
}

// Most rows per chunk whose x rows, planes and output rows fit the scratch
// together (the slot layout of the pipelines), at most M; 0 if not one row fits.
int64_t noalloc_chunk_rows(int64_t M, int64_t K, int64_t N, int32_t G, int32_t P) {
  size_t x_off, planes_off, y_off, slot_bytes;
  const int64_t n_pad = (N + 7) / 8 * 8;
  const int64_t per_row = 2 * K + static_cast<int64_t>(G) * P * K + 4 * n_pad;
  int64_t rows = static_cast<int64_t>(SQ_NOALLOC_SCRATCH_BYTES) / per_row;
  if (rows >= 128) rows = rows / 128 * 128;  // whole GEMM row tiles
  if (rows > M) rows = M;
  // each region is rounded up to 256 bytes: step down until the slot fits
  while (rows > 0 && (!slot_layout(rows, K, N, G, P, &x_off, &planes_off, &y_off, &slot_bytes) ||
                      slot_bytes > SQ_NOALLOC_SCRATCH_BYTES))
    --rows;
  return rows;
}

}  // namespace
}  // namespace sq

using namespace sq;

extern "C" {

size_t sq_host_pipeline_workspace_bytes(int64_t chunk_rows, int64_t max_K, int64_t max_N,
                                        int32_t max_G, int32_t max_P) {
  size_t x_off, planes_off, y_off, slot_bytes;
  if (!slot_layout(chunk_rows, max_K, max_N, max_G, max_P, &x_off, &planes_off, &y_off,
                   &slot_bytes))
    return 0;
  return 2 * slot_bytes;
}

sq_status sq_host_pipeline_create(int64_t chunk_rows, int64_t max_K, int64_t max_N,
                                  int32_t max_G, int32_t max_P, void *workspace,
                                  size_t workspace_bytes, sq_host_pipeline **out) {
  if (out == nullptr) return SQ_ERR_INVALID_ARG;
  *out = nullptr;
  size_t x_off, planes_off, y_off, slot_bytes;
  if (!slot_layout(chunk_rows, max_K, max_N, max_G, max_P, &x_off, &planes_off, &y_off,
                   &slot_bytes))
    return SQ_ERR_INVALID_ARG;
  if (workspace == nullptr || workspace_bytes < 2 * slot_bytes) return SQ_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(workspace) % kAlign != 0) return SQ_ERR_ALIGNMENT;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return SQ_ERR_NO_DEVICE;
  sq_host_pipeline *pl = new (std::nothrow) sq_host_pipeline{};
  if (pl == nullptr) return SQ_ERR_CUDA;
  pl->device = dev;
  pl->chunk_rows = chunk_rows;
  pl->max_K = max_K;
  pl->max_N = max_N;
  pl->max_G = max_G;
  pl->max_P = max_P;
  pl->x_off = x_off;
  pl->planes_off = planes_off;
  pl->y_off = y_off;
  pl->slot_bytes = slot_bytes;
  pl->slot[0] = static_cast<uint8_t *>(workspace);
  pl->slot[1] = pl->slot[0] + slot_bytes;
  bool ok = cudaStreamCreateWithFlags(&pl->s_in, cudaStreamNonBlocking) == cudaSuccess &&
            cudaStreamCreateWithFlags(&pl->s_comp, cudaStreamNonBlocking) == cudaSuccess &&
            cudaStreamCreateWithFlags(&pl->s_out, cudaStreamNonBlocking) == cudaSuccess;
  cudaEvent_t *evs[] = {&pl->ev_start, &pl->ev_done, &pl->ev_in[0], &pl->ev_in[1],
                        &pl->ev_comp[0], &pl->ev_comp[1], &pl->ev_out[0], &pl->ev_out[1]};
  for (cudaEvent_t *e : evs)
    ok = ok && cudaEventCreateWithFlags(e, cudaEventDisableTiming) == cudaSuccess;
  if (!ok) {
    release(pl);
    return SQ_ERR_CUDA;
  }
  *out = pl;
  return SQ_OK;
}

sq_status sq_host_pipeline_destroy(sq_host_pipeline *pl) {
  if (pl == nullptr) return SQ_OK;
  const bool ok = cudaStreamSynchronize(pl->s_in) == cudaSuccess &&
                  cudaStreamSynchronize(pl->s_comp) == cudaSuccess &&
                  cudaStreamSynchronize(pl->s_out) == cudaSuccess;
  release(pl);
  return ok ? SQ_OK : SQ_ERR_CUDA;
}

sq_status sq_dualscale_seglinear_host(sq_host_pipeline *pl, const void *x_host, int64_t M,
                                      int64_t K, int64_t ldx, const float *d,
                                      const float *s_act, const int8_t *wq, const float *s_w,
                                      const void *bias, void *y_host, sq_out_dtype out_dtype,
                                      int64_t N, int64_t ldy, const sq_segments *seg,
                                      sq_stream_t stream) {
  if (pl == nullptr) return SQ_ERR_INVALID_ARG;
  if (out_dtype != SQ_OUT_BF16 && out_dtype != SQ_OUT_F32) return SQ_ERR_INVALID_ARG;
  if (M < 0 || M > INT32_MAX || K < 16 || K % 16 != 0 || N < 1 || ldx < K || ldy < N)
    return SQ_ERR_INVALID_ARG;
  if (K > pl->max_K || N > pl->max_N) return SQ_ERR_INVALID_ARG;
  const int32_t G = seg ? seg->n_groups : 1;
  const int32_t P = (seg && (seg->flags & SQ_FLAG_SINGLE_SCALE)) ? 1 : 2;
  if (G > pl->max_G || P > pl->max_P) return SQ_ERR_INVALID_ARG;
  if (M == 0) return SQ_OK;
  if (x_host == nullptr || y_host == nullptr) return SQ_ERR_INVALID_ARG;
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev != pl->device) return SQ_ERR_INVALID_ARG;

  const size_t elem = out_dtype == SQ_OUT_BF16 ? 2 : 4;
  const int64_t n_pad = (N + 7) / 8 * 8;
  {
    // Every check of the device calls, on the first chunk, before anything is
    // enqueued: later chunks differ only in their row count.
    const int64_t rows = M < pl->chunk_rows ? M : pl->chunk_rows;
    int8_t *planes0 = reinterpret_cast<int8_t *>(pl->slot[0] + pl->planes_off);
    sq_status st = validate_quantize_act(pl->slot[0] + pl->x_off, rows, K, K, d, s_act, seg,
                                         planes0);
    if (st != SQ_OK) return st;
    st = validate_gemm(planes0, wq, s_w, s_act, bias, pl->slot[0] + pl->y_off,
                       out_dtype == SQ_OUT_BF16 ? OUT_BF16 : OUT_F32, rows, N, K, n_pad, seg);
    if (st != SQ_OK) return st;
  }
  cudaStream_t user = reinterpret_cast<cudaStream_t>(stream);
  auto cu = [](cudaError_t e) { return e == cudaSuccess; };
  // After a failure past the first enqueue, wait for the pipeline's streams
  // before returning, so that no copy or kernel of this call is still in
  // flight when the caller sees the error.
  auto fail = [pl](sq_status st) {
    cudaStreamSynchronize(pl->s_in);
    cudaStreamSynchronize(pl->s_comp);
    cudaStreamSynchronize(pl->s_out);
    return st;
  };
  if (!cu(cudaEventRecord(pl->ev_start, user)) ||
      !cu(cudaStreamWaitEvent(pl->s_in, pl->ev_start, 0)) ||
      !cu(cudaStreamWaitEvent(pl->s_comp, pl->ev_start, 0)) ||
      !cu(cudaStreamWaitEvent(pl->s_out, pl->ev_start, 0)))
    return SQ_ERR_CUDA;

  const int64_t n_chunks = (M + pl->chunk_rows - 1) / pl->chunk_rows;
  for (int64_t c = 0; c < n_chunks; ++c) {
    const int s = static_cast<int>(c & 1);
    const int64_t r0 = c * pl->chunk_rows;
    const int64_t rows = (M - r0) < pl->chunk_rows ? (M - r0) : pl->chunk_rows;
    uint8_t *x_dev = pl->slot[s] + pl->x_off;
    int8_t *planes_dev = reinterpret_cast<int8_t *>(pl->slot[s] + pl->planes_off);
    uint8_t *y_dev = pl->slot[s] + pl->y_off;
    // The slot's previous chunk -- chunk c - 2 of this call, or the last chunk
    // an earlier call ran in this slot, whichever stream that call was given --
    // must have been quantized before its rows are overwritten, and copied out
    // before its planes and output are.  Waiting on an event that was never
    // recorded (a fresh pipeline) returns at once.
    if (!cu(cudaStreamWaitEvent(pl->s_in, pl->ev_comp[s], 0))) return fail(SQ_ERR_CUDA);
    if (!cu(cudaMemcpy2DAsync(x_dev, K * 2, static_cast<const uint8_t *>(x_host) + r0 * ldx * 2,
                              ldx * 2, K * 2, rows, cudaMemcpyHostToDevice, pl->s_in)) ||
        !cu(cudaEventRecord(pl->ev_in[s], pl->s_in)) ||
        !cu(cudaStreamWaitEvent(pl->s_comp, pl->ev_in[s], 0)))
      return fail(SQ_ERR_CUDA);
    if (!cu(cudaStreamWaitEvent(pl->s_comp, pl->ev_out[s], 0))) return fail(SQ_ERR_CUDA);
    sq_stream_t comp = reinterpret_cast<sq_stream_t>(pl->s_comp);
    sq_status st = sq_quantize_act(x_dev, rows, K, K, d, s_act, seg, planes_dev, comp);
    if (st != SQ_OK) return fail(st);
    st = sq_dualscale_seglinear_gemm(planes_dev, wq, s_w, s_act, bias, y_dev, out_dtype, rows, N,
                                     K, n_pad, seg, comp);
    if (st != SQ_OK) return fail(st);
    if (!cu(cudaEventRecord(pl->ev_comp[s], pl->s_comp)) ||
        !cu(cudaStreamWaitEvent(pl->s_out, pl->ev_comp[s], 0)) ||
        !cu(cudaMemcpy2DAsync(static_cast<uint8_t *>(y_host) + r0 * ldy * elem, ldy * elem, y_dev,
                              n_pad * elem, N * elem, rows, cudaMemcpyDeviceToHost, pl->s_out)) ||
        !cu(cudaEventRecord(pl->ev_out[s], pl->s_out)))
      return fail(SQ_ERR_CUDA);
  }
  if (!cu(cudaEventRecord(pl->ev_done, pl->s_out)) ||
      !cu(cudaStreamWaitEvent(user, pl->ev_done, 0)))
    return fail(SQ_ERR_CUDA);
  return SQ_OK;
}

sq_status sq_dualscale_seglinear_host_noalloc(const void *x_host, int64_t M, int64_t K,
                                              int64_t ldx, const float *d, const float *s_act,
                                              const int8_t *wq, const float *s_w,
                                              const void *bias, void *y_host,
                                              sq_out_dtype out_dtype, int64_t N, int64_t ldy,
                                              const sq_segments *seg, sq_stream_t stream) {
  if (out_dtype != SQ_OUT_BF16 && out_dtype != SQ_OUT_F32) return SQ_ERR_INVALID_ARG;
  if (M < 0 || M > INT32_MAX || K < 16 || K % 16 != 0 || K > INT32_MAX || N < 1 ||
      N > INT32_MAX || ldx < K || ldy < N)
    return SQ_ERR_INVALID_ARG;
  const int32_t G = seg ? seg->n_groups : 1;
  const int32_t P = (seg && (seg->flags & SQ_FLAG_SINGLE_SCALE)) ? 1 : 2;
  if (G < 1 || G > SQ_MAX_SEGMENTS) return SQ_ERR_INVALID_ARG;
  // One row of x, its planes and its output must fit the fixed scratch.
  const int64_t chunk = noalloc_chunk_rows(M > 0 ? M : 1, K, N, G, P);
  if (chunk < 1) return SQ_ERR_TOO_LARGE;
  if (M == 0) return SQ_OK;
  if (x_host == nullptr || y_host == nullptr) return SQ_ERR_INVALID_ARG;
  uint8_t *scratch = noalloc_scratch();
  if (scratch == nullptr) return SQ_ERR_CUDA;
  size_t x_off, planes_off, y_off, slot_bytes;
  if (!slot_layout(chunk, K, N, G, P, &x_off, &planes_off, &y_off, &slot_bytes))
    return SQ_ERR_INVALID_ARG;
  uint8_t *x_dev = scratch + x_off;
  int8_t *planes_dev = reinterpret_cast<int8_t *>(scratch + planes_off);
  uint8_t *y_dev = scratch + y_off;
  const size_t elem = out_dtype == SQ_OUT_BF16 ? 2 : 4;
  const int64_t n_pad = (N + 7) / 8 * 8;
  // Every check of the device calls, before anything is enqueued: chunks
  // differ only in their row count.
  sq_status st = validate_quantize_act(x_dev, chunk, K, K, d, s_act, seg, planes_dev);
  if (st != SQ_OK) return st;
  st = validate_gemm(planes_dev, wq, s_w, s_act, bias, y_dev,
                     out_dtype == SQ_OUT_BF16 ? OUT_BF16 : OUT_F32, chunk, N, K, n_pad, seg);
  if (st != SQ_OK) return st;
  cudaStream_t user = reinterpret_cast<cudaStream_t>(stream);
  // After a failure past the first enqueue, wait for the caller's stream, so
  // that no copy or kernel of this call is still in flight on return.
  auto fail = [user](sq_status code) {
    cudaStreamSynchronize(user);
    return code;
  };
  // Everything runs on the caller's stream, chunk after chunk through the one
  // scratch region: a chunk's rows are copied in only after the previous
  // chunk's output has been copied out.
  for (int64_t r0 = 0; r0 < M; r0 += chunk) {
    const int64_t rows = (M - r0) < chunk ? (M - r0) : chunk;
    if (cudaMemcpy2DAsync(x_dev, K * 2, static_cast<const uint8_t *>(x_host) + r0 * ldx * 2,
                          ldx * 2, K * 2, rows, cudaMemcpyHostToDevice, user) != cudaSuccess)
      return fail(SQ_ERR_CUDA);
    st = sq_quantize_act(x_dev, rows, K, K, d, s_act, seg, planes_dev, stream);
    if (st != SQ_OK) return fail(st);
    st = sq_dualscale_seglinear_gemm(planes_dev, wq, s_w, s_act, bias, y_dev, out_dtype, rows, N,
                                     K, n_pad, seg, stream);
    if (st != SQ_OK) return fail(st);
    if (cudaMemcpy2DAsync(static_cast<uint8_t *>(y_host) + r0 * ldy * elem, ldy * elem, y_dev,
                          n_pad * elem, N * elem, rows, cudaMemcpyDeviceToHost,
                          user) != cudaSuccess)
      return fail(SQ_ERR_CUDA);
  }
  return SQ_OK;
}

}  // extern "C"
