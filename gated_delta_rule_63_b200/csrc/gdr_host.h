// gdr_host.h -- host-side argument checks shared by the entry points.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/gdr.h"

namespace gdr {

constexpr int kHeadDim = 128;
constexpr int kChunk = 64;
constexpr int kConvK = 4;

inline bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Ranges [a, a + na) and [b, b + nb) in bytes overlap.
inline bool overlaps(const void *a, size_t na, const void *b, size_t nb) {
  if (!a || !b || na == 0 || nb == 0) return false;
  const char *pa = static_cast<const char *>(a), *pb = static_cast<const char *>(b);
  return pa < pb + nb && pb < pa + na;
}

// Heads supported by the kernels: dk = dv = 128, hv % hk == 0, group <= 8.
inline int check_heads(int hk, int hv) {
  if (hk <= 0 || hv <= 0) return GDR_ERR_SHAPE;
  if (hv % hk != 0 || hv / hk > 8) return GDR_ERR_UNSUPPORTED;
  return GDR_OK;
}

// Host copy of cu_seqlens: starts at 0, non-decreasing, total < 2^31.
inline int check_cu_seqlens(const int32_t *cu, int n_seqs) {
  if (!cu) return GDR_ERR_NULL;
  if (n_seqs < 0) return GDR_ERR_SHAPE;
  if (cu[0] != 0) return GDR_ERR_CU_SEQLENS;
  for (int i = 0; i < n_seqs; ++i)
    if (cu[i + 1] < cu[i]) return GDR_ERR_CU_SEQLENS;
  return GDR_OK;
}

// cuTensorMapEncodeTiled, looked up once through the runtime's driver entry
// points (no link against libcuda); null when the driver does not provide it
typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *,
                                  CUtensorMapInterleave, CUtensorMapSwizzle, CUtensorMapL2promotion,
                                  CUtensorMapFloatOOBfill);
EncodeTiledFn tensor_map_encoder();

// Device address of the library's error word on the current device (cached).
int *device_error_ptr();

// Record a host-side failure (step name + CUDA error) for gdr_last_error_string.
void set_last_error(const char *step, cudaError_t e);
void clear_last_error();
const char *t_last_error_ptr();

inline int launch_status(cudaError_t e, const char *step = "kernel launch") {
  if (e == cudaSuccess) return GDR_OK;
  set_last_error(step, e);
  return GDR_ERR_CUDA;
}

inline int last_launch_status(const char *step = "kernel launch") {
  return launch_status(cudaGetLastError(), step);
}

// Launchers implemented in the kernel files (arguments already checked).
int launch_causal_conv(const void *x, const void *w, const void *cs_in, void *cs_out,
                       const int32_t *cu_dev, int n_seqs, int total, int channels, void *y,
                       cudaStream_t s);
int launch_gated_rmsnorm(const void *o, const void *z, const float *w, float eps, int64_t rows,
                         void *y, cudaStream_t s);
int launch_decode(const void *x, const void *conv_w, void *conv_state, const void *a, const void *b,
                  const float *A_log, const float *dt_bias, float scale, int hk, int hv,
                  float *state, const int32_t *slot, int n_slots, void *o, int batch, cudaStream_t s);
// pool of states for gdr_chunk_prefill_slots (see PrefillParams)
struct PrefillPool {
  float *pool;
  int n_slots;
  const int32_t *slot;
  int init_from_pool;
};
int launch_chunk_prefill(const void *q, const void *k, const void *v, int64_t qk_stride,
                         int64_t v_stride, const void *a, const void *b,
                         const float *A_log, const float *dt_bias, float scale, int hk, int hv,
                         const int32_t *cu_dev, const int32_t *cu_host, int n_seqs, int total, int max_chunks,
                         const float *h0, float *hT, void *o, const void *z, const float *norm_w,
                         float eps, void *y, void *workspace, size_t ws_bytes, cudaStream_t s,
                         const PrefillPool *pool = nullptr);
size_t chunk_prefill_workspace_bytes(int n_seqs, int hv, int window_chunks, bool need_carry);
// y[M][N] = x[M][K] W[N][K]^T in bf16 with fp32 accumulation (linear.cu)
int launch_linear(const void *x, const void *w, void *y, int64_t M, int64_t N, int64_t K, cudaStream_t s);
// window schedule of a prefill call on the current device (windows, chunks per window,
// whether the next window's prep runs beside the current chain); GDR_ERR_WORKSPACE when
// not even one chunk per sequence fits
int plan_chunk_prefill(int n_seqs, int hv, int max_chunks, size_t ws_bytes, bool carry_in_ws, bool capturing,
                       int *windows, int *win_chunks, bool *pipelined);

// Conv output of `total` tokens of `channels` bf16 kept in the workspace when the conv is
// fused into the prefill (a whole number of KiB, so the records after it stay aligned).
inline size_t fused_conv_bytes(int total, int channels) {
  const size_t b = static_cast<size_t>(total) * channels * 2;
  return (b + 1023) & ~static_cast<size_t>(1023);
}

}  // namespace gdr
