// gdr_host.cu -- the C ABI of libgdr.so: argument checks, chunk table, error word.
//
// Every entry point validates its arguments on the host and returns a
// gdr_status_t before anything is launched; the launchers live next to their
// kernels.
#include <cuda_runtime.h>
#include <stdint.h>

#include "gdr_common.cuh"
#include "gdr_host.h"

#include <atomic>
#include <cstdio>

namespace gdr {
__device__ int g_device_error = 0;

int *device_error_ptr() {
  static std::atomic<int *> cache[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  int *p = cache[dev].load(std::memory_order_acquire);
  if (!p) {
    void *addr = nullptr;
    if (cudaGetSymbolAddress(&addr, g_device_error) != cudaSuccess) return nullptr;
    p = static_cast<int *>(addr);
    cache[dev].store(p, std::memory_order_release);
  }
  return p;
}
namespace {
thread_local char t_last_error[256] = "";
}

void set_last_error(const char *step, cudaError_t e) {
  snprintf(t_last_error, sizeof(t_last_error), "%s: %s (%d)", step,
           e == cudaSuccess ? "no CUDA error" : cudaGetErrorString(e), static_cast<int>(e));
}
void clear_last_error() { t_last_error[0] = 0; }
const char *t_last_error_ptr() { return t_last_error; }

EncodeTiledFn tensor_map_encoder() {
  static std::atomic<EncodeTiledFn> fn{nullptr};
  EncodeTiledFn f = fn.load(std::memory_order_acquire);
  if (!f) {
    void *ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess || !ptr)
      return nullptr;
    f = reinterpret_cast<EncodeTiledFn>(ptr);
    fn.store(f, std::memory_order_release);
  }
  return f;
}

}  // namespace gdr

using namespace gdr;

extern "C" {

const char *gdr_status_string(int status) {
  switch (status) {
    case GDR_OK: return "GDR_OK";
    case GDR_ERR_NULL: return "GDR_ERR_NULL: a required pointer is NULL";
    case GDR_ERR_SHAPE: return "GDR_ERR_SHAPE: invalid or inconsistent size";
    case GDR_ERR_ALIGN: return "GDR_ERR_ALIGN: tensor pointer not 16-byte aligned";
    case GDR_ERR_CU_SEQLENS: return "GDR_ERR_CU_SEQLENS: offsets must start at 0 and not decrease";
    case GDR_ERR_UNSUPPORTED: return "GDR_ERR_UNSUPPORTED: head dims or grouping not implemented";
    case GDR_ERR_WORKSPACE: return "GDR_ERR_WORKSPACE: workspace missing or too small for one chunk window";
    case GDR_ERR_CUDA: return "GDR_ERR_CUDA: CUDA launch failed";
    case GDR_ERR_TIMEOUT: return "GDR_ERR_TIMEOUT: a bounded wait in a kernel ran out";
    case GDR_ERR_ALIAS: return "GDR_ERR_ALIAS: buffers overlap";
    default: return "GDR_ERR_UNKNOWN";
  }
}

int gdr_abi_version(void) { return 6; }

const char *gdr_last_error_string(void) { return gdr::t_last_error_ptr(); }

int gdr_prepare_chunks(const int32_t *cu, int n_seqs, int chunk, int32_t *chunk_seq,
                       int32_t *chunk_start, int32_t *chunk_len, int max_chunks, int *n_chunks) {
  if (!cu || !n_chunks) return GDR_ERR_NULL;
  if (chunk <= 0 || max_chunks < 0) return GDR_ERR_SHAPE;
  int st = check_cu_seqlens(cu, n_seqs);
  if (st) return st;
  if (max_chunks > 0 && (!chunk_seq || !chunk_start || !chunk_len)) return GDR_ERR_NULL;
  int m = 0;
  for (int n = 0; n < n_seqs; ++n) {
    // number of chunks of sequence n, ceil(len / chunk)
    const int64_t len = static_cast<int64_t>(cu[n + 1]) - cu[n];
    const int64_t nc = (len + chunk - 1) / chunk;
    for (int64_t c = 0; c < nc; ++c) {
      if (m >= max_chunks) {
        *n_chunks = m;
        return GDR_ERR_SHAPE;
      }
      const int64_t start = cu[n] + c * chunk;
      const int64_t rest = cu[n + 1] - start;
      chunk_seq[m] = n;
      chunk_start[m] = static_cast<int32_t>(start);
      chunk_len[m] = static_cast<int32_t>(rest < chunk ? rest : chunk);
      ++m;
    }
  }
  *n_chunks = m;
  return GDR_OK;
}

int gdr_get_device_error(int *error_out, void *stream) {
  if (!error_out) return GDR_ERR_NULL;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int zero = 0, val = 0;
  cudaError_t e = cudaMemcpyFromSymbolAsync(&val, g_device_error, sizeof(int), 0,
                                            cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess)
    e = cudaMemcpyToSymbolAsync(g_device_error, &zero, sizeof(int), 0, cudaMemcpyHostToDevice, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return GDR_ERR_CUDA;
  *error_out = val;
  return GDR_OK;
}

int gdr_causal_conv(const void *x, const void *w, const void *conv_state_in, void *conv_state_out,
                    const int32_t *cu_dev, const int32_t *cu_host, int n_seqs, int channels, void *y,
                    void *stream) {
  clear_last_error();
  if (!cu_host) return GDR_ERR_NULL;
  int st = check_cu_seqlens(cu_host, n_seqs);
  if (st) return st;
  if (channels <= 0 || channels % 8 != 0) return GDR_ERR_SHAPE;
  const int total = n_seqs > 0 ? cu_host[n_seqs] : 0;
  if (n_seqs == 0) return GDR_OK;
  if (!cu_dev || !w) return GDR_ERR_NULL;
  if (total > 0 && (!x || !y)) return GDR_ERR_NULL;
  if (!aligned16(x) || !aligned16(w) || !aligned16(y) || !aligned16(conv_state_in) ||
      !aligned16(conv_state_out))
    return GDR_ERR_ALIGN;
  const size_t state_bytes = static_cast<size_t>(n_seqs) * 3 * channels * 2;
  if (overlaps(conv_state_in, state_bytes, conv_state_out, state_bytes)) return GDR_ERR_ALIAS;
  const size_t act_bytes = static_cast<size_t>(total) * channels * 2;
  if (overlaps(x, act_bytes, y, act_bytes)) return GDR_ERR_ALIAS;
  return launch_causal_conv(x, w, conv_state_in, conv_state_out, cu_dev, n_seqs, total, channels, y,
                            static_cast<cudaStream_t>(stream));
}

int gdr_gated_rmsnorm(const void *o, const void *z, const float *w, float eps, int64_t rows, int d,
                      void *y, void *stream) {
  clear_last_error();
  if (rows < 0) return GDR_ERR_SHAPE;
  if (d != kHeadDim) return GDR_ERR_UNSUPPORTED;
  if (rows == 0) return GDR_OK;
  if (!o || !z || !y) return GDR_ERR_NULL;
  if (!aligned16(o) || !aligned16(z) || !aligned16(y) || !aligned16(w)) return GDR_ERR_ALIGN;
  if (!(eps >= 0.0f)) return GDR_ERR_SHAPE;
  return launch_gated_rmsnorm(o, z, w, eps, rows, y, static_cast<cudaStream_t>(stream));
}

int gdr_decode_step(const void *x, const void *conv_w, void *conv_state, const void *a, const void *b,
                    const float *A_log, const float *dt_bias, float scale, int hk, int hv,
                    float *state, void *o, int batch, void *stream) {
  clear_last_error();
  int st = check_heads(hk, hv);
  if (st) return st;
  if (batch < 0) return GDR_ERR_SHAPE;
  if (batch == 0) return GDR_OK;
  if (!x || !conv_w || !conv_state || !a || !b || !A_log || !dt_bias || !state || !o)
    return GDR_ERR_NULL;
  if (!aligned16(x) || !aligned16(conv_w) || !aligned16(conv_state) || !aligned16(state) ||
      !aligned16(o))
    return GDR_ERR_ALIGN;
  return launch_decode(x, conv_w, conv_state, a, b, A_log, dt_bias, scale, hk, hv, state, nullptr, 0, o,
                       batch, static_cast<cudaStream_t>(stream));
}

int gdr_decode_step_slots(const void *x, const void *conv_w, void *conv_state_pool, const void *a,
                          const void *b, const float *A_log, const float *dt_bias, float scale, int hk,
                          int hv, float *state_pool, int n_slots, const int32_t *slot, void *o, int batch,
                          void *stream) {
  clear_last_error();
  int st = check_heads(hk, hv);
  if (st) return st;
  if (batch < 0 || n_slots < 0) return GDR_ERR_SHAPE;
  if (batch == 0) return GDR_OK;
  if (!x || !conv_w || !a || !b || !A_log || !dt_bias || !slot || !o) return GDR_ERR_NULL;
  // an empty pool makes every row a padding row; the pool pointers are then never read
  if (n_slots > 0 && (!conv_state_pool || !state_pool)) return GDR_ERR_NULL;
  if (!aligned16(x) || !aligned16(conv_w) || !aligned16(conv_state_pool) || !aligned16(state_pool) ||
      !aligned16(o) || (reinterpret_cast<uintptr_t>(slot) & 3u) != 0)
    return GDR_ERR_ALIGN;
  return launch_decode(x, conv_w, conv_state_pool, a, b, A_log, dt_bias, scale, hk, hv, state_pool, slot,
                       n_slots, o, batch, static_cast<cudaStream_t>(stream));
}

size_t gdr_chunk_prefill_workspace_size(int n_seqs, int hv, int window_chunks, int has_final_state) {
  if (n_seqs <= 0 || hv <= 0 || window_chunks <= 0) return 0;
  return chunk_prefill_workspace_bytes(n_seqs, hv, window_chunks, has_final_state == 0);
}

int gdr_linear(const void *x, const void *w, void *y, int64_t M, int64_t N, int64_t K, void *stream) {
  clear_last_error();
  if (M < 0 || N <= 0 || K <= 0 || M > (int64_t{1} << 31) || N > (int64_t{1} << 24) || K > (int64_t{1} << 31))
    return GDR_ERR_SHAPE;
  if (N % 8 != 0 || K % 8 != 0) return GDR_ERR_SHAPE;   // rows of whole 16-byte chunks
  if (M == 0) return GDR_OK;
  if (!x || !w || !y) return GDR_ERR_NULL;
  if (!aligned16(x) || !aligned16(w) || !aligned16(y)) return GDR_ERR_ALIGN;
  const size_t yb = static_cast<size_t>(M) * N * 2;
  if (overlaps(y, yb, x, static_cast<size_t>(M) * K * 2) || overlaps(y, yb, w, static_cast<size_t>(N) * K * 2))
    return GDR_ERR_ALIAS;
  return launch_linear(x, w, y, M, N, K, static_cast<cudaStream_t>(stream));
}

int gdr_chunk_prefill_schedule(const int32_t *cu_host, int n_seqs, int hv, size_t workspace_bytes,
                               int has_final_state, int *windows, int *pipelined) {
  clear_last_error();
  if (!cu_host || !windows || !pipelined) return GDR_ERR_NULL;
  if (hv <= 0 || n_seqs < 0 || (has_final_state != 0 && has_final_state != 1)) return GDR_ERR_SHAPE;
  int st = check_cu_seqlens(cu_host, n_seqs);
  if (st) return st;
  int max_chunks = 0;
  for (int i = 0; i < n_seqs; ++i) {
    const int nc = (cu_host[i + 1] - cu_host[i] + kChunk - 1) / kChunk;
    if (nc > max_chunks) max_chunks = nc;
  }
  int win = 1;
  bool pl = false;
  st = plan_chunk_prefill(n_seqs, hv, max_chunks, workspace_bytes, has_final_state == 0, false, windows, &win, &pl);
  if (st) return st;
  *pipelined = pl ? 1 : 0;
  return GDR_OK;
}

size_t gdr_chunk_prefill_fused_workspace_size(int n_seqs, int hk, int hv, int total_tokens, int window_chunks,
                                              int has_final_state) {
  if (n_seqs <= 0 || hk <= 0 || hv <= 0 || total_tokens < 0 || window_chunks <= 0) return 0;
  return fused_conv_bytes(total_tokens, (2 * hk + hv) * kHeadDim) +
         chunk_prefill_workspace_bytes(n_seqs, hv, window_chunks, has_final_state == 0);
}

int gdr_chunk_prefill(const void *q, const void *k, const void *v, int64_t qk_stride,
                      int64_t v_stride, const void *a, const void *b, const float *A_log,
                      const float *dt_bias, float scale, int hk, int hv, const int32_t *cu_dev,
                      const int32_t *cu_host, int n_seqs, const float *h0, float *hT, void *o,
                      const gdr_prefill_fuse_t *fuse, void *workspace, size_t workspace_bytes,
                      void *stream) {
  clear_last_error();
  int st = check_heads(hk, hv);
  if (st) return st;
  const bool fused_conv = fuse && fuse->x;
  const bool fused_norm = fuse && fuse->z;
  const int channels = (2 * hk + hv) * kHeadDim;
  if (fused_conv) {   // q, k, v are the conv output the call makes: rows of [q | k | v]
    if (q || k || v) return GDR_ERR_SHAPE;
    qk_stride = v_stride = channels;
  }
  if (qk_stride == 0) qk_stride = static_cast<int64_t>(hk) * kHeadDim;
  if (v_stride == 0) v_stride = static_cast<int64_t>(hv) * kHeadDim;
  if (qk_stride < static_cast<int64_t>(hk) * kHeadDim || v_stride < static_cast<int64_t>(hv) * kHeadDim)
    return GDR_ERR_SHAPE;
  if (qk_stride % 8 != 0 || v_stride % 8 != 0) return GDR_ERR_ALIGN;
  if (!cu_host) return GDR_ERR_NULL;
  st = check_cu_seqlens(cu_host, n_seqs);
  if (st) return st;
  if (n_seqs == 0) return GDR_OK;
  const int total = cu_host[n_seqs];
  const bool conv_state_out = fused_conv && fuse->conv_state_out;   // passes through empty sequences too
  if (total == 0 && !hT && !conv_state_out) return GDR_OK;   // nothing to compute, nothing to write
  if (!cu_dev) return GDR_ERR_NULL;
  if (fuse && !fuse->z && fuse->y) return GDR_ERR_NULL;   // y without the gate z
  if (fused_conv && !fuse->conv_w) return GDR_ERR_NULL;
  if (total > 0) {
    if (!a || !b || !A_log || !dt_bias) return GDR_ERR_NULL;
    if (!fused_conv && (!q || !k || !v)) return GDR_ERR_NULL;
    if (!o && !fused_norm) return GDR_ERR_NULL;
    if (fused_norm && !fuse->y) return GDR_ERR_NULL;
  }
  const void *z = fused_norm ? fuse->z : nullptr;
  void *y = fused_norm ? fuse->y : nullptr;
  const float *norm_w = fused_norm ? fuse->norm_w : nullptr;
  const float eps = fused_norm ? fuse->eps : 0.0f;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(h0) ||
      !aligned16(hT) || !aligned16(workspace) || !aligned16(z) || !aligned16(y) || !aligned16(norm_w))
    return GDR_ERR_ALIGN;
  if (fused_conv && (!aligned16(fuse->x) || !aligned16(fuse->conv_w) || !aligned16(fuse->conv_state_in) ||
                     !aligned16(fuse->conv_state_out)))
    return GDR_ERR_ALIGN;
  int max_chunks = 0;
  for (int i = 0; i < n_seqs; ++i) {
    const int nc = (cu_host[i + 1] - cu_host[i] + kChunk - 1) / kChunk;
    if (nc > max_chunks) max_chunks = nc;
  }
  const size_t state_bytes = static_cast<size_t>(n_seqs) * hv * kHeadDim * kHeadDim * 4;
  if (h0 != hT && overlaps(h0, state_bytes, hT, state_bytes)) return GDR_ERR_ALIAS;
  // with the conv fused its output comes first in the workspace, then the chunk records
  const size_t conv_bytes = fused_conv ? fused_conv_bytes(total, channels) : 0;
  const size_t rec_bytes = max_chunks > 0 ? chunk_prefill_workspace_bytes(n_seqs, hv, 1, hT == nullptr) : 0;
  if ((conv_bytes | rec_bytes) != 0 && (!workspace || workspace_bytes < conv_bytes + rec_bytes))
    return GDR_ERR_WORKSPACE;
  if (fused_conv) {
    const size_t cs_bytes = static_cast<size_t>(n_seqs) * 3 * channels * 2;
    const size_t x_bytes = static_cast<size_t>(total) * channels * 2;
    if (overlaps(fuse->conv_state_in, cs_bytes, fuse->conv_state_out, cs_bytes) ||
        overlaps(fuse->x, x_bytes, workspace, conv_bytes))
      return GDR_ERR_ALIAS;
  }
  if (fused_norm && o) {   // o and y are separate outputs
    const size_t out_bytes = static_cast<size_t>(total) * hv * kHeadDim * 2;
    if (overlaps(o, out_bytes, y, out_bytes)) return GDR_ERR_ALIAS;
  }
  if (fused_conv) {
    uint8_t *conv_out = static_cast<uint8_t *>(workspace);
    st = launch_causal_conv(fuse->x, fuse->conv_w, fuse->conv_state_in, fuse->conv_state_out, cu_dev, n_seqs,
                            total, channels, conv_out, static_cast<cudaStream_t>(stream));
    if (st) return st;
    if (total == 0 && !hT) return GDR_OK;
    q = conv_out;
    k = conv_out + static_cast<size_t>(hk) * kHeadDim * 2;
    v = conv_out + static_cast<size_t>(2 * hk) * kHeadDim * 2;
    workspace = conv_out + conv_bytes;
    workspace_bytes -= conv_bytes;
  }
  return launch_chunk_prefill(q, k, v, qk_stride, v_stride, a, b, A_log, dt_bias, scale, hk, hv,
                              cu_dev, cu_host, n_seqs, total, max_chunks, h0, hT, o, z, norm_w, eps, y, workspace,
                              workspace_bytes, static_cast<cudaStream_t>(stream));
}

int gdr_chunk_prefill_slots(const void *q, const void *k, const void *v, int64_t qk_stride, int64_t v_stride,
                            const void *a, const void *b, const float *A_log, const float *dt_bias, float scale,
                            int hk, int hv, const int32_t *cu_dev, const int32_t *cu_host, int n_seqs,
                            float *state_pool, int n_slots, const int32_t *slot, int init_from_pool, void *o,
                            void *workspace, size_t workspace_bytes, void *stream) {
  clear_last_error();
  int st = check_heads(hk, hv);
  if (st) return st;
  if (n_slots < 0 || (init_from_pool != 0 && init_from_pool != 1)) return GDR_ERR_SHAPE;
  if (qk_stride == 0) qk_stride = static_cast<int64_t>(hk) * kHeadDim;
  if (v_stride == 0) v_stride = static_cast<int64_t>(hv) * kHeadDim;
  if (qk_stride < static_cast<int64_t>(hk) * kHeadDim || v_stride < static_cast<int64_t>(hv) * kHeadDim)
    return GDR_ERR_SHAPE;
  if (qk_stride % 8 != 0 || v_stride % 8 != 0) return GDR_ERR_ALIGN;
  if (!cu_host) return GDR_ERR_NULL;
  st = check_cu_seqlens(cu_host, n_seqs);
  if (st) return st;
  if (n_seqs == 0) return GDR_OK;
  if (!cu_dev || !slot) return GDR_ERR_NULL;
  if (n_slots > 0 && !state_pool) return GDR_ERR_NULL;
  const int total = cu_host[n_seqs];
  if (total > 0 && (!q || !k || !v || !a || !b || !A_log || !dt_bias || !o)) return GDR_ERR_NULL;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(state_pool) ||
      !aligned16(workspace) || (reinterpret_cast<uintptr_t>(slot) & 3u) != 0)
    return GDR_ERR_ALIGN;
  int max_chunks = 0;
  for (int i = 0; i < n_seqs; ++i) {
    const int nc = (cu_host[i + 1] - cu_host[i] + kChunk - 1) / kChunk;
    if (nc > max_chunks) max_chunks = nc;
  }
  // the records of a one-chunk window and the carry of sequences without an entry
  const size_t rec_bytes = max_chunks > 0 ? chunk_prefill_workspace_bytes(n_seqs, hv, 1, true) : 0;
  if (rec_bytes != 0 && (!workspace || workspace_bytes < rec_bytes)) return GDR_ERR_WORKSPACE;
  if (n_slots == 0 && total == 0) return GDR_OK;   // no entry to write, nothing to compute
  PrefillPool pool{state_pool, n_slots, slot, init_from_pool};
  return launch_chunk_prefill(q, k, v, qk_stride, v_stride, a, b, A_log, dt_bias, scale, hk, hv, cu_dev, cu_host,
                              n_seqs, total, max_chunks, nullptr, nullptr, o, nullptr, nullptr, 0.0f, nullptr,
                              workspace, workspace_bytes, static_cast<cudaStream_t>(stream), &pool);
}

}  // extern "C"
