// prefill_noalloc.cu -- gdr_chunk_prefill for callers that cannot allocate.
//
// gdr_chunk_prefill needs a device workspace from its caller.  Some callers
// have no way to provide one: a plugin whose host framework owns all device
// memory and hands out no scratch buffers, a fixed-budget deployment that
// must not grow its footprint at run time, or code that runs where CUDA API
// calls such as cudaMalloc are not permitted (a host function enqueued on a
// stream, for instance).  This entry point runs the same kernels on a scratch
// area that is part of the library image itself: a file-scope __device__
// array that every GPU which loads the library holds for the life of the
// process.
#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>
#include <mutex>

#include "gdr_common.cuh"
#include "gdr_host.h"

namespace gdr {
namespace {

// 32 MiB: a one-chunk window for up to 8 sequences of 48 value heads, or an
// eight-chunk window for one sequence.
constexpr size_t kNoAllocScratchBytes = size_t{32} << 20;
static __device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocScratchBytes];

// device address of the scratch on each device, as last looked up
std::atomic<void *> g_scratch_addr[64];
std::mutex g_scratch_mutex;

// The address is looked up again on every call made outside stream capture (the
// lookup is cheap, and a device reset or a new primary context may move the
// module); a call made while the stream is being captured uses the address of
// the last call made outside capture, since capture forbids the lookup.
int scratch_for_current_device(cudaStream_t stream, void **out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return launch_status(e, "prefill (no-alloc): cudaGetDevice");
  if (dev < 0 || dev >= 64) return GDR_ERR_UNSUPPORTED;
  cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
  e = cudaStreamIsCapturing(stream, &cap);
  if (e != cudaSuccess) return launch_status(e, "prefill (no-alloc): cudaStreamIsCapturing");
  if (cap != cudaStreamCaptureStatusNone) {
    void *p = g_scratch_addr[dev].load(std::memory_order_acquire);
    if (!p) {
      set_last_error("prefill (no-alloc): first call on this device made during stream capture; "
                     "make one call outside capture first",
                     cudaSuccess);
      return GDR_ERR_UNSUPPORTED;
    }
    *out = p;
    return GDR_OK;
  }
  std::lock_guard<std::mutex> lock(g_scratch_mutex);
  void *p = nullptr;
  // the symbol's name is a host stand-in; the device address comes from here
  e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
  if (e != cudaSuccess || !p) return launch_status(e, "prefill (no-alloc): cudaGetSymbolAddress");
  g_scratch_addr[dev].store(p, std::memory_order_release);
  *out = p;
  return GDR_OK;
}

}  // namespace
}  // namespace gdr

using namespace gdr;

extern "C" {

size_t gdr_chunk_prefill_noalloc_scratch_bytes(void) { return kNoAllocScratchBytes; }

int gdr_chunk_prefill_noalloc(const void *q, const void *k, const void *v, int64_t qk_token_stride,
                              int64_t v_token_stride, const void *a, const void *b, const float *A_log,
                              const float *dt_bias, float scale, int hk, int hv,
                              const int32_t *cu_seqlens_dev, const int32_t *cu_seqlens_host, int n_seqs,
                              const float *h0, float *hT, void *o, void *stream) {
  clear_last_error();
  if (n_seqs > 0 && hv > 0 &&
      chunk_prefill_workspace_bytes(n_seqs, hv, 1, hT == nullptr) > kNoAllocScratchBytes) {
    set_last_error("prefill (no-alloc): the 32 MiB scratch cannot hold a one-chunk window for "
                   "this many sequences and value heads",
                   cudaSuccess);
    return GDR_ERR_WORKSPACE;
  }
  void *scratch = nullptr;
  int st = scratch_for_current_device(static_cast<cudaStream_t>(stream), &scratch);
  if (st) return st;
  // the scratch needs no initialisation: every record is written before it is read
  return gdr_chunk_prefill(q, k, v, qk_token_stride, v_token_stride, a, b, A_log, dt_bias, scale, hk,
                           hv, cu_seqlens_dev, cu_seqlens_host, n_seqs, h0, hT, o, nullptr, scratch,
                           kNoAllocScratchBytes, stream);
}

}  // extern "C"
