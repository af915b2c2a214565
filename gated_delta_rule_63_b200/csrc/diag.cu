// diag.cu -- a self-test of the kernels' bounded waits.
//
// Every wait of the library's kernels on an mbarrier is bounded: when the
// bound runs out the kernel records GDR_ERR_TIMEOUT in the device error word,
// lets its own copies finish, releases its tensor memory and returns, so the
// context stays usable.  gdr_debug_wait_timeout runs that path on purpose: one
// CTA holds tensor memory and waits, with a short bound, on an mbarrier that
// nothing ever arrives at, using the same wait helpers as the kernels (no copy
// and no MMA is in flight).
#include <cuda_runtime.h>
#include <stdint.h>

#include "gdr_common.cuh"
#include "gdr_host.h"

namespace gdr {
namespace {

constexpr uint32_t kDiagTmemCols = 32;

__global__ void __launch_bounds__(128, 1) wait_timeout_kernel(int kind, unsigned long long limit, int *err,
                                                              int *result) {
  __shared__ __align__(8) uint64_t bar_storage;
  __shared__ uint32_t tmem_holder;
  __shared__ uint32_t abort_flag;
  const uint32_t bar = smem_u32(&bar_storage);
  const int tid = threadIdx.x;
  if (tid == 0) {
    mbar_init(bar, 1);   // one arrival expected; none ever comes
    abort_flag = 0u;
    fence_mbar_init();
  }
  if (tid < 32) {
    tmem_alloc(smem_u32(&tmem_holder), kDiagTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  bool ok = true;
  if (kind == 0) {
    // the poll-count bound of the prep, decode and conv kernels (one thread waits)
    if (tid == 0) ok = mbar_wait(bar, 0, err, static_cast<uint32_t>(limit));
  } else {
    // the clock bound of the state chain: every warp waits and all give up together
    ok = chain_wait(bar, 0, &abort_flag, err, static_cast<long long>(limit));
  }
  ok = __syncthreads_and(ok) != 0;
  if (tid == 0) *result = ok ? 1 : 0;
  tc_fence_before();
  __syncthreads();
  if (tid < 32) tmem_dealloc(tmem_holder, kDiagTmemCols);
}

}  // namespace
}  // namespace gdr

using namespace gdr;

extern "C" int gdr_debug_wait_timeout(int kind, unsigned long long limit, int *result_dev, void *stream) {
  clear_last_error();
  if (!result_dev) return GDR_ERR_NULL;
  if ((kind != 0 && kind != 1) || limit == 0 || limit > (1ull << 31)) return GDR_ERR_SHAPE;
  wait_timeout_kernel<<<1, 128, 0, static_cast<cudaStream_t>(stream)>>>(kind, limit, device_error_ptr(), result_dev);
  return last_launch_status("debug wait timeout: kernel launch");
}
