// linear.cu -- the layer's projections, y = x W^T, on tcgen05 tensor cores.
//
// "33B 只做 18 层 ..." (yfxerp.com) §2 parameter table: a gated delta-rule layer
// projects the hidden state (5120) to q|k|v (10 240 = 2 x 16 x 128 + 48 x 128),
// z (6144), a and b (48 each), and the gated norm's output (6144) back to 5120.
// Each is a dense bf16 product y[m][n] = sum_k x[m][k] W[n][k] (the weight stored
// [out][in], both operands K-major), accumulated in fp32 and rounded to bf16.
//
// Persistent: one CTA per SM takes 128 x 256 output tiles in turn, M-fastest, so
// the CTAs resident together share a few weight tiles and the activations stay in
// L2.  Lane 0 of warp 0 streams the A (128 x 64) and B (256 x 64) tiles of every
// 64-wide K step of every tile it takes into a four-stage shared-memory ring with
// TMA; lane 0 of warp 1 issues four M = 128, N = 256, K = 16 MMAs per step into one
// of two 256-column fp32 TMEM accumulators (tiles alternate) and releases each
// stage with a commit; warps 2..5 (one per TMEM lane quarter) read a finished
// accumulator, store its bf16 rows and hand it back, while the next tile's MMAs
// run on the other.  Rows and columns past M, N and K load as zero (TMA) and are
// not stored.

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <algorithm>
#include <atomic>

#include "gdr_common.cuh"
#include "gdr_host.h"

namespace gdr {
namespace {

constexpr int kLinThreads = 192;             // warp 0 copies, warp 1 products, warps 2..5 epilogue
constexpr int LM = 128, LN = 256, LK = 64;   // output tile, K step (64 bf16 = one 128-byte row)
constexpr int kStages = 4;
constexpr uint32_t L_A = LM * 128;           // bytes of an A tile (128 rows x 128 B)
constexpr uint32_t L_B = LN * 128;           // bytes of a B tile (256 rows x 128 B)
constexpr uint32_t L_STAGE = L_A + L_B;
constexpr uint32_t L_OFF_BAR = kStages * L_STAGE;   // full x 4, empty x 4, acc_full x 2, acc_empty x 2, drain
constexpr uint32_t L_SMEM = L_OFF_BAR + 128 + 1024;
static_assert(L_SMEM <= 232448, "linear shared memory exceeds 227 KB");
constexpr uint32_t L_TM_COLS = 512;                 // two 256-column accumulators

struct LinearParams {
  int64_t M, N, K;
  int tiles_m, tiles;
  uint16_t *y;
  int *err;
};

__global__ void __launch_bounds__(kLinThreads, 1)
linear_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_w,
              const __grid_constant__ LinearParams p) {
  grid_dep_wait();
  grid_dep_launch();
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  const uint32_t sbase = (raw_addr + 1023u) & ~1023u;
  uint8_t *smem = smem_raw + (sbase - raw_addr);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int nk = static_cast<int>((p.K + LK - 1) / LK);
  const uint32_t full = sbase + L_OFF_BAR, empty = full + 8 * kStages;
  const uint32_t acc_full = empty + 8 * kStages, acc_empty = acc_full + 16;   // + 8 * buffer
  const uint32_t drain = acc_empty + 16;
  uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(smem + L_OFF_BAR + 8 * (2 * kStages + 5));
  volatile uint32_t *abort_flag =
      reinterpret_cast<volatile uint32_t *>(smem + L_OFF_BAR + 8 * (2 * kStages + 5) + 4);

  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(full + 8 * s, 1);
      mbar_init(empty + 8 * s, 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(acc_full + 8 * b, 1);
      mbar_init(acc_empty + 8 * b, 4);   // the four epilogue warps
    }
    mbar_init(drain, 1);
    *abort_flag = 0u;
    fence_mbar_init();
    tma_prefetch_desc(&tm_x);
    tma_prefetch_desc(&tm_w);
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(tmem_holder), L_TM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;

  if (warp == 0) {
    if (lane == 0) {
      // ---- producer: K step g (counted over all the CTA's tiles) into stage g % 4 once the
      // MMAs of step g - 4 have read it
      int g = 0, issued = 0;
      bool go = true;
      for (int t = blockIdx.x; t < p.tiles && go; t += gridDim.x) {
        const int32_t m0 = (t % p.tiles_m) * LM, n0 = (t / p.tiles_m) * LN;
        for (int ks = 0; ks < nk; ++ks, ++g) {
          const int s = g % kStages;
          if (g >= kStages && !chain_wait(empty + 8 * s, ((g / kStages) - 1) & 1, abort_flag, p.err)) {
            go = false;
            break;
          }
          const uint32_t st = sbase + s * L_STAGE;
          mbar_arrive_expect_tx(full + 8 * s, L_STAGE);
          tma_load_2d(st, &tm_x, ks * LK, m0, full + 8 * s);
          tma_load_2d(st + L_A, &tm_w, ks * LK, n0, full + 8 * s);
          issued = g + 1;
        }
      }
      // after a timeout the consumer stops: the copies in flight land before the CTA leaves
      // (every earlier copy into a stage was consumed before the stage was refilled)
      for (int c = (issued > kStages ? issued - kStages : 0); c < issued; ++c)
        mbar_wait(full + 8 * (c % kStages), (c / kStages) & 1, p.err, 1u << 16);
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0) {
      // ---- MMA issuer: tile i of this CTA into accumulator i & 1, once the epilogue has
      // handed back that accumulator's tile i - 2
      const uint32_t id = idesc_bf16(LM, LN, false, false);
      int g = 0, i = 0;
      bool go = true;
      for (int t = blockIdx.x; t < p.tiles && go; t += gridDim.x, ++i) {
        const int b = i & 1;
        if (i >= 2 && !chain_wait(acc_empty + 8 * b, ((i >> 1) - 1) & 1, abort_flag, p.err)) break;
        tc_fence_after();
        const uint32_t d = tmem + b * LN;
        for (int ks = 0; ks < nk; ++ks, ++g) {
          const int s = g % kStages;
          if (!chain_wait(full + 8 * s, (g / kStages) & 1, abort_flag, p.err)) {
            go = false;
            break;
          }
          tc_fence_after();
          const uint32_t st = sbase + s * L_STAGE;
#pragma unroll
          for (int kk = 0; kk < LK / 16; ++kk)
            mma_bf16(d, sdesc(st + kk * 32, 16, 1024), sdesc(st + L_A + kk * 32, 16, 1024), id, (ks | kk) != 0);
          mma_commit(empty + 8 * s);
        }
        mma_commit(acc_full + 8 * b);   // the tile's products (or those before a timeout) are done
      }
      mma_commit(drain);   // every product issued is complete before tensor memory is released
      mbar_wait(drain, 0, p.err, 1u << 20);
    }
    __syncwarp();
  } else {
    // ---- epilogue: warp w reads TMEM lane quarter w & 3 (tile rows 32 (w & 3) .. + 31) ----
    const int q = warp & 3;
    int i = 0;
    for (int t = blockIdx.x; t < p.tiles; t += gridDim.x, ++i) {
      const int b = i & 1;
      if (!chain_wait(acc_full + 8 * b, (i >> 1) & 1, abort_flag, p.err)) break;
      __syncwarp();
      tc_fence_after();
      const int64_t m = static_cast<int64_t>(t % p.tiles_m) * LM + 32 * q + lane;
      const int64_t n0 = static_cast<int64_t>(t / p.tiles_m) * LN;
      const uint32_t tl = tmem + (static_cast<uint32_t>(32 * q) << 16) + b * LN;
#pragma unroll 1
      for (int c = 0; c < LN / 32; ++c) {
        float v[32];
        tmem_ld32(tl + 32 * c, v);
        tmem_wait_ld();
        const int64_t n = n0 + 32 * c;
        if (m < p.M) {
          uint16_t *dst = p.y + m * p.N + n;
#pragma unroll
          for (int r = 0; r < 4; ++r)
            if (n + 8 * r < p.N) *reinterpret_cast<uint4 *>(dst + 8 * r) = pack8x2(v + 8 * r);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(acc_empty + 8 * b);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, L_TM_COLS);
}

bool make_map_box(CUtensorMap *m, const void *base, uint64_t cols, uint64_t rows, uint64_t row_stride,
                  uint32_t box_rows) {
  EncodeTiledFn f = tensor_map_encoder();
  if (!f) return false;
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {row_stride * 2};
  const cuuint32_t box[2] = {static_cast<cuuint32_t>(LK), box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return f(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides, box, estr,
           CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
           CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

int launch_linear(const void *x, const void *w, void *y, int64_t M, int64_t N, int64_t K, cudaStream_t s) {
  static std::atomic<uint64_t> done{0};
  static std::atomic<int> sm_count[64];
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return launch_status(e, "linear: cudaGetDevice");
  if (dev < 0 || dev >= 64) return GDR_ERR_UNSUPPORTED;
  const uint64_t bit = uint64_t{1} << dev;
  if (!(done.load(std::memory_order_acquire) & bit)) {
    int sms = 0;
    e = cudaFuncSetAttribute(linear_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, L_SMEM);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return launch_status(e, "linear: set-up");
    sm_count[dev].store(sms, std::memory_order_relaxed);
    done.fetch_or(bit, std::memory_order_acq_rel);
  }
  if (!tensor_map_encoder()) return launch_status(cudaErrorSymbolNotFound, "linear: cuTensorMapEncodeTiled lookup");
  CUtensorMap tx, tw;
  if (!make_map_box(&tx, x, static_cast<uint64_t>(K), static_cast<uint64_t>(M), static_cast<uint64_t>(K), LM) ||
      !make_map_box(&tw, w, static_cast<uint64_t>(K), static_cast<uint64_t>(N), static_cast<uint64_t>(K), LN))
    return launch_status(cudaErrorInvalidValue, "linear: tensor map encoding");
  LinearParams p;
  p.M = M;
  p.N = N;
  p.K = K;
  p.tiles_m = static_cast<int>((M + LM - 1) / LM);
  const int64_t tiles = static_cast<int64_t>(p.tiles_m) * ((N + LN - 1) / LN);
  if (tiles > (int64_t{1} << 31) - 1) return GDR_ERR_SHAPE;
  p.tiles = static_cast<int>(tiles);
  p.y = static_cast<uint16_t *>(y);
  p.err = device_error_ptr();
  const int grid = static_cast<int>(std::min<int64_t>(tiles, sm_count[dev].load(std::memory_order_relaxed)));
  return launch_status(launch_pdl(linear_kernel, dim3(grid), dim3(kLinThreads), L_SMEM, s, 1, tx, tw, p),
                       "linear: kernel launch");
}

}  // namespace gdr
