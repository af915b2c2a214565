// conv.cu -- depthwise causal conv (kernel 4) + SiLU over packed sequences.
//
// "Agnes-3.0-Flash 深度解析：33B 混合注意力多模态模型", 注意力层的细节: a
// kernel-4 causal conv sits in front of the recurrence.  y[t][c] =
// SiLU(sum_j w[c][j] x[t-3+j][c]), fp32 math, bf16 output; inputs before a
// sequence start come from the conv state (oldest first) or are zero.
//
// Memory-bound stencil.  The input is cut into tiles of 64 tokens x 128
// channels; a tile and its 3-row halo (67 rows x 256 bytes) arrive in shared
// memory by one TMA copy.  CTAs are persistent (five per SM) and keep two
// tiles in flight: while one tile is computed the next is loading, so the
// SM's copies stream continuously and x is read from HBM once (the halo rows
// are L2 hits).  Each thread computes 8 channels (one 16-byte vector) of 8
// tokens from a sliding window of unpacked rows and writes y with coalesced
// 16-byte stores.
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <algorithm>
#include <atomic>

#include "gdr_common.cuh"
#include "gdr_host.h"

namespace gdr {
namespace {

constexpr int kThreads = 128;                 // 16 channel groups x 8 token groups
constexpr int kTileT = 64;                    // tokens per tile
constexpr int kTileC = 128;                   // channels per tile
constexpr int kRows = kTileT + 3;             // with the 3-row halo
constexpr uint32_t kRowBytes = kTileC * 2;    // 256
constexpr uint32_t kBufBytes = kRows * kRowBytes;
constexpr int kBufs = 2;                      // tiles in flight per CTA
constexpr int kCtasPerSm = 5;
constexpr uint32_t kSmem = kBufs * kBufBytes + 1024;   // tile buffers, 1 KB alignment slack

struct ConvParams {
  const uint16_t *w;
  const uint16_t *cs_in;
  uint16_t *cs_out;
  const int32_t *cu;
  uint16_t *y;
  int n_seqs;
  int total;
  int channels;
  int n_ctiles;   // channel tiles
  int n_tiles;    // channel tiles x token tiles
  int *err;
};

// SiLU of a pair of values, x / (1 + e^-x), with e^-x = 2^(-x log2 e) from the MUFU's base-2
// exponential and the quotient from its reciprocal; the multiplies and the add run two-wide.
// Very negative x gives an infinite exponential, a zero reciprocal and a signed zero, the limit.
__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ float rcp_approx(float x) {
  float y;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ float2 silu2(float2 x) {
  constexpr float kNegLog2e = -1.4426950408889634f;   // -log2(e)
  const float2 t = __fmul2_rn(x, make_float2(kNegLog2e, kNegLog2e));
  const float2 d = __fadd2_rn(make_float2(ex2_approx(t.x), ex2_approx(t.y)), make_float2(1.0f, 1.0f));
  return __fmul2_rn(x, make_float2(rcp_approx(d.x), rcp_approx(d.y)));
}
// 8 bf16 (one 16-byte vector) as four pairs of floats
__device__ __forceinline__ void unpack8x2(const uint4 &u, float2 *f) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) f[i] = make_float2(__uint_as_float(w[i] << 16), __uint_as_float(w[i] & 0xFFFF0000u));
}

// sequence containing token t: largest n with cu[n] <= t (skipping empty ones)
__device__ int seq_of(const int32_t *cu, int n_seqs, int t) {
  int lo = 0, hi = n_seqs - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (__ldg(cu + mid) <= t) lo = mid; else hi = mid - 1;
  }
  return lo;
}

__device__ __forceinline__ void load_tile(const CUtensorMap *tm, uint32_t dst, uint32_t bar, int tile,
                                          const ConvParams &p) {
  const int ct = tile % p.n_ctiles, tt = tile / p.n_ctiles;
  mbar_arrive_expect_tx(bar, kBufBytes);
  // rows before token 0 and past the last token read as zero
  tma_load_2d(dst, tm, ct * kTileC, tt * kTileT - 3, bar);
}

__global__ void __launch_bounds__(kThreads, kCtasPerSm)
causal_conv_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ ConvParams p) {
  grid_dep_wait();
  grid_dep_launch();
  extern __shared__ uint8_t smem_raw[];
  __shared__ alignas(8) uint64_t s_bar[kBufs];
  const uint32_t sbase = (smem_u32(smem_raw) + 1023u) & ~1023u;
  const int tid = threadIdx.x;
  const int C = p.channels;
  const uint32_t bar0 = smem_u32(&s_bar[0]);

  if (tid == 0) {
    for (int i = 0; i < kBufs; ++i) mbar_init(bar0 + 8 * i, 1);
    fence_mbar_init();
    tma_prefetch_desc(&tm_x);
    for (int i = 0; i < kBufs; ++i) {
      const int tile = blockIdx.x + i * gridDim.x;
      if (tile < p.n_tiles) load_tile(&tm_x, sbase + i * kBufBytes, bar0 + 8 * i, tile, p);
    }
  }
  // empty sequences: their conv state passes through unchanged (first CTA)
  if (blockIdx.x == 0 && p.cs_out) {
    for (int n = 0; n < p.n_seqs; ++n) {
      if (__ldg(p.cu + n + 1) != __ldg(p.cu + n)) continue;
      for (int c = tid * 8; c < C; c += kThreads * 8)
        for (int s = 0; s < 3; ++s) {
          const size_t at = (static_cast<size_t>(n) * 3 + s) * C + c;
          uint4 v = make_uint4(0, 0, 0, 0);
          if (p.cs_in) v = *reinterpret_cast<const uint4 *>(p.cs_in + at);
          *reinterpret_cast<uint4 *>(p.cs_out + at) = v;
        }
    }
  }
  __syncthreads();   // barriers initialised

  const int cg = tid & 15, tg = tid >> 4;   // channel group, token group
  int k = 0;
  for (int tile = blockIdx.x; tile < p.n_tiles; tile += gridDim.x, ++k) {
    const int buf = k % kBufs;
    const uint32_t parity = (k / kBufs) & 1;
    const int ct = tile % p.n_ctiles, tt = tile / p.n_ctiles;
    const int c0 = ct * kTileC + cg * 8;          // first channel of this thread
    const int row0 = tt * kTileT - 3;             // token of tile row 0
    const int tb = tt * kTileT + tg * 8;          // first token of this thread
    const uint32_t tbuf = sbase + buf * kBufBytes + cg * 16;
    const bool ok = mbar_wait(bar0 + 8 * buf, parity, p.err);
    if (ok && c0 < C && tb < p.total) {
      float2 w[4][4];   // tap j, channel pair cp
      {   // w is [C][4]: channels c0..c0+7 occupy 32 contiguous bf16
        const uint4 *wp = reinterpret_cast<const uint4 *>(p.w + static_cast<size_t>(c0) * 4);
        float tmp[32];
#pragma unroll
        for (int i = 0; i < 4; ++i) unpack8(__ldg(wp + i), tmp + 8 * i);
#pragma unroll
        for (int cp = 0; cp < 4; ++cp)
#pragma unroll
          for (int j = 0; j < 4; ++j) w[j][cp] = make_float2(tmp[8 * cp + j], tmp[8 * cp + 4 + j]);
      }
      // sum_j w_j x_j in tap order (a product, then three fused multiply-adds), then SiLU
      auto conv2 = [&](const float2 &x0, const float2 &x1, const float2 &x2, const float2 &x3, int cp) {
        float2 acc = __fmul2_rn(w[0][cp], x0);
        acc = __ffma2_rn(w[1][cp], x1, acc);
        acc = __ffma2_rn(w[2][cp], x2, acc);
        acc = __ffma2_rn(w[3][cp], x3, acc);
        return silu2(acc);
      };
      auto row = [&](int t) { return ld_shared16(tbuf + (t - row0) * kRowBytes); };   // token t's 8 inputs
      int n = seq_of(p.cu, p.n_seqs, tb);
      int seq_start = __ldg(p.cu + n), seq_end = __ldg(p.cu + n + 1);
      if (tb - 3 >= seq_start && tb + 8 < seq_end) {
        // ---- inside one sequence, not its last token: no state, no boundary ----
        float2 xw[4][4];   // sliding window of 4 token rows, channel pairs
#pragma unroll
        for (int j = 0; j < 3; ++j) unpack8x2(row(tb - 3 + j), xw[j]);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          unpack8x2(row(tb + i), xw[(i + 3) & 3]);
          float out[8];
#pragma unroll
          for (int cp = 0; cp < 4; ++cp) {
            const float2 y2 = conv2(xw[i & 3][cp], xw[(i + 1) & 3][cp], xw[(i + 2) & 3][cp], xw[(i + 3) & 3][cp], cp);
            out[2 * cp] = y2.x;
            out[2 * cp + 1] = y2.y;
          }
          *reinterpret_cast<uint4 *>(p.y + static_cast<size_t>(tb + i) * C + c0) = pack8x2(out);
        }
      } else {
        // ---- sequence starts / ends among these tokens ----
        const int te = min(tb + 8, p.total);
#pragma unroll 1
        for (int t = tb; t < te; ++t) {
          while (t >= seq_end) {   // next non-empty sequence
            ++n;
            seq_start = __ldg(p.cu + n);
            seq_end = __ldg(p.cu + n + 1);
          }
          // input at position pos of sequence n: the tile row, or the conv state before the start
          auto tap = [&](int pos) {
            if (pos >= seq_start) return row(pos);
            if (p.cs_in)   // 1..3 positions before the start: the conv state, oldest first
              return *reinterpret_cast<const uint4 *>(
                  p.cs_in + (static_cast<size_t>(n) * 3 + (3 - (seq_start - pos))) * C + c0);
            return make_uint4(0, 0, 0, 0);
          };
          float2 xv[4][4];
#pragma unroll
          for (int j = 0; j < 4; ++j) unpack8x2(tap(t - 3 + j), xv[j]);
          float out[8];
#pragma unroll
          for (int cp = 0; cp < 4; ++cp) {
            const float2 y2 = conv2(xv[0][cp], xv[1][cp], xv[2][cp], xv[3][cp], cp);
            out[2 * cp] = y2.x;
            out[2 * cp + 1] = y2.y;
          }
          *reinterpret_cast<uint4 *>(p.y + static_cast<size_t>(t) * C + c0) = pack8x2(out);
          if (t == seq_end - 1 && p.cs_out) {   // last token: the last three inputs are the new conv state
#pragma unroll
            for (int s = 0; s < 3; ++s)
              *reinterpret_cast<uint4 *>(p.cs_out + (static_cast<size_t>(n) * 3 + s) * C + c0) = tap(t - 2 + s);
          }
        }
      }
    }
    __syncthreads();   // every thread is done with this buffer
    if (tid == 0) {
      const int next = tile + kBufs * gridDim.x;
      if (next < p.n_tiles) load_tile(&tm_x, sbase + buf * kBufBytes, bar0 + 8 * buf, next, p);
    }
  }
}

int conv_grid(int n_tiles) {
  static std::atomic<int> sms[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return -1;
  int n = dev >= 0 && dev < 64 ? sms[dev].load(std::memory_order_relaxed) : 0;
  if (n == 0) {
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) return -1;
    if (dev >= 0 && dev < 64) sms[dev].store(n, std::memory_order_relaxed);
  }
  return std::max(1, std::min(n_tiles, n * kCtasPerSm));
}

}  // namespace

int launch_causal_conv(const void *x, const void *w, const void *cs_in, void *cs_out,
                       const int32_t *cu_dev, int n_seqs, int total, int channels, void *y,
                       cudaStream_t s) {
  static std::atomic<uint64_t> attr_done{0};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return launch_status(e, "conv: cudaGetDevice");
  const uint64_t bit = dev >= 0 && dev < 64 ? (uint64_t{1} << dev) : 0;
  if (!bit || !(attr_done.load(std::memory_order_acquire) & bit)) {
    e = cudaFuncSetAttribute(causal_conv_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(causal_conv_kernel, cudaFuncAttributePreferredSharedMemoryCarveout,
                               cudaSharedmemCarveoutMaxShared);
    if (e != cudaSuccess) return launch_status(e, "conv: shared memory opt-in");
    attr_done.fetch_or(bit, std::memory_order_acq_rel);
  }
  ConvParams p;
  p.w = static_cast<const uint16_t *>(w);
  p.cs_in = static_cast<const uint16_t *>(cs_in);
  p.cs_out = static_cast<uint16_t *>(cs_out);
  p.cu = cu_dev;
  p.y = static_cast<uint16_t *>(y);
  p.n_seqs = n_seqs;
  p.total = total;
  p.channels = channels;
  p.n_ctiles = (channels + kTileC - 1) / kTileC;
  const int64_t n_tiles = static_cast<int64_t>(p.n_ctiles) * ((total + kTileT - 1) / kTileT);
  if (n_tiles > 0x7FFFFFFF) return GDR_ERR_SHAPE;
  p.n_tiles = static_cast<int>(n_tiles);
  p.err = device_error_ptr();
  // x as [total rows][channels] bf16; boxes of 67 rows x 128 channels, no swizzle;
  // with no tokens no tile is loaded and the weights serve as a base address
  EncodeTiledFn enc = tensor_map_encoder();
  if (!enc) return launch_status(cudaErrorSymbolNotFound, "conv: cuTensorMapEncodeTiled lookup");
  CUtensorMap tm;
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(channels), static_cast<cuuint64_t>(total > 0 ? total : 1)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(channels) * 2};
  const cuuint32_t box[2] = {kTileC, kRows};
  const cuuint32_t estr[2] = {1, 1};
  if (enc(&tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(total > 0 ? x : w), dims, strides, box,
          estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return launch_status(cudaErrorInvalidValue, "conv: tensor map encoding");
  const int grid = conv_grid(p.n_tiles);
  if (grid < 0) return launch_status(cudaErrorInvalidDevice, "conv: SM count");
  return launch_status(launch_pdl(causal_conv_kernel, dim3(grid), dim3(kThreads), kSmem, s, 1, tm, p),
                       "conv: kernel launch");
}

}  // namespace gdr
