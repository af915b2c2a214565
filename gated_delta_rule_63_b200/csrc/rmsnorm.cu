// rmsnorm.cu -- gated RMSNorm over rows of 128.
//
// "Agnes-3.0-Flash 深度解析：33B 混合注意力多模态模型", 注意力层的细节: the
// recurrent layer ends in a gated RMS-norm; the z projection of width 6144 =
// 48 x 128 ("33B 只做 18 层 ...", §2 parameter table) supplies the gate.
//     y = o / sqrt(mean(o^2) + eps) * w * SiLU(z)
//
// Memory-bound: 16 threads per row, one 16-byte vector of o and of z each,
// the sum of squares reduced with shuffles inside the 16-lane group.
#include <cuda_runtime.h>
#include <stdint.h>

#include "gdr_common.cuh"
#include "gdr_host.h"

namespace gdr {
namespace {

constexpr int kThreads = 256;
constexpr int kRowsPerBlock = kThreads / 16;

template <bool kWeight>   // a norm weight is given (otherwise ones)
__global__ void __launch_bounds__(kThreads) gated_rmsnorm_kernel(const uint16_t *o, const uint16_t *z,
                                                                 const float *w, float eps,
                                                                 int64_t rows, uint16_t *y) {
  grid_dep_wait();
  grid_dep_launch();
  const int64_t row = static_cast<int64_t>(blockIdx.x) * kRowsPerBlock + (threadIdx.x >> 4);
  const int part = threadIdx.x & 15;   // 8 columns each
  float ov[8], zv[8];
  if (row < rows) {
    unpack8(*reinterpret_cast<const uint4 *>(o + row * 128 + part * 8), ov);
    unpack8(*reinterpret_cast<const uint4 *>(z + row * 128 + part * 8), zv);
  } else {
#pragma unroll
    for (int i = 0; i < 8; ++i) ov[i] = zv[i] = 0.0f;
  }
  float ss = 0.0f;
#pragma unroll
  for (int i = 0; i < 8; ++i) ss += ov[i] * ov[i];
#pragma unroll
  for (int off = 8; off >= 1; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
  const float inv = 1.0f / sqrtf(ss * (1.0f / 128.0f) + eps);
  if (row >= rows) return;
  float sv[8];   // o / rms, times the weight when there is one
#pragma unroll
  for (int i = 0; i < 8; ++i) sv[i] = ov[i] * inv;
  if (kWeight) {
    const float4 w0 = *reinterpret_cast<const float4 *>(w + part * 8);
    const float4 w1 = *reinterpret_cast<const float4 *>(w + part * 8 + 4);
    sv[0] *= w0.x; sv[1] *= w0.y; sv[2] *= w0.z; sv[3] *= w0.w;
    sv[4] *= w1.x; sv[5] *= w1.y; sv[6] *= w1.z; sv[7] *= w1.w;
  }
  float out[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) out[i] = sv[i] * silu_fast(zv[i]);
  *reinterpret_cast<uint4 *>(y + row * 128 + part * 8) = pack8x2(out);
}

}  // namespace

int launch_gated_rmsnorm(const void *o, const void *z, const float *w, float eps, int64_t rows,
                         void *y, cudaStream_t s) {
  const int64_t blocks = (rows + kRowsPerBlock - 1) / kRowsPerBlock;
  if (blocks > 0x7FFFFFFF) return GDR_ERR_SHAPE;
  return launch_status(launch_pdl(w ? gated_rmsnorm_kernel<true> : gated_rmsnorm_kernel<false>, dim3(static_cast<unsigned>(blocks)), dim3(kThreads), 0, s, 1,
                                  static_cast<const uint16_t *>(o), static_cast<const uint16_t *>(z), w, eps,
                                  rows, static_cast<uint16_t *>(y)),
                       "gated norm: kernel launch");
}

}  // namespace gdr
