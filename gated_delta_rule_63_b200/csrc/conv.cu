// conv.cu -- depthwise causal conv (kernel 4) + SiLU over packed sequences.
//
// "Agnes-3.0-Flash 深度解析：33B 混合注意力多模态模型", 注意力层的细节: a
// kernel-4 causal conv sits in front of the recurrence.  y[t][c] =
// SiLU(sum_j w[c][j] x[t-3+j][c]), fp32 math, bf16 output; inputs before a
// sequence start come from the conv state (oldest first) or are zero.
//
// Memory-bound: each thread owns 8 adjacent channels (one 16-byte vector) and
// walks a run of kTokens tokens with a 3-deep sliding window in registers, so
// x is read once (plus a 3-token halo per run) and y written once, both with
// coalesced 16-byte accesses.
#include <cuda_runtime.h>
#include <stdint.h>

#include "gdr_common.cuh"
#include "gdr_host.h"

namespace gdr {
namespace {

constexpr int kThreads = 128;   // threads per block; 8 channels each
constexpr int kTokens = 32;     // tokens per run

struct ConvParams {
  const uint16_t *x;
  const uint16_t *w;
  const uint16_t *cs_in;
  uint16_t *cs_out;
  const int32_t *cu;
  uint16_t *y;
  int n_seqs;
  int total;
  int channels;
};

// sequence containing token t: largest n with cu[n] <= t (skipping empty ones)
__device__ int seq_of(const int32_t *cu, int n_seqs, int t) {
  int lo = 0, hi = n_seqs - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (__ldg(cu + mid) <= t) lo = mid; else hi = mid - 1;
  }
  return lo;
}

__device__ __forceinline__ void load8(const uint16_t *p, float *f) {
  unpack8(*reinterpret_cast<const uint4 *>(p), f);
}

__global__ void __launch_bounds__(kThreads) causal_conv_kernel(ConvParams p) {
  const int C = p.channels;
  const int c0 = (blockIdx.x * kThreads + threadIdx.x) * 8;   // first channel of this thread
  if (c0 >= C) return;
  const int t_begin = blockIdx.y * kTokens;

  float w[4][8];
  {
    // w is [C][4]: channels c0..c0+7 occupy 32 contiguous bf16
    const uint4 *wp = reinterpret_cast<const uint4 *>(p.w + static_cast<size_t>(c0) * 4);
    float tmp[32];
#pragma unroll
    for (int i = 0; i < 4; ++i) unpack8(__ldg(wp + i), tmp + 8 * i);
#pragma unroll
    for (int ch = 0; ch < 8; ++ch)
#pragma unroll
      for (int j = 0; j < 4; ++j) w[j][ch] = tmp[ch * 4 + j];
  }

  // empty sequences: their conv state passes through unchanged (run once)
  if (blockIdx.y == 0 && p.cs_out) {
    for (int n = 0; n < p.n_seqs; ++n) {
      if (__ldg(p.cu + n + 1) != __ldg(p.cu + n)) continue;
      for (int s = 0; s < 3; ++s) {
        uint4 v = make_uint4(0, 0, 0, 0);
        if (p.cs_in) v = *reinterpret_cast<const uint4 *>(p.cs_in + (static_cast<size_t>(n) * 3 + s) * C + c0);
        *reinterpret_cast<uint4 *>(p.cs_out + (static_cast<size_t>(n) * 3 + s) * C + c0) = v;
      }
    }
  }
  if (t_begin >= p.total) return;
  const int t_end = min(t_begin + kTokens, p.total);

  int n = seq_of(p.cu, p.n_seqs, t_begin);
  int seq_start = __ldg(p.cu + n);
  int seq_end = __ldg(p.cu + n + 1);

  // window: win[0] = x[t-3], win[1] = x[t-2], win[2] = x[t-1]
  float win[3][8];
  auto fill_window = [&](int t) {
#pragma unroll
    for (int s = 0; s < 3; ++s) {
      const int pos = t - 3 + s;
      if (pos >= seq_start) {
        load8(p.x + static_cast<size_t>(pos) * C + c0, win[s]);
      } else if (p.cs_in) {
        const int back = seq_start - pos;   // 1..3 positions before the start
        load8(p.cs_in + (static_cast<size_t>(n) * 3 + (3 - back)) * C + c0, win[s]);
      } else {
#pragma unroll
        for (int ch = 0; ch < 8; ++ch) win[s][ch] = 0.0f;
      }
    }
  };
  fill_window(t_begin);

  for (int t = t_begin; t < t_end; ++t) {
    if (t >= seq_end) {   // crossed into the next non-empty sequence
      do {
        ++n;
        seq_start = __ldg(p.cu + n);
        seq_end = __ldg(p.cu + n + 1);
      } while (seq_end <= t);
      fill_window(t);
    }
    float xt[8], out[8];
    load8(p.x + static_cast<size_t>(t) * C + c0, xt);
#pragma unroll
    for (int ch = 0; ch < 8; ++ch) {
      const float acc = w[0][ch] * win[0][ch] + w[1][ch] * win[1][ch] + w[2][ch] * win[2][ch] +
                        w[3][ch] * xt[ch];
      out[ch] = silu_f(acc);
    }
    *reinterpret_cast<uint4 *>(p.y + static_cast<size_t>(t) * C + c0) = pack8(out);
#pragma unroll
    for (int ch = 0; ch < 8; ++ch) {
      win[0][ch] = win[1][ch];
      win[1][ch] = win[2][ch];
      win[2][ch] = xt[ch];
    }
    if (t == seq_end - 1 && p.cs_out) {   // last token: the window is the new conv state
#pragma unroll
      for (int s = 0; s < 3; ++s)
        *reinterpret_cast<uint4 *>(p.cs_out + (static_cast<size_t>(n) * 3 + s) * C + c0) = pack8(win[s]);
    }
  }
}

}  // namespace

int launch_causal_conv(const void *x, const void *w, const void *cs_in, void *cs_out,
                       const int32_t *cu_dev, int n_seqs, int total, int channels, void *y,
                       cudaStream_t s) {
  ConvParams p;
  p.x = static_cast<const uint16_t *>(x);
  p.w = static_cast<const uint16_t *>(w);
  p.cs_in = static_cast<const uint16_t *>(cs_in);
  p.cs_out = static_cast<uint16_t *>(cs_out);
  p.cu = cu_dev;
  p.y = static_cast<uint16_t *>(y);
  p.n_seqs = n_seqs;
  p.total = total;
  p.channels = channels;
  const int groups = channels / 8;
  dim3 grid((groups + kThreads - 1) / kThreads, total > 0 ? (total + kTokens - 1) / kTokens : 1);
  causal_conv_kernel<<<grid, kThreads, 0, s>>>(p);
  return last_launch_status();
}

}  // namespace gdr
