// conv.cu -- depthwise causal conv (kernel 4) + SiLU over packed sequences.
//
// "Agnes-3.0-Flash 深度解析：33B 混合注意力多模态模型", 注意力层的细节: a
// kernel-4 causal conv sits in front of the recurrence.  y[t][c] =
// SiLU(sum_j w[c][j] x[t-3+j][c]), fp32 math, bf16 output; inputs before a
// sequence start come from the conv state (oldest first) or are zero.
//
// Memory-bound: each thread owns 8 adjacent channels (one 16-byte vector) of
// a run of kTokens tokens; the run's rows and its 3-row halo are loaded up
// front so that all its loads are in flight together.  x is read once (plus
// the halo, mostly from L2) and y written once, with coalesced 16-byte
// accesses.
#include <cuda_runtime.h>
#include <stdint.h>

#include "gdr_common.cuh"
#include "gdr_host.h"

namespace gdr {
namespace {

constexpr int kThreads = 128;   // threads per block; 8 channels each
constexpr int kTokens = 8;      // tokens per run

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

// unpack the 8 bf16 of a 16-byte row into floats (one integer op each)
__device__ __forceinline__ void row8(const uint4 &u, float *f) { unpack8(u, f); }

// Each thread: 8 channels x kTokens tokens.  A run that lies inside one
// sequence (the common case) loads all kTokens + 3 input rows up front
// (independent 16-byte loads in flight) and unpacks every row once into a
// sliding window of four; a run that touches a sequence start or end takes
// the general path, whose taps come from the rows of their own sequence, from
// the conv state, or are zero.
__global__ void __launch_bounds__(kThreads) causal_conv_kernel(ConvParams p) {
  grid_dep_wait();
  grid_dep_launch();
  const int C = p.channels;
  const int c0 = (blockIdx.x * kThreads + threadIdx.x) * 8;   // first channel of this thread
  if (c0 >= C) return;
  const int t_begin = blockIdx.y * kTokens;

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
  int n = seq_of(p.cu, p.n_seqs, t_begin);
  int seq_start = __ldg(p.cu + n), seq_end = __ldg(p.cu + n + 1);

  if (t_begin - 3 >= seq_start && t_begin + kTokens < seq_end) {
    // ---- inside one sequence, not its last token: no state, no boundary ----
    uint4 raw[kTokens + 3];   // rows t_begin - 3 .. t_begin + kTokens - 1
#pragma unroll
    for (int i = 0; i < kTokens + 3; ++i)
      raw[i] = __ldg(reinterpret_cast<const uint4 *>(p.x + static_cast<size_t>(t_begin - 3 + i) * C + c0));
    float xw[4][8];
#pragma unroll
    for (int j = 0; j < 3; ++j) row8(raw[j], xw[j]);
#pragma unroll
    for (int i = 0; i < kTokens; ++i) {
      row8(raw[i + 3], xw[(i + 3) & 3]);
      float out[8];
#pragma unroll
      for (int ch = 0; ch < 8; ++ch) {
        const float acc = w[0][ch] * xw[i & 3][ch] + w[1][ch] * xw[(i + 1) & 3][ch] +
                          w[2][ch] * xw[(i + 2) & 3][ch] + w[3][ch] * xw[(i + 3) & 3][ch];
        out[ch] = silu_fast(acc);
      }
      *reinterpret_cast<uint4 *>(p.y + static_cast<size_t>(t_begin + i) * C + c0) = pack8x2(out);
    }
    return;
  }

  // ---- general path: sequence starts / ends inside the run ----
#pragma unroll 1
  for (int i = 0; i < kTokens; ++i) {
    const int t = t_begin + i;
    if (t >= t_end) break;
    while (t >= seq_end) {   // next non-empty sequence
      ++n;
      seq_start = __ldg(p.cu + n);
      seq_end = __ldg(p.cu + n + 1);
    }
    float acc[8];
#pragma unroll
    for (int ch = 0; ch < 8; ++ch) acc[ch] = 0.0f;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int pos = t - 3 + j;
      uint4 v = make_uint4(0, 0, 0, 0);
      if (pos >= seq_start) {   // (re-read: this path is rare and the row sits in L1 / L2)
        v = __ldg(reinterpret_cast<const uint4 *>(p.x + static_cast<size_t>(pos) * C + c0));
      } else if (p.cs_in) {   // before the sequence start: the conv state, oldest first
        const int slot = 3 - (seq_start - pos);   // 1..3 positions before the start
        v = *reinterpret_cast<const uint4 *>(p.cs_in + (static_cast<size_t>(n) * 3 + slot) * C + c0);
      }
      float xv[8];
      unpack8(v, xv);
#pragma unroll
      for (int ch = 0; ch < 8; ++ch) acc[ch] += w[j][ch] * xv[ch];
    }
    float out[8];
#pragma unroll
    for (int ch = 0; ch < 8; ++ch) out[ch] = silu_fast(acc[ch]);
    *reinterpret_cast<uint4 *>(p.y + static_cast<size_t>(t) * C + c0) = pack8x2(out);
    if (t == seq_end - 1 && p.cs_out) {   // last token: the last three inputs are the new conv state
#pragma unroll
      for (int s = 0; s < 3; ++s) {
        const int pos = t - 2 + s;
        uint4 v = make_uint4(0, 0, 0, 0);
        if (pos >= seq_start) {
          v = __ldg(reinterpret_cast<const uint4 *>(p.x + static_cast<size_t>(pos) * C + c0));
        } else if (p.cs_in) {
          v = *reinterpret_cast<const uint4 *>(p.cs_in + (static_cast<size_t>(n) * 3 + (3 - (seq_start - pos))) * C + c0);
        }
        *reinterpret_cast<uint4 *>(p.cs_out + (static_cast<size_t>(n) * 3 + s) * C + c0) = v;
      }
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
  return launch_status(launch_pdl(causal_conv_kernel, grid, dim3(kThreads), 0, s, 1, p), "conv: kernel launch");
}

}  // namespace gdr
