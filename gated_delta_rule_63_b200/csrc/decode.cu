// decode.cu -- one decode step of the gated delta-rule layer.
//
// "33B 只做 18 层：Agnes 3.0 Flash ..." (yfxerp.com) §1.2: when one new token
// resumes from the cached state the layer takes the single-step recurrent call
// with q/k L2-normalised in the kernel; "33B 只做 18 层 ..." (mhpq.cn) §2.1: the
// conv has a single-step form.  Per (sequence, value head):
//     y = SiLU(w0 s0 + w1 s1 + w2 s2 + w3 x), rounded to bf16; state -> (s1, s2, x)
//     q, k <- q / |q|, k / |k|;  g = -exp(A_log) softplus(a + dt_bias);  beta = sigmoid(b)
//     H' = exp(g) H;  u = beta (v - H'^T k);  H <- H' + k u^T;  o = scale H^T q
// where H = S^T is the [dk][dv] fp32 state.  Using o = scale (exp(g) H^T q +
// u (k.q)), both reductions H^T k and H^T q come from ONE read of H, and H is
// written once: 128 KB of HBM traffic per (sequence, head), the whole cost.
//
// Layout of the work: one CTA of 256 threads per (value head, sequence).
// The 64 KB tile of H arrives in shared memory by one bulk copy, issued first
// and in flight while the conv, norms and gates are computed; with registers
// freed from holding the tile, three CTAs share an SM, so about 192 KB of
// state loads are in flight per SM.  Warp w then reads rows 16w..16w+15,
// lane l columns 4l..4l+3 (one float4 per row, each warp-wide access one
// contiguous 512-byte row), once for the reductions and once for the update,
// which is stored straight from registers.  The CTAs of the value heads that
// share a key head form a thread-block cluster: the q/k conv state of that
// key head is read by all of them, then (after a cluster barrier) rolled by
// the first one, so the conv state can be updated in place.
//
// Slot-indexed form (a serving cache: "33B 只做 18 层 ...", §1.2 keeps the
// recurrent and conv states of each request in a per-layer cache): row n of
// the batch reads and writes pool entry slot[n] of the state and conv-state
// pools; x, a, b and o stay indexed by the row.  A slot outside the pool is a
// padding row: the pools are not touched and its o row is zero.
#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>

#include "gdr_common.cuh"
#include "gdr_host.h"

namespace gdr {
namespace {

constexpr int D = kHeadDim;
constexpr int kThreads = 256;
constexpr int kTileBytes = D * D * 4;   // one fp32 state tile

struct DecodeParams {
  const uint16_t *x;
  const uint16_t *conv_w;
  uint16_t *conv_state;
  const uint16_t *a;
  const uint16_t *b;
  const float *A_log;
  const float *dt_bias;
  float scale;
  int hk, hv, group, channels;
  float *state;
  uint16_t *o;
  const int32_t *slot;   // [batch] pool entry of each row (slot form only)
  int n_slots;
  int *err;
};

// Relaxed arrive: what it guards are this thread's reads of the shared q/k conv
// state, and their values have been consumed (the conv outputs are computed) before
// the arrive, so no release fence is needed.
__device__ __forceinline__ void cluster_arrive() {
  asm volatile("barrier.cluster.arrive.relaxed.aligned;\n" ::: "memory");
}
__device__ __forceinline__ void cluster_wait() {
  asm volatile("barrier.cluster.wait.acquire.aligned;\n" ::: "memory");
}

__device__ __forceinline__ void st_stream(float *p, float4 v) {
  __stcs(reinterpret_cast<float4 *>(p), v);
}

template <bool kSlots>
__global__ void __launch_bounds__(kThreads, 3) decode_kernel(DecodeParams p) {
  const int h = blockIdx.x;          // value head
  const int n = blockIdx.y;          // batch row
  const int kh = h / p.group;        // key head shared by `group` value heads
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int C = p.channels;

  __shared__ float s_q[D], s_k[D], s_u[D];
  __shared__ float s_red[8][2][D];   // per-warp partial H^T k and H^T q
  __shared__ float s_sum[3][4];      // per-warp partial |q|^2, |k|^2, q.k
  __shared__ float s_gate[2];        // exp(g), beta
  __shared__ alignas(8) uint64_t s_bar;
  __shared__ int s_ok;
  extern __shared__ float4 s_tile[];   // H, [D][D / 4] float4

  // 1. one bulk copy of the 64 KB state tile into shared memory
  const int row0 = warp * 16;
  const uint32_t bar = smem_u32(&s_bar);
  grid_dep_wait();     // the previous step's state and conv state are complete
  grid_dep_launch();   // the next step's CTAs may take the SMs this grid frees
  int ns = n;          // state / conv-state entry of this row
  bool live = true;    // false: a padding row (the pools stay untouched)
  if (kSlots) {
    ns = __ldg(p.slot + n);
    live = ns >= 0 && ns < p.n_slots;
    if (!live) ns = 0;   // a padding row reads and writes neither pool
  }
  float *S = p.state + (static_cast<size_t>(ns) * p.hv + h) * D * D;
  if (tid == 0 && live) {
    mbar_init(bar, 1);
    fence_mbar_init();
    mbar_arrive_expect_tx(bar, D * D * 4);
    bulk_load(smem_u32(s_tile), S, D * D * 4, bar);
  }

  // 2. conv step of this head's q, k (key head kh) and v channels
  const size_t xoff = static_cast<size_t>(n) * C;
  const size_t soff = static_cast<size_t>(ns) * 3 * C;
  float vq = 0.f, vk = 0.f, vv = 0.f;
  uint16_t new_q = 0, new_k = 0, new_v = 0;   // new newest conv-state entries
  uint16_t keep_q[2] = {0, 0}, keep_k[2] = {0, 0}, keep_v[2] = {0, 0};
  if (tid < D && live) {
    const int cq = kh * D + tid;
    const int ck = p.hk * D + kh * D + tid;
    const int cv = 2 * p.hk * D + h * D + tid;
    auto conv1 = [&](int c, uint16_t &newest, uint16_t *keep) {
      const uint2 wv = *reinterpret_cast<const uint2 *>(p.conv_w + static_cast<size_t>(c) * 4);
      const float w0 = __uint_as_float(wv.x << 16), w1 = __uint_as_float(wv.x & 0xFFFF0000u);
      const float w2 = __uint_as_float(wv.y << 16), w3 = __uint_as_float(wv.y & 0xFFFF0000u);
      const uint16_t s0 = p.conv_state[soff + c];
      const uint16_t s1 = p.conv_state[soff + C + c];
      const uint16_t s2 = p.conv_state[soff + 2 * C + c];
      const uint16_t xb = p.x[xoff + c];
      keep[0] = s1; keep[1] = s2; newest = xb;
      const float acc = w0 * bf_bits2f(s0) + w1 * bf_bits2f(s1) + w2 * bf_bits2f(s2) + w3 * bf_bits2f(xb);
      return round_bf16(silu_f(acc));   // the conv output is a bf16 tensor
    };
    vq = conv1(cq, new_q, keep_q);
    vk = conv1(ck, new_k, keep_k);
    vv = conv1(cv, new_v, keep_v);
  }
  // every CTA of the cluster has read the shared q/k conv state
  cluster_arrive();

  // 3. norms and q.k (threads 0..127 hold one channel each)
  if (tid < D) {
    float a2 = vq * vq, b2 = vk * vk, ab = vq * vk;
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) {
      a2 += __shfl_xor_sync(0xffffffffu, a2, off);
      b2 += __shfl_xor_sync(0xffffffffu, b2, off);
      ab += __shfl_xor_sync(0xffffffffu, ab, off);
    }
    if (lane == 0) { s_sum[0][warp] = a2; s_sum[1][warp] = b2; s_sum[2][warp] = ab; }
  }
  if (tid == 0) {
    s_ok = live && mbar_wait(bar, 0, p.err) ? 1 : 0;   // the tile has landed (bounded wait)
    const float av = bf_bits2f(p.a[static_cast<size_t>(n) * p.hv + h]);
    const float bv = bf_bits2f(p.b[static_cast<size_t>(n) * p.hv + h]);
    const float g = -expf(p.A_log[h]) * softplus_f(av + p.dt_bias[h]);
    s_gate[0] = expf(g);
    s_gate[1] = sigmoid_f(bv);
  }
  __syncthreads();
  const float qq = s_sum[0][0] + s_sum[0][1] + s_sum[0][2] + s_sum[0][3];
  const float kk = s_sum[1][0] + s_sum[1][1] + s_sum[1][2] + s_sum[1][3];
  const float qk = s_sum[2][0] + s_sum[2][1] + s_sum[2][2] + s_sum[2][3];
  const float rq = 1.0f / sqrtf(qq + 1e-6f), rk = 1.0f / sqrtf(kk + 1e-6f);
  const float kq = qk * rq * rk;   // k_hat . q_hat
  const float eg = s_gate[0], beta = s_gate[1];
  if (tid < D) { s_q[tid] = vq * rq; s_k[tid] = vk * rk; }
  __syncthreads();

  const bool ok = s_ok != 0;

  // 4. partial H^T k and H^T q over this warp's 16 rows
  float pk[4] = {0, 0, 0, 0}, pq[4] = {0, 0, 0, 0};
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const float4 r = s_tile[(row0 + i) * (D / 4) + lane];
    const float ki = s_k[row0 + i], qi = s_q[row0 + i];
    pk[0] += r.x * ki; pk[1] += r.y * ki; pk[2] += r.z * ki; pk[3] += r.w * ki;
    pq[0] += r.x * qi; pq[1] += r.y * qi; pq[2] += r.z * qi; pq[3] += r.w * qi;
  }
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    s_red[warp][0][lane * 4 + c] = pk[c];
    s_red[warp][1][lane * 4 + c] = pq[c];
  }
  __syncthreads();

  // 5. u and o per column (threads 0..127)
  if (tid < D) {
    float hk_ = 0.f, hq_ = 0.f;
#pragma unroll
    for (int w = 0; w < 8; ++w) { hk_ += s_red[w][0][tid]; hq_ += s_red[w][1][tid]; }
    const float u = beta * (vv - eg * hk_);
    s_u[tid] = u;
    const float ov = p.scale * (eg * hq_ + u * kq);
    if (ok) p.o[(static_cast<size_t>(n) * p.hv + h) * D + tid] = f2bf_bits(ov);
    else if (!live) p.o[(static_cast<size_t>(n) * p.hv + h) * D + tid] = 0;
  }
  __syncthreads();

  // 6. H <- exp(g) H + k u^T, written once
  const float4 u4 = *reinterpret_cast<const float4 *>(s_u + lane * 4);
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const float ki = s_k[row0 + i];
    float4 v = s_tile[(row0 + i) * (D / 4) + lane];
    v.x = eg * v.x + ki * u4.x;
    v.y = eg * v.y + ki * u4.y;
    v.z = eg * v.z + ki * u4.z;
    v.w = eg * v.w + ki * u4.w;
    if (ok) st_stream(S + (row0 + i) * D + lane * 4, v);
  }

  // 7. roll the conv state: v channels by this CTA, q/k channels by the first
  //    CTA of the cluster once every CTA has read them; a CTA whose state tile
  //    never arrived (bounded wait ran out) leaves its channels as they were
  cluster_wait();
  if (tid < D && live && ok) {
    const int cv = 2 * p.hk * D + h * D + tid;
    p.conv_state[soff + cv] = keep_v[0];
    p.conv_state[soff + C + cv] = keep_v[1];
    p.conv_state[soff + 2 * C + cv] = new_v;
    if (h % p.group == 0) {
      const int cq = kh * D + tid;
      const int ck = p.hk * D + kh * D + tid;
      p.conv_state[soff + cq] = keep_q[0];
      p.conv_state[soff + C + cq] = keep_q[1];
      p.conv_state[soff + 2 * C + cq] = new_q;
      p.conv_state[soff + ck] = keep_k[0];
      p.conv_state[soff + C + ck] = keep_k[1];
      p.conv_state[soff + 2 * C + ck] = new_k;
    }
  }
}

}  // namespace

int launch_decode(const void *x, const void *conv_w, void *conv_state, const void *a, const void *b,
                  const float *A_log, const float *dt_bias, float scale, int hk, int hv,
                  float *state, const int32_t *slot, int n_slots, void *o, int batch, cudaStream_t s) {
  if (batch > 65535) return GDR_ERR_SHAPE;
  DecodeParams p;
  p.x = static_cast<const uint16_t *>(x);
  p.conv_w = static_cast<const uint16_t *>(conv_w);
  p.conv_state = static_cast<uint16_t *>(conv_state);
  p.a = static_cast<const uint16_t *>(a);
  p.b = static_cast<const uint16_t *>(b);
  p.A_log = A_log;
  p.dt_bias = dt_bias;
  p.scale = scale;
  p.hk = hk;
  p.hv = hv;
  p.group = hv / hk;
  p.channels = 2 * hk * D + hv * D;
  p.state = state;
  p.o = static_cast<uint16_t *>(o);
  p.slot = slot;
  p.n_slots = n_slots;
  p.err = device_error_ptr();

  // the shared-memory opt-in, once per device (a bit per device; threads may race to set it,
  // which only repeats the idempotent calls)
  static std::atomic<uint64_t> attr_done{0};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return launch_status(e, "decode: cudaGetDevice");
  const uint64_t bit = dev >= 0 && dev < 64 ? (uint64_t{1} << dev) : 0;
  if (!bit || !(attr_done.load(std::memory_order_acquire) & bit)) {
    e = cudaFuncSetAttribute(decode_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, kTileBytes);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(decode_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, kTileBytes);
    if (e != cudaSuccess) return launch_status(e, "decode: shared memory opt-in");
    attr_done.fetch_or(bit, std::memory_order_acq_rel);
  }
  const unsigned cluster = static_cast<unsigned>(p.group);
  return launch_status(slot ? launch_pdl(decode_kernel<true>, dim3(hv, batch, 1), dim3(kThreads), kTileBytes, s,
                                         cluster, p)
                            : launch_pdl(decode_kernel<false>, dim3(hv, batch, 1), dim3(kThreads), kTileBytes, s,
                                         cluster, p),
                       "decode: kernel launch");
}

}  // namespace gdr
