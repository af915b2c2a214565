// prefill.cu -- chunked prefill of the gated delta rule on tcgen05 tensor cores.
//
// "33B 只做 18 层：Agnes 3.0 Flash ..." (yfxerp.com) §1.2: prefill walks the
// sequence in chunks of 64 and is interchangeable with the per-token form.
// Unrolling S_t = exp(g_t) S_{t-1} (I - beta_t k_t k_t^T) + beta_t v_t k_t^T
// ("Sapiens AI 发布 Agnes-3.0-Flash", delta 规则循环层究竟怎么运作) over a chunk
// of L <= 64 tokens with gamma_i = g_1 + ... + g_i and H = S^T gives
//     A    = strict_lower(beta_i exp(gamma_i - gamma_j) k_i.k_j)
//     T    = (I + A)^-1
//     W    = T diag(beta e^gamma) K,      Ut = T diag(beta) V
//     U    = Ut - W H0
//     O    = scale (diag(e^gamma) Q H0 + (Q K^T . M) U),  M_ij = e^(gamma_i - gamma_j), j <= i
//     H_L  = e^gamma_L H0 + K^T diag(e^(gamma_L - gamma)) U
// with q, k the L2-normalised rows.
//
// Precision plan.  The raw bf16 q, k, v rows are exact MMA operands; the
// 1/|q|, 1/|k| factors, gates and decays are folded into fp32 row/column
// scales of the other operand.  Every fp32 operand that feeds the state
// (T-derived matrices, W, U, H0) is split as hi + lo bf16 and the products
// are accumulated as hi*hi + hi*lo + lo*hi in fp32 TMEM, which keeps about
// 16 significant bits.  The state itself never leaves fp32: thread i holds
// row i of H (its dv slice) in registers from the first chunk to the last.
//
// Work split.  One CTA of 128 threads per (dv slice of 64 columns, value
// head, sequence); the value head h reads key head h / (hv / hk).  Thread t
// owns TMEM lane t; every MMA is M = 128 (cta_group::1) with fp32 TMEM
// accumulators, operands in shared memory in the 128-byte swizzled layout.
// The unit lower-triangular inverse runs on CUDA cores (16x16 diagonal
// blocks by substitution, off-diagonal blocks by block products).
#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>

#include "gdr_common.cuh"
#include "gdr_host.h"

namespace gdr {
namespace {

constexpr int C = kChunk;      // 64 tokens per chunk
constexpr int D = kHeadDim;    // 128
constexpr int N = 64;          // dv columns per CTA
constexpr int NS = D / N;      // dv slices
constexpr int kThreads = 128;

// ---- shared memory plan (byte offsets from a 1024-aligned base) ----------
// OPA: A/B operand rows, two 64-column k-blocks of 256 rows x 128 B each:
//      rows   0.. 63  W_lo      rows  64..127  W_hi
//      rows 128..191  Q (raw)   rows 192..255  K (raw)
constexpr uint32_t OPA_KB = 256 * 128;
constexpr uint32_t ROW_WLO = 0, ROW_WHI = 64, ROW_Q = 128, ROW_K = 192;
constexpr uint32_t OFF_OPA = 0;
// TB: six [64 x 64] bf16 blocks (one 128-B row per token):
//      0 T'_hi, 1 T'_lo, 2 T''_hi, 3 T''_lo, 4 Mq_hi, 5 Mq_lo
//      T' = T diag(beta e^gamma / |k|), T'' = T diag(beta), Mq = (Q K^T . M) / (|q| |k|)
constexpr uint32_t BLK64 = 64 * 128;
constexpr uint32_t OFF_TB = OFF_OPA + 2 * OPA_KB;
constexpr uint32_t OFF_V = OFF_TB + 6 * BLK64;        // V slice [64 tok][64 dv]
constexpr uint32_t OFF_H = OFF_V + BLK64;             // H_hi, H_lo [128 dk][64 dv]
constexpr uint32_t BLK128 = 128 * 128;
constexpr uint32_t OFF_U = OFF_H + 2 * BLK128;        // U_hi, U_lo, U'_hi, U'_lo [64 tok][64 dv]
constexpr int LD = 65;                                // fp32 row stride of A and T
constexpr uint32_t OFF_AF = OFF_U + 4 * BLK64;
constexpr uint32_t OFF_TF = OFF_AF + 64 * LD * 4;
constexpr uint32_t OFF_XF = OFF_TF + 64 * LD * 4;     // block-product scratch, 3 x 16 x 16
constexpr uint32_t OFF_VEC = OFF_XF + 3 * 256 * 4;    // gamma, beta, 1/|k|, 1/|q|, e^gamma, decay-to-end
constexpr uint32_t OFF_BAR = OFF_VEC + 6 * 64 * 4;
constexpr uint32_t SMEM_USED = OFF_BAR + 16;
constexpr uint32_t SMEM_BYTES = SMEM_USED + 1024;    // slack for aligning the base
static_assert(SMEM_BYTES <= 232448, "shared memory plan exceeds 227 KB");

// ---- TMEM columns (fp32, lane = row) ---------------------------------------
constexpr uint32_t TM_COLS = 512;
constexpr uint32_t COL_S = 0;      // [Q K^T ; K K^T]           64 cols
constexpr uint32_t COL_W = 64;     // W (rows 0..63)            128 cols
constexpr uint32_t COL_P = 192;    // [W_hi H ; Q H]            64
constexpr uint32_t COL_P2 = 256;   // W_lo H_hi (rows 0..63)    64
constexpr uint32_t COL_UT = 320;   // Ut (rows 0..63)           64
constexpr uint32_t COL_H = 384;    // K^T U' (rows = dk)        64
constexpr uint32_t COL_O = 448;    // Mq U (rows 64..127)       64

struct PrefillParams {
  const uint16_t *q, *k, *v, *a, *b;
  const float *A_log, *dt_bias;
  float scale;
  int hk, hv, group;
  int64_t qk_stride, v_stride;   // elements between consecutive tokens
  const int32_t *cu;
  const float *h0;
  float *hT;
  uint16_t *o;
  int *err;
#ifdef GDR_PREFILL_DEBUG
  float *dbg;   // diagnostic dump of the first chunk of CTA (0, 0, 0)
#endif
};

#ifdef GDR_PREFILL_DEBUG
float *g_dump = nullptr;
#endif

__device__ __forceinline__ void st_shared16(uint32_t addr, const uint4 &v) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};\n" ::"r"(addr), "r"(v.x), "r"(v.y), "r"(v.z),
               "r"(v.w)
               : "memory");
}
__device__ __forceinline__ uint4 ld_shared16(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];\n"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "r"(addr));
  return v;
}

// write 64 fp32 values as the hi/lo bf16 row `r` of two 128B-swizzled tiles
__device__ __forceinline__ void write_row_split(uint32_t hi_base, uint32_t lo_base, uint32_t r,
                                                const float *vals) {
#pragma unroll
  for (int c = 0; c < 8; ++c) {
    uint4 hi, lo;
    split8(vals + 8 * c, hi, lo);
    st_shared16(hi_base + sw128(r, c), hi);
    st_shared16(lo_base + sw128(r, c), lo);
  }
}

// one thread waits for the MMA barrier phase, the CTA agrees on the outcome
__device__ __forceinline__ bool cta_wait_mma(uint32_t bar, uint32_t &phase, int *err) {
  bool ok = true;
  if (threadIdx.x == 0) ok = mbar_wait(bar, phase, err);
  phase ^= 1u;
  ok = __syncthreads_and(ok) != 0;
  tc_fence_after();
  return ok;
}

__global__ void __launch_bounds__(kThreads, 1) chunk_prefill_kernel(PrefillParams p) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  const uint32_t sbase = (raw_addr + 1023u) & ~1023u;
  uint8_t *smem = smem_raw + (sbase - raw_addr);

  const int slice = blockIdx.x, h = blockIdx.y, n = blockIdx.z;
  const int kh = h / p.group;
  const int tid = threadIdx.x, warp = tid >> 5;
  const int seq_start = p.cu[n], seq_end = p.cu[n + 1];

  float *s_gam = reinterpret_cast<float *>(smem + OFF_VEC);
  float *s_beta = s_gam + 64;
  float *s_rk = s_gam + 128;
  float *s_rq = s_gam + 192;
  float *s_eg = s_gam + 256;     // e^gamma_j
  float *s_ed = s_gam + 320;     // e^(gamma_L - gamma_j) / |k_j|
  float *AF = reinterpret_cast<float *>(smem + OFF_AF);
  float *TF = reinterpret_cast<float *>(smem + OFF_TF);
  float *XF = reinterpret_cast<float *>(smem + OFF_XF);
  const uint32_t bar = sbase + OFF_BAR;
  uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(smem + OFF_BAR + 8);

  if (warp == 0) {
    tmem_alloc(smem_u32(tmem_holder), TM_COLS);
    tmem_relinquish();
  }
  if (tid == 0) {
    mbar_init(bar, 1);
    fence_mbar_init();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  const uint32_t tl = tmem + (static_cast<uint32_t>(warp * 32) << 16);   // this warp's lane quarter
  uint32_t phase = 0;

  // ---- the state: thread tid holds row tid (dk index) of its dv slice ----
  float hreg[N];
  const size_t srow = (static_cast<size_t>(n) * p.hv + h) * D * D + static_cast<size_t>(tid) * D + slice * N;
  if (p.h0) {
#pragma unroll
    for (int j = 0; j < N; j += 4) {
      const float4 v4 = *reinterpret_cast<const float4 *>(p.h0 + srow + j);
      hreg[j] = v4.x; hreg[j + 1] = v4.y; hreg[j + 2] = v4.z; hreg[j + 3] = v4.w;
    }
  } else {
#pragma unroll
    for (int j = 0; j < N; ++j) hreg[j] = 0.0f;
  }
  write_row_split(sbase + OFF_H, sbase + OFF_H + BLK128, tid, hreg);

  const float A_h = expf(p.A_log[h]);
  const float dtb = p.dt_bias[h];
  bool ok = true;
#ifdef GDR_PREFILL_DEBUG
  bool dump = p.dbg && blockIdx.x == 0 && blockIdx.y == 0 && blockIdx.z == 0;
#endif

  for (int t0 = seq_start; t0 < seq_end && ok; t0 += C) {
    const int L = min(C, seq_end - t0);

    // ---- S0: raw q, k rows (key head kh), v slice, gates -------------------
    for (int idx = tid; idx < 64 * 16; idx += kThreads) {
      const int r = idx >> 4, c = idx & 15;
      const bool valid = r < L;
      const size_t tok = static_cast<size_t>(t0 + (valid ? r : 0));
      const uint32_t kb = static_cast<uint32_t>(c >> 3) * OPA_KB;
      cp_async16(sbase + OFF_OPA + kb + sw128(ROW_Q + r, c & 7),
                 p.q + tok * p.qk_stride + kh * D + c * 8, valid ? 16u : 0u);
      cp_async16(sbase + OFF_OPA + kb + sw128(ROW_K + r, c & 7),
                 p.k + tok * p.qk_stride + kh * D + c * 8, valid ? 16u : 0u);
    }
    for (int idx = tid; idx < 64 * 8; idx += kThreads) {
      const int r = idx >> 3, c = idx & 7;
      const bool valid = r < L;
      const size_t tok = static_cast<size_t>(t0 + (valid ? r : 0));
      cp_async16(sbase + OFF_V + sw128(r, c), p.v + tok * p.v_stride + h * D + slice * N + c * 8,
                 valid ? 16u : 0u);
    }
    cp_async_commit();
    if (tid < 64) {
      float g = 0.0f, beta = 0.0f;   // padding rows: no decay, no write
      if (tid < L) {
        const size_t ab = static_cast<size_t>(t0 + tid) * p.hv + h;
        g = -A_h * softplus_f(bf_bits2f(p.a[ab]) + dtb);
        beta = sigmoid_f(bf_bits2f(p.b[ab]));
      }
      s_gam[tid] = g;
      s_beta[tid] = beta;
    }
    cp_async_wait_all();
    fence_proxy_async();
    __syncthreads();

    // ---- S1: cumulative gates, 1/|q|, 1/|k| --------------------------------
    if (tid == 0) {
      float run = 0.0f;
      for (int i = 0; i < 64; ++i) { run += s_gam[i]; s_gam[i] = run; }
    }
    {
      const int r = tid & 63;
      const uint32_t row = (tid < 64 ? ROW_Q : ROW_K) + r;
      float ss = 0.0f;
#pragma unroll
      for (int c = 0; c < 16; ++c) {
        float f[8];
        unpack8(ld_shared16(sbase + OFF_OPA + (c >> 3) * OPA_KB + sw128(row, c & 7)), f);
#pragma unroll
        for (int e = 0; e < 8; ++e) ss += f[e] * f[e];
      }
      (tid < 64 ? s_rq : s_rk)[r] = 1.0f / sqrtf(ss + 1e-6f);
    }
    __syncthreads();
    if (tid < 64) {
      s_eg[tid] = expf(s_gam[tid]);
      s_ed[tid] = expf(s_gam[63] - s_gam[tid]) * s_rk[tid];
    }

    // ---- S2: [Q; K] K^T on the tensor cores --------------------------------
    if (tid == 0) {
      tc_fence_after();
      const uint32_t id = idesc_bf16(128, 64, false, false);
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
        const uint32_t koff = (kk >> 2) * OPA_KB + (kk & 3) * 32;
        mma_bf16(tmem + COL_S, sdesc(sbase + OFF_OPA + koff + ROW_Q * 128, 16, 1024),
                 sdesc(sbase + OFF_OPA + koff + ROW_K * 128, 16, 1024), id, kk > 0);
      }
      mma_commit(bar);
    }
    ok = cta_wait_mma(bar, phase, p.err);
    if (!ok) break;

    // ---- S3: A (fp32) and the masked, decayed, normalised Q K^T ------------
    {
      float sv[64];
      tmem_ld32(tl + COL_S, sv);
      tmem_ld32(tl + COL_S + 32, sv + 32);
      tmem_wait_ld();
      if (tid < 64) {   // row i of Q K^T
        const int i = tid;
        const float gi = s_gam[i], sq = s_rq[i];
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          float m[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const int j = 8 * c + e;
            m[e] = (j <= i) ? sv[j] * sq * s_rk[j] * expf(gi - s_gam[j]) : 0.0f;
          }
          uint4 hi, lo;
          split8(m, hi, lo);
          st_shared16(sbase + OFF_TB + 4 * BLK64 + sw128(i, c), hi);
          st_shared16(sbase + OFF_TB + 5 * BLK64 + sw128(i, c), lo);
        }
      } else {          // row i of K K^T
        const int i = tid - 64;
        const float gi = s_gam[i], bi = s_beta[i] * s_rk[i];
#pragma unroll
        for (int j = 0; j < 64; ++j)
          AF[i * LD + j] = (j < i) ? bi * s_rk[j] * sv[j] * expf(gi - s_gam[j]) : 0.0f;
      }
    }
#ifdef GDR_PREFILL_DEBUG
    if (dump && t0 == seq_start) {
      float sv[64];
      tmem_ld32(tl + COL_S, sv);
      tmem_ld32(tl + COL_S + 32, sv + 32);
      tmem_wait_ld();
      for (int j = 0; j < 64; ++j) p.dbg[tid * 64 + j] = sv[j];
    }
#endif
    tc_fence_before();
    __syncthreads();

    // ---- S4: T = (I + A)^-1 ------------------------------------------------
    if (tid < 64) {   // diagonal 16x16 blocks, one column per thread
      const int bb = tid >> 4, c = tid & 15;
      float x[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        float s = (i == c) ? 1.0f : 0.0f;
#pragma unroll
        for (int j = 0; j < i; ++j) s -= AF[(16 * bb + i) * LD + 16 * bb + j] * x[j];
        x[i] = s;
      }
#pragma unroll
      for (int i = 0; i < 16; ++i) TF[(16 * bb + i) * LD + 16 * bb + c] = x[i];
    }
    __syncthreads();
    for (int d = 1; d < 4; ++d) {   // block diagonal d: T_bc = -T_bb sum_{m=c}^{b-1} A_bm T_mc
      const int nb = 4 - d;
      for (int e = tid; e < nb * 256; e += kThreads) {
        const int blk = e >> 8, bb = d + blk, c = bb - d, i = (e >> 4) & 15, j = e & 15;
        float s = 0.0f;
        for (int m = c; m < bb; ++m)
#pragma unroll
          for (int l = 0; l < 16; ++l) s += AF[(16 * bb + i) * LD + 16 * m + l] * TF[(16 * m + l) * LD + 16 * c + j];
        XF[e] = s;
      }
      __syncthreads();
      for (int e = tid; e < nb * 256; e += kThreads) {
        const int blk = e >> 8, bb = d + blk, c = bb - d, i = (e >> 4) & 15, j = e & 15;
        float s = 0.0f;
#pragma unroll
        for (int l = 0; l < 16; ++l)
          if (l <= i) s -= TF[(16 * bb + i) * LD + 16 * bb + l] * XF[(blk << 8) + l * 16 + j];
        TF[(16 * bb + i) * LD + 16 * c + j] = s;
      }
      __syncthreads();
    }

    // ---- S5: T' = T diag(beta e^gamma / |k|), T'' = T diag(beta), hi/lo ----
    {
      const int i = tid & 63, half = tid >> 6;
#pragma unroll
      for (int cb = 0; cb < 4; ++cb) {
        const int c = half * 4 + cb;
        float t1[8], t2[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const int j = 8 * c + e;
          const float tij = (j <= i) ? TF[i * LD + j] : 0.0f;
          t2[e] = tij * s_beta[j];
          t1[e] = t2[e] * s_eg[j] * s_rk[j];
        }
        uint4 hi, lo;
        split8(t1, hi, lo);
        st_shared16(sbase + OFF_TB + 0 * BLK64 + sw128(i, c), hi);
        st_shared16(sbase + OFF_TB + 1 * BLK64 + sw128(i, c), lo);
        split8(t2, hi, lo);
        st_shared16(sbase + OFF_TB + 2 * BLK64 + sw128(i, c), hi);
        st_shared16(sbase + OFF_TB + 3 * BLK64 + sw128(i, c), lo);
      }
    }
#ifdef GDR_PREFILL_DEBUG
    if (dump && t0 == seq_start) {
      for (int e = tid; e < 64 * 64; e += kThreads) {
        p.dbg[8192 + e] = AF[(e >> 6) * LD + (e & 63)];
        p.dbg[8192 + 4096 + e] = ((e & 63) <= (e >> 6)) ? TF[(e >> 6) * LD + (e & 63)] : 0.0f;
      }
    }
#endif
    fence_proxy_async();
    __syncthreads();

    // ---- S6: W = T' K and Ut = T'' V -----------------------------------------
    if (tid == 0) {
      tc_fence_after();
      const uint32_t idW = idesc_bf16(128, 128, false, true);
      const uint32_t idU = idesc_bf16(128, 64, false, true);
#pragma unroll
      for (int part = 0; part < 2; ++part)
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          mma_bf16(tmem + COL_W, sdesc(sbase + OFF_TB + part * BLK64 + kk * 32, 16, 1024),
                   sdesc(sbase + OFF_OPA + ROW_K * 128 + kk * 2048, OPA_KB, 1024), idW,
                   (part | kk) != 0);
#pragma unroll
      for (int part = 0; part < 2; ++part)
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          mma_bf16(tmem + COL_UT, sdesc(sbase + OFF_TB + (2 + part) * BLK64 + kk * 32, 16, 1024),
                   sdesc(sbase + OFF_V + kk * 2048, BLK64, 1024), idU, (part | kk) != 0);
      mma_commit(bar);
    }
    ok = cta_wait_mma(bar, phase, p.err);
    if (!ok) break;

    // ---- S7: W -> hi/lo operand rows -----------------------------------------
    if (tid < 64) {
#pragma unroll
      for (int kb = 0; kb < 2; ++kb) {
        float w[64];
        tmem_ld32(tl + COL_W + kb * 64, w);
        tmem_ld32(tl + COL_W + kb * 64 + 32, w + 32);
        tmem_wait_ld();
        write_row_split(sbase + OFF_OPA + kb * OPA_KB + ROW_WHI * 128,
                        sbase + OFF_OPA + kb * OPA_KB + ROW_WLO * 128, tid, w);
#ifdef GDR_PREFILL_DEBUG
        if (dump && t0 == seq_start)
          for (int j = 0; j < 64; ++j) p.dbg[16384 + tid * 128 + kb * 64 + j] = w[j];
#endif
      }
    }
    fence_proxy_async();
    tc_fence_before();
    __syncthreads();

    // ---- S8: [W; Q] H0 (hi/lo) -------------------------------------------------
    if (tid == 0) {
      tc_fence_after();
      const uint32_t id = idesc_bf16(128, 64, false, true);
#pragma unroll
      for (int part = 0; part < 3; ++part) {
        // part 0: [W_hi; Q] H_hi   part 1: [W_hi; Q] H_lo   part 2: [W_lo; *] H_hi
        const uint32_t arow = part < 2 ? ROW_WHI : ROW_WLO;
        const uint32_t hb = part == 1 ? OFF_H + BLK128 : OFF_H;
        const uint32_t dcol = part < 2 ? COL_P : COL_P2;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t koff = (kk >> 2) * OPA_KB + (kk & 3) * 32;
          mma_bf16(tmem + dcol, sdesc(sbase + OFF_OPA + koff + arow * 128, 16, 1024),
                   sdesc(sbase + hb + kk * 2048, BLK128, 1024), id, (part == 1 || kk > 0));
        }
      }
      mma_commit(bar);
    }
    ok = cta_wait_mma(bar, phase, p.err);
    if (!ok) break;

    // ---- S9: U = Ut - W H0 and its scaled copy; O_inter --------------------
    float oreg[N];
    if (tid < 64) {
      const int t = tid;
      const float ed = s_ed[t];
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        float ut[32], pw[32], pl[32];
        tmem_ld32(tl + COL_UT + half * 32, ut);
        tmem_ld32(tl + COL_P + half * 32, pw);
        tmem_ld32(tl + COL_P2 + half * 32, pl);
        tmem_wait_ld();
#pragma unroll
        for (int cb = 0; cb < 4; ++cb) {
          float u[8], us[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            u[e] = ut[cb * 8 + e] - pw[cb * 8 + e] - pl[cb * 8 + e];
            us[e] = u[e] * ed;
          }
          const int c = half * 4 + cb;
          uint4 hi, lo;
          split8(u, hi, lo);
          st_shared16(sbase + OFF_U + 0 * BLK64 + sw128(t, c), hi);
          st_shared16(sbase + OFF_U + 1 * BLK64 + sw128(t, c), lo);
          split8(us, hi, lo);
          st_shared16(sbase + OFF_U + 2 * BLK64 + sw128(t, c), hi);
          st_shared16(sbase + OFF_U + 3 * BLK64 + sw128(t, c), lo);
        }
      }
    } else {
      const int i = tid - 64;
      const float f = p.scale * s_eg[i] * s_rq[i];
      tmem_ld32(tl + COL_P, oreg);
      tmem_ld32(tl + COL_P + 32, oreg + 32);
      tmem_wait_ld();
#pragma unroll
      for (int j = 0; j < N; ++j) oreg[j] *= f;
    }
#ifdef GDR_PREFILL_DEBUG
    if (dump && t0 == seq_start) {
      float tmp[64];
      const uint32_t cols[4] = {COL_UT, COL_P, COL_P2, 0};
      for (int q4 = 0; q4 < 3; ++q4) {
        tmem_ld32(tl + cols[q4], tmp);
        tmem_ld32(tl + cols[q4] + 32, tmp + 32);
        tmem_wait_ld();
        for (int j = 0; j < 64; ++j) p.dbg[32768 + q4 * 8192 + tid * 64 + j] = tmp[j];
      }
    }
#endif
    fence_proxy_async();
    tc_fence_before();
    __syncthreads();

    // ---- S10: K^T U' (hi/lo) and Mq U (hi/lo) ----------------------------------
    if (tid == 0) {
      tc_fence_after();
      const uint32_t idH = idesc_bf16(128, 64, true, true);
      const uint32_t idO = idesc_bf16(128, 64, false, true);
#pragma unroll
      for (int part = 0; part < 2; ++part)
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          mma_bf16(tmem + COL_H, sdesc(sbase + OFF_OPA + ROW_K * 128 + kk * 2048, OPA_KB, 1024),
                   sdesc(sbase + OFF_U + (2 + part) * BLK64 + kk * 2048, BLK64, 1024), idH,
                   (part | kk) != 0);
#pragma unroll
      for (int part = 0; part < 3; ++part) {
        // rows 64..127 of the A tile are Mq: start one block earlier
        const uint32_t ablk = part < 2 ? 3 : 4;       // Mq_hi, Mq_hi, Mq_lo
        const uint32_t ub = part == 1 ? 1 : 0;        // U_hi, U_lo, U_hi
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          mma_bf16(tmem + COL_O, sdesc(sbase + OFF_TB + ablk * BLK64 + kk * 32, 16, 1024),
                   sdesc(sbase + OFF_U + ub * BLK64 + kk * 2048, BLK64, 1024), idO,
                   (part | kk) != 0);
      }
      mma_commit(bar);
    }
    ok = cta_wait_mma(bar, phase, p.err);
    if (!ok) break;

    // ---- S11: state update, output -------------------------------------------
    {
      const float eL = s_eg[63];   // padding rows carry gamma_{L-1}
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        float rh[32];
        tmem_ld32(tl + COL_H + half * 32, rh);
        tmem_wait_ld();
#pragma unroll
        for (int j = 0; j < 32; ++j) hreg[half * 32 + j] = eL * hreg[half * 32 + j] + rh[j];
      }
      write_row_split(sbase + OFF_H, sbase + OFF_H + BLK128, tid, hreg);
      if (tid >= 64) {
        const int t = tid - 64;
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          float ro[32];
          tmem_ld32(tl + COL_O + half * 32, ro);
          tmem_wait_ld();
#pragma unroll
          for (int j = 0; j < 32; ++j) oreg[half * 32 + j] += p.scale * ro[j];
        }
        if (t < L) {
          uint16_t *dst = p.o + (static_cast<size_t>(t0 + t) * p.hv + h) * D + slice * N;
#pragma unroll
          for (int c = 0; c < 8; ++c) *reinterpret_cast<uint4 *>(dst + 8 * c) = pack8(oreg + 8 * c);
        }
      }
#ifdef GDR_PREFILL_DEBUG
      if (dump && t0 == seq_start) {
        float tmp[64];
        const uint32_t cols[2] = {COL_H, COL_O};
        for (int q2 = 0; q2 < 2; ++q2) {
          tmem_ld32(tl + cols[q2], tmp);
          tmem_ld32(tl + cols[q2] + 32, tmp + 32);
          tmem_wait_ld();
          for (int j = 0; j < 64; ++j) p.dbg[57344 + q2 * 8192 + tid * 64 + j] = tmp[j];
        }
      }
#endif
    }
    fence_proxy_async();
    tc_fence_before();
    __syncthreads();
  }

  if (p.hT && ok) {
#pragma unroll
    for (int j = 0; j < N; j += 4)
      *reinterpret_cast<float4 *>(p.hT + srow + j) = make_float4(hreg[j], hreg[j + 1], hreg[j + 2], hreg[j + 3]);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, TM_COLS);
}

}  // namespace

int launch_chunk_prefill(const void *q, const void *k, const void *v, int64_t qk_stride,
                         int64_t v_stride, const void *a, const void *b,
                         const float *A_log, const float *dt_bias, float scale, int hk, int hv,
                         const int32_t *cu_dev, int n_seqs, int max_len, const float *h0, float *hT,
                         void *o, const gdr_prefill_fuse_t *fuse, cudaStream_t s) {
  (void)max_len;
  (void)fuse;
  if (n_seqs > 65535 || hv > 65535) return GDR_ERR_SHAPE;
  // the shared-memory opt-in is a per-device function attribute
  static std::atomic<uint64_t> attr_set{0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return GDR_ERR_CUDA;
  const uint64_t bit = dev < 64 ? (uint64_t{1} << dev) : 0;
  if (!bit || !(attr_set.load(std::memory_order_acquire) & bit)) {
    if (cudaFuncSetAttribute(chunk_prefill_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             SMEM_BYTES) != cudaSuccess)
      return GDR_ERR_CUDA;
    attr_set.fetch_or(bit, std::memory_order_acq_rel);
  }
  PrefillParams p;
  p.q = static_cast<const uint16_t *>(q);
  p.k = static_cast<const uint16_t *>(k);
  p.v = static_cast<const uint16_t *>(v);
  p.a = static_cast<const uint16_t *>(a);
  p.b = static_cast<const uint16_t *>(b);
  p.A_log = A_log;
  p.dt_bias = dt_bias;
  p.scale = scale;
  p.hk = hk;
  p.hv = hv;
  p.group = hv / hk;
  p.qk_stride = qk_stride;
  p.v_stride = v_stride;
  p.cu = cu_dev;
  p.h0 = h0;
  p.hT = hT;
  p.o = static_cast<uint16_t *>(o);
  p.err = device_error_ptr();
#ifdef GDR_PREFILL_DEBUG
  p.dbg = g_dump;
#endif
  dim3 grid(NS, hv, n_seqs);
  chunk_prefill_kernel<<<grid, kThreads, SMEM_BYTES, s>>>(p);
  return last_launch_status();
}

}  // namespace gdr

#ifdef GDR_PREFILL_DEBUG
extern "C" GDR_API void gdr_debug_set_prefill_dump(float *dev_ptr) { gdr::g_dump = dev_ptr; }
#endif
