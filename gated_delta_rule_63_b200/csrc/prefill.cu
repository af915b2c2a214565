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
//     O    = scale (diag(e^gamma) Q H0 + Mq U),  Mq = (Q K^T) . M,  M_ij = e^(gamma_i - gamma_j), j <= i
//     H_L  = e^gamma_L H0 + K^T diag(e^(gamma_L - gamma)) U
// with q, k the L2-normalised rows.
//
// Two kernels.  Everything but the state products is independent of the
// state, so it is built for every chunk at once:
//   * prep (one CTA per chunk x value head, fully parallel): norms, gates,
//     K K^T and Q K^T (tensor cores), A, T = (I + A)^-1 (CUDA cores),
//     W = T' K and Ut = T'' V (tensor cores), Mq; results go to a workspace
//     as the exact shared-memory images the chain kernel copies in;
//   * chain (one CTA per dv slice x value head x sequence): two MMA round
//     trips per chunk, [Q; W] H0 then K^T U' and Mq U, with the chunk's
//     operands streamed in by TMA / bulk copies two chunks ahead.
// Long sequences are cut into windows of chunks so that the workspace stays
// bounded; the state crosses windows in fp32.
//
// Precision.  Raw bf16 q, k, v are exact MMA operands; 1/|q|, 1/|k|, gates
// and decays are folded into fp32 row/column scales of the other operand.
// fp32 operands are split hi + lo bf16 and every product keeps the
// hi*hi + hi*lo + lo*hi terms (two terms when one side is a raw input),
// about 16 significant bits; the state itself never leaves fp32.
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <algorithm>
#include <atomic>
#include <mutex>

#include "gdr_common.cuh"
#include "gdr_host.h"

namespace gdr {
namespace {

constexpr int C = kChunk;      // 64 tokens per chunk
constexpr int D = kHeadDim;    // 128
constexpr int N = 64;          // dv columns per chain CTA
constexpr int NS = D / N;      // dv slices
constexpr uint32_t BLK64 = 64 * 128;     // one [64 x 64] bf16 tile, 128-B swizzled rows

// ---- workspace: one record per (sequence, value head, chunk of the window) --
// Images are laid out exactly as the chain kernel's shared memory expects.
constexpr uint32_t WS_W_HI = 0;          // W_hi  [kb 2][64 rows][128 B]
constexpr uint32_t WS_W_LO = 16384;      // W_lo  [kb 2][64 rows][128 B]
constexpr uint32_t WS_MQ = 32768;        // Mq_lo, Mq_hi: 2 x [64 rows][128 B]
constexpr uint32_t WS_UT = 49152;        // Ut fp32 [slice 2][64 rows][64], 16-B chunk j of row r at j ^ (r & 7)
constexpr uint32_t WS_SC = 81920;        // fp32 gamma[64], 1/|q|[64], 1/|k|[64]
constexpr uint32_t WS_REC = 82944;       // record size (81 KiB)

// ---- prep kernel -------------------------------------------------------------
constexpr int kPrepThreads = 256;
// Three prep CTAs share an SM (67 KB of shared memory, 128 TMEM columns and 80
// registers a thread each), so regions are reused as the chunk moves on:
//   k-block kb (16 KB): K rows (8 KB) | Q rows (8 KB); once K K^T and Q K^T are
//     done the Q half stages Mq (lo in kb 0, hi in kb 1), then receives V
//     (dv block kb); after the W product the K half takes W_hi, and after the
//     Ut product the Q half takes W_lo.
//   T region (32 KB): A / T^T and the X^T scratch during the inverse, then
//     T'_hi, T'_lo, T''_hi, T''_lo, then Ut (fp32).
constexpr uint32_t P_KQ_KB = 128 * 128;              // [K rows 0..63 | Q rows 64..127] per k-block
constexpr uint32_t P_OFF_KQ = 0;                     // 2 k-blocks
constexpr uint32_t P_Q_HALF = 64 * 128;              // offset of the Q half in a k-block
constexpr uint32_t P_OFF_T = P_OFF_KQ + 2 * P_KQ_KB; // T'_hi, T'_lo, T''_hi, T''_lo
constexpr int LD = 68;                               // fp32 row stride of AT (rows 16-byte aligned)
constexpr int XLD = 20;                              // fp32 row stride of the 16 x 16 X^T blocks
constexpr int XLD2 = 36;                             // fp32 row stride of the 32 x 32 X^T block
constexpr uint32_t P_OFF_AT = P_OFF_T;               // A below / T^T on and above the diagonal
constexpr uint32_t P_OFF_XF = P_OFF_AT + 64 * LD * 4;
constexpr uint32_t P_OFF_SC = P_OFF_T + 4 * BLK64;   // gamma, rq, rk, beta, e^gamma, block decay, e^g
static_assert(32 * XLD2 >= 3 * 16 * XLD, "X^T scratch holds both block sizes");
static_assert(P_OFF_XF + 32 * XLD2 * 4 <= P_OFF_SC, "the inverse's scratch fits the T region");
constexpr uint32_t P_OFF_BAR = P_OFF_SC + 7 * 64 * 4;   // 4 mbarriers, TMEM base
constexpr uint32_t P_SMEM = P_OFF_BAR + 48 + 1024;
static_assert(P_OFF_T % 1024 == 0, "swizzled tiles need 1 KB alignment");
static_assert(3 * (P_SMEM + 1024) <= 228 * 1024, "three prep CTAs per SM");
constexpr uint32_t P_TM_COLS = 128;                  // [K K^T ; Q K^T] (64 cols), then W, then Ut

// ---- chain kernel ------------------------------------------------------------
constexpr int kChainThreads = 320;                    // warps 0..7 state and output, 8 products, 9 copies
constexpr int kCtrlWarp = 8;
constexpr int kCopyWarp = 9;
// stage: per k-block the rows [W_lo 0..63 | W_hi 64..127 | Q 128..191] (the M = 64 A
// operands of W H0 and Q H0), then K (two dk blocks), then [Mq_lo; Mq_hi]
constexpr uint32_t C_QW_KB = 192 * 128;
constexpr uint32_t C_OFF_K = 2 * C_QW_KB;
constexpr uint32_t C_OFF_MQ = C_OFF_K + 2 * BLK64;
constexpr uint32_t C_STAGE = C_OFF_MQ + 2 * BLK64;   // 80 KiB
constexpr uint32_t BLK128 = 128 * 128;
constexpr uint32_t C_OFF_H = 2 * C_STAGE;            // [H_hi | H_lo], each [128 dk][64 dv]
constexpr uint32_t C_OFF_U = C_OFF_H + 2 * BLK128;   // [U_hi | U_lo | U'_hi | U'_lo], each [64 tok][64 dv]
constexpr uint32_t C_OFF_BAR = C_OFF_U + 4 * BLK64;  // 15 mbarriers, tmem base, abort flag
// fused gated norm: per-row partial sums of squares of this CTA's two column halves
// [parity 2][half 2][64], the other dv slice's row sums [parity 2][64], two mbarriers
constexpr uint32_t C_OFF_NORM = C_OFF_BAR + 128;
constexpr uint32_t C_OFF_PEER = C_OFF_NORM + 2 * 2 * 64 * 4;
constexpr uint32_t C_OFF_PBAR = C_OFF_PEER + 2 * 64 * 4;
constexpr uint32_t C_SMEM = C_OFF_PBAR + 16 + 1024;
static_assert(C_SMEM <= 232448, "chain shared memory exceeds 227 KB");
static_assert((C_QW_KB | C_OFF_K | C_OFF_MQ | C_STAGE | C_OFF_H | C_OFF_U) % 1024 == 0,
              "swizzled tiles need 1 KB alignment");
constexpr uint32_t C_TM_COLS = 512;
constexpr uint32_t C_COL_P = 0;      // M = 64: Q [H_hi | H_lo], Q row 16 q + i in lane 32 q + i
constexpr uint32_t C_COL_PW = 128;   // M = 64: W_hi [H_hi | H_lo] + W_lo [H_hi | -], W row 16 q + i in lane 32 q + i
constexpr uint32_t C_COL_H = 256;    // K^T [U'_hi | U'_lo], lanes = dk
constexpr uint32_t C_COL_O = 384;    // M = 64: Mq_hi [U_hi | U_lo] + Mq_lo [U_hi | -], row 16 q + i in lane 32 q + i

#ifdef GDR_PREFILL_TIMING
// diagnostic build: step timestamps; prep CTA (0,0,0) in row 0, chain CTA
// (0,0,0) chunk c in row 1 + c (32 slots per row).  Kernels read the buffer
// pointer once (PTIME_INIT) so that a marker costs no memory round trip.
__device__ long long *g_prefill_times;
#define PTIME_INIT() long long *const ptime_buf_ = g_prefill_times
#define PTIME_T(row, step, thread)                                         \
  do {                                                                     \
    if (ptime_buf_ && threadIdx.x == (thread) && blockIdx.x == 0 &&        \
        blockIdx.y == 0 && blockIdx.z == 0 && (row) < 64)                  \
      ptime_buf_[(row) * 32 + (step)] = clock64();                         \
  } while (0)
#define PTIME(row, step) PTIME_T(row, step, 0)
#else
#define PTIME_INIT() \
  do {               \
  } while (0)
#define PTIME_T(row, step, thread) \
  do {                             \
  } while (0)
#define PTIME(row, step) \
  do {                   \
  } while (0)
#endif

// cu_seqlens travels in the launch parameters when there are at most kCuParam
// sequences (a constant-bank read instead of a dependent global load at CTA start)
constexpr int kCuParam = 64;

struct PrefillParams {
  int n_seqs;
  int cu_param[kCuParam + 1];
  const uint16_t *a, *b;
  const float *A_log, *dt_bias;
  float scale;
  int hk, hv, group;
  const int32_t *cu;
  uint8_t *ws;          // workspace records
  int win0;             // first chunk (per sequence) of this window
  int win_chunks;       // chunks per window (record stride)
  const float *state_in;
  float *state_out;
  // state pool (gdr_chunk_prefill_slots): sequence n's state lives in entry slot[n] of
  // `pool`; a slot outside [0, n_slots) is a sequence that starts from zero and keeps
  // nothing (its state crosses windows in `carry`)
  const int32_t *slot;   // null: the states are state_in / state_out, indexed by sequence
  int n_slots;
  int pool_init;         // 1: the first window reads the entry, 0: it starts from zero
  float *pool;
  float *carry;
  int last_window;
  uint16_t *o;          // may be null when y is set
  // gated RMSNorm fused into the output (y != null): y = o / sqrt(mean o^2 + eps) w SiLU(z)
  const uint16_t *z;
  const float *norm_w;  // null = ones
  float eps;
  uint16_t *y;
  int *err;
};

// 8 fp32 values -> hi/lo bf16 16-byte chunks at two addresses (shared or global)
__device__ __forceinline__ void st_split8_shared(uint32_t hi_addr, uint32_t lo_addr, const float *v8) {
  uint4 hi, lo;
  split8x2(v8, hi, lo);
  st_shared16(hi_addr, hi);
  st_shared16(lo_addr, lo);
}

// one thread waits (bounded), the CTA agrees on the outcome
__device__ __forceinline__ bool cta_wait(uint32_t bar, uint32_t parity, int *err, bool also = true) {
  bool ok = also;
  if (threadIdx.x == 0 && ok) ok = mbar_wait(bar, parity, err);
  ok = __syncthreads_and(ok) != 0;
  tc_fence_after();
  return ok;
}

__device__ __forceinline__ int cu_at(const PrefillParams &p, int i) {
  return p.n_seqs <= kCuParam ? p.cu_param[i] : __ldg(p.cu + i);
}

__device__ __forceinline__ uint8_t *ws_record(const PrefillParams &p, int n, int h, int cw) {
  return p.ws + ((static_cast<size_t>(n) * p.hv + h) * p.win_chunks + cw) * WS_REC;
}

// =============================================================================
// prep: one chunk of one value head
// =============================================================================
__global__ void __launch_bounds__(kPrepThreads, 3)
prep_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
            const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ PrefillParams p) {
  PTIME_INIT();
  grid_dep_wait();
  grid_dep_launch();
  const int cw = blockIdx.x, h = blockIdx.y, n = blockIdx.z;
  const int seq_start = cu_at(p, n), seq_end = cu_at(p, n + 1);
  const int t0 = seq_start + (p.win0 + cw) * C;
  if (t0 >= seq_end) return;   // the window runs past this sequence (uniform exit)
  const int L = min(C, seq_end - t0);

  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  const uint32_t sbase = (raw_addr + 1023u) & ~1023u;
  uint8_t *smem = smem_raw + (sbase - raw_addr);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int kh = h / p.group;
  float *AT = reinterpret_cast<float *>(smem + P_OFF_AT);
  float *XF = reinterpret_cast<float *>(smem + P_OFF_XF);
  float *s_g = reinterpret_cast<float *>(smem + P_OFF_SC);
  float *s_rq = s_g + 64, *s_rk = s_g + 128, *s_beta = s_g + 192, *s_eg = s_g + 256, *s_eb = s_g + 320;
  float *s_e1 = s_g + 384;   // e^(g_t): one step of decay
  const uint32_t bar_tma = sbase + P_OFF_BAR, bar_mma = sbase + P_OFF_BAR + 8;
  const uint32_t bar_v = sbase + P_OFF_BAR + 16, bar_u = sbase + P_OFF_BAR + 24;
  uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(smem + P_OFF_BAR + 32);
  const uint32_t q_half0 = sbase + P_OFF_KQ + P_Q_HALF, q_half1 = q_half0 + P_KQ_KB;
  uint8_t *rec = ws_record(p, n, h, cw);

  if (tid == 0) {   // the copies go out first
    mbar_init(bar_tma, 1);
    mbar_init(bar_mma, 1);
    mbar_init(bar_v, 1);
    mbar_init(bar_u, 1);
    fence_mbar_init();
    mbar_arrive_expect_tx(bar_tma, 4 * BLK64);
#pragma unroll
    for (int kb = 0; kb < 2; ++kb) {
      tma_load_2d(sbase + P_OFF_KQ + kb * P_KQ_KB, &tm_k, kh * D + kb * 64, t0, bar_tma);
      tma_load_2d(sbase + P_OFF_KQ + kb * P_KQ_KB + P_Q_HALF, &tm_q, kh * D + kb * 64, t0, bar_tma);
    }
  }
  // gate inputs of the chunk's rows (threads 0..63), in flight until the gates are
  // needed after the norms; padding rows get no decay and no write
  uint16_t a_raw = 0, b_raw = 0;
  float a_log = 0.0f, dtb = 0.0f;
  const bool gate_row = tid < L;
  if (gate_row) {
    const size_t ab = static_cast<size_t>(t0 + tid) * p.hv + h;
    a_raw = __ldg(p.a + ab);
    b_raw = __ldg(p.b + ab);
    a_log = __ldg(p.A_log + h);
    dtb = __ldg(p.dt_bias + h);
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(tmem_holder), P_TM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  PTIME(0, 0);
  bool ok = cta_wait(bar_tma, 0, p.err);
  PTIME(0, 1);

  if (ok && L < C) {   // rows past the sequence end hold other tokens: zero them
    const uint32_t nz = static_cast<uint32_t>(C - L) * 16;   // rows x 16-B chunks per tile
    for (uint32_t e = tid; e < 2 * nz; e += kPrepThreads) {   // K and Q (V when it arrives)
      const uint32_t tile = e / nz, rem = e % nz, r = L + rem / 16, cc = rem % 16;
      const uint32_t base = P_OFF_KQ + (cc >> 3) * P_KQ_KB + tile * P_Q_HALF;
      st_shared16(sbase + base + sw128(r, cc & 7), make_uint4(0, 0, 0, 0));
    }
    fence_proxy_async();
    __syncthreads();
  }
  if (ok) {
    // ---- [K; Q] K^T on the raw tiles, while the norms and gates are computed ----------
    if (tid == 0) {
      tc_fence_after();
      const uint32_t id = idesc_bf16(128, 64, false, false);
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
        const uint32_t koff = (kk >> 2) * P_KQ_KB + (kk & 3) * 32;
        mma_bf16(tmem, sdesc(sbase + P_OFF_KQ + koff, 16, 1024),
                 sdesc(sbase + P_OFF_KQ + koff, 16, 1024), id, kk > 0);
      }
      mma_commit(bar_mma);
    }
    // 1/|k| (rows 0..63 of the KQ tile) and 1/|q| (rows 64..127), two threads per row
    const int row = tid >> 1, part = tid & 1;
    float ss = 0.0f;
#pragma unroll
    for (int cc = 0; cc < 8; ++cc) {
      const int c16 = part * 8 + cc;
      float f[8];
      unpack8(ld_shared16(sbase + P_OFF_KQ + (c16 >> 3) * P_KQ_KB + sw128(row, c16 & 7)), f);
#pragma unroll
      for (int e = 0; e < 8; ++e) ss += f[e] * f[e];
    }
    ss += __shfl_xor_sync(0xffffffffu, ss, 1);
    if (part == 0) (row < 64 ? s_rk : s_rq)[row & 63] = 1.0f / sqrtf(ss + 1e-6f);
    // gates: g = -exp(A_log) softplus(a + dt_bias), beta = sigmoid(b) (threads 0..63)
    float g = 0.0f;
    if (tid < 64) {
      float beta = 0.0f;
      if (gate_row) {
        g = -expf(a_log) * softplus_f(bf_bits2f(a_raw) + dtb);
        beta = sigmoid_f(bf_bits2f(b_raw));
      }
      s_beta[tid] = beta;
    }
    // inclusive scan of g over the chunk (threads 0..63)
    float run = g;
    if (tid < 64) {
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const float up = __shfl_up_sync(0xffffffffu, run, off);
        if (lane >= off) run += up;
      }
      if (tid == 31) XF[0] = run;
    }
    __syncthreads();
    if (tid < 64) s_g[tid] = run + (tid >= 32 ? XF[0] : 0.0f);
    __syncthreads();
    if (tid < 64) {
      s_eg[tid] = __expf(s_g[tid]);
      s_eb[tid] = __expf(s_g[tid | 15] - s_g[tid]);   // decay to the end of the 16-block
      s_e1[tid] = __expf(g);
      float *sc = reinterpret_cast<float *>(rec + WS_SC);
      sc[tid] = s_g[tid];
      sc[64 + tid] = s_rq[tid];
      sc[128 + tid] = s_rk[tid];
    }
    fence_proxy_async();
    tc_fence_before();
    __syncthreads();

    PTIME(0, 2);
    ok = cta_wait(bar_mma, 0, p.err);
  }
  if (ok) {
    PTIME(0, 3);
    // ---- A (rows 0..63) and Mq (rows 64..127): 2 threads per row, 32 columns each
    const int q4 = warp & 3, hf = warp >> 2;
    const int row = 32 * q4 + lane;
    float sv[32];
    PTIME(0, 17);
    // per-column factors of this thread's 32 columns: 1/|k_j| and the decay e^(g_i - g_j)
    const int i = row & 63, ib = i >> 4;
    const float gi = s_g[i];
    // e^(g_i - g_j): for a whole earlier 16-block as e^(g_i - g_end) e^(g_end - g_j) (both <= 1);
    // inside the row's own block as a backward running product of one-step decays e^(g_t)
    float colf[32];
#pragma unroll
    for (int b2 = 0; b2 < 2; ++b2) {
      const int blk = 2 * hf + b2;
      const float fi = __expf(gi - s_g[blk * 16 + 15]);   // used for blocks before the row's own only
      float dg[16];
      float run = 0.0f;
#pragma unroll
      for (int e = 15; e >= 0; --e) {
        const int j = blk * 16 + e;
        run = (j == i) ? 1.0f : (e == 15 ? 0.0f : run * s_e1[j + 1]);   // zero above the diagonal
        dg[e] = run;
      }
#pragma unroll
      for (int e4 = 0; e4 < 4; ++e4) {
        const int j0 = blk * 16 + 4 * e4;
        const float4 rk4 = *reinterpret_cast<const float4 *>(s_rk + j0);
        const float4 eb4 = *reinterpret_cast<const float4 *>(s_eb + j0);
        const float rkv[4] = {rk4.x, rk4.y, rk4.z, rk4.w};
        const float ebv[4] = {eb4.x, eb4.y, eb4.z, eb4.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float dec = blk < ib ? fi * ebv[e] : dg[4 * e4 + e];
          colf[b2 * 16 + 4 * e4 + e] = rkv[e] * dec;
        }
      }
    }
    PTIME(0, 11);
    tmem_ld32(tmem + (static_cast<uint32_t>(32 * q4) << 16) + 32 * hf, sv);
    tmem_wait_ld();
    if (row < 64) {   // A_ij = beta_i / |k_i| * (k_i.k_j) / |k_j| * e^(g_i - g_j), j < i
      // (columns j >= i hold junk until T^T overwrites them)
      const float bi = s_beta[i] * s_rk[i];
#pragma unroll
      for (int c4 = 0; c4 < 8; ++c4)
        *reinterpret_cast<float4 *>(AT + i * LD + 32 * hf + 4 * c4) =
            make_float4(bi * sv[4 * c4] * colf[4 * c4], bi * sv[4 * c4 + 1] * colf[4 * c4 + 1],
                        bi * sv[4 * c4 + 2] * colf[4 * c4 + 2], bi * sv[4 * c4 + 3] * colf[4 * c4 + 3]);
    } else {          // Mq_ij = (q_i.k_j) / (|q_i| |k_j|) * e^(g_i - g_j), j <= i
      const float qi = s_rq[i];
#pragma unroll
      for (int c4 = 0; c4 < 4; ++c4) {
        float m[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) m[e] = sv[8 * c4 + e] * qi * colf[8 * c4 + e];
        const uint32_t off = sw128(i, 4 * hf + c4);   // staged in the dead Q halves, stored in bulk
        st_split8_shared(q_half1 + off, q_half0 + off, m);   // Mq_hi, Mq_lo
      }
    }
    PTIME(0, 12);
    fence_proxy_async();
    __syncthreads();
    if (tid == 128) {   // (a thread the inverse below leaves idle)
      bulk_store(rec + WS_MQ, q_half0, BLK64);           // Mq_lo
      bulk_store(rec + WS_MQ + BLK64, q_half1, BLK64);   // Mq_hi
      bulk_commit();
      bulk_wait_read();
      // V (dv block kb into the Q half of k-block kb), in flight during the inverse
      mbar_arrive_expect_tx(bar_v, 2 * BLK64);
      tma_load_2d(q_half0, &tm_v, h * D, t0, bar_v);
      tma_load_2d(q_half1, &tm_v, h * D + 64, t0, bar_v);
    }

    PTIME(0, 4);
    // ---- T = (I + A)^-1, stored transposed on and above the diagonal ----------
    if (tid < 64) {   // diagonal 16x16 blocks, one column per thread
      const int bb = tid >> 4, cc = tid & 15;
      float x[16];
#pragma unroll
      for (int r = 0; r < 16; ++r) {
        float sacc = (r == cc) ? 1.0f : 0.0f;
#pragma unroll
        for (int j = 0; j < r; ++j) sacc -= AT[(16 * bb + r) * LD + 16 * bb + j] * x[j];
        x[r] = sacc;
      }
#pragma unroll
      for (int r = 0; r < 16; ++r)
        if (r >= cc) AT[(16 * bb + cc) * LD + 16 * bb + r] = x[r];
    }
    PTIME(0, 13);
    __syncthreads();
    // off-diagonal blocks.  Level 1: the two 16 x 16 blocks (1, 0) and (3, 2) that complete
    // the 32 x 32 diagonal halves, X_bc = A_bc T_cc, T_bc = -T_bb X_bc, on 64 threads per block with 2 x 2
    // tiles (rows rt, rt + 8; columns jt, jt + 8).  Level 2: the 32 x 32 block below the
    // diagonal of the two 32 x 32 halves T1, T2 (complete after level 1),
    // X = A21 T1, T21 = -T2 X, on all 256 threads with 2 x 2 tiles (rows rt, rt + 16;
    // columns jt, jt + 16).  A rows and T^T rows are read as float4 along k.
    {
      const int blk = tid >> 6, t = tid & 63, rt = t >> 3, jt = t & 7;
      const int bb = 1 + 2 * blk, cb = 2 * blk;
      if (blk < 2) {   // X_bc^T[j][r] into XF
        const float *a0 = AT + (16 * bb + rt) * LD, *a1 = a0 + 8 * LD;
        const float *t0 = AT + (16 * cb + jt) * LD, *t1 = t0 + 8 * LD;   // T^T rows = columns of T
        float x00 = 0.0f, x01 = 0.0f, x10 = 0.0f, x11 = 0.0f;         // x[r][j] for r in {rt, rt+8}, j in {jt, jt+8}
#pragma unroll
        for (int g = 0; g < 4; ++g) {   // T[16c + l][16c + j] is zero for l < j
          const int k = 16 * cb + 4 * g;
          const float4 A0 = *reinterpret_cast<const float4 *>(a0 + k), A1 = *reinterpret_cast<const float4 *>(a1 + k);
          const float4 T0 = *reinterpret_cast<const float4 *>(t0 + k), T1 = *reinterpret_cast<const float4 *>(t1 + k);
          const float av0[4] = {A0.x, A0.y, A0.z, A0.w}, av1[4] = {A1.x, A1.y, A1.z, A1.w};
          const float tv0[4] = {T0.x, T0.y, T0.z, T0.w}, tv1[4] = {T1.x, T1.y, T1.z, T1.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float u0 = (4 * g + e >= jt) ? tv0[e] : 0.0f, u1 = (4 * g + e >= jt + 8) ? tv1[e] : 0.0f;
            x00 += av0[e] * u0; x01 += av0[e] * u1;
            x10 += av1[e] * u0; x11 += av1[e] * u1;
          }
        }
        float *xt = XF + (blk * 16 + jt) * XLD;
        xt[rt] = x00;
        xt[rt + 8] = x10;
        xt[8 * XLD + rt] = x01;
        xt[8 * XLD + rt + 8] = x11;
      }
      __syncthreads();
      if (blk < 2) {   // T_bc[r][j] = -sum_{l <= r} T_bb[r][l] X_bc[l][j], stored as T^T
        const float *xa = XF + (blk * 16 + jt) * XLD, *xb = xa + 8 * XLD;
        const float *tb = AT + (16 * bb) * LD + 16 * bb;               // tb[l * LD + r] = T_bb[r][l]
        float y00 = 0.0f, y01 = 0.0f, y10 = 0.0f, y11 = 0.0f;         // y[r][j]
#pragma unroll
        for (int l = 0; l < 16; ++l) {
          const float t0v = l <= rt ? tb[l * LD + rt] : 0.0f, t1v = l <= rt + 8 ? tb[l * LD + rt + 8] : 0.0f;
          const float x0 = xa[l], x1 = xb[l];
          y00 -= t0v * x0; y01 -= t0v * x1;
          y10 -= t1v * x0; y11 -= t1v * x1;
        }
        float *dst = AT + (16 * cb + jt) * LD + 16 * bb;
        dst[rt] = y00;
        dst[rt + 8] = y10;
        dst[8 * LD + rt] = y01;
        dst[8 * LD + rt + 8] = y11;
      }
      __syncthreads();
      PTIME(0, 14);
    }
    {
      // The triangular factors make half of these products zero; each warp takes two
      // adjacent columns (resp. rows) so that its loops skip the zero k-groups (l-groups)
      // with warp-uniform bounds.
      {   // X^T[j][r] = sum_{k >= j} A[32 + r][k] T[k][j], r, j < 32, into XF (stride XLD2)
        const int rt = lane & 15, jt = 2 * warp + (lane >> 4);   // outputs (rt | rt+16, jt | jt+16)
        const float *a0 = AT + (32 + rt) * LD, *a1 = a0 + 16 * LD;
        const float *t0 = AT + jt * LD, *t1 = t0 + 16 * LD;
        float x00 = 0.0f, x01 = 0.0f, x10 = 0.0f, x11 = 0.0f;   // x[r][j], r in {rt, rt+16}, j in {jt, jt+16}
        const int g0 = warp >> 1, g1 = 4 + (warp >> 1);         // first k-groups holding k >= jt, k >= jt + 16
#pragma unroll 1
        for (int g = g0; g < 8; ++g) {
          const int k0 = 4 * g;
          const float4 A0 = *reinterpret_cast<const float4 *>(a0 + k0), A1 = *reinterpret_cast<const float4 *>(a1 + k0);
          const float4 T0 = *reinterpret_cast<const float4 *>(t0 + k0);
          const float av0[4] = {A0.x, A0.y, A0.z, A0.w}, av1[4] = {A1.x, A1.y, A1.z, A1.w};
          const float tv0[4] = {T0.x, T0.y, T0.z, T0.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {   // T is lower triangular: T[k][j] = 0 for k < j
            const float u0 = (k0 + e >= jt) ? tv0[e] : 0.0f;
            x00 += av0[e] * u0;
            x10 += av1[e] * u0;
          }
          if (g >= g1) {
            const float4 T1 = *reinterpret_cast<const float4 *>(t1 + k0);
            const float tv1[4] = {T1.x, T1.y, T1.z, T1.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const float u1 = (k0 + e >= jt + 16) ? tv1[e] : 0.0f;
              x01 += av0[e] * u1;
              x11 += av1[e] * u1;
            }
          }
        }
        float *xt = XF + jt * XLD2;
        xt[rt] = x00;
        xt[rt + 16] = x10;
        xt[16 * XLD2 + rt] = x01;
        xt[16 * XLD2 + rt + 16] = x11;
      }
      __syncthreads();
      {   // T21[r][j] = -sum_{l <= r} T2[r][l] X[l][j], T2[r][l] = AT[(32 + l) LD + 32 + r]; stored as T^T
        const int rt = 2 * warp + (lane >> 4), jt = lane & 15;   // outputs (rt | rt+16, jt | jt+16)
        const float *xa = XF + jt * XLD2, *xb = xa + 16 * XLD2;
        const float *tb = AT + 32 * LD + 32;
        float y00 = 0.0f, y01 = 0.0f, y10 = 0.0f, y11 = 0.0f;   // y[r][j]
        const int la = warp >> 1, lb = 4 + (warp >> 1);         // last l-groups holding l <= rt, l <= rt + 16
#pragma unroll 1
        for (int l4 = 0; l4 <= lb; ++l4) {
          const float4 X0 = *reinterpret_cast<const float4 *>(xa + 4 * l4), X1 = *reinterpret_cast<const float4 *>(xb + 4 * l4);
          const float x0v[4] = {X0.x, X0.y, X0.z, X0.w}, x1v[4] = {X1.x, X1.y, X1.z, X1.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int l = 4 * l4 + e;
            const float t1v = l <= rt + 16 ? tb[l * LD + rt + 16] : 0.0f;
            y10 -= t1v * x0v[e]; y11 -= t1v * x1v[e];
          }
          if (l4 <= la) {
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int l = 4 * l4 + e;
              const float t0v = l <= rt ? tb[l * LD + rt] : 0.0f;
              y00 -= t0v * x0v[e]; y01 -= t0v * x1v[e];
            }
          }
        }
        float *dst = AT + jt * LD + 32;
        dst[rt] = y00;
        dst[rt + 16] = y10;
        dst[16 * LD + rt] = y01;
        dst[16 * LD + rt + 16] = y11;
      }
      __syncthreads();
      PTIME(0, 15);
    }

    PTIME(0, 5);
    // ---- T' = T diag(beta e^g / |k|), T'' = T diag(beta), hi/lo tiles --------
    {   // tiles with the row index r contiguous (MN-major operands): row j, 16-byte chunk r / 8
      const int j = tid & 63;
      const float f2 = s_beta[j], f1 = f2 * s_eg[j] * s_rk[j];
      float tv[2][8];
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        const int r0 = 8 * ((tid >> 6) + 4 * hh);
        const float4 v0 = *reinterpret_cast<const float4 *>(AT + j * LD + r0);
        const float4 v1 = *reinterpret_cast<const float4 *>(AT + j * LD + r0 + 4);
        tv[hh][0] = v0.x; tv[hh][1] = v0.y; tv[hh][2] = v0.z; tv[hh][3] = v0.w;
        tv[hh][4] = v1.x; tv[hh][5] = v1.y; tv[hh][6] = v1.z; tv[hh][7] = v1.w;
      }
      __syncthreads();   // T^T is read out: the tiles take its place
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        const int rg = (tid >> 6) + 4 * hh, r0 = 8 * rg;
        float t1[8], t2[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const float tij = (r0 + e >= j) ? tv[hh][e] : 0.0f;   // T[r][j], lower triangle
          t1[e] = tij * f1;
          t2[e] = tij * f2;
        }
        const uint32_t off = sw128(j, rg);
        st_split8_shared(sbase + P_OFF_T + off, sbase + P_OFF_T + BLK64 + off, t1);
        st_split8_shared(sbase + P_OFF_T + 2 * BLK64 + off, sbase + P_OFF_T + 3 * BLK64 + off, t2);
      }
    }
    fence_proxy_async();
    ok = cta_wait(bar_v, 0, p.err);   // V has landed in the Q halves
    if (ok && L < C) {   // rows past the sequence end hold other tokens: zero them
      const uint32_t nz = static_cast<uint32_t>(C - L) * 16;
      for (uint32_t e = tid; e < nz; e += kPrepThreads) {
        const uint32_t r = L + e / 16, cc = e % 16;
        st_shared16(q_half0 + (cc >> 3) * P_KQ_KB + sw128(r, cc & 7), make_uint4(0, 0, 0, 0));
      }
      fence_proxy_async();
      __syncthreads();
    }

    PTIME(0, 6);
    // ---- W = T' K (rows in lanes 0..63), then Ut = T'' V (rows in lanes 64..127) in the
    // same TMEM columns once W has been read out.  MN-major A operands of 128 rows: W's
    // second row block and Ut's first are other tiles, whose products land in lanes that
    // are never read
    if (ok && tid == 0) {
      tc_fence_after();
      const uint32_t id = idesc_bf16(128, 128, true, true);
#pragma unroll
      for (int part = 0; part < 2; ++part)
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          mma_bf16(tmem, sdesc(sbase + P_OFF_T + part * BLK64 + kk * 2048, BLK64, 1024),
                   sdesc(sbase + P_OFF_KQ + kk * 2048, P_KQ_KB, 1024), id, (part | kk) != 0);
      mma_commit(bar_mma);
    }
  }
  PTIME(0, 7);
  // ok is uniform across the CTA here; below, the warps of TMEM lanes 0..63 (W) and
  // 64..127 (Ut) wait on their own products
  bool good = ok;
  if (ok) {
    if ((warp & 2) == 0) {
      // warps 0, 1, 4, 5: W rows of k-block kb = warp >> 2; W_hi goes into the K half at
      // once (K is dead once W is done), W_lo into the Q half once Ut has read V there
      const int kb = warp >> 2, r = 32 * (warp & 1) + lane;
      const uint32_t tl = tmem + (static_cast<uint32_t>(32 * (warp & 3)) << 16) + 64 * kb;
      const uint32_t hi_base = sbase + P_OFF_KQ + kb * P_KQ_KB, lo_base = hi_base + P_Q_HALF;
      bool wok = lane == 0 ? mbar_wait(bar_mma, 1, p.err) : true;
      wok = __shfl_sync(0xffffffffu, wok ? 1 : 0, 0) != 0;
      tc_fence_after();
      uint4 lo[8];
      if (wok) {
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          float w[32];
          tmem_ld32(tl + 32 * hh, w);
          tmem_wait_ld();
#pragma unroll
          for (int c4 = 0; c4 < 4; ++c4) {
            uint4 hi;
            split8x2(w + 8 * c4, hi, lo[4 * hh + c4]);
            st_shared16(hi_base + sw128(r, 4 * hh + c4), hi);
          }
        }
      }
      fence_proxy_async();   // W_hi is visible to the bulk copy below
      tc_fence_before();
      const bool all_w = named_sync_or(1, 128, !wok) == false;   // W is out of TMEM
      if (tid == 0 && all_w) {
        tc_fence_after();
        const uint32_t id = idesc_bf16(128, 128, true, true);
#pragma unroll
        for (int part = 0; part < 2; ++part)
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_bf16(tmem, sdesc(sbase + P_OFF_T + (1 + part) * BLK64 + kk * 2048, BLK64, 1024),
                     sdesc(q_half0 + kk * 2048, P_KQ_KB, 1024), id, (part | kk) != 0);
        mma_commit(bar_u);
        // W_hi goes out while Ut is computed
        bulk_store(rec + WS_W_HI, sbase + P_OFF_KQ, BLK64);                     // k-block 0
        bulk_store(rec + WS_W_HI + BLK64, sbase + P_OFF_KQ + P_KQ_KB, BLK64);   // k-block 1
        bulk_commit();
      }
      bool uok = all_w;
      if (lane == 0 && uok) uok = mbar_wait(bar_u, 0, p.err);
      uok = __shfl_sync(0xffffffffu, uok ? 1 : 0, 0) != 0;
      if (uok) {
#pragma unroll
        for (int i = 0; i < 8; ++i) st_shared16(lo_base + sw128(r, i), lo[i]);
      }
      fence_proxy_async();
      good = named_sync_or(1, 128, !uok) == false;
      if (tid == 0 && good) {
        bulk_store(rec + WS_W_LO, q_half0, BLK64);            // k-block 0
        bulk_store(rec + WS_W_LO + BLK64, q_half1, BLK64);    // k-block 1
        bulk_commit();
      }
    } else {
      // warps 2, 3, 6, 7 (lanes 64..127): Ut rows -> fp32 [slice][row][64] over the T tiles
      const int sl = warp >> 2, r = 32 * (warp & 1) + lane;
      const uint32_t tl = tmem + (static_cast<uint32_t>(32 * (warp & 3)) << 16) + 64 * sl;
      const uint32_t dst = sbase + P_OFF_T + (static_cast<uint32_t>(sl) * 64 + r) * 256;
      bool uok = lane == 0 ? mbar_wait(bar_u, 0, p.err) : true;
      uok = __shfl_sync(0xffffffffu, uok ? 1 : 0, 0) != 0;
      tc_fence_after();
      if (uok) {
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          float u[32];
          tmem_ld32(tl + 32 * hh, u);
          tmem_wait_ld();
#pragma unroll
          for (int c4 = 0; c4 < 8; ++c4) {
            const uint32_t j = (8 * hh + c4) ^ (r & 7);
            st_shared16(dst + 16 * j, make_uint4(__float_as_uint(u[4 * c4]), __float_as_uint(u[4 * c4 + 1]),
                                                 __float_as_uint(u[4 * c4 + 2]), __float_as_uint(u[4 * c4 + 3])));
          }
        }
      }
      fence_proxy_async();
      good = named_sync_or(2, 128, !uok) == false;
      if (tid == 64 && good) {
        bulk_store(rec + WS_UT, sbase + P_OFF_T, 4 * BLK64);
        bulk_commit();
      }
    }
  }
  PTIME(0, 9);
  // the threads that issued stores (0: W, 64: Ut) wait until the shared memory is read
  if (tid == 0 || tid == 64) bulk_wait_read();
  tc_fence_before();
  __syncthreads();
  PTIME(0, 10);
  if (warp == 0) tmem_dealloc(tmem, P_TM_COLS);
}

// =============================================================================
// chain: the state of one dv slice of one value head through one window
// =============================================================================
// One CTA per (64-column dv slice, value head, sequence).  The fp32 state slice
// H (128 dk rows x 64 dv columns) stays in registers of warps 0..7: warp w
// holds rows 32 (w & 3) .. + 31 (its TMEM lane quarter), columns
// 32 (w >> 2) .. + 31.  Per chunk:
//   PW = W_hi [H_hi | H_lo] + W_lo [H_hi | -]   (M = 64)             tensor cores
//   P  = Q [H_hi | H_lo]   (M = 64, for Q H0, after PW)               tensor cores
//   U  = Ut - W H0,  U' = U e^(gamma_L - gamma) / |k|                warps 0..7
//   (an M = 64 product puts 16 W rows on each of the four TMEM lane quarters, so the U
//   phase runs on all four SM sub-partitions, 16 rows x 32 columns a warp)
//   H' = K^T [U'_hi | U'_lo]                                         tensor cores
//   H  = e^gamma_L H + H'                                            warps 0..7
//   O  = Mq_hi [U_hi | U_lo] + Mq_lo [U_hi | -]   (M = 64)           tensor cores
//   o  = scale (e^gamma / |q| Q H0 + O)                              warps 0..7
//   (the output products take the U phase's layout: each warp reads 16 output rows x 32
//   columns of its lane quarter, so the output and the fused norm run on all four SM
//   sub-partitions)
// N = 128 products stack the hi and lo parts of one operand side by side, so
// each fp32 product takes two MMA groups instead of three.  Warp 8 issues the
// products on the state's critical path (PW, K^T U'); warp 9 issues the output's
// products (P after PW, O after K^T U', so neither delays the chain in the tensor
// pipe) and every operand copy.  The roles meet only on mbarriers (no CTA-wide
// barrier inside the chunk loop).  Operands arrive two chunks ahead in three
// groups ([Q | W_hi | W_lo], K, Mq) in two stages; warp 9 refills a stage once
// the chunk's O, its last product, is done.  Ut and the chunk scalars are read
// into registers a chunk ahead; the output of a chunk is finished while the
// next chunk's first products run.
// The handoffs (mbarrier: who completes it -> what it allows):
//   full_qw, full_k, full_mq (per stage): a chunk's copies landed -> its products may read them
//   bar_pw:  PW done (commit)           -> every state warp reads W H0 for the U phase
//   bar_p:   P done (commit)            -> every state warp reads Q H0, then may rewrite the H tiles
//   u_ready: U, U' tiles written (8 warps) -> K^T U' and O may be issued
//   bar_h:   K^T U' done (commit)       -> every state warp updates its part of H
//   h_ready: H tiles written (8 warps)  -> the next chunk's PW (then its P, which overwrites P's region)
//   bar_o:   O done (commit)            -> every state warp reads it; the U tiles may be rewritten
//   o_free:  O read (8 warps)           -> the next O may be issued, the Mq stage refilled

// the same for an mbarrier that another CTA of the cluster arrives on; it polls
// (with a short back-off) instead of sleeping in try_wait
__device__ __forceinline__ bool chain_wait_cluster(uint32_t bar, uint32_t parity, volatile uint32_t *abort, int *err) {
  const long long start = clock64();
  while (!*abort) {
    if (mbar_test_wait_cluster(bar, parity)) return true;
    __nanosleep(32);
    if (clock64() - start > (1LL << 32)) {
      *abort = 1u;
      raise_device_error(err, GDR_ERR_TIMEOUT);
      return false;
    }
  }
  return false;
}

template <bool kNorm>   // gated RMSNorm fused into the output (p.y set, cluster of the two dv slices)
__global__ void __launch_bounds__(kChainThreads, 1)
chain_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
             const __grid_constant__ PrefillParams p) {
  PTIME_INIT();
  grid_dep_wait();
  grid_dep_launch();
  const int slice = blockIdx.x, h = blockIdx.y, n = blockIdx.z;
  const int seq_start = cu_at(p, n), seq_end = cu_at(p, n + 1);
  const int n_all = (seq_end - seq_start + C - 1) / C;
  const int c_end = min(n_all, p.win0 + p.win_chunks);
  const int nw = max(0, c_end - p.win0);              // chunks of this window
  if (nw == 0 && p.win0 > 0) return;                  // state already final

  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  const uint32_t sbase = (raw_addr + 1023u) & ~1023u;
  uint8_t *smem = smem_raw + (sbase - raw_addr);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int kh = h / p.group;
  const uint32_t bars = sbase + C_OFF_BAR;
  const uint32_t full_qw = bars, full_k = bars + 16, full_mq = bars + 32;   // + 8 * stage
  const uint32_t bar_p = bars + 48, bar_h = bars + 56, bar_o = bars + 64;  // products complete
  const uint32_t o_free = bars + 72, h_ready = bars + 80, u_ready = bars + 88, bar_drain = bars + 96;
  const uint32_t bar_pw = bars + 104, bar_drain2 = bars + 112;
  uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(smem + C_OFF_BAR + 120);
  volatile uint32_t *abort_flag = reinterpret_cast<volatile uint32_t *>(smem + C_OFF_BAR + 124);
  const bool ctrl = warp == kCtrlWarp, copier = warp == kCopyWarp, state = warp < kCtrlWarp;

  if (warp == 0) {
    tmem_alloc(smem_u32(tmem_holder), C_TM_COLS);
    tmem_relinquish();
  }
  auto t0_of = [&](int cw) { return seq_start + (p.win0 + cw) * C; };
  // copies of chunk cw into stage cw & 1 (lane 0 of the copy warp); issued counts per group
  int iss_qw = 0, iss_k = 0, iss_mq = 0;
  auto load_qw = [&](int cw) {
    const uint32_t st = sbase + (cw & 1) * C_STAGE, fb = full_qw + 8 * (cw & 1);
    const uint8_t *rec = ws_record(p, n, h, cw);
    mbar_arrive_expect_tx(fb, 6 * BLK64);
#pragma unroll
    for (int kb = 0; kb < 2; ++kb) {
      bulk_load(st + kb * C_QW_KB, rec + WS_W_LO + kb * BLK64, BLK64, fb);
      bulk_load(st + kb * C_QW_KB + 64 * 128, rec + WS_W_HI + kb * BLK64, BLK64, fb);
      tma_load_2d(st + kb * C_QW_KB + 128 * 128, &tm_q, kh * D + kb * 64, t0_of(cw), fb);
    }
    iss_qw = cw + 1;
  };
  auto load_k = [&](int cw) {
    const uint32_t st = sbase + (cw & 1) * C_STAGE, fb = full_k + 8 * (cw & 1);
    mbar_arrive_expect_tx(fb, 2 * BLK64);
#pragma unroll
    for (int kb = 0; kb < 2; ++kb) tma_load_2d(st + C_OFF_K + kb * BLK64, &tm_k, kh * D + kb * 64, t0_of(cw), fb);
    iss_k = cw + 1;
  };
  auto load_mq = [&](int cw) {   // Mq_lo | Mq_hi are contiguous in the record
    const uint32_t st = sbase + (cw & 1) * C_STAGE, fb = full_mq + 8 * (cw & 1);
    mbar_arrive_expect_tx(fb, 2 * BLK64);
    bulk_load(st + C_OFF_MQ, ws_record(p, n, h, cw) + WS_MQ, 2 * BLK64, fb);
    iss_mq = cw + 1;
  };
  if (ctrl && lane == 0) {
    // full x 6, products x 3, o_free (8 warps), h_ready (8 warps), u_ready (8 warps), drain, PW,
    // the copy warp's drain
    const uint32_t counts[15] = {1, 1, 1, 1, 1, 1, 1, 1, 1, 8, 8, 8, 1, 1, 1};
    for (int i = 0; i < 15; ++i) mbar_init(bars + 8 * i, counts[i]);
    if (kNorm) {   // the other slice's 64 row sums: 256 transaction bytes per chunk
      mbar_init(sbase + C_OFF_PBAR, 1);
      mbar_init(sbase + C_OFF_PBAR + 8, 1);
    }
    *abort_flag = 0u;
    fence_mbar_init();
  }
  const int q4 = warp & 3, ch = (warp >> 2) & 1;     // lane quarter, column half
  const int row = 32 * q4 + lane;                    // TMEM lane / dk row of the state

  // ---- the state: row `row`, columns 32 ch .. 32 ch + 31 of this dv slice --------------
  float hreg[32];
  // where this sequence's state comes from and goes to
  const float *state_in = p.state_in;
  float *state_out = p.state_out;
  size_t sidx = n;
  if (p.slot) {
    const int e = __ldg(p.slot + n);
    if (e >= 0 && e < p.n_slots) {   // a pool entry, updated in place window by window
      sidx = static_cast<size_t>(e);
      state_in = (p.win0 == 0 && !p.pool_init) ? nullptr : p.pool;
      state_out = p.pool;
    } else {                         // no entry: from zero, through the workspace carry, dropped
      state_in = p.win0 == 0 ? nullptr : p.carry;
      state_out = p.last_window ? nullptr : p.carry;
    }
  }
  const size_t srow = (sidx * p.hv + h) * D * D + static_cast<size_t>(row) * D + slice * N + 32 * ch;
  const size_t crow = (static_cast<size_t>(n) * p.hv + h) * D * D + static_cast<size_t>(row) * D + slice * N + 32 * ch;
  const size_t in_row = (p.slot && state_in == p.carry) ? crow : srow;
  const size_t out_row = (p.slot && state_out == p.carry) ? crow : srow;
  if (state) {
    if (state_in) {
#pragma unroll
      for (int j = 0; j < 32; j += 4) {
        const float4 v4 = *reinterpret_cast<const float4 *>(state_in + in_row + j);
        hreg[j] = v4.x; hreg[j + 1] = v4.y; hreg[j + 2] = v4.z; hreg[j + 3] = v4.w;
      }
    } else {
#pragma unroll
      for (int j = 0; j < 32; ++j) hreg[j] = 0.0f;
    }
  }
  auto write_h = [&]() {
#pragma unroll
    for (int c4 = 0; c4 < 4; ++c4) {
      uint4 hi, lo;
      split8x2(hreg + 8 * c4, hi, lo);
      const uint32_t off = sw128(row, 4 * ch + c4);
      st_shared16(sbase + C_OFF_H + off, hi);
      st_shared16(sbase + C_OFF_H + BLK128 + off, lo);
    }
  };
  tc_fence_before();
  __syncthreads();   // barriers initialised, tensor memory allocated
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  const uint32_t peer = static_cast<uint32_t>(slice) ^ 1u;   // the other dv slice of this head
  if (kNorm) cluster_sync_all();   // both CTAs' barriers exist before either arrives remotely

  if (ctrl) {
    // ============= control warp: the products on the state's critical path =============
    for (int cw = 0; cw < nw; ++cw) {
      const int s = cw & 1;
      const uint32_t par = (cw >> 1) & 1, ph = cw & 1;
      const uint32_t st = sbase + s * C_STAGE;
      // ---- PW = W_hi [H_hi | H_lo] + W_lo [H_hi | -] (M = 64) ----------------------------------
      PTIME_T(1 + cw, 25, 32 * kCtrlWarp);
      chain_wait(full_qw + 8 * s, par, abort_flag, p.err);
      PTIME_T(1 + cw, 28, 32 * kCtrlWarp);
      chain_wait(h_ready, ph, abort_flag, p.err);    // H tiles of this chunk; the last PW and P read
      PTIME_T(1 + cw, 11, 32 * kCtrlWarp);
      tc_fence_after();
      if (lane == 0) {
        const uint32_t idw1 = idesc_bf16(64, 128, false, true), idw2 = idesc_bf16(64, 64, false, true);
        const uint64_t bh = sdesc(sbase + C_OFF_H, BLK128, 1024);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {   // A = rows W_hi
          const uint32_t aoff = (kk >> 2) * C_QW_KB + 64 * 128 + (kk & 3) * 32;
          mma_bf16(tmem + C_COL_PW, sdesc(st + aoff, 16, 1024), bh + ((kk * 2048) >> 4), idw1, kk > 0);
        }
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {   // A = rows W_lo, into the H_hi half
          const uint32_t aoff = (kk >> 2) * C_QW_KB + (kk & 3) * 32;
          mma_bf16(tmem + C_COL_PW, sdesc(st + aoff, 16, 1024), bh + ((kk * 2048) >> 4), idw2, 1);
        }
        mma_commit(bar_pw);
      }
      __syncwarp();
      PTIME_T(1 + cw, 1, 32 * kCtrlWarp);
      // ---- H' = K^T [U'_hi | U'_lo] ----------------------------------------------------------
      chain_wait(u_ready, ph, abort_flag, p.err);
      PTIME_T(1 + cw, 3, 32 * kCtrlWarp);
      chain_wait(full_k + 8 * s, par, abort_flag, p.err);
      PTIME_T(1 + cw, 8, 32 * kCtrlWarp);
      tc_fence_after();
      if (lane == 0) {
        const uint32_t idH = idesc_bf16(128, 128, true, true);
        const uint64_t ak = sdesc(st + C_OFF_K, BLK64, 1024);
        const uint64_t bu = sdesc(sbase + C_OFF_U + 2 * BLK64, BLK64, 1024);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          mma_bf16(tmem + C_COL_H, ak + ((kk * 2048) >> 4), bu + ((kk * 2048) >> 4), idH, kk > 0);
        mma_commit(bar_h);
      }
      __syncwarp();
      PTIME_T(1 + cw, 4, 32 * kCtrlWarp);
    }
    if (lane == 0) {   // its products complete before tensor memory is released
      mma_commit(bar_drain);
      mbar_wait(bar_drain, 0, p.err, 1u << 20);
    }
    __syncwarp();
  } else if (copier) {
    // ====== copy warp: the other products (Q H0, O) and every operand copy ======
    // Each wait here is on work this warp issued or on a handoff that needs it, so no
    // mbarrier can run a phase ahead of the wait.  P goes to the tensor pipe once PW is
    // done and O once K^T U' is done, so neither delays a product of the state chain.
    if (lane == 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      for (int c = 0; c < 2 && c < nw; ++c) {
        load_qw(c);
        load_k(c);
        load_mq(c);
      }
      for (int cw = 0; cw < nw; ++cw) {
        const int s = cw & 1;
        const uint32_t par = (cw >> 1) & 1, ph = cw & 1;
        const uint32_t st = sbase + s * C_STAGE;
        // ---- P = Q [H_hi | H_lo] (M = 64): Q H0, row 16 q + i in lane 32 q + i ------------------
        if (!chain_wait(bar_pw, ph, abort_flag, p.err)) break;
        if (!chain_wait(full_qw + 8 * s, par, abort_flag, p.err)) break;   // (landed: PW read it)
        PTIME_T(1 + cw, 31, 32 * kCopyWarp);
        tc_fence_after();
        {
          const uint32_t id1 = idesc_bf16(64, 128, false, true);
          const uint64_t bh = sdesc(sbase + C_OFF_H, BLK128, 1024);
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {   // A = the Q rows 128..191 of the k-block
            const uint32_t aoff = (kk >> 2) * C_QW_KB + 128 * 128 + (kk & 3) * 32;
            mma_bf16(tmem + C_COL_P, sdesc(st + aoff, 16, 1024), bh + ((kk * 2048) >> 4), id1, kk > 0);
          }
          mma_commit(bar_p);
        }
        PTIME_T(1 + cw, 26, 32 * kCopyWarp);
        // ---- O = Mq_hi [U_hi | U_lo] + Mq_lo [U_hi | -] (M = 64, rows as in P) -------------------
        if (!chain_wait(bar_h, ph, abort_flag, p.err)) break;             // U tiles written, K^T U' first
        PTIME_T(1 + cw, 27, 32 * kCopyWarp);
        if (cw > 0 && !chain_wait(o_free, ph ^ 1, abort_flag, p.err)) break;   // the previous O is read
        PTIME_T(1 + cw, 9, 32 * kCopyWarp);
        if (!chain_wait(full_mq + 8 * s, par, abort_flag, p.err)) break;
        PTIME_T(1 + cw, 10, 32 * kCopyWarp);
        tc_fence_after();
        {
          const uint32_t idO1 = idesc_bf16(64, 128, false, true), idO2 = idesc_bf16(64, 64, false, true);
          const uint64_t bo = sdesc(sbase + C_OFF_U, BLK64, 1024);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)   // A = Mq_hi
            mma_bf16(tmem + C_COL_O, sdesc(st + C_OFF_MQ + BLK64 + kk * 32, 16, 1024), bo + ((kk * 2048) >> 4), idO1,
                     kk > 0);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)   // A = Mq_lo, into the U_hi half
            mma_bf16(tmem + C_COL_O, sdesc(st + C_OFF_MQ + kk * 32, 16, 1024), bo + ((kk * 2048) >> 4), idO2, 1);
          mma_commit(bar_o);
        }
        PTIME_T(1 + cw, 13, 32 * kCopyWarp);
        // ---- stage s takes chunk cw + 2 once every product of chunk cw has read it (PW,
        // waited above; P and O, this thread's, complete with bar_o) -----------------------------
        if (cw + 2 < nw) {
          if (!chain_wait(bar_o, ph, abort_flag, p.err)) break;
          PTIME_T(1 + cw, 14, 32 * kCopyWarp);
          load_qw(cw + 2);
          load_k(cw + 2);
          load_mq(cw + 2);
          PTIME_T(1 + cw, 15, 32 * kCopyWarp);
        }
      }
      // its products complete before tensor memory is released; after a timeout the
      // consumers stop waiting: the last copies land before the CTA leaves (every earlier
      // copy into a stage was consumed before the stage was refilled)
      mma_commit(bar_drain2);
      mbar_wait(bar_drain2, 0, p.err, 1u << 20);
      for (int c = max(0, iss_qw - 2); c < iss_qw; ++c) mbar_wait(full_qw + 8 * (c & 1), (c >> 1) & 1, p.err, 1u << 16);
      for (int c = max(0, iss_k - 2); c < iss_k; ++c) mbar_wait(full_k + 8 * (c & 1), (c >> 1) & 1, p.err, 1u << 16);
      for (int c = max(0, iss_mq - 2); c < iss_mq; ++c) mbar_wait(full_mq + 8 * (c & 1), (c >> 1) & 1, p.err, 1u << 16);
    }
    __syncwarp();
  } else {
    // ======================== state and output warps ========================
    const uint32_t tl = tmem + (static_cast<uint32_t>(32 * q4) << 16) + 32 * ch;
    write_h();
    fence_proxy_async();
    __syncwarp();
    if (lane == 0) mbar_arrive(h_ready);

    // U phase and output (every state warp): chunk row ru = 16 q4 + (lane & 15) of the M = 64
    // products (W rows for U, Q rows for o), dv columns cu .. cu + 15 of this slice (16x32bx2
    // TMEM loads)
    const int ru = 16 * q4 + (lane & 15), cu = 32 * ch + 16 * (lane >> 4);
    // per-chunk data read into registers one chunk ahead: Ut (row ru) and scalars
    float ut[16];
    auto load_ut = [&](int cw) {
      const float4 *src = reinterpret_cast<const float4 *>(ws_record(p, n, h, cw) + WS_UT +
                                                           (static_cast<size_t>(slice) * 64 + ru) * 256);
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float4 v4 = src[((cu >> 2) + j) ^ (ru & 7)];
        ut[4 * j] = v4.x; ut[4 * j + 1] = v4.y; ut[4 * j + 2] = v4.z; ut[4 * j + 3] = v4.w;
      }
    };
    // gamma, 1/|q| and 1/|k| of row ru, gamma_(L-1)
    float nx_gu = 0.0f, nx_ku = 0.0f, nx_s = 0.0f, nx_gL = 0.0f;
    auto load_sc = [&](int cw) {
      const float *sc = reinterpret_cast<const float *>(ws_record(p, n, h, cw) + WS_SC);
      nx_gu = sc[ru];
      nx_s = sc[64 + ru];
      nx_ku = sc[128 + ru];
      nx_gL = sc[63];
    };
    if (nw > 0) {
      load_sc(0);
      load_ut(0);
    }

    float oreg[16];   // o of row ru, columns cu .. cu + 15
    for (int cw = 0; cw < nw; ++cw) {
      const uint32_t ph = cw & 1;
      const int t0 = t0_of(cw), L = min(C, seq_end - t0);
      const float g_u = nx_gu, k_u = nx_ku, sb = nx_s, gL = nx_gL;
      if (cw + 1 < nw) load_sc(cw + 1);
      PTIME(1 + cw, 0);

      {
        // ---- U = Ut - W H0 and U' = U e^(gamma_L - gamma) / |k| (W row ru, 16 columns) ------
        chain_wait(bar_pw, ph, abort_flag, p.err);
        PTIME_T(1 + cw, 22, 64);
        if (cw > 0) chain_wait(bar_o, ph ^ 1, abort_flag, p.err);   // the last O product read U
        __syncwarp();
        tc_fence_after();
        PTIME_T(1 + cw, 23, 64);
        const float ed = __expf(gL - g_u) * k_u;
        const uint32_t tw = tmem + (static_cast<uint32_t>(32 * q4) << 16) + C_COL_PW + 32 * ch;
        float pab[16], pb[16];
        tmem_ld16x2(tw, pab);        // W_hi H_hi + W_lo H_hi
        tmem_ld16x2(tw + 64, pb);    // W_hi H_lo
        tmem_wait_ld();
#pragma unroll
        for (int c4 = 0; c4 < 2; ++c4) {
          float u[8], us[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const int j = 8 * c4 + e;
            u[e] = (ut[j] - pab[j]) - pb[j];
            us[e] = u[e] * ed;
          }
          const uint32_t off = sw128(ru, (cu >> 3) + c4);
          uint4 hi, lo;
          split8x2(u, hi, lo);
          st_shared16(sbase + C_OFF_U + off, hi);
          st_shared16(sbase + C_OFF_U + BLK64 + off, lo);
          split8x2(us, hi, lo);
          st_shared16(sbase + C_OFF_U + 2 * BLK64 + off, hi);
          st_shared16(sbase + C_OFF_U + 3 * BLK64 + off, lo);
        }
        PTIME_T(1 + cw, 24, 64);
        fence_proxy_async();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(u_ready);
        PTIME_T(1 + cw, 12, 64);
        if (cw + 1 < nw) load_ut(cw + 1);
      }
      {
        // ---- Q H0 part of the output (row ru); P read the H tiles, which write_h overwrites ---
        chain_wait(bar_p, ph, abort_flag, p.err);
        __syncwarp();
        tc_fence_after();
        const float f = p.scale * __expf(g_u) * sb;
        const uint32_t tp = tmem + (static_cast<uint32_t>(32 * q4) << 16) + C_COL_P + 32 * ch;
        float pa[16], pb[16];
        tmem_ld16x2(tp, pa);        // Q H_hi
        tmem_ld16x2(tp + 64, pb);   // Q H_lo
        tmem_wait_ld();
#pragma unroll
        for (int j = 0; j < 16; ++j) oreg[j] = (pa[j] + pb[j]) * f;
      }

      // ---- H <- e^gamma_L H + K^T U' ------------------------------------------------------------
      chain_wait(bar_h, ph, abort_flag, p.err);
      __syncwarp();
      tc_fence_after();
      PTIME(1 + cw, 5);
      PTIME_T(1 + cw, 16, 64);
      PTIME_T(1 + cw, 17, 224);
      {
        const float eL = __expf(gL);
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          float ha[16], hb[16];
          tmem_ld16(tl + C_COL_H + 16 * hh, ha);
          tmem_ld16(tl + C_COL_H + 64 + 16 * hh, hb);
          tmem_wait_ld();
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const float2 hn = __ffma2_rn(make_float2(eL, eL), make_float2(hreg[16 * hh + 2 * j], hreg[16 * hh + 2 * j + 1]),
                                         __fadd2_rn(make_float2(ha[2 * j], ha[2 * j + 1]), make_float2(hb[2 * j], hb[2 * j + 1])));
            hreg[16 * hh + 2 * j] = hn.x;
            hreg[16 * hh + 2 * j + 1] = hn.y;
          }
        }
        write_h();
      }
      PTIME(1 + cw, 18);
      PTIME_T(1 + cw, 19, 64);
      fence_proxy_async();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(h_ready);
      PTIME(1 + cw, 6);
      PTIME_T(1 + cw, 20, 64);
      PTIME_T(1 + cw, 21, 224);

      // ---- output: o = scale (e^gamma / |q| Q H0 + O), row ru, overlapping the next chunk ------
      {
        uint4 zr[kNorm ? 2 : 1];   // the norm's gate, this thread's 16 columns of row ru
        const size_t orow = (static_cast<size_t>(t0 + ru) * p.hv + h) * D + slice * N + cu;
        if (kNorm) {
#pragma unroll
          for (int c2 = 0; c2 < 2; ++c2)
            zr[c2] = ru < L ? __ldg(reinterpret_cast<const uint4 *>(p.z + orow) + c2) : make_uint4(0, 0, 0, 0);
          if (tid == 0)   // this chunk's 64 row sums from the other slice: 256 bytes
            mbar_arrive_expect_tx(sbase + C_OFF_PBAR + 8 * (cw & 1), 64 * 4);
        }
        chain_wait(bar_o, ph, abort_flag, p.err);
        PTIME_T(1 + cw, 2, 64);
        __syncwarp();
        tc_fence_after();
        {
          const uint32_t to = tmem + (static_cast<uint32_t>(32 * q4) << 16) + C_COL_O + 32 * ch;
          float oa[16], ob[16];
          tmem_ld16x2(to, oa);        // Mq_hi U_hi + Mq_lo U_hi
          tmem_ld16x2(to + 64, ob);   // Mq_hi U_lo
          tmem_wait_ld();
#pragma unroll
          for (int j = 0; j < 16; ++j) oreg[j] += p.scale * (oa[j] + ob[j]);
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(o_free);
        if (kNorm) {
          // fused gated RMSNorm: the row's 128 values are split over this thread (16), its
          // partner 16 lanes away (16), the two threads of the other column half (32) and the
          // four threads of the other dv slice (64, cluster peer)
          const uint32_t pb = cw & 1;
          float ss = 0.0f;
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            oreg[j] = round_bf16(oreg[j]);   // the norm reads the bf16 o
            ss += oreg[j] * oreg[j];
          }
          ss += __shfl_xor_sync(0xffffffffu, ss, 16);
          float *s_ss = reinterpret_cast<float *>(smem + C_OFF_NORM) + pb * 128;
          if (lane < 16) s_ss[ch * 64 + ru] = ss;
          named_sync(1, 256);   // the eight state warps
          const float own = s_ss[ru] + s_ss[64 + ru];
          const uint32_t peer_slot = smem_u32(smem + C_OFF_PEER) + (pb * 64 + ru) * 4;
          if (ch == 0 && lane < 16)
            st_async_remote(map_peer(peer_slot, peer), own, map_peer(sbase + C_OFF_PBAR + 8 * pb, peer));
          PTIME_T(1 + cw, 29, 64);
          float total = own;
          if (chain_wait_cluster(sbase + C_OFF_PBAR + 8 * pb, (cw >> 1) & 1, abort_flag, p.err))
            total += reinterpret_cast<const float *>(smem + C_OFF_PEER)[pb * 64 + ru];
          PTIME_T(1 + cw, 30, 64);
          const float inv = 1.0f / sqrtf(total * (1.0f / 128.0f) + p.eps);
          if (ru < L) {
            const int col0 = slice * N + cu;
#pragma unroll
            for (int c2 = 0; c2 < 2; ++c2) {
              float zf[8], yv[8];
              unpack8(zr[c2], zf);
#pragma unroll
              for (int e = 0; e < 8; ++e) {
                const float wv = p.norm_w ? __ldg(p.norm_w + col0 + 8 * c2 + e) : 1.0f;
                yv[e] = oreg[8 * c2 + e] * inv * wv * silu_fast(zf[e]);
              }
              *reinterpret_cast<uint4 *>(p.y + orow + 8 * c2) = pack8x2(yv);
              if (p.o) *reinterpret_cast<uint4 *>(p.o + orow + 8 * c2) = pack8x2(oreg + 8 * c2);
            }
          }
        } else if (ru < L) {
#pragma unroll
          for (int c2 = 0; c2 < 2; ++c2) *reinterpret_cast<uint4 *>(p.o + orow + 8 * c2) = pack8x2(oreg + 8 * c2);
        }
        PTIME_T(1 + cw, 7, 64);
      }
    }
  }
  if (kNorm) cluster_sync_all();   // no remote arrivals target a CTA that has left
  tc_fence_before();
  __syncthreads();
  if (state && state_out && *abort_flag == 0u) {
#pragma unroll
    for (int j = 0; j < 32; j += 4)
      *reinterpret_cast<float4 *>(state_out + out_row + j) = make_float4(hreg[j], hreg[j + 1], hreg[j + 2], hreg[j + 3]);
  }
  if (warp == 0) tmem_dealloc(tmem, C_TM_COLS);
}

// ---- host side ---------------------------------------------------------------
// [rows][cols] bf16 with a row stride in elements; 64 x 64 boxes, 128B swizzle;
// rows past `rows` read as zero
bool make_map(CUtensorMap *m, const void *base, uint64_t cols, uint64_t rows, uint64_t row_stride) {
  EncodeTiledFn f = tensor_map_encoder();
  if (!f) return false;
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {row_stride * 2};
  const cuuint32_t box[2] = {64, 64};
  const cuuint32_t estr[2] = {1, 1};
  return f(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides, box, estr,
           CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
           CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// per-device one-time opt-in to large dynamic shared memory
int ensure_smem_attrs() {
  static std::atomic<uint64_t> done{0};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return launch_status(e, "prefill: cudaGetDevice");
  const uint64_t bit = dev < 64 ? (uint64_t{1} << dev) : 0;
  if (bit && (done.load(std::memory_order_acquire) & bit)) return GDR_OK;
  e = cudaFuncSetAttribute(prep_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, P_SMEM);
  if (e == cudaSuccess)   // room for three prep CTAs per SM
    e = cudaFuncSetAttribute(prep_kernel, cudaFuncAttributePreferredSharedMemoryCarveout,
                             cudaSharedmemCarveoutMaxShared);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(chain_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, C_SMEM);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(chain_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, C_SMEM);
  if (e != cudaSuccess) return launch_status(e, "prefill: shared memory opt-in");
  done.fetch_or(bit, std::memory_order_acq_rel);
  return GDR_OK;
}

// ---- pipelined windows -------------------------------------------------------
// When the chains of a call leave SMs idle (fewer than one chain CTA per SM) and the
// sequences span several windows, the prep of window w + 1 runs beside the chain of
// window w: chains on a high-priority stream, preps on a low-priority one, records in two
// buffers used alternately.  The prep CTAs take the SMs the chains leave free and spread
// to all of them once a chain window ends.  Both streams belong to the library (one pair
// per device), fork from the caller's stream and join it again before the call returns,
// so the caller's stream order sees one piece of work.  A call whose stream is being
// captured into a graph keeps the serial schedule.
constexpr int kPipeMinChunks = 16;   // below this the extra chain start-ups cost more than the overlap
constexpr int kPipeEvents = 64;

struct PipeStreams {
  cudaStream_t hi = nullptr, lo = nullptr;
  cudaEvent_t ev[kPipeEvents] = {};
  int next = 0;
  std::mutex lock;   // one call at a time issues on a device's pair
};

int pipe_streams(PipeStreams **out) {
  static PipeStreams per_dev[64];
  static std::mutex init_lock;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return launch_status(e, "prefill: cudaGetDevice");
  if (dev < 0 || dev >= 64) return GDR_ERR_UNSUPPORTED;
  PipeStreams &ps = per_dev[dev];
  std::lock_guard<std::mutex> g(init_lock);
  if (!ps.hi) {
    int least = 0, greatest = 0;
    cudaStream_t hi = nullptr, lo = nullptr;
    e = cudaDeviceGetStreamPriorityRange(&least, &greatest);
    if (e == cudaSuccess) e = cudaStreamCreateWithPriority(&hi, cudaStreamNonBlocking, greatest);
    if (e == cudaSuccess) e = cudaStreamCreateWithPriority(&lo, cudaStreamNonBlocking, least);
    for (int i = 0; i < kPipeEvents && e == cudaSuccess; ++i)
      e = cudaEventCreateWithFlags(&ps.ev[i], cudaEventDisableTiming);
    if (e != cudaSuccess) return launch_status(e, "prefill: pipeline streams");
    ps.lo = lo;
    ps.hi = hi;
  }
  *out = &ps;
  return GDR_OK;
}

int device_sms(int *sms) {
  static std::atomic<int> cached[64];
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return launch_status(e, "prefill: cudaGetDevice");
  if (dev < 0 || dev >= 64) return GDR_ERR_UNSUPPORTED;
  int n = cached[dev].load(std::memory_order_relaxed);
  if (n == 0) {
    e = cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return launch_status(e, "prefill: SM count");
    cached[dev].store(n, std::memory_order_relaxed);
  }
  *sms = n;
  return GDR_OK;
}

}  // namespace

// The window schedule of a call: as many chunks per window as the workspace holds (the
// state crosses windows in hT, in the pool entries, or in the workspace tail), or, pipelined
// (see PipeStreams), two record buffers when the chains leave SMs idle, each buffer at least
// kPipeMinChunks chunks, and at least three windows result.
int plan_chunk_prefill(int n_seqs, int hv, int max_chunks, size_t ws_bytes, bool carry_in_ws, bool capturing,
                       int *windows, int *win_chunks, bool *pipelined) {
  const size_t rec_per_chunk = static_cast<size_t>(n_seqs) * hv * WS_REC;
  const size_t carry = carry_in_ws ? chunk_prefill_workspace_bytes(n_seqs, hv, 0, true) : 0;
  *pipelined = false;
  if (max_chunks <= 0) {
    *windows = 1;
    *win_chunks = 1;
    return GDR_OK;
  }
  if (rec_per_chunk == 0 || ws_bytes < carry + rec_per_chunk) return GDR_ERR_WORKSPACE;
  int win = static_cast<int>(std::min<size_t>({(ws_bytes - carry) / rec_per_chunk, static_cast<size_t>(max_chunks),
                                               size_t{65535}}));
  const size_t fit2 = (ws_bytes - carry) / (2 * rec_per_chunk);
  if (!capturing && max_chunks > 2 * kPipeMinChunks && fit2 >= static_cast<size_t>(kPipeMinChunks) &&
      max_chunks > win) {
    int sms = 0;
    const int st = device_sms(&sms);
    if (st) return st;
    if (static_cast<long long>(n_seqs) * hv * NS < sms) {
      const int win2 = static_cast<int>(std::min<size_t>({fit2, static_cast<size_t>(max_chunks), size_t{65535}}));
      if ((max_chunks + win2 - 1) / win2 >= 3) {
        win = win2;
        *pipelined = true;
      }
    }
  }
  *win_chunks = win;
  *windows = (max_chunks + win - 1) / win;
  return GDR_OK;
}

size_t chunk_prefill_workspace_bytes(int n_seqs, int hv, int window_chunks, bool need_carry) {
  size_t b = static_cast<size_t>(n_seqs) * hv * window_chunks * WS_REC;
  if (need_carry) b += static_cast<size_t>(n_seqs) * hv * D * D * sizeof(float);
  return b;
}

int launch_chunk_prefill(const void *q, const void *k, const void *v, int64_t qk_stride,
                         int64_t v_stride, const void *a, const void *b,
                         const float *A_log, const float *dt_bias, float scale, int hk, int hv,
                         const int32_t *cu_dev, const int32_t *cu_host, int n_seqs, int total, int max_chunks,
                         const float *h0, float *hT, void *o, const void *z, const float *norm_w,
                         float eps, void *y, void *workspace, size_t ws_bytes, cudaStream_t s,
                         const PrefillPool *pool) {
  if (n_seqs > 65535 || hv > 65535) return GDR_ERR_SHAPE;
  int st = ensure_smem_attrs();
  if (st) return st;
  const bool carry_in_ws = hT == nullptr;
  const size_t rec_per_chunk = static_cast<size_t>(n_seqs) * hv * WS_REC;
  if (max_chunks > 0 && !workspace) return GDR_ERR_WORKSPACE;
  // under stream capture the call keeps to the caller's stream: the library's streams are
  // shared by all calls on the device and must not join one caller's graph
  cudaStreamCaptureStatus capture = cudaStreamCaptureStatusNone;
  if (max_chunks > 2 * kPipeMinChunks) {
    const cudaError_t ce = cudaStreamIsCapturing(s, &capture);
    if (ce != cudaSuccess) return launch_status(ce, "prefill: cudaStreamIsCapturing");
  }
  int n_windows = 1, win = 1;
  bool pipelined = false;
  st = plan_chunk_prefill(n_seqs, hv, max_chunks, ws_bytes, carry_in_ws, capture != cudaStreamCaptureStatusNone,
                          &n_windows, &win, &pipelined);
  if (st) return st;
  PipeStreams *ps = nullptr;
  if (pipelined && (st = pipe_streams(&ps))) return st;
  const size_t buf_bytes = rec_per_chunk * win;
  float *carry_buf = carry_in_ws && max_chunks > 0
                         ? reinterpret_cast<float *>(static_cast<uint8_t *>(workspace) + buf_bytes * (pipelined ? 2 : 1))
                         : nullptr;
  CUtensorMap tq, tk, tv;
  const uint64_t rows = total > 0 ? static_cast<uint64_t>(total) : 1;
  // with no tokens no tile is ever loaded; any aligned device address serves as a base
  const void *any = v ? v : (hT ? static_cast<const void *>(hT) : static_cast<const void *>(h0));
  if (!any && pool) any = pool->pool;
  if (!any) return GDR_OK;
  if (!tensor_map_encoder()) return launch_status(cudaErrorSymbolNotFound, "prefill: cuTensorMapEncodeTiled lookup");
  if (!make_map(&tq, q ? q : any, static_cast<uint64_t>(hk) * D, rows, static_cast<uint64_t>(qk_stride)) ||
      !make_map(&tk, k ? k : any, static_cast<uint64_t>(hk) * D, rows, static_cast<uint64_t>(qk_stride)) ||
      !make_map(&tv, v ? v : any, static_cast<uint64_t>(hv) * D, rows, static_cast<uint64_t>(v_stride)))
    return launch_status(cudaErrorInvalidValue, "prefill: tensor map encoding");

  PrefillParams p;
  p.a = static_cast<const uint16_t *>(a);
  p.b = static_cast<const uint16_t *>(b);
  p.A_log = A_log;
  p.dt_bias = dt_bias;
  p.scale = scale;
  p.hk = hk;
  p.hv = hv;
  p.group = hv / hk;
  p.cu = cu_dev;
  p.n_seqs = n_seqs;
  for (int i = 0; i <= kCuParam; ++i) p.cu_param[i] = i <= n_seqs ? cu_host[i] : 0;
  p.ws = static_cast<uint8_t *>(workspace);
  p.win_chunks = win;
  p.o = static_cast<uint16_t *>(o);
  p.z = static_cast<const uint16_t *>(z);
  p.norm_w = norm_w;
  p.eps = eps;
  p.y = static_cast<uint16_t *>(y);
  p.err = device_error_ptr();
  p.slot = pool ? pool->slot : nullptr;
  p.n_slots = pool ? pool->n_slots : 0;
  p.pool_init = pool ? pool->init_from_pool : 0;
  p.pool = pool ? pool->pool : nullptr;
  p.carry = carry_buf;
  auto window_params = [&](int w) {
    PrefillParams pw = p;
    pw.win0 = w * win;
    const bool first = w == 0, last = w == n_windows - 1;
    pw.state_in = first ? h0 : (carry_in_ws ? carry_buf : hT);
    pw.state_out = last ? hT : (carry_in_ws ? carry_buf : hT);
    pw.last_window = last ? 1 : 0;
    if (pipelined) pw.ws = static_cast<uint8_t *>(workspace) + (w & 1) * buf_bytes;
    return pw;
  };
  auto launch_prep = [&](int w, cudaStream_t stream) -> int {
    const PrefillParams pw = window_params(w);
    const int nc = std::min(win, max_chunks - pw.win0);
    if (nc <= 0) return GDR_OK;
    return launch_status(launch_pdl(prep_kernel, dim3(nc, hv, n_seqs), dim3(kPrepThreads), P_SMEM, stream, 1, tq, tk,
                                    tv, pw),
                         "prefill: prep kernel launch");
  };
  auto launch_chain = [&](int w, cudaStream_t stream) -> int {
    const PrefillParams pw = window_params(w);
    // with the fused norm the two dv slices of a head form a cluster and exchange row sums
    return y ? launch_status(launch_pdl(chain_kernel<true>, dim3(NS, hv, n_seqs), dim3(kChainThreads), C_SMEM, stream,
                                        static_cast<unsigned>(NS), tq, tk, pw),
                             "prefill: chain kernel launch")
             : launch_status(launch_pdl(chain_kernel<false>, dim3(NS, hv, n_seqs), dim3(kChainThreads), C_SMEM, stream,
                                        1, tq, tk, pw),
                             "prefill: chain kernel launch");
  };
  if (!pipelined) {
    for (int w = 0; w < n_windows; ++w) {
      if ((st = launch_prep(w, s)) || (st = launch_chain(w, s))) return st;
    }
    return GDR_OK;
  }
  // pipelined: chain w on `hi` after prep w; prep w + 1 on `lo` beside chain w, once chain
  // w - 1 has released the buffer it reuses
  std::lock_guard<std::mutex> g(ps->lock);
  auto record = [&](cudaStream_t from, cudaEvent_t *e) -> int {   // mark `from`'s work so far
    *e = ps->ev[ps->next];
    ps->next = (ps->next + 1) % kPipeEvents;
    return launch_status(cudaEventRecord(*e, from), "prefill: stream ordering");
  };
  auto wait = [&](cudaStream_t to, cudaEvent_t e) -> int {
    return launch_status(cudaStreamWaitEvent(to, e, 0), "prefill: stream ordering");
  };
  cudaEvent_t e = nullptr, chain_prev = nullptr, chain_cur = nullptr;
  if ((st = record(s, &e)) || (st = wait(ps->hi, e)) || (st = wait(ps->lo, e))) return st;
  if ((st = launch_prep(0, ps->lo))) return st;
  for (int w = 0; w < n_windows; ++w) {
    if ((st = record(ps->lo, &e)) || (st = wait(ps->hi, e))) return st;   // prep w is done
    if ((st = launch_chain(w, ps->hi)) || (st = record(ps->hi, &chain_cur))) return st;
    if (w + 1 < n_windows) {
      if (w >= 1 && (st = wait(ps->lo, chain_prev))) return st;   // chain w - 1 read the buffer
      if ((st = launch_prep(w + 1, ps->lo))) return st;
    }
    chain_prev = chain_cur;
  }
  return wait(s, chain_prev);   // the last prep precedes the last chain
}

}  // namespace gdr

#ifdef GDR_PREFILL_TIMING
extern "C" GDR_API int gdr_debug_set_prefill_times(long long *dev_ptr) {
  return cudaMemcpyToSymbol(gdr::g_prefill_times, &dev_ptr, sizeof(dev_ptr)) == cudaSuccess ? 0 : 7;
}
#endif
